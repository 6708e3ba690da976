// fa_kernels.h -- parameter blocks shared by the host launch code and the
// kernels of libfa (internal; not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace fa {

struct FwdParams {
    void* o;            // [B, Hq, Nq, d] (bf16 or fp16)
    float* lse;         // [B, Hq, Nq] or nullptr
    int B, Hq, Hkv, Nq, Nk;
    int G;              // Hq / Hkv
    int n_pairs;        // query tile pairs per tile head: ceil(rows / 256) (ceil(rows / 128) at d = 256)
    // tile heads: with group_rows = 0 each (batch, query head), whose rows are its Nq query
    // positions; with group_rows = 1 each (batch, kv head), whose rows are the G * Nq rows of its
    // G query heads (consecutive in q / o / lse), row r at query position r % Nq
    int group_rows;
    int n_bh;           // B * Hq, or B * Hkv with group rows
    int rows;           // Nq, or G * Nq with group rows
    int d_io;           // head dim of the tensors in memory (<= kernel D, multiple of 32); the
                        // columns d_io..D-1 of the tiles are TMA zero fill and are never stored
    float scale_log2;   // scale * log2(e) (times the Q and K descales for e4m3 inputs)
    float o_scale;      // O = o_scale * U / l: 1, or the V descale for e4m3 inputs
    unsigned* tile_ctr; // [4]: tiles claimed beyond each block's first, blocks done claiming,
                        // owner tag (zero when free; the last block resets all three), padding
    unsigned tile_tag;  // this launch's owner tag (nonzero)
    // key split (fwd_kernel<..., SPLIT = true>): the work units (query tile pair, tile head) in
    // claim order u = 0, 1, ...; units u < full_tiles are one work tile each, every later unit is
    // kv_split work tiles, share s taking the pair's key blocks [s * n / kv_split,
    // (s + 1) * n / kv_split) of its n; the shares' partial results are merged by
    // fwd_combine_kernel (full_tiles = 0: every unit is split)
    int kv_split;
    int full_tiles;
    int pair_rows;      // query rows of a work unit: 256 (128 at d = 256)
    float* part_o;      // [n_bh, kv_split, rows, d_io] fp32: O_s = U_s / l_s of share s
    float* part_lse;    // [n_bh, kv_split, rows] fp32: m_s + log2(l_s), -inf where share s sees no key
};

struct DecodeParams {
    const void* q;           // [B, Hq, Nq, d]  (16-bit elements, bf16 or fp16)
    const void* k;           // [B, Hkv, Nk, d]
    const void* v;
    void* o;                 // [B, Hq, Nq, d]
    float* lse;              // [B, Hq, Nq] or nullptr
    float* part_o;           // [B * Hkv, splits, R, d]  partial O_s (normalised)
    float* part_lse;         // [B * Hkv, splits, R]     partial lse_s
    int B, Hq, Hkv, Nq, Nk;
    int G;                   // Hq / Hkv
    int R;                   // rows per kv group = G * Nq (<= 16)
    int splits;              // key chunks per (b, kv head)
    int chunk;               // keys per chunk (multiple of the key tile)
    int causal;
    int d_io;                // head dim in memory (<= 128, multiple of 32): columns d_io..127 are zero
                             // fill of the K/V tiles, zero in Q, skipped in the MMAs and never stored
    float scale_log2;
    // paged KV cache (decode_split_kernel<true>): K/V are [num_pages, page_size, Hkv, d];
    // the keys of sequence b are block_table[b][key / page_size] * page_size + key % page_size,
    // and sequence b has seq_lens[b] keys (Nk is then the longest allowed length)
    const int* block_table;  // [B, max_pages]
    const int* seq_lens;     // [B]
    int page_size;
    int max_pages;
};

struct BwdParams {
    const void* q;              // [B, Hq, Nq, d]  (16-bit elements, bf16 or fp16)
    const void* k;              // [B, Hkv, Nk, d]
    const void* v;
    const void* o;              // [B, Hq, Nq, d]
    const void* dout;           // [B, Hq, Nq, d]
    const float* lse;           // [B, Hq, Nq]
    void* dq;                   // [B, Hq, Nq, d]
    void* dk;                   // [B, Hkv, Nk, d]
    void* dv;
    float* neg_delta;           // [B, Hq, Nq_pad]  -D_i = -rowsum(dout * o)
    float* neg_lse_log2;        // [B, Hq, Nq_pad]  -LSE_i * log2(e) (-inf for masked and padded rows)
    float* dq_acc;              // [B, Hq, Nq_pad, d] fp32 accumulator
    int B, Hq, Hkv, Nq, Nk;
    int G;
    int Nq_pad;                 // Nq rounded up to the query block
    int d_io;                   // head dim in memory (<= kernel D, multiple of 32); dq_acc keeps D
    int causal;
    float scale;
    float scale_log2;
    // q_split CTAs share each (key block, kv head[, feature half]) unit, each walking
    // its own share of the unit's query steps; all but the last to finish leave their
    // fp32 dK / dV sums in dkv_part, and the last adds them up (q_split = 1: no split)
    int q_split;
    int n_split_units;          // units of the launch (q_split > 1)
    float4* dkv_part;           // [n_split_units][q_split == 2 ? 1 : q_split][2 * dK/dV features / 4][128]
    int* split_cnt;             // [2][n_split_units]: tickets taken, partials written
};

}  // namespace fa
