// fa_kernels.h -- parameter blocks shared by the host launch code and the
// kernels of libfa (internal; not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace fa {

struct FwdParams {
    __nv_bfloat16* o;   // [B, Hq, Nq, d]
    float* lse;         // [B, Hq, Nq] or nullptr
    int B, Hq, Hkv, Nq, Nk;
    int G;              // Hq / Hkv
    int n_pairs;        // ceil(Nq / 256): 256-row query tile pairs per head
    float scale_log2;   // scale * log2(e)
};

struct DecodeParams {
    const __nv_bfloat16* q;  // [B, Hq, Nq, d]
    const __nv_bfloat16* k;  // [B, Hkv, Nk, d]
    const __nv_bfloat16* v;
    __nv_bfloat16* o;        // [B, Hq, Nq, d]
    float* lse;              // [B, Hq, Nq] or nullptr
    float* part_o;           // [B * Hkv, splits, R, d]  partial O_s (normalised)
    float* part_lse;         // [B * Hkv, splits, R]     partial lse_s
    int B, Hq, Hkv, Nq, Nk;
    int G;                   // Hq / Hkv
    int R;                   // rows per kv group = G * Nq (<= 16)
    int splits;              // key chunks per (b, kv head)
    int chunk;               // keys per chunk (multiple of the key tile)
    int causal;
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
    const __nv_bfloat16* q;     // [B, Hq, Nq, d]
    const __nv_bfloat16* k;     // [B, Hkv, Nk, d]
    const __nv_bfloat16* v;
    const __nv_bfloat16* o;     // [B, Hq, Nq, d]
    const __nv_bfloat16* dout;  // [B, Hq, Nq, d]
    const float* lse;           // [B, Hq, Nq]
    __nv_bfloat16* dq;          // [B, Hq, Nq, d]
    __nv_bfloat16* dk;          // [B, Hkv, Nk, d]
    __nv_bfloat16* dv;
    float* delta;               // [B, Hq, Nq_pad]  D_i = rowsum(dout * o)
    float* lse_log2;            // [B, Hq, Nq_pad]  LSE_i * log2(e) (+inf for masked rows)
    float* dq_acc;              // [B, Hq, Nq_pad, d] fp32 accumulator
    int B, Hq, Hkv, Nq, Nk;
    int G;
    int Nq_pad;                 // Nq rounded up to the query block
    int causal;
    float scale;
    float scale_log2;
};

}  // namespace fa
