// fwd.cuh -- forward kernel: O = softmax(scale * Q K^T + mask) V and the per-row
// LSE, tile by tile with the online-softmax state (m, l, U) of the page
// "FlashAttention：为什么少搬数据，反而算得更快", §03 (fix a block of Q, stream the
// K/V blocks past it) and §04 (m_new = max(m_old, max block), rescale the old
// numerator and denominator together by exp(m_old - m_new), add the block).
//
// Layout of one CTA (384 threads = 3 warpgroups, one CTA per SM):
//   * per work tile, two 128-row query tiles of one tile head, Q0 and Q1, staged
//     in shared memory by TMA (128-byte swizzle, 64-column panels); a tile head is
//     a (batch, query head), or a (batch, kv head) whose G query heads' rows
//     share its tiles when each has fewer rows than a tile (group rows);
//   * K and V blocks of 128 keys stream through one ring of NSTAGE tile slots
//     (order K0, V0, K1, V1, ...), each slot guarded by a full / empty mbarrier;
//   * tensor memory (512 columns): S0 | S1 (128 fp32 columns each) | O0 | O1
//     (d fp32 columns each).  P overwrites the first 64 columns of its S tile as
//     packed bf16 pairs and is read from there by the P.V MMA;
//   * warps 0-3 run the softmax of tile 0, warps 4-7 that of tile 1: thread r of
//     a warpgroup owns query row r, which is TMEM lane r;
//   * warp 8 claims the work tiles and issues the TMA loads, warp 9 (one
//     elected thread) the tcgen05.mma ops in the
//     order S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ..., so the softmax of
//     one tile overlaps the MMAs of the other; warps 10-11 only complete the
//     third warpgroup, which hands most of its registers to the softmax ones.
//
// The launch is persistent: one CTA per SM works through the (query tile pair,
// tile head) tiles, heaviest causal tiles first, each CTA claiming its next
// tile from an atomic counter (fwd_tile).  The TMA warp claims it and hands it
// to the other roles through a two-entry ring in shared memory.  TMEM,
// barriers and the K/V ring carry over from tile to tile.  The producer reloads a
// Q slot as soon as the tile's last Q.K^T has read it, and the MMA warp starts
// the next tile's S while the softmax warps still write this tile's O.  The
// start-up of a tile (Q load, first S) and its epilogue therefore overlap the
// neighbouring tiles' work instead of leaving the tensor core idle.
//
// At d = 256 the CTA holds one query tile (kTiles = 1): its O accumulator takes
// 256 TMEM columns, so there is no room for a second tile's S and O, and the
// second softmax warpgroup has no work.  The other 256 columns hold two S
// buffers instead: block j's S goes to buffer j & 1 and the MMA order is
// S(0) S(1) | PV(j) S(j+2) | ..., so each block's Q.K^T runs during the previous
// block's softmax.  K and V then keep fixed ring slots (K in 0, V in 1), loaded
// in the order the MMAs free them, and a softmax that rescales O first waits for
// the previous block's P.V (S(j) no longer follows it).
//
// Key split (SPLIT): where the launch has fewer work tiles than SMs, each tile's
// key blocks are cut into kv_split contiguous shares that run as tiles of their
// own; a share ends with O_s = U_s / l_s in fp32 and lse_s = m_s + log2(l_s), and
// fwd_combine_kernel merges the shares by their lse (the same rescale-and-add as
// between blocks).
//
// Scores are kept in the log2 domain: x = s * scale * log2(e), p = 2^(x - m).
// Rescaling is lazy: the reference max m moves (and U, l are multiplied by
// 2^(m_old - m_new)) only when the block max exceeds it by more than
// kRescaleLog2; until then p <= 2^kRescaleLog2, well inside fp32 and bf16
// range.  O = U / l and LSE = (m + log2 l) ln 2 use the same reference, so the
// result is the same normalised softmax (§04: any common reference gives the
// same answer once numerator and denominator are rescaled together).
#pragma once

#include <type_traits>

#include "sm100.cuh"
#include "fa_kernels.h"

namespace fa {

constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

// F8: Q, K, V are e4m3 bytes and V arrives transposed (d rows of 128 keys),
// see fp8_vt_kernel; otherwise they are 16-bit (T).
template <int D, bool F8 = false>
struct FwdCfg {
    static constexpr int kTiles = (D == 256) ? 1 : 2;    // 128-row query tiles per CTA
    static constexpr int kThreads = 384;
    // registers per thread after the split: 2 x 128 x 208 + 128 x 88 = 384 x 168
    static constexpr uint32_t kRegsSoftmax = 208, kRegsOther = 88;
    static constexpr int kElt = F8 ? 1 : 2;              // bytes per Q/K/V element
    static constexpr int kTileBytes = 128 * D * kElt;    // a 128-row Q or K tile, a V tile
    static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes (one swizzle span)
    static constexpr int kPanels = D * kElt / 128;
    static constexpr int kPanelElems = 128 / kElt;
    static constexpr int kKSteps = D * kElt / 32;        // Q.K^T instructions (32 bytes of d each)
    static constexpr int kStages = F8 ? 10 : (D == 256) ? 2 : (D == 128) ? 5 : 8;
    static constexpr int kBarBytes = 512;
    // part of the exponentials on the FMA pipe (exp2_poly2): pays at d = 128 and for
    // e4m3, where the MUFU unit is the busier one; at d = 64 and 256 all of them on the
    // MUFU measured faster (the FMA-pipe work slows the co-running MMA issue more)
    static constexpr bool kPoly = F8 || D == 128;
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = kTiles * kTileBytes;
    static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + barriers + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static_assert(!F8 || D == 128, "the e4m3 kernel is built for d = 128");
    // setmaxnreg: 168 registers per thread at launch (384 threads); the two softmax
    // warpgroups raise theirs, the third lowers its, within the launch's total
    static_assert(kRegsSoftmax >= 168 && kRegsOther <= 168 && 2 * kRegsSoftmax + kRegsOther <= 3 * 168,
                  "register split");
    static_assert(kTiles == 2 || 2 * 128 + D <= (int)kTmemCols, "one tile: two S buffers and O must fit in TMEM");
};

// 128-key blocks seen by the 128-row query tile at row qt of a tile head with `rows`
// rows, row r at query position r % Nq (rows = Nq: position r)
__device__ __forceinline__ int fwd_blocks_for_tile(int qt, int rows, int Nq, int Nk, bool causal)
{
    const int nkb = (Nk + 127) / 128;
    if (qt >= rows)
        return 0;
    if (!causal)
        return nkb;
    const int last_row = min(qt + 127, rows - 1);
    // the largest query position among the tile's rows
    const int last_pos = (qt / Nq == last_row / Nq) ? last_row % Nq : Nq - 1;
    const int last_key = last_pos + (Nk - Nq);
    if (last_key < 0)
        return 0;
    return min(nkb, last_key / 128 + 1);
}

// Tile counters of the forward launches, four words per slot: tiles claimed
// beyond each block's first, blocks that have stopped claiming, the owner tag
// of the launch using the slot (0 = free), and padding.  Each launch takes the
// next slot (launches in flight on different streams do not share one) and a
// nonzero tag of its own.  Every block first swaps the free owner word for its
// launch's tag; a block that finds another launch's tag there records
// kStatusSlotShared, runs its own first tile only and leaves the slot alone, so
// the other launch's tiles are never taken.  The last block to stop claiming
// sets the counters and then the owner back to zero, so a slot is all zero
// whenever no launch is using it.
constexpr int kFwdCtrSlots = 256;
constexpr int kFwdCtrWords = 4;
__device__ unsigned g_fwd_tile_ctr[kFwdCtrSlots][kFwdCtrWords];

// One work tile: a pair of 128-row query tiles (one at d = 256) of one tile head
// (see FwdParams::group_rows).  Tile i of the launch: pair n_pairs-1 - i / n_bh
// (heaviest causal pairs first; with a key split, i / (n_bh * kv_split)), tile head
// i % n_bh.
struct FwdTile {
    int bh;        // tile head: batch * Hq + head, or batch * Hkv + kv head with group rows
    int kvh;       // batch * Hkv + kv head
    int q0;        // first query row
    int nb0, nb1;  // 128-key blocks seen by query tile 0 / 1 (in this tile's key share)
    int n_iter;    // max of the two
    int kb0;       // first key block of the share (0 without a key split)
    int share;     // key share (0 without a key split)
    int nshares;   // key shares of the tile's unit (1: the whole unit, written straight to o / lse)
};

// The launch has at most one block per SM.  Block c starts with tile c; each
// further tile is the next unclaimed one (the launch's tile counter), so like a
// hardware block scheduler the blocks take the heavy causal tiles first and
// whichever block is free takes the next.  With a key split (SPLIT) tile i is
// share (i / (B*Hq)) % kv_split of its pair's key blocks.
template <int kTiles, bool CAUSAL, bool SPLIT = false>
__device__ __forceinline__ void fwd_tile(const FwdParams& p, int i, FwdTile& w)
{
    const int n_bh = p.n_bh;
    // unit u = (pair n_pairs - 1 - u / n_bh, tile head u % n_bh); units below full_tiles whole
    int u = i, ns = 1;
    w.share = 0;
    if constexpr (SPLIT) {
        if (i >= p.full_tiles) {
            ns = p.kv_split;
            u = p.full_tiles + (i - p.full_tiles) / ns;
            w.share = (i - p.full_tiles) % ns;
        }
    }
    w.nshares = ns;
    const int pair = p.n_pairs - 1 - u / n_bh;
    w.bh = u % n_bh;
    if (p.group_rows) {
        w.kvh = w.bh;
    } else {
        const int b = w.bh / p.Hq, h = w.bh % p.Hq;
        w.kvh = b * p.Hkv + h / p.G;
    }
    w.q0 = pair * 128 * kTiles;
    w.nb0 = fwd_blocks_for_tile(w.q0, p.rows, p.Nq, p.Nk, CAUSAL);
    w.nb1 = (kTiles == 2) ? fwd_blocks_for_tile(w.q0 + 128, p.rows, p.Nq, p.Nk, CAUSAL) : 0;
    w.kb0 = 0;
    if (SPLIT && ns > 1) {
        // blocks [lo, hi) of the pair's n; a tile sees the part of them below its own count
        const int n = max(w.nb0, w.nb1);
        const int lo = (int)(((long long)w.share * n) / ns), hi = (int)(((long long)(w.share + 1) * n) / ns);
        w.kb0 = lo;
        w.nb0 = max(0, min(hi, w.nb0) - lo);
        w.nb1 = max(0, min(hi, w.nb1) - lo);
    }
    w.n_iter = max(w.nb0, w.nb1);
}

// A consumer warp's read of the u-th tile index: wait until the producer has
// published it, read it, and give the ring entry back (one arrival per warp).
__device__ __forceinline__ int fwd_take_tile(uint64_t* bar_tfull, uint64_t* bar_tfree, volatile int* tile_ring,
                                             int u, int lane, volatile int* abort_flag, bool& ok)
{
    ok = __all_sync(0xffffffffu, mbar_wait(&bar_tfull[u & 1], (uint32_t)(u >> 1) & 1u, abort_flag));
    if (!ok)
        return 0;
    const int tile = tile_ring[u & 1];
    __syncwarp();
    if (lane == 0)
        mbar_arrive(&bar_tfree[u & 1]);
    return tile;
}

// SPLIT: key split (kv_split shares per pair, partial results to part_o / part_lse);
// without it the kernel carries none of the split's code
template <int D, bool CAUSAL, typename T = __nv_bfloat16, bool F8 = false, bool SPLIT = false>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, FwdParams p)
{
    using C = FwdCfg<D, F8>;
    griddep_launch_dependents();   // the merge of a key split may be scheduled
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sKV = smem + C::kOffKV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    // Barrier phases run on across the tiles of the block: every role counts
    // the completions it has waited for (Q loads per tile slot, K/V ring loads,
    // blocks per tile slot, tiles per tile slot) and waits on their parity.
    uint64_t* bar_q = bars;                            // [2]  Q tile landed
    uint64_t* bar_qfree = bar_q + 2;                   // [2]  last Q.K^T of a tile done: Q slot reusable
    uint64_t* bar_full = bar_qfree + 2;                // [S]  ring slot landed
    uint64_t* bar_empty = bar_full + C::kStages;       // [S]  ring slot released
    uint64_t* bar_s = bar_empty + C::kStages;          // [2]  S tile ready in TMEM
    uint64_t* bar_p = bar_s + 2;                       // [2][2] P half h (and O rescale) written
    uint64_t* bar_o = bar_p + 4;                       // [2]  last P.V of a tile done
    uint64_t* bar_drain = bar_o + 2;                   // [1]  MMA drain on abort
    uint64_t* bar_tfull = bar_drain + 1;               // [2]  tile index published in tile_ring[u & 1]
    uint64_t* bar_tfree = bar_tfull + 2;               // [2]  tile index read by the MMA and softmax warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tfree + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* tile_ring = abort_flag + 1;          // [2]  tile indices (>= n_tiles: no more)
    static_assert((17 + 2 * C::kStages) * 8 + 16 <= C::kBarBytes, "barrier area too small");
    const int n_units = p.n_pairs * p.n_bh;
    const int n_tiles = SPLIT ? p.full_tiles + (n_units - p.full_tiles) * p.kv_split : n_units;

    const int warp = warp_id(), lane = lane_id();
    const int delta = p.Nk - p.Nq;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bar_q[t], 1);
            mbar_init(&bar_qfree[t], 1);
            mbar_init(&bar_s[t], 1);
            mbar_init(&bar_p[2 * t], 4);
            mbar_init(&bar_p[2 * t + 1], 4);
            mbar_init(&bar_o[t], 1);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(bar_drain, 1);
        for (int u = 0; u < 2; ++u) {
            mbar_init(&bar_tfull[u], 1);
            mbar_init(&bar_tfree[u], 9);   // the MMA warp and the eight softmax warps
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // after the e4m3 V transpose the kernel is a programmatic dependent of it: V^T (and
    // everything else) is read only once that kernel has completed; a no-op in a plain launch
    griddep_wait();
    FwdTile w;

    // Each role runs inside the branch that sets its register budget.
    if (warp >= 8) {
      regs_dec<C::kRegsOther>();
      if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int nq0 = 0, nq1 = 0;   // Q loads so far into tile slot 0 / 1
            int kvi = 0;            // K/V ring loads so far
            int kn = 0, vn = 0;     // one-tile blocks: K loads (slot 0) and V loads (slot 1) so far
            bool ok = true;
            int tile = (int)blockIdx.x;
            // take the counter slot for this launch, or find it held by another one
            const unsigned owner = atomicCAS(p.tile_ctr + 2, 0u, p.tile_tag);
            const bool own_slot = (owner == 0u || owner == p.tile_tag);
            if (!own_slot)
                atomicOr(&g_status, kStatusSlotShared);
            for (int u = 0; ok; ++u) {
                // publish the tile to the other roles (a ring of two entries)
                if (!(ok = mbar_wait(&bar_tfree[u & 1], ((uint32_t)(u >> 1) & 1u) ^ 1u, abort_flag)))
                    break;
                tile_ring[u & 1] = tile;
                mbar_arrive(&bar_tfull[u & 1]);
                if (tile >= n_tiles)
                    break;
                fwd_tile<C::kTiles, CAUSAL, SPLIT>(p, tile, w);
                for (int t = 0; t < 2 && ok; ++t) {
                    if ((t ? w.nb1 : w.nb0) == 0)
                        continue;
                    const int nq = t ? nq1 : nq0;
                    // the slot still holds the previous tile's Q until its last Q.K^T is done
                    if (nq > 0 && !(ok = mbar_wait(&bar_qfree[t], (uint32_t)((nq - 1) & 1), abort_flag)))
                        break;
                    mbar_arrive_expect_tx(&bar_q[t], C::kTileBytes);
                    for (int pn = 0; pn < C::kPanels; ++pn)
                        tma_load_3d(sQ + t * C::kTileBytes + pn * C::kPanelBytes, &tmQ, &bar_q[t],
                                    pn * C::kPanelElems, w.q0 + 128 * t, w.bh);
                    if (t)
                        ++nq1;
                    else
                        ++nq0;
                }
                if constexpr (C::kTiles == 1) {
                    // K blocks in slot 0, V blocks in slot 1, loaded in the order the MMA
                    // warp frees them: it issues S(0), S(1), P.V(0), S(2), P.V(1), ...,
                    // so K(j + 2) may land once S(j + 1) has read K(j + 1), and V(j + 1)
                    // once P.V(j) has read V(j)
                    auto load_kv = [&](int j, int kv) -> bool {
                        int& cnt = kv ? vn : kn;
                        if (!mbar_wait(&bar_empty[kv], ((uint32_t)cnt & 1u) ^ 1u, abort_flag))
                            return false;
                        uint8_t* dst = sKV + kv * C::kTileBytes;
                        mbar_arrive_expect_tx(&bar_full[kv], C::kTileBytes);
                        for (int pn = 0; pn < C::kPanels; ++pn)
                            tma_load_3d(dst + pn * C::kPanelBytes, kv ? &tmV : &tmK, &bar_full[kv],
                                        pn * C::kPanelElems, (w.kb0 + j) * 128, w.kvh);
                        ++cnt;
                        return true;
                    };
                    const int n = w.n_iter;
                    if (n > 0)
                        ok = load_kv(0, 0) && load_kv(0, 1) && (n < 2 || load_kv(1, 0));
                    for (int j = 0; ok && j < n; ++j) {
                        if (j + 2 < n && !(ok = load_kv(j + 2, 0)))
                            break;
                        if (j + 1 < n && !(ok = load_kv(j + 1, 1)))
                            break;
                    }
                } else
                for (int j = 0; ok && j < w.n_iter; ++j) {
                    for (int kv = 0; kv < 2; ++kv) {
                        const int slot = kvi % C::kStages;
                        const uint32_t round = (uint32_t)(kvi / C::kStages);
                        if (!(ok = mbar_wait(&bar_empty[slot], (round & 1u) ^ 1u, abort_flag)))
                            break;
                        uint8_t* dst = sKV + slot * C::kTileBytes;
                        mbar_arrive_expect_tx(&bar_full[slot], C::kTileBytes);
                        if (F8 && kv)   // V^T: d rows of keys j*128 .. j*128+127
                            tma_load_3d(dst, &tmV, &bar_full[slot], (w.kb0 + j) * 128, 0, w.kvh);
                        else
                            for (int pn = 0; pn < C::kPanels; ++pn)
                                tma_load_3d(dst + pn * C::kPanelBytes, kv ? &tmV : &tmK, &bar_full[slot],
                                            pn * C::kPanelElems, (w.kb0 + j) * 128, w.kvh);
                        ++kvi;
                    }
                }
                // Claim the next tile once this one's loads are all issued, a couple of
                // key blocks before its end: blocks claim in the order they run out of
                // work (a block that claimed at its start would take a second tile
                // before knowing whether its first is long), and the claim's latency
                // hides behind the rest of the tile.
                tile = own_slot ? (int)gridDim.x + (int)atomicAdd(p.tile_ctr, 1u) : n_tiles;
            }
            // this block claims no more tiles; the last one to get here (finished or
            // aborted) resets the launch's counter slot, the owner word last.  A block
            // that found the slot held by another launch touches nothing: its launch
            // never counts all its blocks, so the slot stays marked until
            // fa_check_device_status() clears every slot after reporting the conflict.
            if (own_slot) {
                __threadfence();
                if (atomicAdd(p.tile_ctr + 1, 1u) == gridDim.x - 1) {
                    __threadfence();
                    atomicExch(p.tile_ctr, 0u);
                    atomicExch(p.tile_ctr + 1, 0u);
                    __threadfence();
                    atomicExch(p.tile_ctr + 2, 0u);
                }
            }
            if (*abort_flag) {
                // let the last load of every slot and of both Q slots land before the block exits
                for (int i = max(0, kvi - C::kStages); i < kvi; ++i)
                    mbar_wait_limited(&bar_full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u,
                                      FA_WAIT_LIMIT_CYCLES);
                if (kn > 0)
                    mbar_wait_limited(&bar_full[0], (uint32_t)((kn - 1) & 1), FA_WAIT_LIMIT_CYCLES);
                if (vn > 0)
                    mbar_wait_limited(&bar_full[1], (uint32_t)((vn - 1) & 1), FA_WAIT_LIMIT_CYCLES);
                if (nq0 > 0)
                    mbar_wait_limited(&bar_q[0], (uint32_t)((nq0 - 1) & 1), FA_WAIT_LIMIT_CYCLES);
                if (nq1 > 0)
                    mbar_wait_limited(&bar_q[1], (uint32_t)((nq1 - 1) & 1), FA_WAIT_LIMIT_CYCLES);
            }
        }
      } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs this loop; one elected lane issues each MMA)
        {
            // e4m3 is format code 0 of kind::f8f6f4; V^T makes both P.V operands K-major
            constexpr uint32_t fmt = F8 ? 0u : Elt<T>::kMmaFmt;
            const uint32_t idS = idesc_f16kind(fmt, 128, 128, false, false);
            const uint32_t idPV = idesc_f16kind(fmt, 128, D, false, !F8);
            const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
            auto tS = [&](int t) { return tmem + 128u * (uint32_t)t; };
            auto tO = [&](int t) { return tmem + 256u + (uint32_t)(D * t); };

            // base descriptors; a byte offset `o` inside an operand is added as o >> 4
            // to the start-address field (addresses stay below 256 KB, no carry)
            const uint64_t dQ_k = sdesc_sw128(sQa, 16, 1024);                   // Q tiles, K-major
            const uint64_t dKV_k = sdesc_sw128(sKVa, 16, 1024);                 // ring as K (K-major)
            const uint64_t dKV_mn = sdesc_sw128(sKVa, C::kPanelBytes, 1024);    // ring as V (MN-major)
            auto off = [](uint32_t bytes) { return (uint64_t)(bytes >> 4); };
            auto slot_off = [&](int idx) { return (uint32_t)((idx % C::kStages) * C::kTileBytes); };
            auto phase = [&](int idx) { return (uint32_t)((idx / C::kStages) & 1); };
            // S(t) = Q(t) K^T for the K block at ring index ik
            auto issue_S = [&](int t, int ik) {
                const uint32_t ko = slot_off(ik);
                const uint32_t qo = (uint32_t)(t * C::kTileBytes);
                constexpr int kUnrollS = C::kKSteps <= 4 ? C::kKSteps : 4;   // fewer live descriptors
#pragma unroll kUnrollS
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t o = (uint32_t)((kk >> 2) * C::kPanelBytes + (kk & 3) * 32);
                    mma_ss_k<F8>(tS(t), dQ_k + off(qo + o), dKV_k + off(ko + o), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit_w(&bar_s[t]);
            };
            // O(t) += P V for keys 64*half .. 64*half+63 of block j (P columns 32*half ..
            // 32*half+31), V at ring index iv; block 0 of a tile overwrites O
            auto issue_PV = [&](int t, int j, int iv, int half) {
                const uint32_t vo = slot_off(iv);
                if constexpr (F8) {
                    // P: four e4m3 per column, 8 columns per 32 keys; V^T rows are 128 keys
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const int kk = 2 * half + k2;
                        mma_ts_f8_w(tO(t), tS(t) + (uint32_t)(kk * 8), dKV_k + off(vo + (uint32_t)(kk * 32)),
                                    idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * half + k4;
                        mma_ts_w(tO(t), tS(t) + (uint32_t)(kk * 8), dKV_mn + off(vo + (uint32_t)(kk * 2048)),
                                 idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                }
            };

            bool ok = true;
            // phase bits: 1 << t = parity of the Q loads of tile slot t waited for so far,
            // 4 << t = parity of the blocks of slot t in earlier tiles (bar_p phases)
            uint32_t ph = 0;
            int kvi = 0;            // ring index of the tile's first K block
            // one-tile blocks: K and V blocks read so far (slots 0 and 1), and the blocks of
            // earlier tiles whose S went to S buffer 0 / 1 (bar_p phases)
            int kc = 0, vc = 0;
            int su[2] = {0, 0};
            for (int u = 0; ok; ++u) {
                const int tile = fwd_take_tile(bar_tfull, bar_tfree, tile_ring, u, lane, abort_flag, ok);
                if (!ok || tile >= n_tiles)
                    break;
                fwd_tile<C::kTiles, CAUSAL, SPLIT>(p, tile, w);
                for (int t = 0; t < 2 && ok; ++t) {
                    if ((t ? w.nb1 : w.nb0) == 0)
                        continue;
                    ok = mbar_wait_w(&bar_q[t], (ph >> t) & 1u, abort_flag);
                    ph ^= 1u << t;
                }
                tc_fence_after();
                if constexpr (C::kTiles == 1) {
                    // S of block j goes to S buffer j & 1 (TMEM columns 128 (j & 1) ..), so
                    // S(j + 1) runs while block j's softmax reads S(j): the order is S(0),
                    // S(1), P.V(0), S(2), P.V(1), ... and the tensor core waits for a
                    // softmax only when P.V(j) would run ahead of it
                    const int n = w.n_iter;
                    auto issue_S1 = [&](int j) -> bool {
                        if (!mbar_wait_w(&bar_full[0], (uint32_t)(kc & 1), abort_flag))
                            return false;
                        tc_fence_after();
                        constexpr int kUnrollS = C::kKSteps <= 4 ? C::kKSteps : 4;   // fewer live descriptors
#pragma unroll kUnrollS
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            const uint32_t o = (uint32_t)((kk >> 2) * C::kPanelBytes + (kk & 3) * 32);
                            mma_ss_k<F8>(tS(j & 1), dQ_k + off(o), dKV_k + off(o), idS, kk > 0 ? 1u : 0u);
                        }
                        mma_commit_w(&bar_empty[0]);   // K slot free
                        mma_commit_w(&bar_s[j & 1]);
                        if (j == n - 1)
                            mma_commit_w(&bar_qfree[0]);   // the tile's last Q.K^T
                        ++kc;
                        return true;
                    };
                    if (ok && n > 0)
                        ok = issue_S1(0) && (n < 2 || issue_S1(1));
                    for (int j = 0; ok && j < n; ++j) {
                        const int b = j & 1;
                        if (!(ok = mbar_wait_w(&bar_full[1], (uint32_t)(vc & 1), abort_flag)))
                            break;
                        tc_fence_after();
                        const uint32_t pp = (uint32_t)((su[b] + (j >> 1)) & 1);
                        for (int hf = 0; hf < 2 && ok; ++hf) {
                            if (!(ok = mbar_wait_w(&bar_p[2 * b + hf], pp, abort_flag)))
                                break;
                            tc_fence_after();
                            // O += P V for keys 64 hf .. 64 hf + 63 of block j (V in slot 1)
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                const int kk = 4 * hf + k4;
                                mma_ts_w(tO(0), tS(b) + (uint32_t)(kk * 8),
                                         dKV_mn + off((uint32_t)C::kTileBytes + (uint32_t)(kk * 2048)), idPV,
                                         (j > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        if (!ok)
                            break;
                        mma_commit_w(&bar_empty[1]);   // V slot free
                        ++vc;
                        mma_commit_w(&bar_o[1]);       // P.V(j) done: block j + 1 may rescale O
                        if (j == n - 1)
                            mma_commit_w(&bar_o[0]);
                        if (j + 2 < n && !(ok = issue_S1(j + 2)))
                            break;
                    }
                    su[0] += (n + 1) / 2;
                    su[1] += n / 2;
                    continue;
                }
                const int k0 = kvi;
                if (ok && w.n_iter > 0) {
                    ok = mbar_wait_w(&bar_full[k0 % C::kStages], phase(k0), abort_flag);
                    tc_fence_after();
                    if (ok) {
                        for (int t = 0; t < 2; ++t)
                            if ((t ? w.nb1 : w.nb0) > 0) {
                                issue_S(t, k0);
                                if ((t ? w.nb1 : w.nb0) == 1)
                                    mma_commit_w(&bar_qfree[t]);
                            }
                        mma_commit_w(&bar_empty[k0 % C::kStages]);
                    }
                }
                for (int j = 0; ok && j < w.n_iter; ++j) {
                    const int iv = k0 + 2 * j + 1, ik = k0 + 2 * j + 2;
                    if (!(ok = mbar_wait_w(&bar_full[iv % C::kStages], phase(iv), abort_flag)))
                        break;
                    tc_fence_after();
                    bool k_ready = false;
                    for (int t = 0; t < 2 && ok; ++t) {
                        const int nbt = t ? w.nb1 : w.nb0;
                        if (j < nbt) {
                            const uint32_t pp = ((ph >> (2 + t)) ^ (uint32_t)j) & 1u;
                            for (int hf = 0; hf < 2 && ok; ++hf) {
                                if (!(ok = mbar_wait_w(&bar_p[2 * t + hf], pp, abort_flag)))
                                    break;
                                tc_fence_after();
                                issue_PV(t, j, iv, hf);
                            }
                            if (!ok)
                                break;
                            if (j == nbt - 1)
                                mma_commit_w(&bar_o[t]);
                        }
                        if (j + 1 < nbt) {
                            if (!k_ready) {
                                if (!(ok = mbar_wait_w(&bar_full[ik % C::kStages], phase(ik), abort_flag)))
                                    break;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_S(t, ik);
                            if (j + 2 == nbt)   // that was the tile's last Q(t).K^T
                                mma_commit_w(&bar_qfree[t]);
                        }
                    }
                    if (!ok)
                        break;
                    mma_commit_w(&bar_empty[iv % C::kStages]);
                    if (k_ready)
                        mma_commit_w(&bar_empty[ik % C::kStages]);
                }
                kvi = k0 + 2 * w.n_iter;
                ph ^= (((uint32_t)w.nb0 & 1u) << 2) | (((uint32_t)w.nb1 & 1u) << 3);
            }
            if (!ok) {
                mma_commit_w(bar_drain);
                mbar_wait_limited(bar_drain, 0, FA_WAIT_LIMIT_CYCLES);
            }
        }
      }
    } else {
        regs_inc<C::kRegsSoftmax>();
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int r = ((warp & 3) << 5) + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * (uint32_t)t;
        const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(D * t);
        const float sl2 = p.scale_log2;
        int bt = 0;   // blocks of earlier tiles (bar_s phases)
        int no = 0;   // earlier tiles with at least one block (bar_o phases)
        int su[2] = {0, 0};   // one-tile blocks: blocks of earlier tiles in S buffer 0 / 1
        bool ok = true;

        for (int u = 0; ok; ++u) {
            const int tile = fwd_take_tile(bar_tfull, bar_tfree, tile_ring, u, lane, abort_flag, ok);
            if (!ok || tile >= n_tiles)
                break;
            fwd_tile<C::kTiles, CAUSAL, SPLIT>(p, tile, w);
            const int qi = w.q0 + 128 * t + r;   // row of the tile head
            const int nb = t ? w.nb1 : w.nb0;
            const int qlim = (p.group_rows ? qi % p.Nq : qi) + delta;   // last key its query position sees
            float m_ref = -INFINITY, l = 0.f;

            for (int j = 0; j < nb; ++j) {
                // one-tile blocks alternate between two S buffers (TMEM columns 0 and 128)
                const int sb = C::kTiles == 1 ? (j & 1) : t;
                const uint32_t tSb = C::kTiles == 1 ? tmem + lane_off + 128u * (uint32_t)sb : tS;
                const uint32_t sph = C::kTiles == 1 ? (uint32_t)((su[sb] + (j >> 1)) & 1) : (uint32_t)((bt + j) & 1);
                ok = mbar_wait(&bar_s[sb], sph, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld128(tSb, sr);
                float s[128];
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    s[c] = __uint_as_float(sr[c]);

                const int kb = (w.kb0 + j) * 128;
                const bool need_mask = (kb + 128 > p.Nk) || (CAUSAL && kb + 127 > qlim);
                if (need_mask) {
                    const int lim = CAUSAL ? min(p.Nk - 1, qlim) : p.Nk - 1;
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (kb + c > lim)
                            s[c] = -INFINITY;
                }
                // row max: two independent chains of three-input max
                float mxa = fmaxf(s[0], s[1]), mxb = fmaxf(s[2], s[3]);
#pragma unroll
                for (int c = 4; c < 128; c += 4) {
                    mxa = fmax3(mxa, s[c], s[c + 1]);
                    mxb = fmax3(mxb, s[c + 2], s[c + 3]);
                }
                const float m_blk = fmaxf(mxa, mxb) * sl2;
                float a = 1.f;
                bool resc = false;
                if (m_blk > m_ref + kRescaleLog2) {
                    a = ex2_approx(m_ref - m_blk);
                    resc = (j > 0);
                    m_ref = m_blk;
                    l *= a;
                }
                if (__any_sync(0xffffffffu, resc)) {
                    if constexpr (C::kTiles == 1) {
                        // S(j) ran ahead of P.V(j - 1): O may be rescaled once that is done
                        ok = mbar_wait(&bar_o[1], (uint32_t)((bt + j - 1) & 1), abort_flag);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok)
                            break;
                        tc_fence_after();
                    }
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tO + (uint32_t)c0, o);
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
                        tmem_st32(tO + (uint32_t)c0, o);
                    }
                }
                const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                const float2 sl22 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
                float2 acc = make_float2(0.f, 0.f);
                // One exp2 per score: the MUFU unit would be as busy as the tensor
                // core at d = 128, so there (kPoly) in blocks without masked scores
                // one pair in four goes to the FMA-pipe exp2 instead (masked -inf
                // scores always take ex2.approx, which returns exactly 0 for them).
                const bool soft = C::kPoly && !__any_sync(0xffffffffu, need_mask);
                auto half_block_f8 = [&](int hf, auto use_poly) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int e = 64 * hf + 4 * c;
                        const float2 x0 = ffma2(make_float2(s[e], s[e + 1]), sl22, nm2);
                        const float2 x1 = ffma2(make_float2(s[e + 2], s[e + 3]), sl22, nm2);
                        const float2 p0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
                        float2 p1;
                        if (decltype(use_poly)::value && (c & 1) == 1)
                            p1 = exp2_poly2(x1);
                        else
                            p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
                        acc = fadd2(acc, fadd2(p0, p1));
                        pk[c] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
                    }
                    tmem_st16(tSb + (uint32_t)(16 * hf), pk);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bar_p[2 * sb + hf]);
                };
                auto half_block_16 = [&](int hf, auto use_poly) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = 64 * hf + 2 * c;
                        const float2 x = ffma2(make_float2(s[e], s[e + 1]), sl22, nm2);
                        float2 pv;
                        if (decltype(use_poly)::value && (c & 3) == 3)
                            pv = exp2_poly2(x);
                        else
                            pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        acc = fadd2(acc, pv);
                        pk[c] = Elt<T>::pack(pv.x, pv.y);
                    }
                    tmem_st32(tSb + (uint32_t)(32 * hf), pk);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bar_p[2 * sb + hf]);
                };
                auto half_block = [&](int hf, auto use_poly) {
                    if constexpr (F8)
                        half_block_f8(hf, use_poly);
                    else
                        half_block_16(hf, use_poly);
                };
                // P in two halves of 64 keys: the MMA warp starts P.V on the first
                // half while the second is still being exponentiated
                if (soft) {
                    half_block(0, std::true_type{});
                    half_block(1, std::true_type{});
                } else {
                    half_block(0, std::false_type{});
                    half_block(1, std::false_type{});
                }
                l += acc.x + acc.y;
            }

            if (!ok)
                break;

            // ---- epilogue: O = U / l (bf16), LSE = (m + log2 l) ln 2
            const bool row_valid = (C::kTiles == 2 || t == 0) && qi < p.rows;   // one-tile blocks: warps 4-7 idle
            const size_t row = (size_t)w.bh * (size_t)p.rows + (size_t)qi;   // the same flat row either way
            if (nb > 0) {
                ok = mbar_wait(&bar_o[t], (uint32_t)(no & 1), abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                ++no;
                if (!ok)
                    break;
                tc_fence_after();
                const float inv_l = (l > 0.f) ? p.o_scale / l : 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < p.d_io; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + (uint32_t)c0, o);
                    if (SPLIT && w.nshares > 1) {
                        // this share's normalised partial O_s in fp32
                        if (row_valid) {
                            const size_t prow = ((size_t)w.bh * p.kv_split + w.share) * p.rows + qi;
                            float4* dst = reinterpret_cast<float4*>(p.part_o + prow * p.d_io + c0);
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv_l, __uint_as_float(o[4 * c + 1]) * inv_l,
                                                     __uint_as_float(o[4 * c + 2]) * inv_l, __uint_as_float(o[4 * c + 3]) * inv_l);
                        }
                        continue;
                    }
                    if (row_valid) {
                        uint32_t wv[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            wv[c] = Elt<T>::pack(__uint_as_float(o[2 * c]) * inv_l,
                                                 __uint_as_float(o[2 * c + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.o) + row * p.d_io + c0);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            dst[c] = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                    }
                }
                // O(t) is read out: the next tile's first P.V may overwrite it once this
                // warpgroup's P of that tile is signalled (after the fence in the P write)
                tc_fence_before();
                if (SPLIT && w.nshares > 1) {
                    if (row_valid)
                        p.part_lse[((size_t)w.bh * p.kv_split + w.share) * p.rows + qi] =
                            (l > 0.f) ? m_ref + __log2f(l) : -INFINITY;
                } else if (row_valid && p.lse) {
                    p.lse[row] = (l > 0.f) ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
                }
            } else if (SPLIT && w.nshares > 1 && row_valid) {
                // no key of this share for any row of the tile: its partial carries no weight
                p.part_lse[((size_t)w.bh * p.kv_split + w.share) * p.rows + qi] = -INFINITY;
            } else if (row_valid) {
                // no visible key for any row of this tile
                uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.o) + row * p.d_io);
#pragma unroll 1
                for (int c = 0; c < p.d_io / 8; ++c)
                    dst[c] = make_uint4(0u, 0u, 0u, 0u);
                if (p.lse)
                    p.lse[row] = -INFINITY;
            }
            bt += nb;
            su[0] += (nb + 1) / 2;
            su[1] += nb / 2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Merge of the key shares of a split forward (one warp per query row): with
// w_s = 2^(lse_s - M), M = max_s lse_s, O = sum_s w_s O_s / sum_s w_s and
// LSE = (M + log2 sum_s w_s) ln 2 -- the rescale-and-add of the online softmax
// (page "FlashAttention：为什么少搬数据，反而算得更快", §04) applied to whole
// shares.  Shares with lse_s = -inf (no key) are skipped; a row no share sees
// gets O = 0 and LSE = -inf.
template <typename T = __nv_bfloat16>
__global__ void __launch_bounds__(128) fwd_combine_kernel(FwdParams p)
{
    griddep_wait();   // the partials are complete once the forward has finished
    const long long row = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long long)p.n_bh * p.rows)
        return;
    const long long bh = row / p.rows, i = row % p.rows;
    // rows of the whole units (written straight to o / lse by the forward) are final
    const long long unit = (long long)(p.n_pairs - 1 - (int)(i / p.pair_rows)) * p.n_bh + bh;
    if (unit < p.full_tiles)
        return;
    const int ns = p.kv_split;   // <= 32: lane s holds share s's lse and weight
    const float ls = lane < ns ? p.part_lse[((size_t)bh * ns + lane) * p.rows + i] : -INFINITY;
    float M = ls;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wl = (M != -INFINITY && ls != -INFINITY) ? ex2_approx(ls - M) : 0.f;
    float L = wl;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        L += __shfl_xor_sync(0xffffffffu, L, off);
    // lane l merges columns [n*l, n*l + n) of the row, n = d_io / 32 (<= 8): one or
    // two 16-byte loads per share and lane where n is 4 or 8
    const int n = p.d_io / 32;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        acc[k] = 0.f;
    const float* o0 = p.part_o + (((size_t)bh * ns) * p.rows + i) * p.d_io + (size_t)n * lane;
    const size_t share_stride = (size_t)p.rows * p.d_io;
#pragma unroll 4
    for (int s = 0; s < ns; ++s) {
        const float w = __shfl_sync(0xffffffffu, wl, s);
        if (w == 0.f)   // no key in this share (its O_s was never written) or a negligible one
            continue;
        const float* os = o0 + (size_t)s * share_stride;
        if (n == 4) {
            const float4 v = *reinterpret_cast<const float4*>(os);
            acc[0] = fmaf(w, v.x, acc[0]);
            acc[1] = fmaf(w, v.y, acc[1]);
            acc[2] = fmaf(w, v.z, acc[2]);
            acc[3] = fmaf(w, v.w, acc[3]);
        } else if (n == 8) {
            const float4 v = *reinterpret_cast<const float4*>(os), u = *reinterpret_cast<const float4*>(os + 4);
            acc[0] = fmaf(w, v.x, acc[0]);
            acc[1] = fmaf(w, v.y, acc[1]);
            acc[2] = fmaf(w, v.z, acc[2]);
            acc[3] = fmaf(w, v.w, acc[3]);
            acc[4] = fmaf(w, u.x, acc[4]);
            acc[5] = fmaf(w, u.y, acc[5]);
            acc[6] = fmaf(w, u.z, acc[6]);
            acc[7] = fmaf(w, u.w, acc[7]);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < n)
                    acc[k] = fmaf(w, os[k], acc[k]);
        }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    T* o = static_cast<T*>(p.o) + (size_t)row * p.d_io + (size_t)n * lane;
    if (n == 4) {
        *reinterpret_cast<uint2*>(o) = make_uint2(Elt<T>::pack(acc[0] * inv, acc[1] * inv),
                                                  Elt<T>::pack(acc[2] * inv, acc[3] * inv));
    } else if (n == 8) {
        *reinterpret_cast<uint4*>(o) = make_uint4(Elt<T>::pack(acc[0] * inv, acc[1] * inv),
                                                  Elt<T>::pack(acc[2] * inv, acc[3] * inv),
                                                  Elt<T>::pack(acc[4] * inv, acc[5] * inv),
                                                  Elt<T>::pack(acc[6] * inv, acc[7] * inv));
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < n)
                o[k] = Elt<T>::from_float(acc[k] * inv);
    }
    if (lane == 0 && p.lse)
        p.lse[row] = (L > 0.f) ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace fa
