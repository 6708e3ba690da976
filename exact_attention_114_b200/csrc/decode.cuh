// decode.cuh -- split-KV forward for the decode shape (few query rows per kv
// head; page "FlashAttention：为什么少搬数据，反而算得更快", §09: a single query
// position whose scores are 1 x history) and the log-sum-exp combine.
//
// Split pass: one CTA per (batch, kv head, key chunk).  The key chunk streams
// through shared memory exactly once for all R = (Hq / Hkv) * Nq query rows of
// the group, so K/V are read from HBM once per kv head, not once per query
// head.  The pass is bound by HBM bandwidth, so the contraction uses plain warp
// MMAs (m16n8k16, bf16 -> fp32) and the effort goes into the memory pipeline:
//   * warp 4 issues TMA loads of 64-key K and V tiles (128-byte swizzle) into a
//     ring of kStages slots;
//   * warps 0-3 each take 16 keys of every tile and run their own online
//     softmax (§04 recurrence, log2 domain) for all R rows (padded to 16);
//   * at the end the four per-warp states are merged in shared memory with the
//     same rescale-and-add rule and written as a partial (O_s, lse_s), or as the
//     final output when there is a single chunk.
// Combine: lse = ln sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s (§04 rule in
// log form), one warp per output row.
//
// Paged variant (PAGED = true): the KV cache is a pool of pages, [num_pages,
// page_size, Hkv, d], shared by all sequences (the pages are only "where the KV
// is stored", §09); a block table maps each sequence's logical pages to
// physical ones and every sequence has its own length.  Only the producer
// changes: it looks up the page of each 64-key tile and issues a 4-D TMA load.
#pragma once

#include "sm100.cuh"
#include "fa_kernels.h"

namespace fa {

struct DecCfg {
    static constexpr int kThreads = 160;        // 4 consumer warps + 1 producer warp
    static constexpr int kKeys = 64;            // keys per tile
    static constexpr int kTileBytes = 64 * 128 * 2;   // one K or V tile (d = 128)
    static constexpr int kPanelBytes = 64 * 128;      // 64 keys x 64 bf16
    static constexpr int kStages = 3;
    static constexpr int kOffRing = 0;
    static constexpr int kOffBar = kStages * 2 * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + 128 + 1024;
};

// D += A B with 16-bit A/B (bf16 or fp16) and fp32 accumulators
template <typename T>
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    if constexpr (Elt<T>::kMmaFmt == 1u)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// byte offset of (key row, 16-byte chunk) inside a 64-key tile stored as two
// 128-byte-swizzled panels of 64 columns
__device__ __forceinline__ uint32_t dec_tile_off(int key, int chunk)
{
    const int panel = chunk >> 3, c = chunk & 7;
    return (uint32_t)(panel * DecCfg::kPanelBytes + key * 128 + ((c ^ (key & 7)) << 4));
}

// NARROW: the head has fewer than 128 columns (p.d_io); the full-width kernel
// compiles without the column checks.
template <bool PAGED, typename T = __nv_bfloat16, bool NARROW = false>
__global__ void __launch_bounds__(160, 2)   // two CTAs per SM (shared memory allows exactly two)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        DecodeParams p)
{
    griddep_launch_dependents();   // the combine may be scheduled
    const int d_io = NARROW ? p.d_io : 128;
    using C = DecCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_empty = bar_full + C::kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_empty + C::kStages);

    const int warp = warp_id(), lane = lane_id();
    const int split = (int)blockIdx.x % p.splits;
    const int kvh = (int)blockIdx.x / p.splits;     // b * Hkv + kv head
    const int b = kvh / p.Hkv, hk = kvh % p.Hkv;
    // keys of this sequence (a paged sequence's own length, clamped to what its table can hold)
    const int Nk_b = PAGED ? max(0, min(__ldg(p.seq_lens + b), p.max_pages * p.page_size)) : p.Nk;
    const int k_begin = split * p.chunk;
    const int k_end = min(Nk_b, k_begin + p.chunk);
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + C::kKeys - 1) / C::kKeys : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            for (int t = 0; t < n_tiles; ++t) {
                const int slot = t % C::kStages;
                const uint32_t round = (uint32_t)(t / C::kStages);
                if (!mbar_wait(&bar_empty[slot], (round & 1u) ^ 1u, abort_flag))
                    break;
                uint8_t* dk = smem + C::kOffRing + slot * 2 * C::kTileBytes;
                uint8_t* dv = dk + C::kTileBytes;
                // the second 64-column panel only when the head has columns there
                const bool two = d_io > 64;
                mbar_arrive_expect_tx(&bar_full[slot], (two ? 4 : 2) * C::kPanelBytes);
                const int key0 = k_begin + t * C::kKeys;
                if (PAGED) {
                    // a 64-key tile never straddles a page (page_size is a multiple of 64);
                    // an out-of-range page id reads zeros (TMA bounds), never another buffer
                    const int page = __ldg(p.block_table + (size_t)b * p.max_pages + key0 / p.page_size);
                    const int off = key0 % p.page_size;
                    tma_load_4d(dk, &tmK, &bar_full[slot], 0, hk, off, page);
                    tma_load_4d(dv, &tmV, &bar_full[slot], 0, hk, off, page);
                    if (two) {
                        tma_load_4d(dk + C::kPanelBytes, &tmK, &bar_full[slot], 64, hk, off, page);
                        tma_load_4d(dv + C::kPanelBytes, &tmV, &bar_full[slot], 64, hk, off, page);
                    }
                } else {
                    tma_load_3d(dk, &tmK, &bar_full[slot], 0, key0, kvh);
                    tma_load_3d(dv, &tmV, &bar_full[slot], 0, key0, kvh);
                    if (two) {
                        tma_load_3d(dk + C::kPanelBytes, &tmK, &bar_full[slot], 64, key0, kvh);
                        tma_load_3d(dv + C::kPanelBytes, &tmV, &bar_full[slot], 64, key0, kvh);
                    }
                }
            }
            if (*abort_flag) {
                const int last = n_tiles;
                for (int t = max(0, last - C::kStages); t < last; ++t)
                    mbar_wait_limited(&bar_full[t % C::kStages], (uint32_t)(t / C::kStages) & 1u,
                                      FA_WAIT_LIMIT_CYCLES);
            }
        }
        return;  // the producer takes no part in the merge below
    }

    // ------------------------------------------------------------------ consumers
    const int g = lane >> 2, tq = lane & 3;   // mma fragment coordinates
    const float sl2 = p.scale_log2;
    // query rows of this group: row r -> head hk * G + r / Nq, query i = r % Nq
    uint32_t qa[8][4];
    {
        const int rows[2] = {g, g + 8};
        for (int ks = 0; ks < 8; ++ks)
            for (int e = 0; e < 4; ++e) qa[ks][e] = 0u;
        for (int hr = 0; hr < 2; ++hr) {
            const int r = rows[hr];
            if (r >= p.R)
                continue;
            const int h = hk * p.G + r / p.Nq, i = r % p.Nq;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                static_cast<const T*>(p.q) + (((size_t)b * p.Hq + h) * p.Nq + i) * d_io);
            for (int ks = 0; ks < 8; ++ks) {
                if (ks * 16 >= d_io)
                    break;
                qa[ks][hr] = __ldg(qrow + ks * 8 + tq);          // cols 16ks + 2tq, +1
                qa[ks][hr + 2] = __ldg(qrow + ks * 8 + 4 + tq);  // cols 16ks + 8 + 2tq, +1
            }
        }
    }
    // per-row causal limit (last visible key) for the two rows this thread holds
    int lim[2];
    for (int hr = 0; hr < 2; ++hr) {
        const int r = g + 8 * hr;
        const int i = (r < p.R) ? r % p.Nq : 0;
        lim[hr] = p.causal ? min(k_end - 1, i + Nk_b - p.Nq) : k_end - 1;
    }

    float o[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
        o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool ok = true;

    for (int t = 0; t < n_tiles; ++t) {
        const int slot = t % C::kStages;
        ok = mbar_wait(&bar_full[slot], (uint32_t)(t / C::kStages) & 1u, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            break;
        const uint32_t kbase = smem_u32(smem + C::kOffRing + slot * 2 * C::kTileBytes);
        const uint32_t vbase = kbase + C::kTileBytes;
        const int key_w = warp * 16;   // this warp's 16 keys within the tile

        // S (16 rows x 16 keys) = Q K^T
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int mi = lane >> 3, rr = lane & 7;
            const int key = key_w + (mi >> 1) * 8 + rr;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                if (ks * 16 >= d_io)   // columns past the head: not loaded
                    break;
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + dec_tile_off(key, 2 * ks + (mi & 1)), b0, b1, b2, b3);
                mma_16816<T>(s[0], qa[ks], b0, b1);
                mma_16816<T>(s[1], qa[ks], b2, b3);
            }
        }
        // mask: keys past the chunk / causal limit
        const int key0 = k_begin + t * C::kKeys + key_w;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + nt * 8 + 2 * tq + (e & 1);
                if (key > lim[e >> 1])
                    s[nt][e] = -INFINITY;
            }
        // online softmax for rows g (e = 0, 1) and g + 8 (e = 2, 3)
        uint32_t pa[4];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float mx = fmaxf(fmaxf(s[0][2 * hr], s[0][2 * hr + 1]), fmaxf(s[1][2 * hr], s[1][2 * hr + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m[hr], mx * sl2);
            const float a = (m_new == -INFINITY) ? 1.f : ex2_approx(m[hr] - m_new);
            const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;
            m[hr] = m_new;
            const float p00 = ex2_approx(fmaf(s[0][2 * hr], sl2, neg_m));
            const float p01 = ex2_approx(fmaf(s[0][2 * hr + 1], sl2, neg_m));
            const float p10 = ex2_approx(fmaf(s[1][2 * hr], sl2, neg_m));
            const float p11 = ex2_approx(fmaf(s[1][2 * hr + 1], sl2, neg_m));
            l[hr] = l[hr] * a + (p00 + p01 + p10 + p11);
            pa[hr] = Elt<T>::pack(p00, p01);       // keys 2tq, 2tq+1
            pa[hr + 2] = Elt<T>::pack(p10, p11);   // keys 8 + 2tq, +1
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                o[nd][2 * hr] *= a;
                o[nd][2 * hr + 1] *= a;
            }
        }
        // O (16 rows x 128) += P (16 x 16 keys) V (16 keys x 128)
        {
            const int mi = lane >> 3, rr = lane & 7;
            const int key = key_w + (mi & 1) * 8 + rr;
#pragma unroll
            for (int nd = 0; nd < 16; nd += 2) {
                if (nd * 8 >= d_io)   // output columns past the head stay zero
                    break;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vbase + dec_tile_off(key, nd + (mi >> 1)), b0, b1, b2, b3);
                mma_16816<T>(o[nd], pa, b0, b1);
                mma_16816<T>(o[nd + 1], pa, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bar_empty[slot]);
    }

    // ---- merge the four warps' states (shared memory reused; all tiles consumed)
    named_bar_sync(1, 128);
    float* sm_m = reinterpret_cast<float*>(smem);            // [4][16]
    float* sm_l = sm_m + 64;                                  // [4][16]
    float* sm_o = sm_l + 64;                                  // [4][16][128]
    if (ok) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float lt = l[hr];
            lt += __shfl_xor_sync(0xffffffffu, lt, 1);
            lt += __shfl_xor_sync(0xffffffffu, lt, 2);
            const int r = g + 8 * hr;
            if (tq == 0) {
                sm_m[warp * 16 + r] = m[hr];
                sm_l[warp * 16 + r] = lt;
            }
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                float* dst = sm_o + (warp * 16 + r) * 128 + nd * 8 + 2 * tq;
                dst[0] = o[nd][2 * hr];
                dst[1] = o[nd][2 * hr + 1];
            }
        }
    }
    named_bar_sync(1, 128);
    if (*abort_flag)
        return;
    const int dcol = threadIdx.x;   // 0..127
    for (int r = 0; r < p.R; ++r) {
        float M = -INFINITY;
        for (int w = 0; w < 4; ++w)
            M = fmaxf(M, sm_m[w * 16 + r]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < 4; ++w) {
                const float sc = ex2_approx(sm_m[w * 16 + r] - M);
                L += sm_l[w * 16 + r] * sc;
                acc += sm_o[(w * 16 + r) * 128 + dcol] * sc;
            }
        }
        const float on = (L > 0.f) ? acc / L : 0.f;
        const float lse = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
        if (p.splits == 1) {
            const int h = hk * p.G + r / p.Nq, i = r % p.Nq;
            const size_t row = ((size_t)b * p.Hq + h) * p.Nq + i;
            if (dcol < d_io)
                static_cast<T*>(p.o)[row * d_io + dcol] = Elt<T>::from_float(on);
            if (dcol == 0 && p.lse)
                p.lse[row] = lse;
        } else {
            const size_t prow = ((size_t)kvh * p.splits + split) * p.R + r;
            p.part_o[prow * 128 + dcol] = on;
            if (dcol == 0)
                p.part_lse[prow] = lse;
        }
    }
}

// One warp per output row (b, kv head, r): merge the partials of all splits.
template <typename T = __nv_bfloat16>
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeParams p)
{
    griddep_wait();   // the partials are complete once the split pass has finished
    const int warp = (int)(blockIdx.x * 4 + (threadIdx.x >> 5));
    const int lane = threadIdx.x & 31;
    const int total = p.B * p.Hkv * p.R;
    if (warp >= total)
        return;
    const int r = warp % p.R;
    const int kvh = warp / p.R;
    const int b = kvh / p.Hkv, hk = kvh % p.Hkv;
    const size_t base = (size_t)kvh * p.splits * p.R + r;
    float M = -INFINITY;
    for (int s = lane; s < p.splits; s += 32)
        M = fmaxf(M, p.part_lse[base + (size_t)s * p.R]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float L = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < p.splits; ++s) {
            const size_t prow = base + (size_t)s * p.R;
            const float ls = p.part_lse[prow];
            const float w = __expf(ls - M);
            L += w;
            const float4 v = *reinterpret_cast<const float4*>(p.part_o + prow * 128 + lane * 4);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
        }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const int h = hk * p.G + r / p.Nq, i = r % p.Nq;
    const size_t row = ((size_t)b * p.Hq + h) * p.Nq + i;
    uint2 w2;
    w2.x = Elt<T>::pack(acc[0] * inv, acc[1] * inv);
    w2.y = Elt<T>::pack(acc[2] * inv, acc[3] * inv);
    if (lane * 4 < p.d_io)
        *reinterpret_cast<uint2*>(static_cast<T*>(p.o) + row * p.d_io + lane * 4) = w2;
    if (lane == 0 && p.lse)
        p.lse[row] = (L > 0.f) ? M + __logf(L) : -INFINITY;
}

}  // namespace fa
