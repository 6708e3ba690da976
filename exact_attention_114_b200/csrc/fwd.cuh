// fwd.cuh -- forward kernel: O = softmax(scale * Q K^T + mask) V and the per-row
// LSE, tile by tile with the online-softmax state (m, l, U) of the page
// "FlashAttention：为什么少搬数据，反而算得更快", §03 (fix a block of Q, stream the
// K/V blocks past it) and §04 (m_new = max(m_old, max block), rescale the old
// numerator and denominator together by exp(m_old - m_new), add the block).
//
// Layout of one CTA (384 threads = 3 warpgroups, one CTA per SM):
//   * two 128-row query tiles of one (batch, head), Q0 and Q1, staged once in
//     shared memory by TMA (128-byte swizzle, 64-column panels);
//   * K and V blocks of 128 keys stream through one ring of NSTAGE tile slots
//     (order K0, V0, K1, V1, ...), each slot guarded by a full / empty mbarrier;
//   * tensor memory (512 columns): S0 | S1 (128 fp32 columns each) | O0 | O1
//     (d fp32 columns each).  P overwrites the first 64 columns of its S tile as
//     packed bf16 pairs and is read from there by the P.V MMA;
//   * warps 0-3 run the softmax of tile 0, warps 4-7 that of tile 1: thread r of
//     a warpgroup owns query row r, which is TMEM lane r;
//   * warp 8 issues the TMA loads, warp 9 (one thread) the tcgen05.mma ops in the
//     order S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ..., so the softmax of
//     one tile overlaps the MMAs of the other; warps 10-11 only complete the
//     third warpgroup, which hands most of its registers to the softmax ones.
//
// At d = 256 the CTA holds one query tile (kTiles = 1): its O accumulator takes
// 256 TMEM columns, so there is no room for a second tile's S and O; the second
// softmax warpgroup then has no work, and the MMA order is S(0) | PV(j) S(j+1).
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
    // registers per thread after the split: 2 x 128 x 208 + 128 x 80 <= 384 x 168
    static constexpr uint32_t kRegsSoftmax = 208, kRegsOther = 80;
    static constexpr int kElt = F8 ? 1 : 2;              // bytes per Q/K/V element
    static constexpr int kTileBytes = 128 * D * kElt;    // a 128-row Q or K tile, a V tile
    static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes (one swizzle span)
    static constexpr int kPanels = D * kElt / 128;
    static constexpr int kPanelElems = 128 / kElt;
    static constexpr int kKSteps = D * kElt / 32;        // Q.K^T instructions (32 bytes of d each)
    static constexpr int kStages = F8 ? 10 : (D == 256) ? 2 : (D == 128) ? 5 : 8;
    static constexpr int kBarBytes = F8 ? 512 : 256;
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = kTiles * kTileBytes;
    static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + barriers + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static_assert(!F8 || D == 128, "the e4m3 kernel is built for d = 128");
    static_assert(kTiles == 2 || 128 + D <= (int)kTmemCols, "one tile: S and O must fit in TMEM");
};

__device__ __forceinline__ int fwd_blocks_for_tile(int qt, int Nq, int Nk, bool causal)
{
    const int nkb = (Nk + 127) / 128;
    if (qt >= Nq)
        return 0;
    if (!causal)
        return nkb;
    const int last_row = min(qt + 127, Nq - 1);
    const int last_key = last_row + (Nk - Nq);
    if (last_key < 0)
        return 0;
    return min(nkb, last_key / 128 + 1);
}

template <int D, bool CAUSAL, typename T = __nv_bfloat16, bool F8 = false>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, FwdParams p)
{
    using C = FwdCfg<D, F8>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sKV = smem + C::kOffKV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars;                            // [2]  Q tile landed
    uint64_t* bar_full = bar_q + 2;                    // [S]  ring slot landed
    uint64_t* bar_empty = bar_full + C::kStages;       // [S]  ring slot released
    uint64_t* bar_s = bar_empty + C::kStages;          // [2]  S tile ready in TMEM
    uint64_t* bar_p = bar_s + 2;                       // [2][2] P half h (and O rescale) written
    uint64_t* bar_o = bar_p + 4;                       // [2]  last P.V of a tile done
    uint64_t* bar_drain = bar_o + 2;                   // [1]  MMA drain on abort
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();

    // ---- work item: (query tile pair, batch, head); heaviest causal pairs first
    const int n_bh = p.B * p.Hq;
    const int pair = p.n_pairs - 1 - (int)(blockIdx.x / n_bh);
    const int bh = (int)(blockIdx.x % n_bh);
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int kvh = b * p.Hkv + h / p.G;
    const int q0 = pair * 128 * C::kTiles;
    const int delta = p.Nk - p.Nq;
    int nblk[2];
    nblk[0] = fwd_blocks_for_tile(q0, p.Nq, p.Nk, CAUSAL);
    nblk[1] = (C::kTiles == 2) ? fwd_blocks_for_tile(q0 + 128, p.Nq, p.Nk, CAUSAL) : 0;
    const int n_iter = max(nblk[0], nblk[1]);

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bar_q[t], 1);
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

    // Each role runs inside the branch that sets its register budget.
    if (warp >= 8) {
      regs_dec<C::kRegsOther>();
      if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int t = 0; t < 2; ++t) {
                if (nblk[t] == 0)
                    continue;
                mbar_arrive_expect_tx(&bar_q[t], C::kTileBytes);
                for (int pn = 0; pn < C::kPanels; ++pn)
                    tma_load_3d(sQ + t * C::kTileBytes + pn * C::kPanelBytes, &tmQ, &bar_q[t],
                                pn * C::kPanelElems, q0 + 128 * t, bh);
            }
            int slot = 0;
            uint32_t round = 0;
            int issued = 0;
            for (int j = 0; j < n_iter; ++j) {
                bool ok = true;
                for (int kv = 0; kv < 2; ++kv) {
                    if (!mbar_wait(&bar_empty[slot], (round & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = sKV + slot * C::kTileBytes;
                    mbar_arrive_expect_tx(&bar_full[slot], C::kTileBytes);
                    if (F8 && kv)   // V^T: d rows of keys j*128 .. j*128+127
                        tma_load_3d(dst, &tmV, &bar_full[slot], j * 128, 0, kvh);
                    else
                        for (int pn = 0; pn < C::kPanels; ++pn)
                            tma_load_3d(dst + pn * C::kPanelBytes, kv ? &tmV : &tmK, &bar_full[slot],
                                        pn * C::kPanelElems, j * 128, kvh);
                    ++issued;
                    if (++slot == C::kStages) {
                        slot = 0;
                        ++round;
                    }
                }
                if (!ok)
                    break;
            }
            if (*abort_flag) {
                // let the last load of every slot land before the block exits
                for (int i = max(0, issued - C::kStages); i < issued; ++i)
                    mbar_wait_limited(&bar_full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u,
                                      FA_WAIT_LIMIT_CYCLES);
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
            const uint32_t tS[2] = {tmem, tmem + 128u};
            const uint32_t tO[2] = {tmem + 256u, tmem + 256u + (uint32_t)D};
            bool ok = true;
            for (int t = 0; t < 2 && ok; ++t)
                if (nblk[t] > 0)
                    ok = mbar_wait_w(&bar_q[t], 0, abort_flag);
            tc_fence_after();

            // base descriptors; a byte offset `o` inside an operand is added as o >> 4
            // to the start-address field (addresses stay below 256 KB, no carry)
            const uint64_t dQ_k = sdesc_sw128(sQa, 16, 1024);                   // Q tiles, K-major
            const uint64_t dKV_k = sdesc_sw128(sKVa, 16, 1024);                 // ring as K (K-major)
            const uint64_t dKV_mn = sdesc_sw128(sKVa, C::kPanelBytes, 1024);    // ring as V (MN-major)
            auto off = [](uint32_t bytes) { return (uint64_t)(bytes >> 4); };
            auto slot_off = [&](int idx) { return (uint32_t)((idx % C::kStages) * C::kTileBytes); };
            auto phase = [&](int idx) { return (uint32_t)((idx / C::kStages) & 1); };
            auto issue_S = [&](int t, int j) {
                const uint32_t ko = slot_off(2 * j);
                const uint32_t qo = (uint32_t)(t * C::kTileBytes);
                constexpr int kUnrollS = C::kKSteps <= 8 ? C::kKSteps : 4;   // d = 256: fewer live descriptors
#pragma unroll kUnrollS
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t o = (uint32_t)((kk >> 2) * C::kPanelBytes + (kk & 3) * 32);
                    mma_ss_k<F8>(tS[t], dQ_k + off(qo + o), dKV_k + off(ko + o), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit_w(&bar_s[t]);
            };
            // keys 64*half .. 64*half+63 of block j (P columns 32*half .. 32*half+31)
            auto issue_PV = [&](int t, int j, int half) {
                const uint32_t vo = slot_off(2 * j + 1);
                if constexpr (F8) {
                    // P: four e4m3 per column, 8 columns per 32 keys; V^T rows are 128 keys
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const int kk = 2 * half + k2;
                        mma_ts_f8_w(tO[t], tS[t] + (uint32_t)(kk * 8), dKV_k + off(vo + (uint32_t)(kk * 32)),
                                    idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * half + k4;
                        mma_ts_w(tO[t], tS[t] + (uint32_t)(kk * 8), dKV_mn + off(vo + (uint32_t)(kk * 2048)),
                                 idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                }
            };

            if (ok && n_iter > 0) {
                ok = mbar_wait_w(&bar_full[0], 0, abort_flag);
                tc_fence_after();
                if (ok) {
                    for (int t = 0; t < 2; ++t)
                        if (nblk[t] > 0)
                            issue_S(t, 0);
                    mma_commit_w(&bar_empty[0]);
                }
            }
            for (int j = 0; ok && j < n_iter; ++j) {
                const int iv = 2 * j + 1, ik = 2 * j + 2;
                if (!(ok = mbar_wait_w(&bar_full[iv % C::kStages], phase(iv), abort_flag)))
                    break;
                tc_fence_after();
                bool k_ready = false;
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j < nblk[t]) {
                        for (int hf = 0; hf < 2 && ok; ++hf) {
                            if (!(ok = mbar_wait_w(&bar_p[2 * t + hf], (uint32_t)(j & 1), abort_flag)))
                                break;
                            tc_fence_after();
                            issue_PV(t, j, hf);
                        }
                        if (!ok)
                            break;
                        if (j == nblk[t] - 1)
                            mma_commit_w(&bar_o[t]);
                    }
                    if (j + 1 < nblk[t]) {
                        if (!k_ready) {
                            if (!(ok = mbar_wait_w(&bar_full[ik % C::kStages], phase(ik), abort_flag)))
                                break;
                            tc_fence_after();
                            k_ready = true;
                        }
                        issue_S(t, j + 1);
                    }
                }
                if (!ok)
                    break;
                mma_commit_w(&bar_empty[iv % C::kStages]);
                if (k_ready)
                    mma_commit_w(&bar_empty[ik % C::kStages]);
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
        const int qi = q0 + 128 * t + r;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * (uint32_t)t;
        const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(D * t);
        const int nb = t ? nblk[1] : nblk[0];
        const int qlim = qi + delta;
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;

        for (int j = 0; j < nb; ++j) {
            ok = mbar_wait(&bar_s[t], (uint32_t)(j & 1), abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            uint32_t sr[128];
            tmem_ld128(tS, sr);
            float s[128];
#pragma unroll
            for (int c = 0; c < 128; ++c)
                s[c] = __uint_as_float(sr[c]);

            const int kb = j * 128;
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
            // core at d = 128, so in blocks without masked scores one pair in
            // four goes to the FMA-pipe exp2 instead (masked -inf scores always
            // take ex2.approx, which returns exactly 0 for them).
            const bool soft = !__any_sync(0xffffffffu, need_mask);
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
                tmem_st16(tS + (uint32_t)(16 * hf), pk);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bar_p[2 * t + hf]);
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
                tmem_st32(tS + (uint32_t)(32 * hf), pk);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bar_p[2 * t + hf]);
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

        // ---- epilogue: O = U / l (bf16), LSE = (m + log2 l) ln 2
        const bool row_valid = (C::kTiles == 2 || t == 0) && qi < p.Nq;   // one-tile CTAs: warps 4-7 idle
        const size_t row = (size_t)bh * (size_t)p.Nq + (size_t)qi;
        if (nb > 0 && ok) {
            ok = mbar_wait(&bar_o[t], 0, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                const float inv_l = (l > 0.f) ? p.o_scale / l : 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < p.d_io; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + (uint32_t)c0, o);
                    if (row_valid) {
                        uint32_t w[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            w[c] = Elt<T>::pack(__uint_as_float(o[2 * c]) * inv_l,
                                               __uint_as_float(o[2 * c + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.o) + row * p.d_io + c0);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    }
                }
                if (row_valid && p.lse)
                    p.lse[row] = (l > 0.f) ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
            }
        } else if (nb == 0 && row_valid) {
            // no visible key for any row of this tile
            uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.o) + row * p.d_io);
#pragma unroll 1
            for (int c = 0; c < p.d_io / 8; ++c)
                dst[c] = make_uint4(0u, 0u, 0u, 0u);
            if (p.lse)
                p.lse[row] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
