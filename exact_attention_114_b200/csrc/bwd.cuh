// bwd.cuh -- backward pass by recomputation (page "FlashAttention：为什么少搬数据，
// 反而算得更快", §05: rebuild each needed block of P from the saved row
// statistic instead of reading a stored P).  For L = sum(dO * O):
//   P = exp(scale q.k - LSE),  dV += P^T dO,  dP = dO V^T,  D = rowsum(dO * O),
//   dS = P * (dP - D),  dK += scale dS^T Q,  dQ += scale dS K.
//
// Three kernels:
//   bwd_pre   one warp per query row: D_i, LSE_i * log2(e) (+inf for rows that
//             see no key, so their P is 0), and zero the fp32 dQ accumulator.
//   bwd_main  one CTA per (batch, kv head, 128-key block), key-stationary:
//             K and V stay in shared memory while the CTA walks every query
//             head of the group and every 64-row query block that can see the
//             keys (causal blocks above the diagonal are skipped).  dK and dV
//             accumulate in tensor memory across the whole group, so the GQA
//             reduction over query heads needs no atomics.
//   bwd_post  dQ = bf16(scale * accumulator).
//
// Query split: when there are too few (key block, kv head) units to fill the SMs, or
// their count leaves a last round of CTAs with most SMs idle, q_split CTAs share a
// unit, each walking a contiguous share of its (query head, query block) steps.  Their
// dK / dV sums meet in an fp32 workspace: each takes a ticket when its steps are done;
// all but the last store their sums (16-byte columns, lane after lane) and count
// themselves; the last waits for that count (bounded), adds the partials in a fixed
// order and writes dK / dV.  The last waits only for CTAs that have finished their
// steps, so the wait cannot depend on a CTA that is not yet running.
//
// bwd_main roles (384 threads = 3 warpgroups):
//   warps 0-3  thread r = key r = TMEM lane r: read S^T and dP^T rows from TMEM,
//              write P^T (bf16) back over S^T in TMEM and dS^T (bf16) into
//              shared memory; final dK/dV epilogue.
//   warps 4-7  thread c = dQ^T row c (feature c): move dQ^T from TMEM to a
//              shared [32 x d] fp32 tile (two halves per step) and add it to
//              the dQ accumulator with bulk asynchronous reduce-adds.
//   warp 8     TMA loads (K, V once; Q, dO, LSE, D per step, three slots so a
//              step's loads are issued two steps ahead).
//   warps 10-11 complete the third warpgroup (which gives registers away).
//   warp 9     one thread issues the tcgen05.mma ops, per step `it`:
//                S^T(it+1) = K Q^T, dP^T(it+1) = V dO^T  (as soon as warps 0-3
//                                                        have loaded step it's)
//                dV += P^T(it) dO  (P^T read from tensor memory),
//                dK += dS^T(it) Q, dQ^T(it) = K^T dS^T(it)
//              so the softmax of step it+1 overlaps the gradient MMAs of it;
//              S^T / P^T and dS^T are double-buffered so neither side waits
//              for the other's previous step.
// Tensor memory (512 columns): dK | dV (d each) | S^T/P^T x2 (64 each) | dP^T 64
// | dQ^T 64  (for d = 64 the last 128 columns are unused).
//
// Head size 256: dK and dV of a 128-key block would fill all 512 columns, so
// the features are split in two halves.  A CTA owns (key block, kv head,
// feature half fh): S^T and dP^T still contract over all 256 features (the
// two CTAs of a key block both recompute them), while dV, dK and dQ^T cover
// only features 128 fh .. 128 fh + 127, with the tensor-memory layout of
// d = 128.  K and V of the block take 128 KB of shared memory, which leaves no
// room for a dQ staging tile: the drain warps add dQ^T to the accumulator
// straight from registers with fp32 reductions (one 128-byte row segment per
// warp instruction, paced so that they do not crowd the MMA warp's barrier
// checks out of the memory pipe).  A step's Q / dO are staged by feature half:
// the other CTA's half (Q and dO), which only S^T and dP^T read, is refilled for
// the next step as soon as those MMAs are done; this CTA's Q half (read by S^T
// and dK) sits in two buffers and lands a step ahead; its dO half (read by dP^T
// and dV) sits in one buffer and is refilled once dV is done, while dK, dQ^T and
// the own-half S^T run.  One dS^T buffer.
#pragma once

#include "sm100.cuh"
#include "fa_kernels.h"

namespace fa {

// ----------------------------------------------------------------------------
// bulk (non-tensor) async copies
// ----------------------------------------------------------------------------
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes)
{
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void red_add_f32(float* dst, float x)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst), "f"(x) : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ----------------------------------------------------------------------------
// bwd_pre: -D = -rowsum(dO * O), -LSE in log2 units (stored negated: the main
// kernel adds them), zero the dQ accumulator
// ----------------------------------------------------------------------------
template <int D, typename T = __nv_bfloat16>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdParams p)
{
    // one warp per two rows of B * Hq * Nq_pad (both rows' loads issued before
    // either is reduced); lane l owns columns E*l .. E*l+E-1
    constexpr int E = D / 32;   // elements per lane
    griddep_launch_dependents();   // bwd_main may start its set-up and K / V loads
    const int lane = threadIdx.x & 31;
    const int total = p.B * p.Hq * p.Nq_pad;
    const int row0 = (int)(blockIdx.x * 16 + (threadIdx.x >> 5) * 2);
    const T* po = static_cast<const T*>(p.o);
    const T* pd = static_cast<const T*>(p.dout);
    float s[2] = {0.f, 0.f};
    if (p.q_split > 1) {
        for (int i = (int)(blockIdx.x * blockDim.x + threadIdx.x); i < 2 * p.n_split_units;
             i += (int)(gridDim.x * blockDim.x))
            p.split_cnt[i] = 0;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = row0 + r;
        if (row >= total)
            continue;
        float* acc = p.dq_acc + (size_t)row * D + lane * E;
        if constexpr (E == 8) {
            reinterpret_cast<float4*>(acc)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(acc)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else if constexpr (E == 4) {
            *reinterpret_cast<float4*>(acc) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            *reinterpret_cast<float2*>(acc) = make_float2(0.f, 0.f);
        }
        const int bh = row / p.Nq_pad, i = row - bh * p.Nq_pad;
        if (i >= p.Nq || lane * E >= p.d_io)   // padded row, or padded columns of a narrower head
            continue;
        const size_t src = ((size_t)bh * p.Nq + i) * p.d_io + lane * E;
        if constexpr (E == 8) {
            const uint4 a = *reinterpret_cast<const uint4*>(po + src);
            const uint4 c = *reinterpret_cast<const uint4*>(pd + src);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = Elt<T>::unpack(aw[e]), y = Elt<T>::unpack(cw[e]);
                s[r] = fmaf(x.x, y.x, s[r]);
                s[r] = fmaf(x.y, y.y, s[r]);
            }
        } else if constexpr (E == 4) {
            const uint2 a = *reinterpret_cast<const uint2*>(po + src);
            const uint2 c = *reinterpret_cast<const uint2*>(pd + src);
            const float2 x0 = Elt<T>::unpack(a.x), y0 = Elt<T>::unpack(c.x);
            const float2 x1 = Elt<T>::unpack(a.y), y1 = Elt<T>::unpack(c.y);
            s[r] = fmaf(x0.x, y0.x, s[r]);
            s[r] = fmaf(x0.y, y0.y, s[r]);
            s[r] = fmaf(x1.x, y1.x, s[r]);
            s[r] = fmaf(x1.y, y1.y, s[r]);
        } else {
            const float2 x = Elt<T>::unpack(*reinterpret_cast<const uint32_t*>(po + src));
            const float2 y = Elt<T>::unpack(*reinterpret_cast<const uint32_t*>(pd + src));
            s[r] = fmaf(x.x, y.x, s[r]);
            s[r] = fmaf(x.y, y.y, s[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            s[r] += __shfl_xor_sync(0xffffffffu, s[r], off);
    }
    if (lane < 2) {
        const int row = row0 + lane;
        if (row < total) {
            const float sr = lane ? s[1] : s[0];
            const int bh = row / p.Nq_pad, i = row - bh * p.Nq_pad;
            if (i >= p.Nq) {
                p.neg_delta[row] = 0.f;
                p.neg_lse_log2[row] = -INFINITY;
            } else {
                p.neg_delta[row] = -sr;
                const float l = p.lse[(size_t)bh * p.Nq + i];
                p.neg_lse_log2[row] = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
            }
        }
    }
}

// ----------------------------------------------------------------------------
// bwd_post: dQ = 16-bit(scale * accumulator).  Grid (row chunks, batch * head):
// one warp per two rows, lane l converting columns 4l .. 4l+3 (d <= 128), no
// per-element index division.
// ----------------------------------------------------------------------------
template <int D, typename T = __nv_bfloat16>
__global__ void __launch_bounds__(256) bwd_post_kernel(BwdParams p)
{
    griddep_wait();   // the accumulator is complete once bwd_main has finished
    const int lane = threadIdx.x & 31;
    const long long BH = (long long)p.B * p.Hq;
    const int i_step = (int)gridDim.x * 16;
#pragma unroll 1
    for (int c = lane * 4; c < p.d_io; c += 128)   // one pass per 128 columns
    for (long long bh = blockIdx.y; bh < BH; bh += gridDim.y) {
        const float* acc = p.dq_acc + bh * p.Nq_pad * D + c;
        T* dq = static_cast<T*>(p.dq) + bh * p.Nq * p.d_io + c;
        for (int i0 = (int)(blockIdx.x * 16 + (threadIdx.x >> 5) * 2); i0 < p.Nq; i0 += i_step) {
            const bool two = i0 + 1 < p.Nq;
            const float4 a0 = *reinterpret_cast<const float4*>(acc + (size_t)i0 * D);
            float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (two)
                a1 = *reinterpret_cast<const float4*>(acc + (size_t)(i0 + 1) * D);
            uint2 w;
            w.x = Elt<T>::pack(a0.x * p.scale, a0.y * p.scale);
            w.y = Elt<T>::pack(a0.z * p.scale, a0.w * p.scale);
            *reinterpret_cast<uint2*>(dq + (size_t)i0 * p.d_io) = w;
            if (two) {
                w.x = Elt<T>::pack(a1.x * p.scale, a1.y * p.scale);
                w.y = Elt<T>::pack(a1.z * p.scale, a1.w * p.scale);
                *reinterpret_cast<uint2*>(dq + (size_t)(i0 + 1) * p.d_io) = w;
            }
        }
    }
}

// ----------------------------------------------------------------------------
// bwd_main
// ----------------------------------------------------------------------------
template <int D>
struct BwdCfg {
    static constexpr int kThreads = 384;
    // registers per thread after the split: 128 x (208 + 112 + 144) <= 384 x 168
    static constexpr uint32_t kRegsDS = 208, kRegsDQ = 112, kRegsOther = 144;
    static constexpr int kFeatSplit = (D == 256) ? 2 : 1;   // CTAs per (key block, kv head)
    static constexpr int kDO = D / kFeatSplit;               // dK / dV / dQ features of one CTA
    static constexpr bool kStagedDQ = (D <= 128);            // dQ through a shared staging tile
    static constexpr int kKPanel = 128 * 128;          // 128 keys x 64 bf16
    static constexpr int kKTile = (D / 64) * kKPanel;  // K or V block
    static constexpr int kQPanel = 64 * 128;           // 64 rows x 64 bf16
    static constexpr int kQTile = (D / 64) * kQPanel;  // Q or dO block
    // d = 256: a step's Q / dO by feature half (kQTileH bytes each): the other CTA's
    // half (Q, dO: read by S^T / dP^T only), this CTA's Q half in two buffers (read
    // by S^T and dK) and its dO half in one (read by dP^T and dV); -lse_log2 / -delta
    // in a separate pair of buffers; one dS^T buffer
    static constexpr bool kHalves = (D == 256);
    static constexpr int kQTileH = kHalves ? 2 * kQPanel : kQTile;   // Q or dO of one feature half
    static constexpr int kSlot = 2 * kQTile + 1024;    // d <= 128: Q, dO, -lse_log2[64], -delta[64]
    static constexpr int kSlots = 3;                   // d <= 128: step slots in flight (TMA latency cover)
    static constexpr int kOffOther = 0, kOffQOwn = 2 * kQTileH, kOffDOOwn = 4 * kQTileH;   // d = 256, in the slot area
    static constexpr int kSlotArea = kHalves ? 5 * kQTileH : kSlots * kSlot;
    static constexpr int kPTile = 128 * 128;           // dS^T: 128 keys x 64 q bf16
    static constexpr int kDSBufs = kHalves ? 1 : 2;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kKTile;
    static constexpr int kOffZero = kOffV + kKTile;                 // zero panel (D = 64 only)
    static constexpr int kOffSlots = kOffZero + (D == 64 ? kKPanel : 0);
    static constexpr int kOffVec = kOffSlots + kSlotArea;           // d = 256: [2][-lse_log2 64, -delta 64]
    static constexpr int kOffDS = kOffVec + (kHalves ? 1024 : 0);   // dS^T buffers
    static constexpr int kOffDQ = kOffDS + kDSBufs * kPTile;        // fp32 [32][D] staging (half a step)
    static constexpr int kOffBar = kOffDQ + (kStagedDQ ? 32 * D * 4 : 0);
    static constexpr int kSmemBytes = kOffBar + 256 + 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColDK = 0, kColDV = kDO, kColS = 2 * kDO, kColDP = 2 * kDO + 128,
                              kColDQ = 2 * kDO + 192;
    static_assert(kSmemBytes <= 232448, "shared memory per block");
    // setmaxnreg: the launch gives every thread 168 registers (384 threads, one
    // block per SM); .dec may only lower a warpgroup's count and .inc only raise
    // it, and the three counts must add up to the launch's total
    static_assert(kRegsDQ <= 168 && kRegsOther <= 168 && kRegsDS >= 168, "register split direction");
    static_assert(kRegsDS + kRegsDQ + kRegsOther <= 3 * 168, "register split total");
    static_assert(kColDQ + 64 <= kTmemCols || D == 64, "tensor memory columns");
};

__device__ __forceinline__ void bwd_q_range(const BwdParams& p, int kb, int& qb0, int& nqb)
{
    const int nqb_all = p.Nq_pad / 64;
    qb0 = 0;
    if (p.causal) {
        // first query block containing a row i with kb*128 <= i + (Nk - Nq)
        const int first_row = kb * 128 - (p.Nk - p.Nq);
        qb0 = first_row <= 0 ? 0 : first_row / 64;
    }
    nqb = max(0, nqb_all - qb0);
}

// byte offset of (row, 16-byte chunk) in a tile of 128-byte swizzled rows
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk)
{
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// SPLIT: the launch shares units between CTAs (q_split > 1); without it the kernel
// carries none of the split's code
template <int D, bool CAUSAL, typename T = __nv_bfloat16, bool SPLIT = false>
__global__ void __launch_bounds__(384, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    BwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_kv = bars;            // K, V landed
    uint64_t* bar_full = bars + 1;      // [kSlots] step slot landed
    uint64_t* bar_sdp = bars + 7;       // S^T and dP^T of a step in TMEM
    // A parity wait tells phase k from phase k + 2 apart only if the waiter can never be
    // two phases behind.  The compute warps may finish step it + 1 before the MMA warp
    // looks at step it, and the TMA warp waits for step it - 3's gradients while steps
    // it - 2 and it - 1 run on: so bar_ds alternates between two barriers and bar_gdone
    // between four, and no waiter is ever two phases behind on the barrier it waits on.
    uint64_t* bar_ds = bars + 8;        // [2] P^T (TMEM), dS^T (smem) of step it written: [it & 1] (count 4)
    // [4] gradient MMAs of step it done ([it & 3]): dQ^T(it) is in TMEM, the dS^T
    // buffer (it & 1) and step slot (it % kSlots) are free again
    uint64_t* bar_gdone = bars + 10;
    uint64_t* bar_dqfree = bars + 14;   // dQ^T read out of TMEM (count 4)
    uint64_t* bar_final = bars + 15;    // all MMAs done
    uint64_t* bar_sdp_read = bars + 16; // S^T, dP^T of a step loaded into registers (count 4)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
    // d = 256: bar_full[0] the other half landed, [1 + b] Q own in buffer b, [3] dO own;
    // the other half read by the step's S^T / dP^T, Q own in buffer b by its dK
    // ([b]: one barrier per buffer, so a buffer's next read waits for its next load),
    // dO own by its dV
    uint64_t* bar_h0free = bars + 18;
    uint64_t* bar_qfree = bars + 19;   // [2]
    uint64_t* bar_dofree = bars + 21;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* split_word = reinterpret_cast<int*>(bars + 22);   // query split: the ticket, to the compute warps

    griddep_launch_dependents();   // bwd_post may take the SMs this launch frees
    const int warp = warp_id(), lane = lane_id();
    const int nsp = SPLIT ? p.q_split : 1;                         // CTAs per unit
    const int units = p.B * p.Hkv * C::kFeatSplit;                 // units per key block
    const int kb = (int)blockIdx.x / (units * nsp);   // small key blocks (most work) first
    const int ui = ((int)blockIdx.x % (units * nsp)) / nsp;
    const int sp = (int)blockIdx.x % nsp;                          // share of the unit's steps
    const int kvh = ui / C::kFeatSplit;
    const int fh = ui % C::kFeatSplit;   // feature half (head size 256)
    const int b = kvh / p.Hkv, hk = kvh % p.Hkv;
    int qb0, nqb;
    bwd_q_range(p, kb, qb0, nqb);
    if (!CAUSAL) {
        qb0 = 0;
        nqb = p.Nq_pad / 64;
    }
    // steps it_lo .. it_lo + n_it - 1 of the unit's G * nqb (query head, query block) steps
    const int n_all = p.G * nqb;
    const int it_lo = (int)(((long long)sp * n_all) / nsp);
    const int n_it = (int)(((long long)(sp + 1) * n_all) / nsp) - it_lo;

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < (C::kHalves ? 4 : C::kSlots); ++s)
            mbar_init(&bar_full[s], 1);
        mbar_init(bar_sdp, 1);
        mbar_init(&bar_ds[0], 4);
        mbar_init(&bar_ds[1], 4);
        mbar_init(bar_sdp_read, 4);
        for (int i = 0; i < 4; ++i)
            mbar_init(&bar_gdone[i], 1);
        mbar_init(bar_dqfree, 4);
        mbar_init(bar_final, 1);
        mbar_init(bar_h0free, 1);
        mbar_init(&bar_qfree[0], 1);
        mbar_init(&bar_qfree[1], 1);
        mbar_init(bar_dofree, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (D == 64) {
        // zero panel: rows 64..127 of K^T for the dQ^T MMA (M is 128)
        uint4* z = reinterpret_cast<uint4*>(smem + C::kOffZero);
        for (int i = threadIdx.x; i < C::kKPanel / 16; i += blockDim.x)
            z[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The launch may overlap the end of bwd_pre (programmatic launch), which writes -lse_log2,
    // -delta, the zeroed dQ accumulator and the split counters: every thread waits for it
    // here, except the TMA thread, which first issues the K / V loads (inputs bwd_pre leaves
    // alone) and then waits.
    if (warp != 8 || lane != 0)
        griddep_wait();

    auto step_coords = [&](int it, int& h, int& qb) {
        const int g = it_lo + it;
        h = hk * p.G + g / nqb;
        qb = qb0 + g % nqb;
    };

    // Each role runs inside the branch that sets its register budget.
    if (warp >= 8) {
      regs_dec<C::kRegsOther>();
      if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmDO);
            mbar_arrive_expect_tx(bar_kv, 2 * C::kKTile);
            for (int pn = 0; pn < D / 64; ++pn) {
                tma_load_3d(smem + C::kOffK + pn * C::kKPanel, &tmK, bar_kv, pn * 64, kb * 128, kvh);
                tma_load_3d(smem + C::kOffV + pn * C::kKPanel, &tmV, bar_kv, pn * 64, kb * 128, kvh);
            }
            griddep_wait();
            if constexpr (C::kHalves) {
                // part 0: the other CTA's feature half (Q and dO), read only by the step's
                // S^T / dP^T; part 1: this CTA's Q half (buffer st & 1) with the step's
                // -lse_log2 / -delta; part 2: its dO half.  Loads go out in the order their
                // buffers are freed: the other half of step st + 1, the dO half of st, the
                // Q half of st + 1.
                int issued[3] = {0, 0, 0};
                auto load_part = [&](int st, int part) {
                    int h, qb;
                    step_coords(st, h, qb);
                    const int bh = b * p.Hq + h;
                    const int pn0 = 2 * (part ? fh : 1 - fh);   // first 64-feature panel of the half
                    uint64_t* bar = &bar_full[part == 0 ? 0 : part == 1 ? 1 + (st & 1) : 3];
                    uint8_t* dst = smem + C::kOffSlots +
                                   (part == 0 ? C::kOffOther : part == 1 ? C::kOffQOwn + (st & 1) * C::kQTileH
                                                                         : C::kOffDOOwn);
                    mbar_arrive_expect_tx(bar, (part ? 1 : 2) * C::kQTileH + (part == 1 ? 512 : 0));
                    for (int j = 0; j < 2; ++j) {
                        if (part != 2)
                            tma_load_3d(dst + j * C::kQPanel, &tmQ, bar, (pn0 + j) * 64, qb * 64, bh);
                        if (part != 1)
                            tma_load_3d(dst + (part ? 0 : C::kQTileH) + j * C::kQPanel, &tmDO, bar,
                                        (pn0 + j) * 64, qb * 64, bh);
                    }
                    if (part == 1) {
                        const size_t vrow = (size_t)bh * p.Nq_pad + (size_t)qb * 64;
                        uint8_t* vec = smem + C::kOffVec + (st & 1) * 512;
                        bulk_load(vec, p.neg_lse_log2 + vrow, 256, bar);
                        bulk_load(vec + 256, p.neg_delta + vrow, 256, bar);
                    }
                    ++issued[part];
                };
                if (n_it > 0)
                    for (int part = 0; part < 3; ++part)
                        load_part(0, part);
                if (n_it > 1)
                    load_part(1, 1);   // the second Q buffer starts free
                for (int st = 0; st < n_it; ++st) {
                    // the other half of step st + 1 once step st's S^T / dP^T have read it
                    if (st + 1 < n_it) {
                        if (!mbar_wait(bar_h0free, (uint32_t)(st & 1), abort_flag))
                            break;
                        load_part(st + 1, 0);
                    }
                    if (st > 0) {
                        // the dO half of step st once step st - 1's dV has read it
                        if (!mbar_wait(bar_dofree, (uint32_t)((st - 1) & 1), abort_flag))
                            break;
                        load_part(st, 2);
                        // the Q half of step st + 1 into the buffer step st - 1's dK has read
                        if (st + 1 < n_it) {
                            if (!mbar_wait(&bar_qfree[(st - 1) & 1], (uint32_t)(((st - 1) >> 1) & 1), abort_flag))
                                break;
                            load_part(st + 1, 1);
                        }
                    }
                }
                if (*abort_flag) {
                    mbar_wait_limited(bar_kv, 0, FA_WAIT_LIMIT_CYCLES);
                    // the last load of each buffer: part 1 alternates between two barriers
                    if (issued[0] > 0)
                        mbar_wait_limited(&bar_full[0], (uint32_t)((issued[0] - 1) & 1), FA_WAIT_LIMIT_CYCLES);
                    for (int i = max(0, issued[1] - 2); i < issued[1]; ++i)
                        mbar_wait_limited(&bar_full[1 + (i & 1)], (uint32_t)((i >> 1) & 1), FA_WAIT_LIMIT_CYCLES);
                    if (issued[2] > 0)
                        mbar_wait_limited(&bar_full[3], (uint32_t)((issued[2] - 1) & 1), FA_WAIT_LIMIT_CYCLES);
                }
            } else {
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int s = it % C::kSlots;
                // the slot was last used by step it - kSlots: wait for its gradient MMAs
                if (it >= C::kSlots) {
                    const int prev = it - C::kSlots;
                    if (!mbar_wait(&bar_gdone[prev & 3], (uint32_t)((prev >> 2) & 1), abort_flag))
                        break;
                }
                int h, qb;
                step_coords(it, h, qb);
                const int bh = b * p.Hq + h;
                uint8_t* slot = smem + C::kOffSlots + s * C::kSlot;
                mbar_arrive_expect_tx(&bar_full[s], 2 * C::kQTile + 512);
                for (int pn = 0; pn < D / 64; ++pn) {
                    tma_load_3d(slot + pn * C::kQPanel, &tmQ, &bar_full[s], pn * 64, qb * 64, bh);
                    tma_load_3d(slot + C::kQTile + pn * C::kQPanel, &tmDO, &bar_full[s], pn * 64, qb * 64, bh);
                }
                const size_t vrow = (size_t)bh * p.Nq_pad + (size_t)qb * 64;
                bulk_load(slot + 2 * C::kQTile, p.neg_lse_log2 + vrow, 256, &bar_full[s]);
                bulk_load(slot + 2 * C::kQTile + 256, p.neg_delta + vrow, 256, &bar_full[s]);
                ++issued;
            }
            if (*abort_flag) {
                mbar_wait_limited(bar_kv, 0, FA_WAIT_LIMIT_CYCLES);
                for (int i = max(0, issued - C::kSlots); i < issued; ++i)
                    mbar_wait_limited(&bar_full[i % C::kSlots], (uint32_t)((i / C::kSlots) & 1),
                                      FA_WAIT_LIMIT_CYCLES);
            }
            }
        }
      } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs this loop; one elected lane issues each MMA)
        {
            constexpr uint32_t fmt = Elt<T>::kMmaFmt;
            const uint32_t id_sdp = idesc_f16kind(fmt, 128, 64, false, false);      // S^T, dP^T
            const uint32_t id_grad = idesc_f16kind(fmt, 128, C::kDO, false, true);  // dV, dK
            const uint32_t id_dq = idesc_f16kind(fmt, 128, 64, true, true);         // dQ^T
            const uint32_t tDK = tmem + C::kColDK, tDV = tmem + C::kColDV, tS = tmem + C::kColS,
                           tDP = tmem + C::kColDP, tDQ = tmem + C::kColDQ;
            // base descriptors; a byte offset `o` inside an operand is added as o >> 4
            // to the start-address field (addresses stay below 256 KB, no carry)
            const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);      // K as K-major A
            const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::kOffV), 16, 1024);      // V as K-major A
            // K^T as the M = 128 (feature) MN-major operand of dQ^T: the second 64-feature
            // panel is 16 KB on for d = 128 (and for the feature half of d = 256), the
            // zero panel for d = 64
            const uint32_t lbo_kt = (D >= 128) ? (uint32_t)C::kKPanel : (uint32_t)(C::kOffZero - C::kOffK);
            const uint64_t dK_mn =
                sdesc_sw128(smem_u32(smem + C::kOffK + fh * 2 * C::kKPanel), lbo_kt, 1024);
            // the feature half's two panels of a Q / dO tile (the B operands of dK / dV)
            const uint32_t fo = (uint32_t)(fh * 2 * C::kQPanel);
            const uint64_t dSlot_k = sdesc_sw128(smem_u32(smem + C::kOffSlots), 16, 1024);   // Q / dO K-major
            const uint64_t dSlot_mn = sdesc_sw128(smem_u32(smem + C::kOffSlots), C::kQPanel, 1024);
            const uint64_t dDS_mn = sdesc_sw128(smem_u32(smem + C::kOffDS), C::kPTile, 1024);
            auto off = [](uint32_t bytes) { return (uint64_t)(bytes >> 4); };

            auto issue_sdp = [&](int it) {
                const uint32_t so = (uint32_t)((it % C::kSlots) * C::kSlot);
                const uint32_t tSb = tS + (uint32_t)(64 * (it & 1));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ok_ = (uint32_t)((kk >> 2) * C::kKPanel + (kk & 3) * 32);
                    const uint32_t oq = (uint32_t)((kk >> 2) * C::kQPanel + (kk & 3) * 32);
                    mma_ss_w(tSb, dK_k + off(ok_), dSlot_k + off(so + oq), id_sdp, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ok_ = (uint32_t)((kk >> 2) * C::kKPanel + (kk & 3) * 32);
                    const uint32_t oq = (uint32_t)((kk >> 2) * C::kQPanel + (kk & 3) * 32);
                    mma_ss_w(tDP, dV_k + off(ok_), dSlot_k + off(so + C::kQTile + oq), id_sdp, kk > 0 ? 1u : 0u);
                }
                mma_commit_w(bar_sdp);
            };

            // step it's S^T / dP^T are in registers: the next step's may overwrite dP^T
            // and the other S^T buffer once its Q / dO have landed
            auto next_sdp = [&](int it) -> bool {
                const int in = it + 1;
                if (!mbar_wait_w(bar_sdp_read, (uint32_t)(it & 1), abort_flag))
                    return false;
                if (!mbar_wait_w(&bar_full[in % C::kSlots], (uint32_t)((in / C::kSlots) & 1), abort_flag))
                    return false;
                issue_sdp(in);
                return true;
            };
            // d = 256: S^T / dP^T of step it over one half slot (hs 0: the other CTA's
            // features, K dimension first; hs 1: this CTA's own, accumulating on top)
            // d = 256: S^T (dp false) or dP^T (dp true) of step it over one feature half:
            // hs 0 the other CTA's features, K dimension first; hs 1 this CTA's own,
            // accumulating on top (Q own in buffer it & 1, dO own in its one buffer)
            auto mma_half = [&](int it, int hs, bool dp) {
                const uint32_t tdst = dp ? tDP : tS + (uint32_t)(64 * (it & 1));
                const uint64_t a0 = dp ? dV_k : dK_k;
                const uint32_t so = (uint32_t)(hs == 0 ? C::kOffOther + (dp ? C::kQTileH : 0)
                                               : dp ? C::kOffDOOwn : C::kOffQOwn + (it & 1) * C::kQTileH);
                const int pn0 = 2 * (hs ? fh : 1 - fh);
#pragma unroll 4   // fewer live descriptors
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ok_ = (uint32_t)((pn0 + (kk >> 2)) * C::kKPanel + (kk & 3) * 32);
                    const uint32_t oq = (uint32_t)((kk >> 2) * C::kQPanel + (kk & 3) * 32);
                    mma_ss_w(tdst, a0 + off(ok_), dSlot_k + off(so + oq), id_sdp, (hs || kk > 0) ? 1u : 0u);
                }
            };
            // bar_full[part] of step it landed: part 0 the other half, 1 Q own, 2 dO own
            auto wait_part = [&](int it, int part) -> bool {
                uint64_t* bar = &bar_full[part == 0 ? 0 : part == 1 ? 1 + (it & 1) : 3];
                const uint32_t ph = (uint32_t)((part == 1 ? (it >> 1) : it) & 1);
                if (!mbar_wait_w(bar, ph, abort_flag))
                    return false;
                tc_fence_after();
                return true;
            };
            // this CTA's half of step it: S^T on Q own, dP^T on dO own, then the signal
            auto own_half = [&](int it) -> bool {
                if (!wait_part(it, 1))
                    return false;
                mma_half(it, 1, false);
                if (!wait_part(it, 2))
                    return false;
                mma_half(it, 1, true);
                mma_commit_w(bar_sdp);
                return true;
            };
            bool ok = mbar_wait_w(bar_kv, 0, abort_flag);
            if constexpr (C::kHalves) {
            // per step it: S^T / dP^T of step it + 1 over the other half (under step it's
            // exponentials); step it's dV (frees the dO half), dK (frees its Q buffer)
            // and dQ^T; then step it + 1's own half: its Q half was loaded a step ahead,
            // and its dO half's load runs under dK, dQ^T and the own-half S^T
            if (ok && n_it > 0) {
                ok = wait_part(0, 0);
                if (ok) {
                    mma_half(0, 0, false);
                    mma_half(0, 0, true);
                    mma_commit_w(bar_h0free);
                    ok = own_half(0);
                }
            }
            for (int it = 0; ok && it < n_it; ++it) {
                if (it + 1 < n_it) {
                    // step it's dP^T in registers, and the other half of step it + 1 landed
                    if (!(ok = mbar_wait2_w(bar_sdp_read, (uint32_t)(it & 1), &bar_full[0],
                                            (uint32_t)((it + 1) & 1), abort_flag)))
                        break;
                    tc_fence_after();
                    mma_half(it + 1, 0, false);
                    mma_half(it + 1, 0, true);
                    mma_commit_w(bar_h0free);
                }
                // dS of step it written, and dQ^T of step it - 1 read out (for it = 0 the
                // second check is of the phase before the barrier's first, complete)
                if (!(ok = mbar_wait2_w(&bar_ds[it & 1], (uint32_t)((it >> 1) & 1), bar_dqfree,
                                        (uint32_t)((it - 1) & 1), abort_flag)))
                    break;
                tc_fence_after();
                const uint32_t tP = tS + (uint32_t)(64 * (it & 1));
                const uint32_t oq = (uint32_t)(C::kOffQOwn + (it & 1) * C::kQTileH);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts_w(tDV, tP + (uint32_t)(kk * 8), dSlot_mn + off(C::kOffDOOwn + kk * 2048), id_grad,
                             (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit_w(bar_dofree);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts_w(tDK, tP + 32u + (uint32_t)(kk * 8), dSlot_mn + off(oq + kk * 2048), id_grad,
                             (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit_w(&bar_qfree[it & 1]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss_w(tDQ, dK_mn + off(kk * 2048), dDS_mn + off(kk * 2048), id_dq, kk > 0 ? 1u : 0u);
                mma_commit_w(&bar_gdone[it & 3]);
                if (it + 1 < n_it && !(ok = own_half(it + 1)))
                    break;
            }
            } else {
            if (ok && n_it > 0) {
                ok = mbar_wait_w(&bar_full[0], 0, abort_flag);
                if (ok)
                    issue_sdp(0);
            }
            for (int it = 0; ok && it < n_it; ++it) {
                if (it + 1 < n_it && !(ok = next_sdp(it)))
                    break;
                if (!(ok = mbar_wait_w(&bar_ds[it & 1], (uint32_t)((it >> 1) & 1), abort_flag)))
                    break;
                tc_fence_after();
                if (it > 0) {
                    if (!(ok = mbar_wait_w(bar_dqfree, (uint32_t)((it - 1) & 1), abort_flag)))
                        break;
                    tc_fence_after();
                }
                const uint32_t so = (uint32_t)((it % C::kSlots) * C::kSlot);
                const uint32_t dso = (uint32_t)((it & 1) * C::kPTile);
                const uint32_t tP = tS + (uint32_t)(64 * (it & 1));   // P^T: 32 columns of bf16 pairs
                // dV += P^T dO ; dK += dS^T Q   (K dimension = 64 query rows)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
                    mma_ts_w(tDV, tP + (uint32_t)(kk * 8), dSlot_mn + off(so + C::kQTileH + fo + kk * 2048), id_grad,
                             acc);
                    mma_ts_w(tDK, tP + 32u + (uint32_t)(kk * 8), dSlot_mn + off(so + fo + kk * 2048), id_grad, acc);
                }
                // dQ^T = K^T dS^T   (K dimension = 128 keys)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss_w(tDQ, dK_mn + off(kk * 2048), dDS_mn + off(dso + kk * 2048), id_dq, kk > 0 ? 1u : 0u);
                mma_commit_w(&bar_gdone[it & 3]);
            }
            }
            mma_commit_w(bar_final);
            if (!ok)
                mbar_wait_limited(bar_final, 0, FA_WAIT_LIMIT_CYCLES);
        }
      }
    } else if (warp < 4) {
        regs_inc<C::kRegsDS>();
        // ------------------------------------------------------------ P^T / dS^T
        const int r = warp * 32 + lane;                 // key within the block
        const int key = kb * 128 + r;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::kColS, tDP = tmem + lane_off + C::kColDP;
        const float sl2 = p.scale_log2;
        const int delta_q = p.Nk - p.Nq;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            int h, qb;
            step_coords(it, h, qb);
            ok = mbar_wait(bar_sdp, (uint32_t)(it & 1), abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            // -LSE * log2(e) and -D of the step's 64 query rows, read four at a time: each
            // load is a broadcast, and 16-byte ones take a quarter of the shared-memory cycles
            const float4* nlse4 = reinterpret_cast<const float4*>(
                C::kHalves ? smem + C::kOffVec + (it & 1) * 512
                           : smem + C::kOffSlots + (it % C::kSlots) * C::kSlot + 2 * C::kQTile);
            const float4* ndlt4 = nlse4 + 16;
            const uint32_t tSb = tS + (uint32_t)(64 * (it & 1));
            uint32_t sr[64], dr[64];
            tmem_ld64x2(tSb, tDP, sr, dr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_sdp_read);
            // query rows qb*64 + c see this key iff key < Nk and (causal) key <= row + Nk - Nq
            const int q_first = qb * 64;
            const int min_row = CAUSAL ? key - delta_q : INT_MIN;   // rows >= min_row see the key
            const bool key_ok = key < p.Nk;
            uint32_t pp[32], dd[32];
            const float2 sl22 = make_float2(sl2, sl2);
            // rows >= min_row see the key; whole 64-row block visible in most steps
            const bool all_vis = key_ok && (q_first >= min_row);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                const float4 nl4 = nlse4[c4], nd4 = ndlt4[c4];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int c = 4 * c4 + 2 * h2;
                    const float2 nl = h2 ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
                    const float2 nd = h2 ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
                    const float2 x =
                        ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl22, nl);
                    float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    if (!all_vis) {
                        pv.x = (key_ok && q_first + c >= min_row) ? pv.x : 0.f;
                        pv.y = (key_ok && q_first + c + 1 >= min_row) ? pv.y : 0.f;
                    }
                    // dS = P * (dP - D)
                    const float2 dd2 = fadd2(make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])), nd);
                    const float2 ds2 = fmul2(pv, dd2);
                    pp[c >> 1] = Elt<T>::pack(pv.x, pv.y);
                    dd[c >> 1] = Elt<T>::pack(ds2.x, ds2.y);
                }
            }
            // P^T over this step's S^T columns (the dV MMA reads it from there)
            tmem_st32(tSb, pp);
            // dS^T into this step's buffer, free once the gradient MMAs of the step that
            // used it last (it - 2; it - 1 with the single buffer of d = 256) are done
            if (it >= C::kDSBufs) {
                const int prev = it - C::kDSBufs;
                ok = mbar_wait(&bar_gdone[prev & 3], (uint32_t)((prev >> 2) & 1), abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
            }
            uint8_t* sDS = smem + C::kOffDS + (it % C::kDSBufs) * C::kPTile;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(sDS + sw128_off(r, ch)) =
                    make_uint4(dd[4 * ch], dd[4 * ch + 1], dd[4 * ch + 2], dd[4 * ch + 3]);
            fence_proxy_async_smem();
            // dS^T also over the other 32 S^T columns: the dK MMA reads it from there
            // (A in TMEM), which takes its 16 KB per step off the shared-memory reads
            tmem_st32(tSb + 32u, dd);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bar_ds[it & 1]);
        }
        // ---- epilogue: dK = scale * acc, dV = acc  (bf16).  With q_split > 1 each CTA
        // of the unit holds the sums over its own steps: the first q_split - 1 to get
        // here leave theirs in fp32 in the workspace, and the last adds them in.
        if (ok) {
            ok = mbar_wait(bar_final, 0, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
        }
        int ticket = nsp - 1;   // the last CTA of the unit (the only one without a split)
        // the unit's counters, from the block index again (nothing kept live over the steps)
        const int unit_e = SPLIT ? (int)(ctaid_x() / (uint32_t)nsp) : 0;
        int* n_written = SPLIT ? p.split_cnt + p.n_split_units + unit_e : nullptr;
        if (SPLIT && nsp > 1) {
            ok = named_bar_and(3, 128, ok);   // the four warps go on together
            if (threadIdx.x == 0)
                *split_word = atomicAdd(&p.split_cnt[unit_e], 1);
            named_bar_sync(3, 128);
            ticket = *split_word;
            if (ok && ticket == nsp - 1) {
                // the others took their tickets after their last step and only store
                // and count from there, so this wait ends unless one of them gave up
                bool got = true;
                if (threadIdx.x == 0) {
                    const long long t0 = clock64();
                    while (ld_acquire_gpu(n_written) < nsp - 1) {
                        if (clock64() - t0 > FA_WAIT_LIMIT_CYCLES) {
                            atomicOr(&g_status, kStatusTimeout);
                            got = false;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                ok = named_bar_and(3, 128, got);
                __threadfence();
            }
        }
        if (ok) {
            tc_fence_after();
            const bool key_ok = key < p.Nk;
            const int d_io = p.d_io;
            constexpr int kPart4 = 2 * C::kDO / 4 * 128;   // float4 per partial
            // partial slots: one per unit for two shares (the last CTA adds the other's to
            // its own, and a + b = b + a); one per share for more, all stored and added in
            // share order, so that dK / dV do not depend on which CTA finishes last
            const int nslot = nsp == 2 ? 1 : nsp;
            const int my_slot = (!SPLIT || nsp == 2) ? 0 : (int)(ctaid_x() % (uint32_t)nsp);
            float4* part = SPLIT ? p.dkv_part + (size_t)unit_e * (size_t)nslot * kPart4 + r : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < C::kDO; c0 += 32) {
                const int col = fh * C::kDO + c0;   // feature of the tensors in memory
                if (col >= d_io)   // padded columns of a narrower head
                    break;
                const size_t krow = ((size_t)kvh * p.Nk + key) * d_io + fh * C::kDO;
                uint32_t a[32], v[32];
                if (n_it > 0) {
                    tmem_ld32(tmem + lane_off + C::kColDK + c0, a);
                    tmem_ld32(tmem + lane_off + C::kColDV + c0, v);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        a[c] = v[c] = 0u;
                }
                // a partial is [dK chunks | dV chunks][128 keys] of 4 floats: lane r of a
                // warp stores or loads the 16 bytes after lane r - 1's (each thread reads
                // back only what it or another CTA's thread r stored)
                const int ck = c0 / 4, cv = C::kDO / 4 + c0 / 4;
                if (SPLIT && nsp > 1) {
                    if (ticket < nsp - 1 || nsp > 2) {
                        float4* out = part + (size_t)my_slot * kPart4;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            __stcg(out + (ck + j) * 128, make_float4(__uint_as_float(a[4 * j]), __uint_as_float(a[4 * j + 1]),
                                                                     __uint_as_float(a[4 * j + 2]), __uint_as_float(a[4 * j + 3])));
                            __stcg(out + (cv + j) * 128, make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
                        }
                    }
                    if (ticket < nsp - 1)
                        continue;
                    // the last: two shares add the other's partial to this one; more start
                    // from share 0's and add the rest in order (this CTA's own included)
#pragma unroll 1
                    for (int o = (nsp == 2 ? 0 : 1); o < nslot; ++o) {
                        const float4* in = part + (size_t)o * kPart4;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 x = __ldcg(in + (ck + j) * 128), y = __ldcg(in + (cv + j) * 128);
                            if (nsp > 2 && o == 1) {
                                const float4 x0 = __ldcg(part + (ck + j) * 128), y0 = __ldcg(part + (cv + j) * 128);
                                a[4 * j] = __float_as_uint(x0.x);
                                a[4 * j + 1] = __float_as_uint(x0.y);
                                a[4 * j + 2] = __float_as_uint(x0.z);
                                a[4 * j + 3] = __float_as_uint(x0.w);
                                v[4 * j] = __float_as_uint(y0.x);
                                v[4 * j + 1] = __float_as_uint(y0.y);
                                v[4 * j + 2] = __float_as_uint(y0.z);
                                v[4 * j + 3] = __float_as_uint(y0.w);
                            }
                            a[4 * j] = __float_as_uint(__uint_as_float(a[4 * j]) + x.x);
                            a[4 * j + 1] = __float_as_uint(__uint_as_float(a[4 * j + 1]) + x.y);
                            a[4 * j + 2] = __float_as_uint(__uint_as_float(a[4 * j + 2]) + x.z);
                            a[4 * j + 3] = __float_as_uint(__uint_as_float(a[4 * j + 3]) + x.w);
                            v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + y.x);
                            v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + y.y);
                            v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + y.z);
                            v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + y.w);
                        }
                    }
                }
                if (key_ok) {
                    uint32_t wk[16], wv[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        wk[c] = Elt<T>::pack(__uint_as_float(a[2 * c]) * p.scale, __uint_as_float(a[2 * c + 1]) * p.scale);
                        wv[c] = Elt<T>::pack(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
                    }
                    uint4* dk4 = reinterpret_cast<uint4*>(static_cast<T*>(p.dk) + krow + c0);
                    uint4* dv4 = reinterpret_cast<uint4*>(static_cast<T*>(p.dv) + krow + c0);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        dk4[c] = make_uint4(wk[4 * c], wk[4 * c + 1], wk[4 * c + 2], wk[4 * c + 3]);
                        dv4[c] = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                    }
                }
            }
        }
        if (SPLIT && nsp > 1 && ticket < nsp - 1) {
            // publish the partial: every thread's stores, then the count (also after a
            // give-up, so that the last CTA does not wait out its limit)
            __threadfence();
            named_bar_sync(3, 128);
            if (threadIdx.x == 0)
                atomicAdd(n_written, 1);
        }
    } else {
        regs_dec<C::kRegsDQ>();
        // ------------------------------------------------------------ dQ^T drain (warps 4-7)
        const int wq = warp - 4;
        const int f = wq * 32 + lane;              // feature index = TMEM lane
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tDQ = tmem + lane_off + C::kColDQ;
        float* stage = reinterpret_cast<float*>(smem + C::kOffDQ);   // [32][D]
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            int h, qb;
            step_coords(it, h, qb);
            ok = mbar_wait(&bar_gdone[it & 3], (uint32_t)((it >> 2) & 1), abort_flag);
            // all four drain warps decide together: the named barriers below need all of them
            ok = named_bar_and(2, 128, ok);
            if (!ok)
                break;
            tc_fence_after();
            if constexpr (!C::kStagedDQ) {
                // fp32 reductions straight from registers: for query row c the 32 lanes
                // of a warp add 32 consecutive features, one 128-byte segment per
                // instruction (this CTA's feature half of the accumulator row); the
                // 64 query columns are read in two halves of 32
                float* dst = p.dq_acc + ((size_t)(b * p.Hq + h) * p.Nq_pad + (size_t)qb * 64) * D +
                             fh * C::kDO + f;
                uint32_t a[32];
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    tmem_ld32(tDQ + (uint32_t)(32 * hq), a);
                    if (hq == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(bar_dqfree);
                    }
                    // paced: a short pause after every 8 reductions keeps them from filling
                    // the memory pipe that the MMA warp's barrier checks go through (the
                    // drain has most of a step to finish)
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        red_add_f32(dst + (size_t)(32 * hq + c) * D, __uint_as_float(a[c]));
                        if ((c & 7) == 7)
                            __nanosleep(64);
                    }
                }
                continue;
            }
            uint32_t a[64];
            tmem_ld64(tDQ, a);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_dqfree);
            // two halves of 32 query rows through a 16 KB staging tile
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                // the previous bulk reduce must have finished reading the staging tile
                if (threadIdx.x == 128)
                    bulk_wait_read0();
                named_bar_sync(2, 128);
                if (f < D) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        stage[c * D + f] = __uint_as_float(a[32 * hf + c]);
                }
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (threadIdx.x == 128) {
                    const size_t row0 = ((size_t)(b * p.Hq + h) * p.Nq_pad + (size_t)qb * 64 + 32 * hf) * D;
                    bulk_reduce_add_f32(p.dq_acc + row0, stage, 32 * D * 4);
                    bulk_commit();
                }
            }
        }
        if (threadIdx.x == 128)
            bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
