// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument checks,
// TMA descriptor set-up, kernel selection and launches on the caller's stream.
//
// All kernels live in this one translation unit so that they share the device
// status word g_status without relocatable device code.
#include "fa.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <queue>
#include <vector>
#include <string>
#include <type_traits>
#include <utility>

#include "bwd.cuh"
#include "decode.cuh"
#include "fa_kernels.h"
#include "fp8.cuh"
#include "fwd.cuh"

namespace {

constexpr int kAbiVersion = 1;
constexpr float kLog2e = 1.4426950408889634f;

thread_local std::string t_error;

void set_error(const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_error = buf;
}

fa_status_t cuda_fail(cudaError_t e, const char* what)
{
    set_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return FA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// argument checks (no CUDA call is made before these pass)
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status_t check_ptr(const void* p, const char* name)
{
    if (p == nullptr) {
        set_error("%s is NULL", name);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (!aligned16(p)) {
        set_error("%s is not 16-byte aligned", name);
        return FA_ERR_INVALID_ARGUMENT;
    }
    return FA_OK;
}

fa_status_t check_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) {
        set_error("sizes must be >= 1 (B=%d Hq=%d Hkv=%d Nq=%d Nk=%d)", B, Hq, Hkv, Nq, Nk);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (Hq % Hkv != 0) {
        set_error("Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (d < 1) {
        set_error("d=%d must be >= 1", d);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (causal != 0 && causal != 1) {
        set_error("causal=%d must be 0 or 1", causal);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (!(std::isfinite(scale) && scale > 0.f)) {
        set_error("scale must be finite and > 0");
        return FA_ERR_INVALID_ARGUMENT;
    }
    // index ranges: row counts and TMA coordinates are 32-bit
    if ((long long)B * Hq * ((long long)Nq + 256) > (1ll << 31) - 1 ||
        (long long)B * Hkv * ((long long)Nk + 256) > (1ll << 31) - 1) {
        set_error("problem too large for 32-bit row indices");
        return FA_ERR_UNSUPPORTED;
    }
    if (d < 32 || d > 256 || d % 32 != 0) {
        set_error("d=%d is not supported (a multiple of 32 up to 256)", d);
        return FA_ERR_UNSUPPORTED;
    }
    return FA_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

template <typename T>
constexpr CUtensorMapDataType tma_type()
{
    return std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// 3-D map over a [outer][rows][inner] tensor of `elt` -byte elements, box
// {box_inner, box_rows, 1} with box_inner * elt = 128 bytes (the 128-byte
// swizzle span); elements past `inner` or `rows` read as zero.
fa_status_t make_map_box(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                         uint32_t elt, uint32_t box_inner, uint32_t box_rows, CUtensorMapDataType dt)
{
    EncodeTiledFn enc = get_encode();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable");
        return FA_ERR_CUDA;
    }
    cuuint64_t dims[3] = {inner, rows, outer};
    cuuint64_t strides[2] = {inner * elt, inner * rows * elt};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

// 16-bit tensor [outer][rows][inner], box {64, box_rows, 1}
fa_status_t make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                     uint32_t box_rows, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
{
    return make_map_box(m, base, inner, rows, outer, 2, 64, box_rows, dt);
}

// 4-D map over a paged KV pool [pages][page_size][Hkv][d] (bf16), box {64, 1, 64, 1}
// (one kv head, 64 keys of one page), 128-byte swizzle.
fa_status_t make_map_paged(CUtensorMap* m, const void* base, uint64_t d, uint64_t Hkv, uint64_t page_size,
                           uint64_t pages, CUtensorMapDataType dt)
{
    EncodeTiledFn enc = get_encode();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable");
        return FA_ERR_CUDA;
    }
    cuuint64_t dims[4] = {d, Hkv, page_size, pages};
    cuuint64_t strides[3] = {d * 2, Hkv * d * 2, page_size * Hkv * d * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled (paged) failed (%d)", (int)r);
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

// Raise a kernel's dynamic shared memory limit once per (kernel, device).
fa_status_t ensure_smem(const void* kernel, int bytes)
{
    static std::mutex mu;
    static std::map<const void*, unsigned long long> done;   // kernel -> bit per device (< 64)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(mu);
    unsigned long long& mask = done[kernel];
    if (dev < 64 && (mask >> dev) & 1ull)
        return FA_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute");
    if (dev < 64)
        mask |= 1ull << dev;
    return FA_OK;
}

fa_status_t check_launch(const char* what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, what);
    return FA_OK;
}

// Launch `kern` as a programmatic dependent of the kernel before it on the stream, which
// is always one of this library's own launches of the same call: its blocks may be
// scheduled, and run their set-up, while that kernel's last blocks finish.  Each such
// kernel calls griddep_wait() before it reads anything that kernel writes, and the
// kernel before it calls griddep_launch_dependents() at its start.
template <typename... P, typename... A>
fa_status_t launch_dependent(const char* what, void (*kern)(P...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, A&&... args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
    if (e != cudaSuccess)
        return cuda_fail(e, what);
    return check_launch(what);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

// ---------------------------------------------------------------------------
// forward (tiled kernel)
// ---------------------------------------------------------------------------
// Kernel head dim for a head dim d of the tensors (a multiple of 32): the next of
// 64, 128, 256, the missing columns being zero fill of the TMA boxes (zero
// columns add nothing to Q K^T, and P V gives zero there, never stored).
int kernel_d(int d) { return d <= 64 ? 64 : d <= 128 ? 128 : 256; }

// The forward is persistent: one block per SM (its shared memory allows no
// second), together working through the n_pairs * n_bh (* kv_split) tiles.
unsigned fwd_grid(const fa::FwdParams& p)
{
    const long long units = (long long)p.n_pairs * p.n_bh;
    const long long tiles = p.kv_split > 1 ? p.full_tiles + (units - p.full_tiles) * p.kv_split : units;
    return (unsigned)std::max<long long>(1, std::min<long long>(tiles, sm_count()));
}

// stream-ordered scratch from the library's memory pool (defined below)
cudaError_t scratch_alloc(void** out, size_t bytes, cudaStream_t s);

// Tile heads of the tiled forward.  A query head with fewer rows than a work tile
// (Nq < 128 * tiles per CTA) would leave most of its tiles' rows idle and read its kv
// head's K/V once per query head; so where a kv head serves several query heads (G > 1)
// their G * Nq rows, consecutive in q / o / lse, share the kv head's tiles ("group rows").
struct FwdGeom {
    int group_rows, n_bh, rows, n_pairs;
};

FwdGeom fwd_geom(int B, int Hq, int Hkv, int Nq, int d)
{
    const int kt = kernel_d(d) == 256 ? 1 : 2;
    const int G = Hq / Hkv;
    FwdGeom g;
    g.group_rows = (G > 1 && Nq < 128 * kt) ? 1 : 0;
    g.n_bh = g.group_rows ? B * Hkv : B * Hq;
    g.rows = g.group_rows ? G * Nq : Nq;
    g.n_pairs = (g.rows + 128 * kt - 1) / (128 * kt);
    return g;
}

// 128-key blocks seen by the 128-row query tile at row qt of a tile head with `rows`
// rows, row r at query position r % Nq (as the kernel's fwd_blocks_for_tile)
int host_blocks_for_tile(int qt, int rows, int Nq, int Nk, int causal)
{
    const int nkb = (Nk + 127) / 128;
    if (qt >= rows)
        return 0;
    if (!causal)
        return nkb;
    const int last_row = std::min(qt + 127, rows - 1);
    const int last_pos = (qt / Nq == last_row / Nq) ? last_row % Nq : Nq - 1;
    const long long last_key = (long long)last_pos + (Nk - Nq);
    return last_key < 0 ? 0 : (int)std::min<long long>(nkb, last_key / 128 + 1);
}

// Key split of the tiled forward.  The persistent launch claims its work units (query tile
// pair, tile head) heaviest first; a unit costs its key blocks plus about 2 block times of
// fixed work (Q load, first S, epilogue).  With few units, or a last round that fills few
// SMs, units are cut into s contiguous shares of their key blocks (each share a work tile of
// its own, writing an fp32 partial that fwd_combine_kernel merges): either every unit, or only
// the units after the last full round of whole units (full_tiles of them stay whole and write
// o / lse directly).  Each choice is scored by simulating the greedy claiming on the SMs, plus
// the merge: about 8 block times of launch and fixed work and the partials' traffic (written
// and read, 13 MB per block time at the copy bandwidth).  A split is taken where it saves at
// least 5%; launches with more than 8 units per SM are balanced enough by the claiming alone.
// A tail split keeps to 2 shares when K and V take more than 64 MB: the whole units of a kv
// head stream its keys together and mostly hit in L2, while the shares of one unit read
// different key ranges at once (4 shares on a 2048-row chunk against 32K keys: no gain, with
// 8% in the simulation).  The choice depends only on the units' key-block counts, the head
// size, the SM count and whether K / V pass 64 MB; it is cached under those (up to 4096 entries,
// then the cache starts over).  Candidates whose even-spread lower bound cannot beat the best so
// far are not simulated, and a plan of at most one tile per SM needs no simulation.
struct FwdSplit {
    int shares, full;
};

FwdSplit fwd_split_plan(const FwdGeom& g, int B, int Hkv, int Nq, int Nk, int d, int causal, int sms)
{
    const long long n_units = (long long)g.n_pairs * g.n_bh;
    if (n_units > 8LL * sms || n_units < 1)
        return {1, (int)n_units};
    const int kt = kernel_d(d) == 256 ? 1 : 2;
    // the plan depends on the sizes only through the units' key-block counts
    const double kv_bytes = 4.0 * B * Hkv * (double)Nk * d;   // K and V, 16-bit
    const bool kv_beyond_l2 = kv_bytes > 64.0 * (1 << 20);
    std::vector<long long> key{g.n_bh, kt, d, sms, kv_beyond_l2};
    for (int pr = 0; pr < g.n_pairs; ++pr) {
        int n = 0;
        for (int t = 0; t < kt; ++t)
            n = std::max(n, host_blocks_for_tile(pr * 128 * kt + 128 * t, g.rows, Nq, Nk, causal));
        key.push_back(n);
    }
    static std::mutex mu;
    static std::map<std::vector<long long>, FwdSplit> cache;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = cache.find(key);
        if (it != cache.end())
            return it->second;
    }
    auto unit_len = [&](long long u) { return (int)key[5 + (size_t)(g.n_pairs - 1 - u / g.n_bh)]; };
    const double fixed = 2.0, merge_fixed = 8.0, bytes_per_block = 13.0e6;
    std::vector<double> lens;
    // the work tiles of a plan, in claim order
    auto items = [&](long long full, int sh) {
        lens.clear();
        for (long long u = 0; u < n_units; ++u) {
            const int n = unit_len(u);
            if (u < full || sh == 1) {
                lens.push_back(n + fixed);
            } else {
                for (int k = 0; k < sh; ++k)
                    lens.push_back((double)(((long long)(k + 1) * n) / sh - ((long long)k * n) / sh) + fixed);
            }
        }
    };
    // greedy claiming on `sms` CTAs: the last finish (one round: the longest tile)
    auto simulate = [&]() {
        double last = 0;
        if ((int)lens.size() <= sms) {
            for (double x : lens)
                last = std::max(last, x);
            return last;
        }
        std::priority_queue<double, std::vector<double>, std::greater<double>> done;
        for (double x : lens) {
            double start = 0;
            if ((int)done.size() == sms) {
                start = done.top();
                done.pop();
            }
            done.push(start + x);
            last = std::max(last, start + x);
        }
        return last;
    };
    items(n_units, 1);
    const double base = simulate();
    FwdSplit best{1, (int)n_units};
    double best_cost = base;
    static const int kShares[] = {2, 3, 4, 6, 8, 12, 16};
    const long long fulls[2] = {0, (n_units / sms) * sms};
    for (long long full : fulls) {
        if (full >= n_units || (full > 0 && full == fulls[0]))
            continue;
        int longest = 0;
        double total = 0;
        for (long long u = 0; u < n_units; ++u) {
            total += unit_len(u);
            if (u >= full)
                longest = std::max(longest, unit_len(u));
        }
        for (int sh : kShares) {
            const double part_bytes = (double)(n_units - full) * sh * 128 * kt * d * 4.0;
            if (longest < 2 * sh || part_bytes > 256.0 * (1 << 20) ||
                (full > 0 && sh > 2 && kv_beyond_l2))
                break;
            const double extra = merge_fixed + 2.0 * part_bytes / bytes_per_block;
            // no plan beats its lower bound, the work spread evenly over all SMs, and
            // the bound grows with the share count
            const double n_items = (double)full + (double)(n_units - full) * sh;
            const double bound = (total + n_items * fixed) / sms + extra;
            if (bound >= best_cost || bound >= 0.95 * base)
                break;
            items(full, sh);
            const double cost = simulate() + extra;
            if (cost < best_cost && cost < 0.95 * base) {
                best = {sh, (int)full};
                best_cost = cost;
            }
        }
    }
    std::lock_guard<std::mutex> lk(mu);
    if (cache.size() >= 4096)
        cache.clear();
    cache[key] = best;
    return best;
}

// Test hook state: a slot every tiled forward launch is pinned to (-1: rotate).
std::atomic<int> g_pinned_slot{-1};

// The launch's tile counter: the next slot of fa::g_fwd_tile_ctr (zero between
// launches: the kernel's last block resets it) and the launch's owner tag, a
// nonzero number unique among the last 2^32 - 1 launches of the process.
// Slots rotate, so concurrent launches on different streams get different ones;
// a launch that still finds its slot held by another reports kStatusSlotShared.
fa_status_t fwd_tile_counter(unsigned** ctr, unsigned* tag)
{
    static std::atomic<unsigned> seq{0};
    void* base = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&base, fa::g_fwd_tile_ctr);
    if (e != cudaSuccess)
        return cuda_fail(e, "tile counter address");
    const unsigned n = seq.fetch_add(1u, std::memory_order_relaxed);
    const int pinned = g_pinned_slot.load(std::memory_order_relaxed);
    const unsigned slot = pinned >= 0 ? (unsigned)pinned : n % fa::kFwdCtrSlots;
    *ctr = static_cast<unsigned*>(base) + fa::kFwdCtrWords * slot;
    *tag = n % 0xFFFFFFFFu + 1u;
    return FA_OK;
}

// The tiled forward's launch: with a key split (p.kv_split > 1) the shares' fp32 partials
// go to stream-ordered scratch and fwd_combine_kernel merges them into o / lse.
template <typename T, typename Kern>
fa_status_t launch_fwd_tiles(Kern kern, int threads, int smem, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, fa::FwdParams& p, cudaStream_t stream,
                             bool after_kernel = false)
{
    void* ws = nullptr;
    if (p.kv_split > 1) {
        // indexed by tile head and share: [n_bh][kv_split][rows] (only split units' rows used)
        const size_t rows = (size_t)p.n_bh * p.kv_split * p.rows;
        const size_t o_bytes = align256(rows * p.d_io * 4);
        cudaError_t e = scratch_alloc(&ws, o_bytes + align256(rows * 4), stream);
        if (e != cudaSuccess)
            return cuda_fail(e, "scratch allocation (forward key-split partials)");
        p.part_o = static_cast<float*>(ws);
        p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + o_bytes);
    }
    fa_status_t st;
    if (after_kernel && p.kv_split <= 1) {
        // straight after a kernel of the same call (the e4m3 V transpose)
        st = launch_dependent("fwd_kernel launch", kern, dim3(fwd_grid(p)), dim3(threads), (size_t)smem, stream,
                              mq, mk, mv, p);
    } else {
        kern<<<fwd_grid(p), threads, smem, stream>>>(mq, mk, mv, p);
        st = check_launch("fwd_kernel launch");
    }
    if (p.kv_split > 1) {
        if (st == FA_OK) {
            const long long rows = (long long)p.n_bh * p.rows;
            st = launch_dependent("fwd_combine_kernel launch", fa::fwd_combine_kernel<T>,
                                  dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, stream, p);
        }
        cudaError_t e = cudaFreeAsync(ws, stream);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

template <int D, bool CAUSAL, typename T>
fa_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Nq, int Nk, int d, float scale, cudaStream_t stream)
{
    using C = fa::FwdCfg<D>;
    CUtensorMap mq, mk, mv;
    fa_status_t st;
    const FwdGeom g = fwd_geom(B, Hq, Hkv, Nq, d);
    // q as [tile heads][rows][d]: with group rows a kv head's G query heads are one run of rows
    if ((st = make_map(&mq, q, d, g.rows, (uint64_t)g.n_bh, 128, tma_type<T>())) != FA_OK) return st;
    if ((st = make_map(&mk, k, d, Nk, (uint64_t)B * Hkv, 128, tma_type<T>())) != FA_OK) return st;
    if ((st = make_map(&mv, v, d, Nk, (uint64_t)B * Hkv, 128, tma_type<T>())) != FA_OK) return st;
    const FwdSplit sp = fwd_split_plan(g, B, Hkv, Nq, Nk, d, CAUSAL, sm_count());
    const int kv_split = sp.shares;
    auto kern = kv_split > 1 ? fa::fwd_kernel<D, CAUSAL, T, false, true> : fa::fwd_kernel<D, CAUSAL, T, false, false>;
    if ((st = ensure_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes)) != FA_OK) return st;
    fa::FwdParams p;
    p.o = o;
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.group_rows = g.group_rows;
    p.n_bh = g.n_bh;
    p.rows = g.rows;
    p.n_pairs = g.n_pairs;
    p.d_io = d;
    p.scale_log2 = scale * kLog2e;
    p.o_scale = 1.f;
    p.kv_split = kv_split;
    p.full_tiles = sp.full;
    p.pair_rows = 128 * C::kTiles;
    p.part_o = nullptr;
    p.part_lse = nullptr;
    if ((st = fwd_tile_counter(&p.tile_ctr, &p.tile_tag)) != FA_OK)
        return st;
    return launch_fwd_tiles<T>(kern, C::kThreads, C::kSmemBytes, mq, mk, mv, p, stream);
}

// ---------------------------------------------------------------------------
// forward with e4m3 inputs (d = 128): V^T into the workspace, then the tiled
// kernel on kind::f8f6f4
// ---------------------------------------------------------------------------
constexpr int kF8D = 128;

size_t fp8_nk_pad(int Nk) { return ((size_t)Nk + 15) / 16 * 16; }

size_t fp8_workspace_bytes(int B, int Hkv, int Nk) { return align256((size_t)B * Hkv * kF8D * fp8_nk_pad(Nk)); }

template <bool CAUSAL>
fa_status_t launch_fwd_fp8(const void* q, const void* k, const void* v, void* vt, void* o, float* lse, int B,
                           int Hq, int Hkv, int Nq, int Nk, float scale_log2, float o_scale, cudaStream_t stream)
{
    using C = fa::FwdCfg<kF8D, true>;
    const int nk_pad = (int)fp8_nk_pad(Nk);
    const dim3 tgrid((unsigned)((nk_pad + 63) / 64), (unsigned)(B * Hkv));
    fa::fp8_vt_kernel<kF8D><<<tgrid, 256, 0, stream>>>(static_cast<const uint8_t*>(v), static_cast<uint8_t*>(vt),
                                                      Nk, nk_pad);
    fa_status_t st;
    if ((st = check_launch("fp8_vt_kernel launch")) != FA_OK) return st;
    constexpr CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const FwdGeom g = fwd_geom(B, Hq, Hkv, Nq, kF8D);
    CUtensorMap mq, mk, mv;
    if ((st = make_map_box(&mq, q, kF8D, g.rows, (uint64_t)g.n_bh, 1, 128, 128, u8)) != FA_OK) return st;
    if ((st = make_map_box(&mk, k, kF8D, Nk, (uint64_t)B * Hkv, 1, 128, 128, u8)) != FA_OK) return st;
    // V^T [B * Hkv][d][nk_pad]: box of 128 keys x d rows
    if ((st = make_map_box(&mv, vt, nk_pad, kF8D, (uint64_t)B * Hkv, 1, 128, kF8D, u8)) != FA_OK) return st;
    const FwdSplit sp = fwd_split_plan(g, B, Hkv, Nq, Nk, kF8D, CAUSAL, sm_count());
    const int kv_split = sp.shares;
    auto kern = kv_split > 1 ? fa::fwd_kernel<kF8D, CAUSAL, __nv_bfloat16, true, true>
                             : fa::fwd_kernel<kF8D, CAUSAL, __nv_bfloat16, true, false>;
    if ((st = ensure_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes)) != FA_OK) return st;
    fa::FwdParams p;
    p.o = o;
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.group_rows = g.group_rows;
    p.n_bh = g.n_bh;
    p.rows = g.rows;
    p.n_pairs = g.n_pairs;
    p.d_io = kF8D;
    p.scale_log2 = scale_log2;
    p.o_scale = o_scale;
    p.kv_split = kv_split;
    p.full_tiles = sp.full;
    p.pair_rows = 256;
    p.part_o = nullptr;
    p.part_lse = nullptr;
    if ((st = fwd_tile_counter(&p.tile_ctr, &p.tile_tag)) != FA_OK)
        return st;
    return launch_fwd_tiles<__nv_bfloat16>(kern, C::kThreads, C::kSmemBytes, mq, mk, mv, p, stream, true);
}

template <typename T>
fa_status_t fwd_tiled_t(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Nq, int Nk, int d, float scale, int causal, cudaStream_t s)
{
    if (kernel_d(d) == 256)
        return causal ? launch_fwd<256, true, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s)
                      : launch_fwd<256, false, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s);
    if (kernel_d(d) == 128)
        return causal ? launch_fwd<128, true, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s)
                      : launch_fwd<128, false, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s);
    return causal ? launch_fwd<64, true, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s)
                  : launch_fwd<64, false, T>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, s);
}

fa_status_t fwd_tiled(int dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int causal, cudaStream_t s)
{
    return dtype == FA_DTYPE_FP16 ? fwd_tiled_t<__half>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, s)
                                  : fwd_tiled_t<__nv_bfloat16>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, s);
}

// ---------------------------------------------------------------------------
// split-KV decode
// ---------------------------------------------------------------------------
constexpr int kDecodeMaxRows = 16;
constexpr int kDecodeCtasPerSm = 2;

// The split-KV kernels work at width 128; narrower heads (32, 64, 96) leave the
// rest of the tiles as TMA zero fill and skip it in the MMAs.
constexpr int kDecodeWidth = 128;
bool decode_shape(int Hq, int Hkv, int Nq, int d)
{
    return d <= kDecodeWidth && (long long)Nq * (Hq / Hkv) <= kDecodeMaxRows;
}

// Number of key chunks: the first count whose CTAs fill whole waves of the GPU
// to 95% (at least 256 keys per chunk), else the best fill found.
int decode_splits(int B, int Hkv, int Nk, int requested)
{
    const int max_splits = std::max(1, (Nk + fa::DecCfg::kKeys - 1) / fa::DecCfg::kKeys);
    if (requested > 0)
        return std::min(requested, max_splits);
    const long long units = (long long)B * Hkv;
    const long long slots = (long long)sm_count() * kDecodeCtasPerSm;
    const int cap = std::max(1, std::min(64, Nk / 256));
    int best = 1;
    double best_eff = 0.0;
    for (int s = 1; s <= cap; ++s) {
        const long long ctas = units * s;
        const long long waves = (ctas + slots - 1) / slots;
        const double eff = (double)ctas / (double)(waves * slots);
        if (eff >= 0.95)
            return s;
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = s;
        }
    }
    return best;
}

struct DecodePlan {
    int splits, chunk;
    size_t o_bytes, lse_bytes;
    size_t total() const { return splits > 1 ? align256(o_bytes) + align256(lse_bytes) : 0; }
};

DecodePlan decode_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int requested)
{
    DecodePlan pl;
    int s = decode_splits(B, Hkv, Nk, requested);
    const int kt = fa::DecCfg::kKeys;
    pl.chunk = ((Nk + s - 1) / s + kt - 1) / kt * kt;
    pl.splits = (Nk + pl.chunk - 1) / pl.chunk;
    const size_t R = (size_t)Nq * (Hq / Hkv);
    pl.o_bytes = (size_t)B * Hkv * pl.splits * R * kDecodeWidth * sizeof(float);
    (void)d;
    pl.lse_bytes = (size_t)B * Hkv * pl.splits * R * sizeof(float);
    return pl;
}

struct PagedDesc {
    const int* block_table;
    const int* seq_lens;
    int page_size, num_pages, max_pages;
};

template <typename T>
fa_status_t launch_decode_t(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                            int Hkv, int Nq, int Nk, int d, float scale, int causal, const DecodePlan& pl, void* ws,
                            cudaStream_t stream, const PagedDesc* pg)
{
    using C = fa::DecCfg;
    CUtensorMap mk, mv;
    fa_status_t st;
    if (pg) {
        if ((st = make_map_paged(&mk, k, d, Hkv, pg->page_size, pg->num_pages, tma_type<T>())) != FA_OK) return st;
        if ((st = make_map_paged(&mv, v, d, Hkv, pg->page_size, pg->num_pages, tma_type<T>())) != FA_OK) return st;
    } else {
        if ((st = make_map(&mk, k, d, Nk, (uint64_t)B * Hkv, 64, tma_type<T>())) != FA_OK) return st;
        if ((st = make_map(&mv, v, d, Nk, (uint64_t)B * Hkv, 64, tma_type<T>())) != FA_OK) return st;
    }
    auto kern = d < 128 ? (pg ? fa::decode_split_kernel<true, T, true> : fa::decode_split_kernel<false, T, true>)
                        : (pg ? fa::decode_split_kernel<true, T, false> : fa::decode_split_kernel<false, T, false>);
    if ((st = ensure_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes)) != FA_OK) return st;
    fa::DecodeParams p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.lse = lse;
    p.part_o = pl.splits > 1 ? static_cast<float*>(ws) : nullptr;
    p.part_lse = pl.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + align256(pl.o_bytes)) : nullptr;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.R = Nq * p.G;
    p.splits = pl.splits;
    p.chunk = pl.chunk;
    p.causal = causal;
    p.d_io = d;
    p.scale_log2 = scale * kLog2e;
    p.block_table = pg ? pg->block_table : nullptr;
    p.seq_lens = pg ? pg->seq_lens : nullptr;
    p.page_size = pg ? pg->page_size : 0;
    p.max_pages = pg ? pg->max_pages : 0;
    const long long grid = (long long)B * Hkv * pl.splits;
    kern<<<(unsigned)grid, C::kThreads, C::kSmemBytes, stream>>>(mk, mv, p);
    if ((st = check_launch("decode_split_kernel launch")) != FA_OK) return st;
    if (pl.splits > 1) {
        const long long rows = (long long)B * Hkv * p.R;
        if ((st = launch_dependent("decode_combine_kernel launch", fa::decode_combine_kernel<T>,
                                   dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, stream, p)) != FA_OK)
            return st;
    }
    return FA_OK;
}

fa_status_t launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int Nq, int Nk, int d, float scale, int causal, const DecodePlan& pl, void* ws,
                          cudaStream_t stream, const PagedDesc* pg = nullptr, int dtype = FA_DTYPE_BF16)
{
    if (dtype == FA_DTYPE_FP16)
        return launch_decode_t<__half>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, pl, ws, stream, pg);
    return launch_decode_t<__nv_bfloat16>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, pl, ws, stream, pg);
}

// ---------------------------------------------------------------------------
// split-KV without allocation: partials live in a fixed device array
// ---------------------------------------------------------------------------
// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_splitkv_scratch[FA_SPLITKV_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn get_ctx_current()
{
    static std::once_flag once;
    static CtxGetCurrentFn fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

// Device address of g_splitkv_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up with the
// device current, once per device and context, and cached.  The cache is keyed
// on the current CUDA context as well as the device: after cudaDeviceReset the
// runtime makes a new context, the module (and the array) is loaded again, and
// the address is looked up again instead of reusing the old one.
// Stream-ordered scratch of the calls that allocate their own: a memory pool of the
// library per device (per context: a new one after cudaDeviceReset) that keeps up to
// kScratchKeepBytes between calls.  The device's default pool gives its free memory back
// at every synchronisation, so each call after one would map fresh pages again (about
// 0.2 ms per call measured).  While the stream is being captured into a graph the
// allocation is left to cudaMallocAsync, whose graph memory nodes are the documented path.
constexpr uint64_t kScratchKeepBytes = 1ull << 30;

cudaError_t scratch_alloc(void** out, size_t bytes, cudaStream_t s)
{
    static std::mutex mu;
    static cudaMemPool_t pool_of[64] = {};
    static CUcontext ctx_of[64] = {};
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
        cudaGetLastError();
        cap = cudaStreamCaptureStatusActive;
    }
    int dev = 0;
    CtxGetCurrentFn get_ctx = get_ctx_current();
    CUcontext ctx = nullptr;
    if (cap != cudaStreamCaptureStatusNone || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 ||
        !get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return cudaMallocAsync(out, bytes, s);
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (pool_of[dev] == nullptr || ctx_of[dev] != ctx) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.handleTypes = cudaMemHandleTypeNone;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t p = nullptr;
            if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
                cudaGetLastError();
                return cudaMallocAsync(out, bytes, s);
            }
            uint64_t keep = kScratchKeepBytes;
            cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
            pool_of[dev] = p;
            ctx_of[dev] = ctx;
        }
        pool = pool_of[dev];
    }
    return cudaMallocFromPoolAsync(out, bytes, pool, s);
}

fa_status_t noalloc_scratch(void** out)
{
    static std::mutex mu;
    static void* addr[64] = {};
    static CUcontext ctx_of[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) {
        set_error("device ordinal %d out of range", dev);
        return FA_ERR_UNSUPPORTED;
    }
    CtxGetCurrentFn get_ctx = get_ctx_current();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) {
        set_error("cuCtxGetCurrent is unavailable");
        return FA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (ctx == nullptr || addr[dev] == nullptr || ctx_of[dev] != ctx) {
        // the lookup also sets up the runtime's context on this device if this
        // thread had none yet; the context is read again after it
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_splitkv_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress (split-KV scratch)");
        if (get_ctx(&ctx) != CUDA_SUCCESS) {
            set_error("cuCtxGetCurrent failed");
            return FA_ERR_CUDA;
        }
        addr[dev] = p;
        ctx_of[dev] = ctx;
    }
    *out = addr[dev];
    return FA_OK;
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------
struct BwdPlan {
    int Nq_pad;
    size_t delta_off, lse_off, acc_off, total;   // total: without a query split
    // query split (q_split[causal] CTAs per unit): fp32 dK / dV partials and the two
    // counters per unit, after the accumulator, sized for the larger of the two splits
    int q_split[2], n_units;
    size_t part_off, cnt_off, total_split;
};

// CTAs that share each (key block, kv head[, feature half]) unit's query steps.  A unit of
// key block kb has G * (visible 64-row query blocks) steps; a CTA costs its steps plus a
// fixed part (set-up, pipeline fill, dK / dV epilogue: about 8.5 step times) and, when
// split, about 0.8 step times per fp32 partial it stores or adds.  Without a causal mask
// all units are alike and the launch takes ceil(CTAs / SMs) rounds of one CTA; with it
// the estimate is the larger of the total work over the SMs and the longest CTA.  The
// split of least estimated time is taken if it saves at least 3% (each CTA keeps at
// least 16 steps): it fills the SMs when there are few units, and evens out a last
// round that would leave most of them idle.
int bwd_q_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, int sms)
{
    const int kd = kernel_d(d);
    const int n_kb = (Nk + 127) / 128;
    const double per_kb = (double)B * Hkv * (kd == 256 ? 2 : 1);
    const int G = Hq / Hkv, nqb_all = (Nq + 63) / 64;
    double total = 0, longest = 0;
    for (int kb = 0; kb < n_kb; ++kb) {
        int qb0 = 0;
        if (causal) {
            const int first_row = kb * 128 - (Nk - Nq);
            qb0 = first_row <= 0 ? 0 : first_row / 64;
        }
        const double steps = (double)G * std::max(0, nqb_all - qb0);
        total += steps * per_kb;
        longest = std::max(longest, steps);
    }
    static const int kSplits[] = {1, 2, 3, 4, 6, 8};
    int best = 1;
    double best_cost = 0;
    for (int s : kSplits) {
        if (s > 1 && longest < 16.0 * s)
            break;
        const double fixed = 8.5 + (s > 1 ? 0.8 * (s - 1) : 0.0);
        const double ctas = n_kb * per_kb * s;
        const double cost = causal ? std::max((total + ctas * fixed) / sms, longest / s + fixed)
                                   : std::ceil(ctas / sms) * (longest / s + fixed);
        if (s == 1 || cost < 0.97 * best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    return best;
}

BwdPlan bwd_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d)
{
    BwdPlan pl;
    pl.Nq_pad = (Nq + 63) / 64 * 64;
    const size_t rows = (size_t)B * Hq * pl.Nq_pad;
    pl.delta_off = 0;
    pl.lse_off = align256(rows * 4);
    pl.acc_off = pl.lse_off + align256(rows * 4);
    pl.total = pl.acc_off + align256(rows * kernel_d(d) * 4);   // accumulator rows of the kernel width
    const int kd = kernel_d(d);
    pl.n_units = ((Nk + 127) / 128) * B * Hkv * (kd == 256 ? 2 : 1);
    const int sms = sm_count();
    pl.q_split[0] = bwd_q_split(B, Hq, Hkv, Nq, Nk, d, 0, sms);
    pl.q_split[1] = bwd_q_split(B, Hq, Hkv, Nq, Nk, d, 1, sms);
    const int most = std::max(pl.q_split[0], pl.q_split[1]);
    // partial slots per unit: one for two shares, one per share for more
    const int slots = most == 1 ? 0 : most == 2 ? 1 : most;
    const size_t part_bytes = (size_t)pl.n_units * slots * 2 * std::min(kd, 128) * 128 * 4;
    pl.part_off = pl.total;
    pl.cnt_off = pl.part_off + align256(part_bytes);
    pl.total_split = most > 1 ? pl.cnt_off + align256((size_t)pl.n_units * 2 * 4) : pl.total;
    return pl;
}

template <int D, bool CAUSAL, typename T>
fa_status_t launch_bwd(const fa::BwdParams& p, const void* q, const void* k, const void* v, const void* dout,
                       cudaStream_t stream)
{
    using C = fa::BwdCfg<D>;
    fa_status_t st;
    const long long rows = (long long)p.B * p.Hq * p.Nq_pad;
    fa::bwd_pre_kernel<D, T><<<(unsigned)((rows + 15) / 16), 256, 0, stream>>>(p);
    if ((st = check_launch("bwd_pre_kernel launch")) != FA_OK) return st;

    CUtensorMap mq, mk, mv, mdo;
    constexpr CUtensorMapDataType dt = tma_type<T>();
    if ((st = make_map(&mq, q, p.d_io, p.Nq, (uint64_t)p.B * p.Hq, 64, dt)) != FA_OK) return st;
    if ((st = make_map(&mdo, dout, p.d_io, p.Nq, (uint64_t)p.B * p.Hq, 64, dt)) != FA_OK) return st;
    if ((st = make_map(&mk, k, p.d_io, p.Nk, (uint64_t)p.B * p.Hkv, 128, dt)) != FA_OK) return st;
    if ((st = make_map(&mv, v, p.d_io, p.Nk, (uint64_t)p.B * p.Hkv, 128, dt)) != FA_OK) return st;
    auto kern = p.q_split > 1 ? fa::bwd_main_kernel<D, CAUSAL, T, true> : fa::bwd_main_kernel<D, CAUSAL, T, false>;
    if ((st = ensure_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes)) != FA_OK) return st;
    const long long grid = (long long)((p.Nk + 127) / 128) * p.B * p.Hkv * C::kFeatSplit * p.q_split;
    if ((st = launch_dependent("bwd_main_kernel launch", kern, dim3((unsigned)grid), dim3(C::kThreads),
                               C::kSmemBytes, stream, mq, mk, mv, mdo, p)) != FA_OK)
        return st;

    // 16 rows per block; the y dimension walks batch * head (looping past 65535)
    const dim3 pgrid((unsigned)std::max(1, std::min((p.Nq + 15) / 16, 4096)),
                     (unsigned)std::max<long long>(1, std::min<long long>((long long)p.B * p.Hq, 65535)));
    return launch_dependent("bwd_post_kernel launch", fa::bwd_post_kernel<D, T>, pgrid, dim3(256), 0, stream, p);
}

template <typename T>
fa_status_t bwd_dispatch(const fa::BwdParams& p, const void* q, const void* k, const void* v, const void* dout,
                         int kd, int causal, cudaStream_t s)
{
    if (kd == 256)
        return causal ? launch_bwd<256, true, T>(p, q, k, v, dout, s) : launch_bwd<256, false, T>(p, q, k, v, dout, s);
    if (kd == 128)
        return causal ? launch_bwd<128, true, T>(p, q, k, v, dout, s) : launch_bwd<128, false, T>(p, q, k, v, dout, s);
    return causal ? launch_bwd<64, true, T>(p, q, k, v, dout, s) : launch_bwd<64, false, T>(p, q, k, v, dout, s);
}

// ---------------------------------------------------------------------------
// timeout self-test
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(long long limit_cycles)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        fa::mbar_init(&bar, 1);
        fa::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing arrives on this barrier: the wait must run out and report it
        if (!fa::mbar_wait_limited(&bar, 0, limit_cycles))
            atomicOr(&fa::g_status, fa::kStatusTimeout);
    }
}

}  // namespace

// ===========================================================================
// exported entry points
// ===========================================================================
extern "C" {

int fa_abi_version(void) { return kAbiVersion; }

const char* fa_status_string(fa_status_t s)
{
    switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARGUMENT: return "FA_ERR_INVALID_ARGUMENT";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_SLOT_CONFLICT: return "FA_ERR_SLOT_CONFLICT";
    }
    return "FA_ERR_UNKNOWN";
}

const char* fa_last_error_message(void) { return t_error.c_str(); }

static fa_status_t fwd_entry(int dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                             int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream)
{
    t_error.clear();
    fa_status_t st;
    if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16) {
        set_error("dtype=%d is not FA_DTYPE_BF16 or FA_DTYPE_FP16", dtype);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
        (st = check_ptr(o, "o")))
        return st;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
        set_error("lse is not 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal)) != FA_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!decode_shape(Hq, Hkv, Nq, d))
        return fwd_tiled(dtype, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, s);
    const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, d, 0);
    void* ws = nullptr;
    if (pl.total() > 0) {
        cudaError_t e = scratch_alloc(&ws, pl.total(), s);
        if (e != cudaSuccess)
            return cuda_fail(e, "scratch allocation (split-KV partials)");
    }
    st = launch_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, pl, ws, s, nullptr, dtype);
    if (ws) {
        cudaError_t e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int Nq, int Nk, int d, float scale, int causal, void* stream)
{
    return fwd_entry(FA_DTYPE_BF16, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

fa_status_t fa_fwd_ex(fa_dtype_t dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream)
{
    return fwd_entry((int)dtype, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

size_t fa_fwd_fp8_workspace_size(int B, int Hkv, int Nk, int d)
{
    if (B < 1 || Hkv < 1 || Nk < 1 || d != kF8D)
        return 0;
    return fp8_workspace_bytes(B, Hkv, Nk);
}

fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k,
                       float descale_v, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       float scale, int causal, void* workspace, size_t workspace_bytes, void* stream)
{
    t_error.clear();
    fa_status_t st;
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
        (st = check_ptr(o, "o")))
        return st;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
        set_error("lse is not 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    const float ds[3] = {descale_q, descale_k, descale_v};
    for (float x : ds)
        if (!(std::isfinite(x) && x > 0.f)) {
            set_error("descale factors must be finite and > 0");
            return FA_ERR_INVALID_ARGUMENT;
        }
    if ((st = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal)) != FA_OK)
        return st;
    if (d != kF8D) {
        set_error("the e4m3 forward takes d = 128 (got %d)", d);
        return FA_ERR_UNSUPPORTED;
    }
    if ((long long)B * Hkv > 65535) {   // grid.y of the V transpose
        set_error("the e4m3 forward takes B * Hkv <= 65535");
        return FA_ERR_UNSUPPORTED;
    }
    const float scale_log2 = scale * descale_q * descale_k * kLog2e;
    if (!(std::isfinite(scale_log2) && scale_log2 > 0.f)) {
        set_error("scale * descale_q * descale_k is not a positive finite fp32 value");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
        set_error("workspace is not 256-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    const size_t need = fp8_workspace_bytes(B, Hkv, Nk);
    if (workspace && workspace_bytes < need) {
        set_error("workspace has %zu bytes, %zu needed", workspace_bytes, need);
        return FA_ERR_WORKSPACE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* ws = workspace;
    if (!ws) {
        cudaError_t e = scratch_alloc(&ws, need, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "scratch allocation (V^T workspace)");
    }
    st = causal ? launch_fwd_fp8<true>(q, k, v, ws, o, lse, B, Hq, Hkv, Nq, Nk, scale_log2, descale_v, s)
                : launch_fwd_fp8<false>(q, k, v, ws, o, lse, B, Hq, Hkv, Nq, Nk, scale_log2, descale_v, s);
    if (!workspace) {
        cudaError_t e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

size_t fa_fwd_splitkv_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || d < 1 || num_splits < 0)
        return 0;
    return decode_plan(B, Hq, Hkv, Nq, Nk, d, num_splits).total();
}

fa_status_t fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                           int Hkv, int Nq, int Nk, int d, float scale, int causal, int num_splits,
                           void* workspace, size_t workspace_bytes, void* stream)
{
    t_error.clear();
    fa_status_t st;
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
        (st = check_ptr(o, "o")))
        return st;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
        set_error("lse is not 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal)) != FA_OK)
        return st;
    if (num_splits < 0 || num_splits > 256) {
        set_error("num_splits=%d must be in [0, 256]", num_splits);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (!decode_shape(Hq, Hkv, Nq, d)) {
        set_error("split-KV needs d <= 128 and Nq * Hq / Hkv <= %d", kDecodeMaxRows);
        return FA_ERR_UNSUPPORTED;
    }
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
        set_error("workspace is not 256-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, d, num_splits);
    void* ws = workspace;
    bool owned = false;
    if (pl.total() > 0) {
        if (ws == nullptr) {
            cudaError_t e = scratch_alloc(&ws, pl.total(), s);
            if (e != cudaSuccess)
                return cuda_fail(e, "scratch allocation (split-KV partials)");
            owned = true;
        } else if (workspace_bytes < pl.total()) {
            set_error("workspace has %zu bytes, %zu needed", workspace_bytes, pl.total());
            return FA_ERR_WORKSPACE;
        }
    }
    st = launch_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, pl, ws, s);
    if (owned) {
        cudaError_t e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

fa_status_t fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                   int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                                   int num_splits, void* stream)
{
    t_error.clear();
    fa_status_t st;
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
        (st = check_ptr(o, "o")))
        return st;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
        set_error("lse is not 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal)) != FA_OK)
        return st;
    if (num_splits < 0 || num_splits > 256) {
        set_error("num_splits=%d must be in [0, 256]", num_splits);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (!decode_shape(Hq, Hkv, Nq, d)) {
        set_error("split-KV needs d <= 128 and Nq * Hq / Hkv <= %d", kDecodeMaxRows);
        return FA_ERR_UNSUPPORTED;
    }
    DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, d, num_splits);
    // an automatic split count is lowered until the partials fit (one split
    // needs no scratch at all); an explicit count that does not fit is refused
    while (num_splits == 0 && pl.splits > 1 && pl.total() > (size_t)FA_SPLITKV_NOALLOC_SCRATCH_BYTES)
        pl = decode_plan(B, Hq, Hkv, Nq, Nk, d, pl.splits - 1);
    if (pl.total() > (size_t)FA_SPLITKV_NOALLOC_SCRATCH_BYTES) {
        set_error("this shape needs %zu bytes of split-KV scratch but the fixed scratch holds %zu; "
                  "use fewer splits or fa_fwd_splitkv with a caller workspace",
                  pl.total(), (size_t)FA_SPLITKV_NOALLOC_SCRATCH_BYTES);
        return FA_ERR_WORKSPACE;
    }
    void* ws = nullptr;
    if (pl.total() > 0 && (st = noalloc_scratch(&ws)) != FA_OK)
        return st;
    // every partial the combine reads is written by the split pass of this same
    // call, so nothing in the scratch has to be cleared first
    return launch_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, pl, ws,
                         static_cast<cudaStream_t>(stream));
}

size_t fa_fwd_paged_workspace_size(int B, int Hq, int Hkv, int Nq, int page_size, int max_pages_per_seq, int d,
                                   int num_splits)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Hq % Hkv != 0 || d < 1 || num_splits < 0 || page_size < 1 ||
        max_pages_per_seq < 1 || (long long)page_size * max_pages_per_seq > (1ll << 30))
        return 0;
    return decode_plan(B, Hq, Hkv, Nq, page_size * max_pages_per_seq, d, num_splits).total();
}

static fa_status_t paged_entry(int dtype, const void* q, const void* k_cache, const void* v_cache,
                               const int* block_table, const int* seq_lens, void* o, float* lse, int B, int Hq,
                               int Hkv, int Nq, int d, int page_size, int num_pages, int max_pages_per_seq,
                               float scale, int causal, int num_splits, void* workspace, size_t workspace_bytes,
                               void* stream)
{
    t_error.clear();
    fa_status_t st;
    if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16) {
        set_error("dtype=%d is not FA_DTYPE_BF16 or FA_DTYPE_FP16", dtype);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k_cache, "k_cache")) || (st = check_ptr(v_cache, "v_cache")) ||
        (st = check_ptr(o, "o")))
        return st;
    if (!block_table || !seq_lens || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u)) {
        set_error("block_table and seq_lens must be non-NULL and 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
        set_error("lse is not 4-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (page_size < 64 || page_size % 64 != 0 || num_pages < 1 || max_pages_per_seq < 1 ||
        (long long)page_size * max_pages_per_seq > (1ll << 30) || (long long)num_pages * page_size > (1ll << 31)) {
        set_error("page_size must be a positive multiple of 64; num_pages, max_pages_per_seq >= 1");
        return FA_ERR_INVALID_ARGUMENT;
    }
    const int max_len = page_size * max_pages_per_seq;
    if ((st = check_shape(B, Hq, Hkv, Nq, max_len, d, scale, causal)) != FA_OK)
        return st;
    if (num_splits < 0 || num_splits > 256) {
        set_error("num_splits=%d must be in [0, 256]", num_splits);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (!decode_shape(Hq, Hkv, Nq, d)) {
        set_error("paged decode needs d <= 128 and Nq * Hq / Hkv <= %d", kDecodeMaxRows);
        return FA_ERR_UNSUPPORTED;
    }
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
        set_error("workspace is not 256-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, max_len, d, num_splits);
    void* ws = workspace;
    bool owned = false;
    if (pl.total() > 0) {
        if (ws == nullptr) {
            cudaError_t e = scratch_alloc(&ws, pl.total(), s);
            if (e != cudaSuccess)
                return cuda_fail(e, "scratch allocation (paged split-KV partials)");
            owned = true;
        } else if (workspace_bytes < pl.total()) {
            set_error("workspace has %zu bytes, %zu needed", workspace_bytes, pl.total());
            return FA_ERR_WORKSPACE;
        }
    }
    PagedDesc pg{block_table, seq_lens, page_size, num_pages, max_pages_per_seq};
    st = launch_decode(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nq, max_len, d, scale, causal, pl, ws, s, &pg,
                       dtype);
    if (owned) {
        cudaError_t e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

fa_status_t fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                         const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                         int page_size, int num_pages, int max_pages_per_seq, float scale, int causal,
                         int num_splits, void* workspace, size_t workspace_bytes, void* stream)
{
    return paged_entry(FA_DTYPE_BF16, q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, Nq, d,
                       page_size, num_pages, max_pages_per_seq, scale, causal, num_splits, workspace,
                       workspace_bytes, stream);
}

fa_status_t fa_fwd_paged_ex(fa_dtype_t dtype, const void* q, const void* k_cache, const void* v_cache,
                            const int* block_table, const int* seq_lens, void* o, float* lse, int B, int Hq,
                            int Hkv, int Nq, int d, int page_size, int num_pages, int max_pages_per_seq,
                            float scale, int causal, int num_splits, void* workspace, size_t workspace_bytes,
                            void* stream)
{
    return paged_entry((int)dtype, q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, Nq, d,
                       page_size, num_pages, max_pages_per_seq, scale, causal, num_splits, workspace,
                       workspace_bytes, stream);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || d < 1 || d > 256)
        return 0;
    return bwd_plan(B, Hq, Hkv, Nq, Nk, d).total_split;
}

int fa_fwd_kv_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || d < 1 || d > 256 || d % 32 != 0 ||
        (causal != 0 && causal != 1))
        return 0;
    if (decode_shape(Hq, Hkv, Nq, d))
        return 1;
    return fwd_split_plan(fwd_geom(B, Hq, Hkv, Nq, d), B, Hkv, Nq, Nk, d, causal, sm_count()).shares;
}

int fa_bwd_query_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || d < 1 || d > 256 ||
        (causal != 0 && causal != 1))
        return 0;
    return bwd_plan(B, Hq, Hkv, Nq, Nk, d).q_split[causal];
}

static fa_status_t bwd_entry(int dtype, const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                             int Nq, int Nk, int d, float scale, int causal, void* workspace,
                             size_t workspace_bytes, void* stream)
{
    t_error.clear();
    fa_status_t st;
    if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16) {
        set_error("dtype=%d is not FA_DTYPE_BF16 or FA_DTYPE_FP16", dtype);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
        (st = check_ptr(o, "o")) || (st = check_ptr(dout, "dout")) || (st = check_ptr(lse, "lse")) ||
        (st = check_ptr(dq, "dq")) || (st = check_ptr(dk, "dk")) || (st = check_ptr(dv, "dv")))
        return st;
    if ((st = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal)) != FA_OK)
        return st;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
        set_error("workspace is not 256-byte aligned");
        return FA_ERR_INVALID_ARGUMENT;
    }
    const BwdPlan pl = bwd_plan(B, Hq, Hkv, Nq, Nk, d);
    if (workspace && workspace_bytes < pl.total) {
        set_error("workspace has %zu bytes, %zu needed", workspace_bytes, pl.total);
        return FA_ERR_WORKSPACE;
    }
    // the query split needs the partials' room too: a smaller workspace runs without it
    const int q_split = (!workspace || workspace_bytes >= pl.total_split) ? pl.q_split[causal ? 1 : 0] : 1;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* ws = workspace;
    bool owned = false;
    if (!ws) {
        cudaError_t e = scratch_alloc(&ws, q_split > 1 ? pl.total_split : pl.total, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "scratch allocation (backward workspace)");
        owned = true;
    }
    fa::BwdParams p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    char* w = static_cast<char*>(ws);
    p.neg_delta = reinterpret_cast<float*>(w + pl.delta_off);
    p.neg_lse_log2 = reinterpret_cast<float*>(w + pl.lse_off);
    p.dq_acc = reinterpret_cast<float*>(w + pl.acc_off);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.Nq_pad = pl.Nq_pad;
    p.d_io = d;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    p.q_split = q_split;
    p.n_split_units = pl.n_units;
    p.dkv_part = q_split > 1 ? reinterpret_cast<float4*>(w + pl.part_off) : nullptr;
    p.split_cnt = q_split > 1 ? reinterpret_cast<int*>(w + pl.cnt_off) : nullptr;
    st = dtype == FA_DTYPE_FP16 ? bwd_dispatch<__half>(p, q, k, v, dout, kernel_d(d), causal, s)
                                : bwd_dispatch<__nv_bfloat16>(p, q, k, v, dout, kernel_d(d), causal, s);
    if (owned) {
        cudaError_t e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == FA_OK)
            st = cuda_fail(e, "cudaFreeAsync");
    }
    return st;
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                   int causal, void* workspace, size_t workspace_bytes, void* stream)
{
    return bwd_entry(FA_DTYPE_BF16, q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                     workspace, workspace_bytes, stream);
}

fa_status_t fa_bwd_ex(fa_dtype_t dtype, const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                      int Nq, int Nk, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                      void* stream)
{
    return bwd_entry((int)dtype, q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                     workspace, workspace_bytes, stream);
}

fa_status_t fa_check_device_status(void* stream)
{
    t_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int h = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&h, fa::g_status, sizeof h, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(fa::g_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e, "reading the device status word");
    if (h & fa::kStatusSlotShared) {
        // A slot may have been left marked by the launch that lost it: once every
        // launch on the device has finished, all slots are cleared.
        void* base = nullptr;
        e = cudaDeviceSynchronize();
        if (e == cudaSuccess)
            e = cudaGetSymbolAddress(&base, fa::g_fwd_tile_ctr);
        if (e == cudaSuccess)
            e = cudaMemset(base, 0, sizeof(fa::g_fwd_tile_ctr));
        if (e == cudaSuccess)
            e = cudaDeviceSynchronize();
        if (e != cudaSuccess)
            return cuda_fail(e, "clearing the forward tile-counter slots");
        set_error("a tiled forward launch found its tile-counter slot held by another launch in flight "
                  "(more than 256 tiled forwards at once); its output is incomplete");
        return FA_ERR_SLOT_CONFLICT;
    }
    if (h & fa::kStatusTimeout) {
        set_error("a bounded device wait ran out");
        return FA_ERR_TIMEOUT;
    }
    return FA_OK;
}

fa_status_t fa_testhook_tile_slot(int slot, unsigned preset_owner)
{
    t_error.clear();
    if (slot < -1 || slot >= fa::kFwdCtrSlots) {
        set_error("slot=%d must be -1 or in [0, %d)", slot, fa::kFwdCtrSlots);
        return FA_ERR_INVALID_ARGUMENT;
    }
    if (slot >= 0 && preset_owner != 0u) {
        void* base = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&base, fa::g_fwd_tile_ctr);
        if (e == cudaSuccess)
            e = cudaMemcpy(static_cast<unsigned*>(base) + fa::kFwdCtrWords * slot + 2, &preset_owner,
                           sizeof preset_owner, cudaMemcpyHostToDevice);
        if (e != cudaSuccess)
            return cuda_fail(e, "presetting a tile-counter slot owner");
    }
    g_pinned_slot.store(slot, std::memory_order_relaxed);
    return FA_OK;
}

fa_status_t fa_selftest_wait_timeout(unsigned timeout_us, void* stream)
{
    t_error.clear();
    int dev = 0, khz = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "querying the clock rate");
    const long long cycles = (long long)timeout_us * (long long)(khz > 0 ? khz : 2000000) / 1000;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    selftest_wait_kernel<<<1, 32, 0, s>>>(cycles);
    fa_status_t st = check_launch("selftest_wait_kernel launch");
    if (st != FA_OK)
        return st;
    return fa_check_device_status(stream);
}

}  // extern "C"
