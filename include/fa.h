/*
 * fa.h -- C ABI of libfa, exact scaled-dot-product attention for NVIDIA B200
 * (sm_100a).
 *
 * The operation (page "FlashAttention：为什么少搬数据，反而算得更快", §02, the
 * S = QK^T / P = softmax(S) / O = PV table, with scale and causal mask present):
 *
 *     O = softmax(scale * Q K^T + mask) V,   LSE_i = ln sum_j exp(scale q_i . k_j)
 *
 * computed tile by tile with the running statistics (m, l, U) of §04 so that S
 * and P never reach device memory, and the backward of §05, which recomputes P
 * block by block from the saved LSE.  MHA, MQA and GQA are selected by Hq / Hkv
 * (page "FlashAttention技术原理详解"): query head h reads key/value head
 * h / (Hq / Hkv).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are dense, row-major, "BHSD": q, o, dout, dq are [B, Hq, Nq, d];
 *    k, v, dk, dv are [B, Hkv, Nk, d]; lse is [B, Hq, Nq].  q/k/v/o/dout/dq/dk/dv
 *    hold bf16 (fp16 through the *_ex calls), lse holds fp32 (natural log of
 *    the scaled scores).
 *  - Every tensor pointer is a DEVICE pointer, non-NULL and 16-byte aligned.
 *  - d is a multiple of 32 up to 256 (page "AI infra 一层全看懂(五) Flash
 *    Attention", §五, gives 64 to 128 as the usual head dimension; other sizes
 *    run on the 64, 128 or 256 kernels with the missing columns zero-filled on
 *    chip; d > 128 uses one 128-row query tile per CTA in the forward and two
 *    CTAs per key block, one per half of the features, in the backward).  The
 *    split-KV and paged calls take d up to 128, the e4m3 call d = 128 only.
 *    Hq must be a multiple of Hkv.
 *    B, Hq, Hkv, Nq, Nk >= 1.
 *  - causal is 0 or 1.  With causal = 1, key j is visible to query i iff
 *    j <= i + (Nk - Nq) (the mask is aligned to the bottom-right corner; for
 *    Nq = Nk this is the usual lower triangle).  A query row that sees no key
 *    gets O = 0, LSE = -inf and zero gradients.
 *  - stream is a cudaStream_t (NULL = the legacy default stream).  All work is
 *    enqueued on it; no call synchronises the stream or the device.  A call's
 *    first kernel is a plain launch: it starts after all earlier work on the
 *    stream.  Its later kernels (the backward's main and post passes, the merge of
 *    split partials, the e4m3 forward after its V transpose) are programmatic
 *    dependent launches.  They may start their
 *    set-up while the kernel before them finishes, but they read nothing that
 *    kernel writes until it has completed.  Later work on the stream starts after
 *    the whole call, as usual.
 *  - Ownership: the caller owns every buffer; the library keeps no pointer
 *    after a call returns and frees nothing it did not allocate.
 *  - Scratch: a call that allocates its own scratch (workspace NULL, or the
 *    split-KV / key-split partials of fa_fwd) takes it stream-ordered from a
 *    memory pool of the library (one per device and context) and frees it
 *    stream-ordered on the same stream.  The pool keeps up to 1 GiB of freed
 *    memory for later calls (the device's default pool returns its memory at
 *    every synchronisation, and mapping it again cost about 0.2 ms per call);
 *    during stream capture the allocation uses cudaMallocAsync instead.
 *  - Errors: arguments are checked before anything is enqueued; a bad argument
 *    returns FA_ERR_INVALID_ARGUMENT or FA_ERR_UNSUPPORTED with nothing launched.
 *    A CUDA launch or allocation failure returns FA_ERR_CUDA;
 *    fa_last_error_message() describes the last failure of the calling thread.
 *  - Every wait inside a kernel is bounded.  A wait that runs out records
 *    FA_ERR_TIMEOUT in a per-device status word and the kernel returns early;
 *    fa_check_device_status() reads and clears it.
 *  - Results are equal to the definition up to floating-point ordering, not
 *    bit for bit (§04 calls the tiled result equivalent, not identical).  Every
 *    output is bitwise repeatable from run to run except dq, which is added up
 *    across key blocks by reductions in L2 whose order varies.
 */
#ifndef LIBFA_FA_H
#define LIBFA_FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARGUMENT = 1, /* NULL / misaligned pointer, bad size or flag */
    FA_ERR_UNSUPPORTED = 2,      /* valid but not implemented (e.g. d = 80) */
    FA_ERR_WORKSPACE = 3,        /* workspace given but smaller than required */
    FA_ERR_CUDA = 4,             /* a CUDA runtime / driver call failed */
    FA_ERR_TIMEOUT = 5,          /* a bounded device wait ran out */
    FA_ERR_SLOT_CONFLICT = 6     /* a tiled forward found its tile-counter slot in use (see fa_fwd) */
} fa_status_t;

/* Element type of the 16-bit tensors (q, k, v, o, dout, dq, dk, dv). */
typedef enum {
    FA_DTYPE_BF16 = 0,
    FA_DTYPE_FP16 = 1
} fa_dtype_t;

/* Version of this ABI (incremented on any signature change). */
int fa_abi_version(void);

/* Static string for a status code. */
const char* fa_status_string(fa_status_t status);

/* Text of the last failure on the calling thread ("" if none). */
const char* fa_last_error_message(void);

/*
 * Forward pass (§03 tiling, §04 online softmax).
 *   q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] (bf16, read only)
 *   o [B,Hq,Nq,d] bf16 (written), lse [B,Hq,Nq] fp32 (written; may be NULL when
 *   the caller does not need it).
 *   scale multiplies q.k (usually 1/sqrt(d)); it must be finite and > 0.
 * Shapes with few query rows per kv head (Nq * Hq / Hkv <= 16, the decode shape
 * of §09) and d <= 128 run the split-KV kernels; their partial results need scratch, which
 * this call allocates and frees stream-ordered on `stream` (see Scratch
 * above).  Use fa_fwd_splitkv() to pass the scratch instead.
 * Other shapes run one persistent block per SM over work tiles of 256 query
 * rows (128 at d > 128).  Where a kv head serves several query heads and each
 * has fewer rows than a tile, the G * Nq rows of the kv head's query heads
 * share its tiles (row r at query position r % Nq), so K/V are read once per
 * kv head.  Where the work tiles would leave SMs idle (fewer tiles than SMs,
 * or a last round that fills few of them), the key blocks of every tile, or
 * of the tiles after the last full round, are cut into fa_fwd_kv_split(...)
 * contiguous shares that run as separate tiles; their partial results (fp32 O
 * and LSE per share, in scratch this call allocates and frees stream-ordered
 * on `stream`) are merged by a second kernel as the online softmax merges
 * blocks (§04).  The blocks share a tile
 * counter, one of 256 slots in the library's device memory that launches take
 * in turn; the launch's last block resets it.  So at most 256 tiled forward
 * launches (this call, fa_fwd_ex, fa_fwd_fp8) may be in flight on one device
 * at once.  Each launch marks its slot with a tag of its own; a launch whose
 * blocks find the slot held by another launch takes no tile from it, leaves
 * its own output incomplete and records FA_ERR_SLOT_CONFLICT in the device
 * status word, which the next fa_check_device_status() reports (so an overrun
 * is reported, never a silently wrong O).  A launch captured in a CUDA graph
 * keeps its slot and tag on every replay.
 */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   void* stream);

/*
 * fa_fwd for either 16-bit element type: q, k, v, o hold `dtype` elements
 * (FA_DTYPE_BF16 is exactly fa_fwd).  Everything else as fa_fwd; an unknown
 * dtype returns FA_ERR_INVALID_ARGUMENT.
 */
fa_status_t fa_fwd_ex(fa_dtype_t dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                      void* stream);

/*
 * Forward with e4m3 (FP8) inputs.  The pages list an FP8 path as the lower-
 * precision trade-off of the Hopper-generation kernel that needs its error
 * kept under control (page "FlashAttention：为什么少搬数据，反而算得更快",
 * §07); they give no recipe, so this call takes the plainest one:
 *   q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d]: one e4m3 byte per element (OCP FP8
 *   E4M3: bias 7, no infinities), dense BHSD, read only.  The values are
 *   code * descale_{q,k,v} (one fp32 scale per tensor, finite and > 0).
 *   S = scale * (Q K^T) accumulates exactly in fp32; P = exp(S - m) is rounded
 *   to e4m3 for the P.V product (fp32 accumulation); the row sum l uses the
 *   fp32 P.  o [B,Hq,Nq,d] is bf16 (written); lse [B,Hq,Nq] fp32 (or NULL).
 *   d must be 128 (else FA_ERR_UNSUPPORTED).  Masking and shapes as fa_fwd,
 *   always on the tiled kernel (decode shapes too), with fa_fwd's group rows
 *   and key split (whose partials are fp32 scratch allocated and freed
 *   stream-ordered, outside `workspace`).
 *   workspace: device scratch of fa_fwd_fp8_workspace_size(B, Hkv, Nk, d)
 *   bytes, 256-byte aligned, for V transposed to [B,Hkv,d,Nk rounded up to
 *   16]; NULL makes the call allocate it stream-ordered.  A smaller one returns
 *   FA_ERR_WORKSPACE with nothing launched.
 * Error bound against exact attention of the dequantised inputs: |O - O_ref|
 * <= sum_j err(p_ij) |v_j| / l_i per element, err(p) = max(p / 16, 2^-10) (the
 * e4m3 rounding of P), plus fp32 and bf16 output rounding.
 */
size_t fa_fwd_fp8_workspace_size(int B, int Hkv, int Nk, int d);

fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k,
                       float descale_v, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk,
                       int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * Split-KV forward for the decode shape (§09: a single query position, scores
 * of shape 1 x history).  The keys of every (batch, kv head) are cut into
 * num_splits contiguous chunks; each chunk yields a partial (O_s, lse_s) for all
 * Hq / Hkv query heads of the group, and a combine kernel merges them with the
 * rescale-and-add rule of §04 in log form:
 *     lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 *   Requires Nq * (Hq / Hkv) <= 16 and d <= 128.
 *   num_splits: 0 picks a value from the shape; otherwise 1..256.
 *   workspace: device scratch of at least fa_fwd_splitkv_workspace_size(...)
 *   bytes, 256-byte aligned; NULL makes the call allocate it stream-ordered.
 */
size_t fa_fwd_splitkv_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                     int num_splits);
fa_status_t fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                           int causal, int num_splits, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * Decode over a paged KV cache (§09: paged KV management is independent of the
 * attention computation -- it only decides where K and V are stored).
 *   k_cache, v_cache: [num_pages, page_size, Hkv, d] bf16 (fp16 through
 *     fa_fwd_paged_ex), one pool shared by
 *     all sequences (heads innermost).
 *   block_table: int32 [B, max_pages_per_seq] (device); logical page n of
 *     sequence b is physical page block_table[b * max_pages_per_seq + n].
 *   seq_lens: int32 [B] (device); sequence b has seq_lens[b] keys, at most
 *     page_size * max_pages_per_seq (values are clamped to that range; a page id
 *     outside [0, num_pages) reads zeros).
 *   q, o: [B, Hq, Nq, d] bf16; lse [B, Hq, Nq] fp32 or NULL.  With causal = 1 the
 *     Nq query rows of sequence b are its last Nq positions (bottom-right mask
 *     against seq_lens[b]).
 *   page_size: a multiple of 64.  d <= 128, Nq * Hq / Hkv <= 16.
 *   num_splits / workspace as for fa_fwd_splitkv, sized with
 *   fa_fwd_paged_workspace_size().
 */
size_t fa_fwd_paged_workspace_size(int B, int Hq, int Hkv, int Nq, int page_size, int max_pages_per_seq,
                                   int d, int num_splits);
fa_status_t fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                         const int* block_table, const int* seq_lens, void* o, float* lse,
                         int B, int Hq, int Hkv, int Nq, int d, int page_size, int num_pages,
                         int max_pages_per_seq, float scale, int causal, int num_splits,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_fwd_paged for either 16-bit element type: q, o, k_cache and v_cache hold
 * `dtype` elements (FA_DTYPE_BF16 is exactly fa_fwd_paged).  An unknown dtype
 * returns FA_ERR_INVALID_ARGUMENT.
 */
fa_status_t fa_fwd_paged_ex(fa_dtype_t dtype, const void* q, const void* k_cache, const void* v_cache,
                            const int* block_table, const int* seq_lens, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int d, int page_size, int num_pages,
                            int max_pages_per_seq, float scale, int causal, int num_splits,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Split-KV forward that allocates nothing (the paper has no counterpart; this
 * is a deployment variant of fa_fwd_splitkv).
 *
 * For callers that may not allocate device memory on their call path -- for
 * example an inference runtime's plugin whose enqueue step must not allocate,
 * a host program whose allocator owns the whole device memory budget, or a
 * latency-critical loop where growing a stream-ordered pool would stall.
 * Arguments, shapes and results are those of fa_fwd_splitkv; only the
 * workspace argument is gone.  The per-split partials go to one fixed device
 * array of FA_SPLITKV_NOALLOC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library holds until the process exits.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 *   - With num_splits = 0 the split count is chosen as for fa_fwd_splitkv and
 *     then lowered until the partials fit the array (a single split needs no
 *     scratch), so the automatic choice never fails for lack of scratch.  An
 *     explicit num_splits whose partials need more than
 *     FA_SPLITKV_NOALLOC_SCRATCH_BYTES (fa_fwd_splitkv_workspace_size() with
 *     the same arguments) is rejected with FA_ERR_WORKSPACE before anything is
 *     launched; fewer splits need less.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it, keyed on
 *     the device and its current CUDA context, so a call after cudaDeviceReset
 *     (a new context, the array loaded again) looks the address up again; make
 *     the first call on a device, and the first after a reset, before any
 *     stream capture.
 *   - All calls share the one array and it keeps the previous call's contents.
 *     Nothing in it needs clearing (each call writes every partial it reads),
 *     but calls that can overlap on the GPU -- on different streams, or on
 *     different host threads -- race on it and must be serialised by the caller.
 */
#define FA_SPLITKV_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
fa_status_t fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                                   int causal, int num_splits, void* stream);

/*
 * Backward pass (§05: recompute each needed block of P from the saved LSE).
 *   q, k, v, o, dout (bf16) and lse (fp32) as produced by fa_fwd with the same
 *   scale and causal flag.
 *   dq [B,Hq,Nq,d], dk/dv [B,Hkv,Nk,d] (bf16, written).  dk/dv are summed over
 *   the Hq / Hkv query heads of each kv group.
 *   workspace: device scratch of fa_bwd_workspace_size(...) bytes, 256-byte
 *   aligned (it holds D = rowsum(dout * o), the fp32 dq accumulator and, for
 *   the query split below, fp32 dk / dv partials); NULL makes the call
 *   allocate it stream-ordered.  A workspace smaller than that but large
 *   enough without the partials (D, LSE and the accumulator) runs unsplit.
 *   Query split: where there are too few (key block, kv head) units to fill
 *   the GPU, or their count would leave a last round of CTAs with most SMs
 *   idle, fa_bwd_query_split(...) CTAs share each unit's query steps and the
 *   last of them adds the others' partials in a fixed order, so dk / dv still
 *   repeat bitwise from call to call.
 *   For d > 128 the features are split in two halves: each key block is
 *   handled by two CTAs that both recompute S and dP over all d features and
 *   each accumulate their half of dk, dv and dq.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/*
 * Key shares per split work tile that fa_fwd / fa_fwd_ex use on the current
 * device: 1 for no key split (also for the decode shapes, which run the
 * split-KV decode kernels), 2 to 16 where a split of every tile, or of the
 * tiles after the last full round, is estimated (by simulating the persistent
 * launch's claiming) to save at least 5%.  0 for sizes fa_fwd would refuse.
 */
int fa_fwd_kv_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);

/*
 * The number of CTAs that fa_bwd / fa_bwd_ex share each (key block, kv head)
 * unit between on the current device, given fa_bwd_workspace_size(...) bytes
 * of workspace (or none, so that the call allocates it): 1 (no split), 2, 3,
 * 4, 6 or 8.  The choice depends only on the sizes, the causal flag and the
 * device's SM count.  0 for sizes that fa_bwd would refuse.
 */
int fa_bwd_query_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);
fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd for either 16-bit element type: q, k, v, o, dout, dq, dk, dv hold
 * `dtype` elements (FA_DTYPE_BF16 is exactly fa_bwd).  The workspace size does
 * not depend on the element type.
 */
fa_status_t fa_bwd_ex(fa_dtype_t dtype, const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Reads and clears the device status word of the current device.  Synchronises
 * `stream` (the only call that does).  Returns FA_OK; FA_ERR_SLOT_CONFLICT if a
 * tiled forward found its tile-counter slot held by another launch since the
 * last check (the call then waits for the whole device, cudaDeviceSynchronize,
 * and clears every slot, so call it when no forward of the results you still
 * trust is in flight); FA_ERR_TIMEOUT if a bounded wait in a kernel ran out; or
 * FA_ERR_CUDA.
 */
fa_status_t fa_check_device_status(void* stream);

/*
 * Test hook (not for production use; the pages have no counterpart): pins
 * every later tiled forward launch of the process to tile-counter slot `slot`
 * (0..255), or restores the rotation with slot = -1.  With a slot given and
 * preset_owner != 0, first writes preset_owner into that slot's owner word
 * (synchronous copy), as if a launch with that tag held the slot: the next
 * launch pinned there must then report FA_ERR_SLOT_CONFLICT.  Returns
 * FA_ERR_INVALID_ARGUMENT for a slot outside -1..255, FA_ERR_CUDA if the copy
 * fails.
 */
fa_status_t fa_testhook_tile_slot(int slot, unsigned preset_owner);

/*
 * Self-test of the bounded-wait machinery: launches one block that waits on a
 * barrier nothing will arrive on, with a limit of timeout_us microseconds.
 * The kernel gives up, records FA_ERR_TIMEOUT and returns; the device stays
 * usable.  Returns what fa_check_device_status() then reports (FA_ERR_TIMEOUT
 * when the machinery works).  Synchronises `stream`.
 */
fa_status_t fa_selftest_wait_timeout(unsigned timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBFA_FA_H */
