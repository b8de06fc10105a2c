/*
 * lora.h — C ABI of the B200 (sm_100a) multi-LoRA shrink / expand library
 * (liblora_b200.so).
 *
 * The operation, per LoRA-wrapped linear layer y = x W^T of a mixed batch in
 * which every token t carries an adapter-slot index idx[t] (-1 = base model
 * only, no LoRA contribution):
 *
 *   shrink   buf[i][t][j]     = sum_d x[t][d] * A_i[idx[t]][j][d]       (fp32)
 *   expand   y[t][off_i + o] += scale * sum_j buf_i[t][j] * B_i[idx[t]][o][j]
 *
 * Sources: "[Hardware][TPU][V1] Better tpu multilora compilation"
 * (vllm-project/vllm pull 16989), the ref_bgmv baseline function in the
 * discussion (gather the per-token adapter matrix, multiply the token's
 * vector by it); "Add multi-LoRA support" (vllm-project/vllm pull 1804),
 * Features list (LoRA and base-only requests in one batch, fixed GPU adapter
 * slots, BGMV kernels, CUDA-graph friendly) and Limitations list (BGMV is not
 * efficient for prefill, SGMV lost accuracy to a half-precision intermediate,
 * maximum rank 64); "[LoRA] LoRA cuda graph specialization"
 * (vllm-project/vllm pull 25914), Implementation list (no LoRA work at all,
 * not even zeroing the intermediate, when no adapter is active).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensors are row-major.  fp16/bf16 elements (lora_dtype) for x, A, B
 *    and y; fp32 for the intermediate buf; int32 for indices and segments.
 *  - "device" pointers point to memory of the current CUDA device; "host"
 *    pointers to ordinary host memory that is only read during the call.
 *  - The caller owns every buffer.  The library never allocates, frees or
 *    synchronises in the compute calls; work is enqueued on `stream` (NULL =
 *    the legacy default stream) in stream order, so the calls can be captured
 *    in a CUDA graph.
 *  - Every call returns a status and never aborts.  Host-side argument checks
 *    return LORA_ERR_INVALID_ARG / _UNSUPPORTED / _MISALIGNED before anything
 *    is enqueued.  A failed launch returns LORA_ERR_CUDA.  Device code never
 *    traps: an adapter index outside [-1, S) is treated as -1 and counted in
 *    the workspace, and lora_check_errors() reports it as LORA_ERR_BAD_INDEX.
 *  - Limits: 1 <= n_slices <= LORA_MAX_SLICES, r in {8, 16, 32, 64}
 *    (pull 1804 caps the rank at 64; pad a smaller rank with zero rows of A
 *    and zero columns of B, which is exact), 1 <= S <= LORA_MAX_SLOTS,
 *    0 <= T <= LORA_MAX_TOKENS, D and every D_out a multiple of 8,
 *    all base pointers 16-byte aligned, ldx / ldy multiples of 8 elements,
 *    y_col_off entries multiples of 8.
 *  - x, buf and y must not overlap.
 */
#ifndef LORA_B200_H
#define LORA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LORA_OK = 0,
  LORA_ERR_INVALID_ARG = -1,  /* null pointer, negative size, bad slice list */
  LORA_ERR_UNSUPPORTED = -2,  /* rank / slot count / slice count outside the limits */
  LORA_ERR_MISALIGNED = -3,   /* pointer, stride or offset breaks the 16-byte rule */
  LORA_ERR_CUDA = -4,         /* a CUDA launch or query failed */
  LORA_ERR_BAD_INDEX = -5     /* device saw an adapter index outside [-1, S) or bad segments */
} lora_status;

typedef enum { LORA_F16 = 0, LORA_BF16 = 1 } lora_dtype;

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* lora_stream_t;

#define LORA_MAX_SLICES 8
#define LORA_MAX_SLOTS 1024
#define LORA_MAX_TOKENS (1 << 22)

/*
 * Bytes of device workspace ("meta") that lora_group and the compute calls
 * need for a batch of T tokens over S slots: an error counter, the per-slot
 * token offsets, the token permutation and the work list.  About
 * 4*(T + S) + 16*(T/16 + S) + 512 bytes.  Returns 0 for sizes outside the
 * limits.  The workspace must be zero-filled once before its first use
 * (cudaMemsetAsync, or lora_workspace_reset); after that the library keeps
 * it consistent.
 */
LORA_API size_t lora_workspace_bytes(int T, int S);

/* Zero the workspace on `stream` (clears the error counter). */
LORA_API lora_status lora_workspace_reset(void* meta, size_t meta_bytes, lora_stream_t stream);

/*
 * Per-slot ranks ("Add multi-LoRA support", Features list: LoRAs of different
 * ranks in one batch).  The stacks keep the call's rank r for every slot; a
 * slot whose adapter has a smaller rank k fills only the first k rows of
 * A_i[g] and the first k columns of B_i[g] and leaves the rest zero.  This
 * records each slot's k in the workspace, so that the kernels skip the padded
 * rows and columns (neither read nor multiplied) instead of multiplying
 * zeros; the buf columns past a slot's rank are written as 0.
 *
 *   ranks   device int32 [S]: slot g's rank; 0, or a value >= the call's r,
 *           means r.  Values are rounded up to a multiple of 8 (the padding
 *           up to that multiple must be zero).  NULL clears the ranks.
 *   meta    a workspace of at least lora_workspace_bytes(T, S) for the calls
 *           that will use it; the ranks stay in it across lora_group calls
 *           until changed, or until lora_workspace_reset.
 * Enqueued on `stream` as one small kernel (capturable).  The fused one-launch
 * path of lora_bgmv and lora_shrink_laned read the whole stack and ignore the
 * ranks (the padding is zero, so their results are the same).
 */
LORA_API lora_status lora_set_slot_ranks(int S, const int32_t* ranks, void* meta,
                                         size_t meta_bytes, lora_stream_t stream);

/*
 * Group-by-slot metadata for one batch (the token-index tensor moved to the
 * device, as in pull 16989's review thread, then sorted by slot on the
 * device).  A stable counting sort of the tokens by idx[t]: tokens of slot 0
 * in increasing token order, then slot 1, ..., then the tokens without an
 * adapter; the per-slot offsets; and a work list of (slot, up to 16 tokens)
 * items that the per-token (BGMV) shrink and expand consume.
 *
 *   T, S        tokens in the batch, adapter slots.
 *   idx         device int32 [T]; -1 = no adapter; others outside [-1, S)
 *               are counted as bad and treated as -1.
 *   meta        device workspace of at least lora_workspace_bytes(T, S)
 *               bytes, 256-byte aligned; overwritten (except the error
 *               counter, which accumulates).
 *
 * Build it once per batch; every layer's lora_shrink / lora_expand of that
 * batch may then reuse it.  One kernel, one CTA.
 */
LORA_API lora_status lora_group(int T, int S, const int32_t* idx, void* meta, size_t meta_bytes,
                       lora_stream_t stream);

/*
 * BGMV shrink (per-token adapters), one launch for all slices:
 *   buf[i][t][j] = sum_d x[t][d] * A_i[idx[t]][j][d]  for tokens with an adapter,
 *   buf[i][t][j] = 0                                   for tokens without one.
 *
 *   x           device [T, ldx] (ldx >= D), dtype elements.
 *   A           host array of n_slices device pointers; A[i] is [S, r, D]
 *               contiguous (slot-major stack of rank-r down-projections).
 *   idx         device int32 [T], this batch's adapter indices: the same
 *               tensor (and contents) lora_group grouped into `meta`.
 *   buf         device fp32 [n_slices, T, r], fully overwritten.  The sums
 *               accumulate in fp32 and are stored in fp32 (pull 1804 names a
 *               half-precision intermediate as the accuracy problem).
 *   has_active  host flag: 0 means the caller knows no token has an adapter;
 *               the call then returns LORA_OK with nothing enqueued and buf
 *               untouched (pull 25914: no LoRA kernels, no zeroing).
 *   meta        the workspace lora_group filled from idx on this stream (or
 *               one ordered before it).
 * The grouping is checked against idx token by token: a token whose index
 * differs from the group the workspace put it in (a workspace grouped from
 * another batch) is not written, and the mismatch is counted, so that
 * lora_check_errors returns LORA_ERR_BAD_INDEX; a stale grouping never yields
 * a silently wrong row.
 * With r >= 16 and T >= 16 * S the slot groups of the grouping run on tcgen05
 * tensor cores (x rows gathered through the grouping permutation); otherwise
 * on CUDA cores.
 */
LORA_API lora_status lora_shrink(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                        const void* x, int64_t ldx, const void* const* A, const int32_t* idx,
                        float* buf, int has_active, const void* meta, size_t meta_bytes,
                        lora_stream_t stream);

/*
 * Laned shrink: the same result as lora_group + lora_shrink, with no grouping
 * and no sort.  After the LoRA laning of the TPU kernels in "[Hardware][TPU]
 * [V1] Better tpu multilora compilation" (several adapters side by side in
 * one register, one pass for tokens of different adapters): the stack A_i
 * [S, r, D] is read as one [S*r, D] matrix of "lanes", every token is
 * contracted with every lane on tcgen05 tensor cores (M = tokens, N = S*r,
 * K = D, fp32 accumulator in tensor memory), and each token keeps the r lanes
 * of its own slot: buf[i][t][j] = C[t][idx[t]*r + j].  The contraction does S
 * times the useful multiply-adds; for small ranks and slot counts that stays
 * far below the tensor-core roofline while x and A are read once, in dense
 * tiles.
 *
 *   Arguments as for lora_shrink; idx is read directly (no lora_group);
 *   indices outside [-1, S) are treated as -1 and counted.
 *   meta   a workspace of at least 256 bytes whose error counters are used
 *          (any lora_workspace_bytes-sized workspace will do).
 * D must be a multiple of 8 and x 16-byte aligned with ldx a multiple of 8
 * (tensor-map rules); otherwise LORA_ERR_MISALIGNED / LORA_ERR_UNSUPPORTED.
 */
LORA_API lora_status lora_shrink_laned(lora_dtype dtype, int T, int D, int r, int S,
                                       int n_slices, const void* x, int64_t ldx,
                                       const void* const* A, const int32_t* idx, float* buf,
                                       int has_active, void* meta, size_t meta_bytes,
                                       lora_stream_t stream);

/*
 * BGMV expand into fused output slices (q/k/v, gate/up), one launch:
 *   y[t][y_col_off[i] + o] = round(y[t][y_col_off[i] + o]
 *                                  + scale * sum_j buf_i[t][j] * B_i[idx[t]][o][j])
 * for tokens with an adapter, with the sum in fp32 and one round-to-nearest-
 * even into dtype; rows of tokens without an adapter are not read or written.
 *
 *   buf               device fp32; slice i's [T, r] block starts at
 *                     buf + i * buf_slice_stride (0 = one intermediate shared by
 *                     every slice, for a shared A).
 *   B                 host array of n_slices device pointers; B[i] is
 *                     [S, D_out[i], r] contiguous.
 *   D_out             host int32 [n_slices], output width of each slice.
 *   scale             LoRA scaling factor (per-adapter scales: fold into B).
 *   y                 device [T, ldy] dtype, updated in place.
 *   idx               device int32 [T], as for lora_shrink (checked against
 *                     the grouping the same way: a mismatched row of y is not
 *                     written, and is counted).
 *   y_col_off         host int64 [n_slices], first column of each slice in y;
 *                     slices must not overlap.
 *   has_active, meta  as for lora_shrink.
 * Tensor cores or CUDA cores as for lora_shrink.
 */
LORA_API lora_status lora_expand(lora_dtype dtype, int T, int r, int S, int n_slices,
                        const float* buf, int64_t buf_slice_stride, const void* const* B,
                        const int32_t* D_out, const int32_t* idx, float scale, void* y,
                        int64_t ldy, const int64_t* y_col_off, int has_active, const void* meta,
                        size_t meta_bytes, lora_stream_t stream);

/*
 * Whole per-token (BGMV) LoRA of one batch in one call: lora_group, then
 * lora_shrink, then lora_expand, with the same results (buf and y).  When the
 * shape fits (T <= 4096 and the slot's tiles fit in shared memory) this is ONE
 * kernel launch: each thread-block cluster owns one (slot, slice), finds its
 * tokens itself, and keeps the fp32 intermediate on chip between the shrink
 * and the expand (it is still written to buf).  Otherwise it runs the three
 * launches.  Sources as for lora_shrink / lora_expand.
 *
 *   A, shared_A   shared_A = 0: A holds n_slices stacks (one per output slice);
 *                 shared_A = 1: A[0] is one stack used by every slice.
 *   buf           device fp32 [n_A, T, r], n_A = shared_A ? 1 : n_slices;
 *                 receives the intermediate (required).
 *   idx           device int32 [T] as for lora_group.
 *   flags         LORA_FLAG_PDL_EARLY: A, B and idx are not written by the
 *                 kernel launched just before this call on `stream`, so the
 *                 call may read them before that kernel has finished
 *                 (programmatic dependent launch): the one-launch kernel reads
 *                 A and idx early, the grouping of the three-launch path reads
 *                 and counts idx early and exchanges the counts of its CTAs
 *                 through its own words of the workspace (words that no other
 *                 kernel reads), so that kernel must not write the workspace
 *                 either; x, y and the grouping held in the workspace are
 *                 always read or written after it.  0: nothing is read before
 *                 it finishes.
 *                 LORA_FLAG_GROUPED: the workspace already holds the grouping
 *                 of this idx (lora_group, or an earlier lora_bgmv of the same
 *                 batch, on this stream), as when the projections of one
 *                 decoder layer share a batch: the three-launch path makes
 *                 two launches (shrink, expand) and no grouping.  The grouping
 *                 is checked against idx row by row as in lora_shrink, so a
 *                 stale one is reported, never used silently.  The one-launch
 *                 kernel finds its tokens itself and ignores the flag.
 *   meta          workspace as for lora_group (its error counters are used;
 *                 the three-launch path also keeps the grouping there).
 *   Other arguments as for lora_shrink / lora_expand.
 */
#define LORA_FLAG_PDL_EARLY 1u
#define LORA_FLAG_GROUPED 2u
LORA_API lora_status lora_bgmv(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                               const void* x, int64_t ldx, const void* const* A, int shared_A,
                               const void* const* B, const int32_t* D_out, float scale, void* y,
                               int64_t ldy, const int64_t* y_col_off, float* buf,
                               const int32_t* idx, int has_active, unsigned flags, void* meta,
                               size_t meta_bytes, lora_stream_t stream);

/* Kernel launches lora_bgmv makes for this shape (1 fused, 3 otherwise), or a
 * negative status for invalid sizes.  Host only; nothing is enqueued. */
LORA_API int lora_bgmv_launches(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                                const int32_t* D_out);

/*
 * SGMV shrink (segment-grouped, for prefill): contiguous runs of tokens share
 * one adapter.  Same result as lora_shrink with idx[t] = seg_adapter[s] for
 * seg_starts[s] <= t < seg_starts[s+1] ("Add multi-LoRA support", Limitations
 * list: SGMV is the prefill kernel; here its intermediate stays fp32).
 *
 *   seg_starts   device int32 [n_seg + 1]: 0 = seg_starts[0] <= ... <=
 *                seg_starts[n_seg] = T (empty segments allowed).
 *   seg_adapter  device int32 [n_seg]; -1 allowed; repeats allowed.
 *   n_seg        host count, 0 <= n_seg <= T + 1 (n_seg = 0 requires T = 0).
 *   meta         workspace of at least lora_workspace_bytes(T, S) bytes (its
 *                error counter and work list are used).
 * Malformed segments are counted as bad (LORA_ERR_BAD_INDEX from
 * lora_check_errors); the rows they would cover are then unspecified, but no
 * access leaves the buffers.  Runs on tcgen05 tensor cores when r >= 16 and
 * n_seg <= 2048, else on CUDA cores.
 */
LORA_API lora_status lora_shrink_segment(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                                const void* x, int64_t ldx, const void* const* A,
                                const int32_t* seg_starts, const int32_t* seg_adapter,
                                int n_seg, float* buf, int has_active, void* meta,
                                size_t meta_bytes, lora_stream_t stream);

/* SGMV expand: lora_expand with the adapters given by segments, as above. */
LORA_API lora_status lora_expand_segment(lora_dtype dtype, int T, int r, int S, int n_slices,
                                const float* buf, int64_t buf_slice_stride,
                                const void* const* B, const int32_t* D_out,
                                const int32_t* seg_starts, const int32_t* seg_adapter,
                                int n_seg, float scale, void* y, int64_t ldy,
                                const int64_t* y_col_off, int has_active, void* meta,
                                size_t meta_bytes, lora_stream_t stream);

/*
 * SGMV shrink + expand of one prefill batch in one call ("Add multi-LoRA
 * support", Limitations list: SGMV is the prefill kernel): lora_shrink_segment
 * into buf, then lora_expand_segment from it, with A either one stack per
 * slice or (shared_A != 0) one stack whose intermediate every slice expands
 * (buf then holds one slice).  The result equals the two calls; inside this
 * call the expand's previous launch is known to be this library's shrink,
 * which writes only buf, so the tensor-core expand sets up its schedule and
 * issues its first B and y tiles while the shrink finishes and waits for it
 * only before reading buf (programmatic dependent launch).
 *   Arguments as for lora_shrink_segment / lora_expand_segment and lora_bgmv
 *   (buf: device fp32 [n_A, T, r], n_A = shared_A ? 1 : n_slices).
 */
LORA_API lora_status lora_sgmv(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                               const void* x, int64_t ldx, const void* const* A, int shared_A,
                               const void* const* B, const int32_t* D_out, float scale, void* y,
                               int64_t ldy, const int64_t* y_col_off, float* buf,
                               const int32_t* seg_starts, const int32_t* seg_adapter, int n_seg,
                               int has_active, void* meta, size_t meta_bytes,
                               lora_stream_t stream);

/*
 * Synchronise `stream`, read and clear the workspace's error counter.
 * Returns LORA_ERR_BAD_INDEX if any call since the last check saw an index
 * outside [-1, S) or malformed segments, LORA_ERR_CUDA if the stream reports
 * an error, else LORA_OK.  Not for use inside stream capture.
 */
LORA_API lora_status lora_check_errors(void* meta, size_t meta_bytes, lora_stream_t stream);

/*
 * Allocation-free per-token shrink: lora_group + lora_shrink in one call, with
 * the grouping workspace kept in a fixed array inside the library instead of
 * caller memory.  The paper has no counterpart; it exists for callers that
 * cannot allocate device memory (code that runs where cudaMalloc is not
 * available or not allowed, such as a host that only hands out the input and
 * output buffers) and so cannot supply `meta`.
 *
 *   Arguments as for lora_shrink, plus idx (device int32 [T]) as for
 *   lora_group; no meta.  Same result as lora_group + lora_shrink.
 *   Limits: T <= LORA_NOALLOC_MAX_TOKENS and S <= LORA_MAX_SLOTS, else
 *   LORA_ERR_UNSUPPORTED before anything is enqueued.
 *   The array is LORA_NOALLOC_SCRATCH_BYTES of device memory that every GPU
 *   which loads the library holds until the process exits.  The first call on
 *   a device looks up the array's device address (once per device); make that
 *   first call before any stream capture.  No cudaMalloc / cudaFree or other
 *   allocating routine is called.
 *   Every call shares the one array and it keeps the last call's contents:
 *   each call clears its header and rebuilds the rest, so calls that overlap
 *   on the GPU (different streams, or different host threads on one device)
 *   race and give wrong results; order them.  Indices outside [-1, S) are
 *   treated as -1 and are not reported (there is no caller workspace to hold
 *   the error counter).
 */
#define LORA_NOALLOC_MAX_TOKENS 8192
#define LORA_NOALLOC_SCRATCH_BYTES 246784
LORA_API lora_status lora_shrink_noalloc(lora_dtype dtype, int T, int D, int r, int S,
                                         int n_slices, const void* x, int64_t ldx,
                                         const void* const* A, const int32_t* idx, float* buf,
                                         int has_active, lora_stream_t stream);

/* Static, human-readable name of a status. */
LORA_API const char* lora_status_string(lora_status status);

/* Build identification: "liblora_b200 sm_100a <version>". */
LORA_API const char* lora_build_info(void);

/* Kernel launches this library has made in this process (all devices and
 * streams), counting a launch recorded into a stream capture once; a graph
 * replay launches nothing through the library and adds nothing.  For
 * instrumentation: the difference across a call is the number of kernels
 * that call enqueued. */
LORA_API unsigned long long lora_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LORA_B200_H */
