/*
 * fa2.h -- C ABI of the B200 (sm_100a) exact tiled attention library.
 *
 * The operation is exact scaled-dot-product attention, forward and backward,
 * computed tile by tile so that the N x N score matrix never goes to HBM:
 *   "FlashAttention (v2)" glossary page, definition paragraph (tiles held in
 *   on-chip memory, the full score matrix never written to HBM, the result not
 *   approximated) and results paragraph (output matches standard attention);
 *   "FlashAttention-2" summary page, How It Works items 1-2 (work split along
 *   the sequence as well as batch and heads; scaling done once at the end);
 *   "FlashAttention-2: Faster Attention with Better Parallelism and Work
 *   Partitioning" reproduction page, closing paragraph (key blocks entirely
 *   above the diagonal are never computed; only the diagonal block of each
 *   row of blocks needs the elementwise mask) and
 *   Figures 5-6 (forward and backward attention are the benchmarked passes).
 *
 * For each head (b, h) and rows i, keys j in [0, N):
 *   S = scale * Q K^T (causal: S_ij = -inf for j > i),  P = softmax_rows(S),
 *   O = P V,  LSE_i = ln sum_j exp(S_ij)  (natural log).
 * Backward, for an upstream gradient dO:
 *   D_i = sum_c dO_ic O_ic,  dP = dO V^T,  dS = P o (dP - D),
 *   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
 *
 * Conventions shared by every call:
 *  - Tensors q, k, v, o, dO, dq, dk, dv are bf16, contiguous [B, H, N, d]
 *    (row-major; d innermost). Q and K/V have the same length N
 *    (self-attention). lse is fp32 [B, H, N].
 *  - d must be 64 or 128. 1 <= N <= 65535 * 128 (any N; the last tile is masked).
 *    B >= 1, H >= 1, B * H <= 65535.
 *  - scale must be finite and >= 0 (typically 1/sqrt(d)).
 *  - All pointers are device pointers (HBM), 16-byte aligned (the kernels load
 *    tiles with the Tensor Memory Accelerator, which requires it).
 *  - The caller owns every buffer, including the backward workspace. The
 *    library never allocates or frees device memory and never synchronises the
 *    stream (fa2_get_device_status is the one exception, documented there).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    means the legacy default stream). Arguments are checked on the host before
 *    any launch; on any error nothing is launched and nothing is written.
 */
#ifndef FA2_B200_H_
#define FA2_B200_H_

#include <stddef.h>

#if defined(__GNUC__)
#define FA2_API __attribute__((visibility("default")))
#else
#define FA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA2_OK = 0,
  FA2_ERR_INVALID_ARG = 1, /* null pointer, N/B/H < 1, bad scale, workspace too small */
  FA2_ERR_UNSUPPORTED = 2, /* d not in {64, 128}, B*H > 65535, or no sm_100 device */
  FA2_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned */
  FA2_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, tensor map) */
  FA2_ERR_TIMEOUT = 5,     /* a kernel gave up on a bounded wait (see fa2_get_device_status) */
  FA2_ERR_CONFLICT = 6     /* a forward found its work counter reset by a later launch (ditto) */
} fa2_status;

/*
 * Forward pass: o = softmax(scale * q k^T [causal]) v and lse (natural log).
 * Defined by the "FlashAttention (v2)" glossary page, definition paragraph
 * (attention computed tile by tile in on-chip memory, the score matrix never
 * written to HBM, no approximation) and the "FlashAttention-2" summary page,
 * How It Works items 1-2 (query blocks spread over the GPU as well as batch
 * and heads; the softmax normalisation applied once at the end); causal block
 * skipping from the reproduction page's closing paragraph.
 * q, k, v: inputs [B,H,N,d] bf16. o: output [B,H,N,d] bf16. lse: output
 * [B,H,N] fp32, kept for the backward pass. causal: 0 or 1 (j <= i allowed).
 * Work: pairs of 128-row query blocks x batch*head, taken from a work counter by
 * a persistent grid of one CTA per SM. Enqueues on `stream` an 8-byte memset of
 * that counter (cuMemsetD32Async: the launch's tag in both halves; one of 256
 * counters inside the library, used in turn) and one kernel launch. Launches
 * ordered on one stream are always independent. Launches that may overlap on
 * the GPU (other streams) are independent as long as fewer than 256 are in
 * flight at once; beyond that a launch can find its counter reset by a later
 * one: it then stops early and fa2_get_device_status reports FA2_ERR_CONFLICT
 * (its o and lse, and the later launch's, are then not to be trusted). A forward
 * enqueued under stream capture takes its counter from a second ring of 256
 * that eager calls never use, and keeps it for every replay of the graph:
 * replays of one graph must not overlap one another on the GPU. The first call
 * on a device (and the first after a cudaDeviceReset) looks up the counters'
 * device address (cudaGetSymbolAddress): make it outside stream capture.
 */
FA2_API fa2_status fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * (No counterpart on the pages, which describe no interface: the backward's
 * scratch memory is caller-owned so that the library never allocates.)
 * Bytes of device workspace fa2_backward needs for these sizes: an fp32 dQ
 * accumulator [B,H,Np,d], two fp32 row vectors [B,H,Np] (D = rowsum(dO o O)
 * and the log2-scaled LSE), with Np = N rounded up to 128, and 16 bytes for the
 * main kernel's work-item counter. Returns 0 for invalid sizes.
 */
FA2_API size_t fa2_backward_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass: the gradients of the forward pass with respect to q, k and v,
 * recomputing the probabilities from the saved LSE rather than storing them.
 * The pages benchmark this pass ("FlashAttention-2: Faster Attention with
 * Better Parallelism and Work Partitioning" reproduction page, Figure 6a-d
 * captions: backward speed against sequence length, head dimension 64 and 128,
 * with and without the causal mask) but print no equations; the chain-rule
 * gradients above are this library's reading.
 * Inputs q, k, v, o (the forward output), lse (the forward
 * LSE), dO (gradient of the loss w.r.t. o). Outputs dq, dk, dv [B,H,N,d] bf16.
 * o and lse must come from fa2_forward on the same q, k, v, causal and scale;
 * they are trusted as given. workspace: caller-owned device memory of at least
 * fa2_backward_workspace_size() bytes, 16-byte aligned; its contents on entry
 * do not matter and on exit are unspecified. Three launches on `stream`:
 * preprocess (D, log2 LSE, zero dQ accumulator), the key-block-parallel main
 * kernel (dK, dV, and dQ accumulated with fp32 reductions), and the dQ
 * conversion to bf16.
 */
FA2_API fa2_status fa2_backward(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dO, void* dq, void* dk, void* dv,
                        int B, int H, int N, int d, int causal, float scale,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * How the backward produces dQ (the pages' two options; the default is chosen
 * by measurement, see fa2_backward_dq_strategy):
 *  FA2_DQ_REDUCE    the key-block kernel adds each step's dQ into an fp32
 *                   accumulator in the workspace with reductions; a third
 *                   kernel converts it to bf16.
 *  FA2_DQ_SEPARATE  the key-block kernel computes dK, dV only; a separate
 *                   query-parallel kernel recomputes S, P, dP, dS per query
 *                   block and accumulates dQ on chip (no atomics, bitwise
 *                   reproducible dQ, 40% more tensor work).
 */
typedef enum { FA2_DQ_AUTO = 0, FA2_DQ_REDUCE = 1, FA2_DQ_SEPARATE = 2 } fa2_dq_strategy;

/* The strategy FA2_DQ_AUTO uses for these sizes (FA2_DQ_REDUCE or FA2_DQ_SEPARATE). */
FA2_API int fa2_backward_dq_strategy(int B, int H, int N, int d, int causal);

/*
 * fa2_backward with an explicit dQ strategy (FA2_DQ_*; anything else is
 * FA2_ERR_INVALID_ARG). Same arguments, workspace and results otherwise.
 * fa2_backward(...) is fa2_backward_ex(..., FA2_DQ_AUTO, stream).
 */
FA2_API fa2_status fa2_backward_ex(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                   int B, int H, int N, int d, int causal, float scale,
                                   void* workspace, size_t workspace_bytes, int dq_strategy,
                                   void* stream);

/*
 * The three stages fa2_backward launches, callable one at a time (same
 * arguments and checks as fa2_backward; run them in this order on one stream,
 * with the same workspace, to get exactly fa2_backward's result):
 *  fa2_backward_preprocess  D = rowsum(dO o O), LSE * log2(e), dQ accumulator
 *                           and work-item counter zeroed; padding rows get
 *                           D = 0 and LSE = +inf.
 *  fa2_backward_main        dK, dV (bf16 outputs) and the fp32 dQ accumulator;
 *                           one persistent CTA per SM takes (key tile, head)
 *                           items from the counter.
 *  fa2_backward_dq_convert  dq = bf16(scale * accumulator).
 * Splitting them lets a caller time or overlap the stages individually.
 */
FA2_API fa2_status fa2_backward_preprocess(const void* o, const float* lse, const void* dO,
                                           int B, int H, int N, int d, void* workspace,
                                           size_t workspace_bytes, void* stream);
FA2_API fa2_status fa2_backward_main(const void* q, const void* k, const void* v, const void* dO,
                                     void* dk, void* dv, int B, int H, int N, int d, int causal,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     void* stream);
FA2_API fa2_status fa2_backward_dq_convert(void* dq, int B, int H, int N, int d, float scale,
                                           void* workspace, size_t workspace_bytes, void* stream);
/*
 * The FA2_DQ_SEPARATE stages, after fa2_backward_preprocess:
 *  fa2_backward_main_dkdv   dK, dV only (the key-block kernel without dQ).
 *  fa2_backward_dq          dq = scale * dS K by the query-parallel kernel
 *                           (reads D and LSE from the workspace).
 */
FA2_API fa2_status fa2_backward_main_dkdv(const void* q, const void* k, const void* v,
                                          const void* dO, void* dk, void* dv, int B, int H, int N,
                                          int d, int causal, float scale, void* workspace,
                                          size_t workspace_bytes, void* stream);
FA2_API fa2_status fa2_backward_dq(const void* q, const void* k, const void* v, const void* dO,
                                   void* dq, int B, int H, int N, int d, int causal, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace. (The pages
 * describe no counterpart; this is a deployment convenience of this library.)
 *
 * For callers that cannot allocate device memory when they run the backward:
 * applications that reserve all device memory at start-up and may not call
 * cudaMalloc later, plugins whose host forbids allocation (and the device
 * synchronisation it can cause) on the hot path, or C callers without an
 * allocator to size a workspace with. Same arguments, checks and results as
 * fa2_backward, minus workspace/workspace_bytes: the scratch (fp32 dQ
 * accumulator, D, log2-scaled LSE) lives in a fixed device array of
 * FA2_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.
 *  - Returns FA2_ERR_UNSUPPORTED, without launching anything, when
 *    fa2_backward_workspace_size(B, H, N, d) > FA2_NOALLOC_SCRATCH_BYTES
 *    (for example B*H*N*d above about 16 million elements).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - All calls share the one array: calls whose kernels overlap on the GPU
 *    (different streams without ordering between them) race on it and give
 *    wrong results. Calls ordered on one stream are safe; each call
 *    re-initialises the parts that must start at zero.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define FA2_NOALLOC_SCRATCH_BYTES (64u << 20)
FA2_API fa2_status fa2_backward_noalloc(const void* q, const void* k, const void* v,
                                        const void* o, const float* lse, const void* dO,
                                        void* dq, void* dk, void* dv, int B, int H, int N, int d,
                                        int causal, float scale, void* stream);

/*
 * Different query and key lengths (cross attention): q, o, dO, dq are
 * [B, H, Nq, d], k, v, dk, dv [B, H, Nk, d], lse [B, H, Nq]; the workspace is
 * fa2_backward_workspace_size(B, H, Nq, d) bytes. With causal = 1 the mask is
 * aligned to the bottom-right corner of the Nq x Nk score matrix: query i sees
 * keys j <= i + Nk - Nq (the pages only use Nq = Nk, where this is j <= i;
 * the bottom-right reading is ours). Causal with Nq > Nk (rows without keys)
 * returns FA2_ERR_UNSUPPORTED, like d not in {64, 128}. Otherwise the same
 * arguments, checks, kernels and errors as fa2_forward / fa2_backward (the
 * backward uses the dQ-reduction strategy); fa2_forward and fa2_backward are
 * these with Nq = Nk = N.
 */
FA2_API fa2_status fa2_forward_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int B, int H, int Nq, int Nk, int d, int causal, float scale,
                                  void* stream);
FA2_API fa2_status fa2_backward_qk(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                   int B, int H, int Nq, int Nk, int d, int causal, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward and backward from HOST buffers: the form of the computation for
 * callers whose tensors live in host memory (and how end-to-end throughput,
 * host<->device copies included, is measured). The pages' method itself is the
 * two device passes above; this only schedules them with the copies.
 *
 *  Inputs  q, k, v, dO: host, bf16 [B, H, N, d] contiguous.
 *  Outputs o (bf16), lse (fp32 [B, H, N]), dq, dk, dv (bf16): host.
 *  Same mask, scale, d and size rules as fa2_forward / fa2_backward.
 *
 * The B*H heads are processed in chunks of `heads_per_chunk` heads (0 = B*H/8
 * rounded up). Chunk c's inputs are copied in, its forward and backward run,
 * and its outputs are copied out on three library-owned streams, up to three
 * chunks in flight, so that the copies in both directions overlap each other
 * and the kernels. Host buffers should be page-locked (cudaHostAlloc /
 * cudaHostRegister); with pageable memory the copies are correct but do not
 * overlap.
 *
 * `device_workspace` (caller-owned device memory, 256-byte aligned, at least
 * fa2_forward_backward_host_workspace_size(B, H, N, d, heads_per_chunk)
 * bytes) holds the chunks' device copies and backward workspaces.
 *
 * Ordering: the work starts after everything enqueued on `stream` before the
 * call and the call returns as soon as it is enqueued; work enqueued on
 * `stream` afterwards (a synchronisation, a read of the outputs) runs after all
 * of it has completed, copies to host included. Calls on one device are
 * serialised internally (they share the library's streams); do not let the
 * host arrays or the workspace change until `stream` has passed the call.
 * Errors: FA2_ERR_INVALID_ARG (null pointer, heads_per_chunk < 0, workspace too
 * small), FA2_ERR_MISALIGNED (workspace), FA2_ERR_UNSUPPORTED (d, sizes,
 * device), FA2_ERR_CUDA (a copy or launch failed; outputs then undefined).
 */
FA2_API size_t fa2_forward_backward_host_workspace_size(int B, int H, int N, int d,
                                                        int heads_per_chunk);
FA2_API fa2_status fa2_forward_backward_host(const void* q, const void* k, const void* v,
                                             const void* dO, void* o, float* lse, void* dq,
                                             void* dk, void* dv, int B, int H, int N, int d,
                                             int causal, float scale, int heads_per_chunk,
                                             void* device_workspace, size_t workspace_bytes,
                                             void* stream);

/* Static, NUL-terminated name of a status code. */
FA2_API const char* fa2_status_string(int status);

/*
 * Synchronises `stream` and reports whether any kernel of this library on the
 * current device recorded an error since the last clear: FA2_ERR_TIMEOUT (a
 * bounded wait ran out) or FA2_ERR_CONFLICT (a forward's work counter was reset
 * by a later launch while it ran; see fa2_forward); then *info, if non-NULL,
 * holds a site code. Returns FA2_OK if none, FA2_ERR_CUDA if the
 * synchronisation itself failed.
 */
FA2_API fa2_status fa2_get_device_status(void* stream, int* info);

/* Clears the device-side status word of the current device (synchronous). */
FA2_API fa2_status fa2_clear_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* FA2_B200_H_ */
