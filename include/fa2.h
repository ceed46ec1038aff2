/*
 * fa2.h -- C ABI of the B200 (sm_100a) exact-attention forward library.
 *
 * The operation (FlashAttention-2, Tri Dao, arXiv 2307.08691; arXiv abstract
 * page, "Abstract"; iplexlaw blog "FlashAttention-2: making long-context
 * attention run efficiently on GPUs", sections "Tiling preserves the attention
 * calculation" and "Three changes improve GPU utilisation"):
 *
 *   for every batch b, head h and query row i,
 *     s_ij  = scale * <q_i, k_j>           for allowed keys j
 *     LSE_i = ln sum_j exp(s_ij)
 *     O_i   = sum_j exp(s_ij - LSE_i) v_j
 *   allowed(i) = all keys (causal = 0) or keys j <= i (causal != 0).
 *
 * The result is exact attention (no approximation): the kernel walks the keys
 * in tiles with an online softmax and never writes the N x N score matrix to
 * device memory; only floating-point rounding differs from the plain
 * definition.
 *
 * Layout: q, k, v, o are bf16 tensors of shape [B, H, N, d], contiguous
 * row-major (d fastest).  lse is fp32 [B, H, N], contiguous, natural log.
 *
 * Ownership: the caller allocates and owns every buffer; the library never
 * allocates device memory in fa2_fwd and keeps no pointer after a call returns.
 *
 * Errors: every entry point returns an fa2_status.  Argument errors are
 * detected on the host before anything is launched, so nothing is written.
 * fa2_fwd is asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 * means the legacy default stream): a status of FA2_OK means the kernel was
 * launched.  Kernel-side failures (a bounded wait that gave up) are recorded
 * in a device status word and reported by fa2_sync_status.
 */
#ifndef FA2_H_
#define FA2_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA2_OK = 0,
  FA2_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, aliasing, non-finite scale */
  FA2_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (e.g. d not in {32,64,96,128,256}) */
  FA2_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed; see fa2_last_error_detail() */
  FA2_ERR_TIMEOUT = 4      /* a kernel's bounded wait gave up (reported by fa2_sync_status) */
} fa2_status;

/*
 * Exact attention forward (the hot path).
 *
 *   q, k, v : device pointers, bf16 [B,H,N,d], contiguous, 16-byte aligned.
 *   o       : device pointer, bf16 [B,H,N,d], contiguous, 16-byte aligned;
 *             written.  Must not overlap q, k, v or lse.
 *   lse     : device pointer, fp32 [B,H,N], contiguous, 4-byte aligned;
 *             written with the natural-log logsumexp of the scaled scores.
 *   B, H, N : >= 1; B <= 65535, H <= 65535, B*H < 2^31, N <= 16776960.
 *             Any such N works (a ragged last tile is masked).
 *   d       : head dimension, 32, 64, 96, 128 or 256 (others ->
 *             FA2_ERR_UNSUPPORTED).  32 and 96 run on the 64- and 128-column
 *             kernels with the extra columns zero-filled on load and clipped
 *             on store; 256 runs on the one-query-tile kernel of
 *             fa2_fwd_splitkv with 64-key tiles (a single key range).
 *   causal  : 0 = every key; non-zero = key j allowed only for query i >= j.
 *   scale   : multiplier of q.k, finite and > 0 (the usual choice is
 *             1/sqrt(d)); other values -> FA2_ERR_INVALID_ARG.
 *   stream  : cudaStream_t as void* (NULL = legacy default stream).
 */
int fa2_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
            int causal, float scale, void* stream);

/*
 * The same operation on HOST buffers (end-to-end call).  q, k, v are read
 * from host memory (pinned memory gives full copy bandwidth), o and lse are
 * written to host memory, and the call returns after the results have landed.
 * `workspace` is a caller-owned device buffer of at least
 * fa2_fwd_host_workspace_bytes(B,H,N,d) bytes, 256-byte aligned, that holds
 * the device copies.  The work is split into up to 8 chunks of whole batches
 * (or of heads when B < 8): uploads run on `stream`, each chunk's kernel on a
 * compute stream and its downloads on a download stream of the library's own
 * (created once per device on first use, kept until the process ends), so
 * copies in both directions overlap the kernels; results are identical to
 * one fa2_fwd call.  Concurrent calls on one device are serialised.  Returns
 * FA2_ERR_TIMEOUT if a kernel reported a timeout; after any error every
 * queued copy and kernel has completed before the call returns.
 */
int fa2_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace fa2_fwd_host needs for this shape (0 on bad sizes). */
size_t fa2_fwd_host_workspace_bytes(int B, int H, int N, int d);

/*
 * Synchronise `stream`, then read and clear the device status word.  Returns
 * FA2_ERR_TIMEOUT if any kernel launched since the last call gave up a bounded
 * wait, FA2_ERR_CUDA if the synchronisation failed, else FA2_OK.
 *
 * The status word is one per device for the whole process, not one per
 * stream or per call: a time-out in a kernel on any stream of the current
 * device is reported to whichever caller reads the word first (this call, or
 * fa2_fwd_host, which calls it), and that read clears it for everyone.  Code
 * that shares a device between independent users and needs to attribute a
 * time-out must serialise its calls with their fa2_sync_status reads.
 */
int fa2_sync_status(void* stream);

/*
 * Test hook for the failure path: launch the attention kernel (same
 * arguments as fa2_fwd, every supported d; d = 256 runs the one-tile kernel
 * of fa2_fwd_splitkv) with the query-tile load withheld, so every wait on it
 * runs out after `timeout_ns` nanoseconds (1 .. 2e9).  The kernel then sets the status
 * word and exits cleanly (tensor memory released, no copy left in flight);
 * fa2_sync_status returns FA2_ERR_TIMEOUT.  Outputs are unspecified.
 */
int fa2_fwd_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                           int N, int d, int causal, float scale, unsigned long long timeout_ns, void* stream);

/*
 * Exact attention of few queries against many keys: decoding, or a chunk of
 * new queries after a cached prefix.  The pages separate the processing of a
 * long prompt from token-by-token generation, whose bottlenecks differ
 * (iplexlaw blog "FlashAttention-2: making long-context attention run
 * efficiently on GPUs", section "Document the implementation difference").
 * With few query rows, one CTA per query tile and head would leave most SMs
 * idle, so the keys are split into ranges: one CTA per (128-row query tile,
 * batch*head, key range) computes that range's partial output and
 * logsumexp, and a second kernel merges them exactly
 * (LSE = ln sum_r exp(LSE_r), O = sum_r exp(LSE_r - LSE) O_r).  With at
 * most 32 query rows and d <= 128 the same split is also applied inside each
 * CTA: every softmax warp takes a quarter of each key tile for all the rows
 * and the four quarters merge exactly before the range result is written.
 *
 *   q       : device pointer, bf16 [B,H,Nq,d], contiguous, 16-byte aligned.
 *   k, v    : device pointers, bf16 [B,H,Nk,d], contiguous, 16-byte aligned.
 *   o       : device pointer, bf16 [B,H,Nq,d]; written.
 *   lse     : device pointer, fp32 [B,H,Nq], 4-byte aligned; written (natural
 *             log of the sum of exp of the scaled scores over allowed keys).
 *   Nq, Nk  : 1 <= Nq <= Nk.  Query row i is sequence position Nk - Nq + i
 *             (the last Nq positions); with Nq == Nk this is fa2_fwd.
 *   B, H    : >= 1 with B*H <= 65535.
 *   d       : 32, 64, 96, 128 or 256 (others -> FA2_ERR_UNSUPPORTED).
 *   causal  : 0 = every key; non-zero = key j allowed for query row i only if
 *             j <= Nk - Nq + i.
 *   scale   : finite and > 0.
 *   n_splits: number of key ranges; 0 lets the library choose: the fewest
 *             ranges that give at least 0.8 x (SM count) CTAs, keeping at
 *             least 4 key tiles per range.  A request is capped at 128 and at
 *             the number of 128-key tiles; fa2_fwd_splitkv_splits returns the
 *             count used.
 *   workspace, workspace_bytes: caller-owned device buffer, 256-byte aligned,
 *             of at least fa2_fwd_splitkv_workspace_bytes(...) bytes (same
 *             sizes and n_splits), holding the fp32 partial outputs and
 *             logsumexps between the two kernels.  It must not overlap any
 *             other argument.  Concurrent calls need separate workspaces.
 *             With a single range the kernel writes o and lse itself, no
 *             merge runs, the required size is 0 and workspace may be NULL.
 *   stream  : cudaStream_t as void*; the kernels are queued on it.
 * Argument errors are reported before anything is launched; kernel-side
 * timeouts through fa2_sync_status.  The library allocates nothing.
 */
int fa2_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                    int d, int causal, float scale, int n_splits, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Test hook for the failure path of fa2_fwd_splitkv (same arguments, plus
 * `timeout_ns`, 1 .. 2e9): the range kernel runs with its query load withheld,
 * so its waits run out after `timeout_ns` nanoseconds; with two or more key
 * ranges the merge kernel still runs after it, on the unspecified partials.
 * Every CTA records the time-out, drains its own copies and MMAs, releases
 * tensor memory and returns; fa2_sync_status returns FA2_ERR_TIMEOUT.
 * Outputs are unspecified.  Covers the quarter mode (Nq <= 32) as well.
 */
int fa2_fwd_splitkv_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                   int Nq, int Nk, int d, int causal, float scale, int n_splits, void* workspace,
                                   size_t workspace_bytes, unsigned long long timeout_ns, void* stream);

/* Key ranges fa2_fwd_splitkv uses for these sizes and request (0 on bad sizes). */
int fa2_fwd_splitkv_splits(int B, int H, int Nq, int Nk, int d, int n_splits);

/*
 * Workspace bytes fa2_fwd_splitkv needs for these sizes and request: 0 when a
 * single range is used (no workspace needed) and 0 on bad sizes, which
 * fa2_fwd_splitkv_splits tells apart (it returns 0 only on bad sizes).
 */
size_t fa2_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_splits);

/*
 * Backward pass of exact attention: the gradients dQ, dK, dV for an upstream
 * gradient dO, given the forward's inputs, its output O and its LSE (iplexlaw
 * blog "FlashAttention-2: making long-context attention run efficiently on
 * GPUs", section "Tiling preserves the attention calculation": outputs and
 * gradients are compared with tolerances).  With P = exp(scale*QK^T - LSE):
 *     D = rowsum(dO o O), dV = P^T dO, dS = P o (dO V^T - D),
 *     dQ = scale * dS K,  dK = scale * dS^T Q.
 * P is recomputed tile by tile from LSE; the N x N matrices never reach
 * device memory.
 *
 *   q, k, v, o, dout : device pointers, bf16 [B,H,N,d], contiguous,
 *                      16-byte aligned (o and lse as written by fa2_fwd with
 *                      the same q, k, v, causal and scale).
 *   lse     : device pointer, fp32 [B,H,N], natural log, 4-byte aligned.
 *   dq, dk, dv : device pointers, bf16 [B,H,N,d]; written.  They must not
 *             overlap each other, the inputs or the workspace.
 *   B, H, N, d, causal, scale : as for fa2_fwd (d 32, 64, 96, 128 or 256;
 *             scale > 0).
 *   workspace, workspace_bytes : caller-owned device buffer, 256-byte
 *             aligned, of at least fa2_bwd_workspace_bytes(B,H,N,d) bytes;
 *             it carries per-row -LSE*log2(e) and rowsum(dO o O) from the
 *             first kernel to the second.  Concurrent calls need separate
 *             workspaces.
 *   stream  : cudaStream_t as void*; two kernels are queued on it (three
 *             at d = 256: the dQ kernel streams 64-key tiles, and dV and dK
 *             are computed by two passes over 64-query tiles, since their
 *             accumulators and the two score tiles exceed tensor memory).
 * Argument errors are reported before anything is launched; kernel-side
 * timeouts through fa2_sync_status.
 */
int fa2_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
            void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
            size_t workspace_bytes, void* stream);

/* Workspace bytes fa2_bwd needs for this shape (0 on bad sizes). */
size_t fa2_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Test hook for the failure path of fa2_bwd (same arguments, plus `kernel`
 * and `timeout_ns`, 1 .. 2e9).  kernel = 0: the dQ kernel runs with its Q/dO
 * tile load withheld; kernel = 1: the dK/dV kernel runs with its K/V tile load
 * withheld (both passes at d = 256).  That kernel's waits run out after `timeout_ns`; it records the
 * time-out, drains its own copies and MMAs, releases tensor memory and
 * returns; the other kernel runs normally.  fa2_sync_status returns
 * FA2_ERR_TIMEOUT.  Gradients are unspecified.  kernel outside {0, 1} ->
 * FA2_ERR_INVALID_ARG.
 */
int fa2_bwd_inject_timeout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal,
                           float scale, void* workspace, size_t workspace_bytes, int kernel,
                           unsigned long long timeout_ns, void* stream);

/*
 * fa2_fwd_splitkv without a workspace argument, for callers that cannot
 * allocate device memory: a plug-in running inside a host application whose
 * memory pool owns the whole device (a serving process or a framework's
 * caching allocator), where a direct cudaMalloc would bypass that pool or be
 * refused, and latency-critical loops where an allocation could stall the
 * device.  The pages have no counterpart: this is a property of the library,
 * not of the method.
 *
 * Arguments, layout and results are those of fa2_fwd_splitkv.  The partial
 * outputs go to a scratch array inside the library (a file-scope device
 * array of FA2_SPLITKV_STATIC_SCRATCH_BYTES = 16 MiB that every GPU which
 * loads the library holds until the process exits).  The library allocates
 * nothing on this path: no cudaMalloc, no cudaFree, no allocating library
 * call.
 *
 *   - A request whose partials need more than 16 MiB (see
 *     fa2_fwd_splitkv_workspace_bytes) returns FA2_ERR_INVALID_ARG before
 *     anything is launched; fewer key ranges need less, and one range needs
 *     none.
 *   - The first call on each device that needs the scratch looks up the
 *     array's device address there (cudaGetSymbolAddress) and caches it;
 *     make that first call before any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents.
 *     Nothing in it has to start at zero (each call writes every partial
 *     before its merge reads it), but calls that overlap on the GPU (on other
 *     streams or from other host threads) race on it: serialise them.
 */
#define FA2_SPLITKV_STATIC_SCRATCH_BYTES (16u << 20)
int fa2_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                           int Nk, int d, int causal, float scale, int n_splits, void* stream);

/* Static description of a status code. */
const char* fa2_strerror(int status);

/* Detail of the most recent failure on the calling host thread ("" if none). */
const char* fa2_last_error_detail(void);

/* Library ABI version (major * 100 + minor). */
int fa2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA2_H_ */
