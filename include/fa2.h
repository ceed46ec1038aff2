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
  FA2_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (e.g. d not in {64,128}) */
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
 *   B, H, N : >= 1; B <= 65535, H <= 65535.  Any N >= 1 (a ragged last tile
 *             is masked).
 *   d       : head dimension, 64 or 128 (others -> FA2_ERR_UNSUPPORTED).
 *   causal  : 0 = every key; non-zero = key j allowed only for query i >= j.
 *   scale   : multiplier of q.k (finite; the usual choice is 1/sqrt(d)).
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
 * the device copies.  Returns FA2_ERR_TIMEOUT if the kernel reported a
 * timeout.
 */
int fa2_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace fa2_fwd_host needs for this shape (0 on bad sizes). */
size_t fa2_fwd_host_workspace_bytes(int B, int H, int N, int d);

/*
 * Synchronise `stream`, then read and clear the device status word.  Returns
 * FA2_ERR_TIMEOUT if any kernel launched since the last call gave up a bounded
 * wait, FA2_ERR_CUDA if the synchronisation failed, else FA2_OK.
 */
int fa2_sync_status(void* stream);

/*
 * Test hook for the failure path: launch the attention kernel (same
 * arguments as fa2_fwd) with the query-tile load withheld, so every wait on it
 * runs out after `timeout_ns` nanoseconds.  The kernel then sets the status
 * word and exits cleanly (tensor memory released, no copy left in flight);
 * fa2_sync_status returns FA2_ERR_TIMEOUT.  Outputs are unspecified.
 */
int fa2_fwd_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                           int N, int d, int causal, float scale, unsigned long long timeout_ns, void* stream);

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
