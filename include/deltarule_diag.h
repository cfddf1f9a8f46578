/*
 * deltarule_diag.h -- diagnostic entry points of libdeltarule (not part of the
 * operation itself; the pages have no counterpart).  They run a named kernel
 * in place of the library's choice, so that the kernels can be compared on the
 * same problem, exercise the tensor-core building blocks of the prefill kernel
 * in isolation so that a layout or descriptor fault is found before it hides
 * inside the full kernel, and run the kernels' bounded waits out on purpose.
 */
#ifndef DELTARULE_DIAG_H
#define DELTARULE_DIAG_H

#include <stddef.h>

#include "deltarule.h"

#ifndef DR_API
#if defined(__GNUC__)
#define DR_API __attribute__((visibility("default")))
#else
#define DR_API
#endif
#endif

#ifdef __cplusplus
extern "C" {
#endif

/*
 * dr_chunk_fwd through a named kernel instead of the library's choice, so
 * that the kernels can be compared with one another on the same problem:
 *   variant 0  the library's choice (what dr_chunk_fwd runs)
 *   variant 1  the tensor-core kernel with one CTA per 64-column value slice
 *              (bf16 I/O, dk = 128, chunk 64, dv a multiple of 64); the
 *              library's choice for such shapes when dv != 128
 *   variant 2  the CUDA-core kernel (every supported shape; the library's
 *              choice for fp32 I/O and for chunk 16 and 32)
 *   variant 3  the two-CTA cluster kernel (bf16 I/O, dk = dv = 128, chunk
 *              64); the library's choice for such shapes with more heads
 *              than resident four-CTA clusters
 *   variant 4  the four-CTA cluster kernel (same shapes); the library's
 *              choice for them otherwise
 * Arguments, layouts, ownership and errors are those of dr_chunk_fwd, with
 * a workspace of dr_diag_chunk_fwd_workspace(variant, p) bytes; a variant
 * that cannot take the problem returns DR_ERR_UNSUPPORTED before anything
 * is enqueued.  Every variant computes the same operation.
 */
DR_API size_t dr_diag_chunk_fwd_workspace(int variant, const dr_problem *p);
DR_API int dr_diag_chunk_fwd_variant(int variant, const dr_problem *p, const void *q, const void *k,
                                     const void *v, const float *alpha, const float *beta_k,
                                     const float *beta_v, const float *S0, void *o, float *S_T,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * dr_decode_step (s == NULL) or dr_decode_step_osdn (s != NULL) through a
 * named kernel:
 *   variant 0  the library's choice
 *   variant 1  one CTA per head
 *   variant 2  four CTAs per head, 32 value columns each (dk = dv = 128)
 *   variant 3  the persistent streaming kernel, two CTAs per SM, the next
 *              head's state copied ahead into shared memory (dk = dv = 128)
 * All variants perform the same operations in the same order per value
 * column, so they give the same bits.  Arguments and errors as in
 * dr_decode_step; an unsupported variant returns DR_ERR_UNSUPPORTED.
 */
DR_API int dr_diag_decode_step_variant(int variant, const dr_problem *p, const void *q, const void *k,
                                       const void *v, const float *alpha, const float *beta_k,
                                       const float *beta_v, const float *s, float *S, void *o,
                                       void *stream);

/*
 * dr_backward through a named kernel instead of the library's choice:
 *   variant 0  the library's choice (what dr_backward runs)
 *   variant 1  the token-sequential kernel (fp32 arithmetic throughout; every
 *              supported shape; the library's choice for fp32 I/O and for
 *              head sizes other than dk = dv = 128)
 *   variant 2  the chunkwise kernel on the tensor cores (bf16 I/O, dk = dv =
 *              128): a forward pass that keeps the state at the start of every
 *              chunk, then the chunks from the last to the first
 * Arguments, layouts and errors are those of dr_backward; the workspace must
 * hold dr_diag_backward_workspace(variant, p) bytes.  An unsupported variant
 * returns DR_ERR_UNSUPPORTED before anything is enqueued.
 */
DR_API size_t dr_diag_backward_workspace(int variant, const dr_problem *p);
DR_API int dr_diag_backward_variant(int variant, const dr_problem *p, const void *q, const void *k,
                                    const void *v, const float *alpha, const float *beta_k,
                                    const float *beta_v, const float *s, const float *S0,
                                    const void *dout, const float *dS_T, float *dq, float *dk,
                                    float *dv, float *dalpha, float *dbeta_k, float *dbeta_v,
                                    float *ds, float *dS0, void *workspace, size_t workspace_bytes,
                                    void *stream);

/*
 * D[128 x N] = A[128 x K] * B[K x N] on one CTA through tcgen05.mma (16-bit
 * inputs: bf16 if bf16 != 0, else fp16; fp32 accumulate), with A staged
 * K-major (a_mn = 0) or MN-major (a_mn = 1)
 * and B staged K-major (b_mn = 0) or MN-major (b_mn = 1) in 128-byte-swizzled
 * shared memory, the result read back from tensor memory.
 * A, B: row-major 16-bit device buffers; D: row-major fp32 device buffer;
 * workspace: >= 256 bytes of device memory (status word, same meaning as in
 * dr_workspace_status).  N, K in {64, 128}.  Returns a dr_status code.
 */
DR_API int dr_diag_umma_selftest(int N, int K, int a_mn, int b_mn, int bf16, const void *A, const void *B,
                                 float *D, void *workspace, void *stream);

/*
 * T = (I + A)^-1 for the strictly lower-triangular part of a 64 x 64 matrix A
 * (the UT transform of one chunk), computed by one of the prefill kernels'
 * warp-MMA routines (fp16 operands, fp32 accumulation):
 *   variant 0  the ring prefill's (operands in its swizzled tile layout,
 *              result kept in registers)
 *   variant 1  the one-CTA prefill's (padded row-major arrays)
 * A: row-major fp32 device buffer (its diagonal and upper part are ignored);
 * T: row-major fp32 device buffer that the caller zeroes first (only the lower
 * blocks are written).  Returns a dr_status code (DR_ERR_INVALID_ARG for an
 * unknown variant).
 */
DR_API int dr_diag_tri_inverse(int variant, const float *A, float *T, void *stream);

/*
 * The bounded waits of the prefill kernels, run out on purpose: every CTA waits
 * on an mbarrier that nothing completes, through the prefill kernels' own wait
 * helpers (cluster_scope = 0: one CTA, CTA-scope wait; cluster_scope != 0: a
 * cluster of two CTAs, cluster-scope acquire).  Each wait gives up after
 * limit_ns of wall time (0 < limit_ns <= 1e9, else DR_ERR_INVALID_ARG), sets the
 * timeout bit of the status word in `workspace` (>= 256 bytes of device memory;
 * dr_workspace_status then returns DR_ERR_TIMEOUT) and stores the nanoseconds
 * it waited in waited_ns[cta] (device buffer of 2 entries, or NULL).  The
 * kernel exits normally and the context stays usable.  Asynchronous on
 * `stream`; returns a dr_status code for the launch.
 */
DR_API int dr_diag_wait_timeout(int cluster_scope, unsigned long long limit_ns, void *workspace,
                                unsigned long long *waited_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DELTARULE_DIAG_H */
