/*
 * deltarule_diag.h -- diagnostic entry points of libdeltarule (not part of the
 * operation itself; the pages have no counterpart).  They exercise the
 * tensor-core building blocks of the prefill kernel in isolation so that a
 * layout or descriptor fault is found before it hides inside the full kernel.
 */
#ifndef DELTARULE_DIAG_H
#define DELTARULE_DIAG_H

#include <stddef.h>

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
 * (the UT transform of one chunk), computed by the warp-MMA routine of the
 * prefill kernel (fp16 operands, fp32 accumulation).  A: row-major fp32 device
 * buffer (its diagonal and upper part are ignored); T: row-major fp32 device
 * buffer that the caller zeroes first (only the lower blocks are written).
 * Returns a dr_status code.
 */
DR_API int dr_diag_tri_inverse(const float *A, float *T, void *stream);

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
