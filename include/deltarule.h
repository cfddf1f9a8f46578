/*
 * deltarule.h -- C ABI of the gated delta-rule forward pass on NVIDIA B200 (sm_100a).
 *
 * The operation (one independent recurrence per batch row b and head h):
 *
 *   b_t = sqrt(beta_k_t) (.) k_t                              erase key
 *   w_t = beta_v_t (.) v_t   if beta_v is given,
 *         sqrt(beta_k_t) (.) v_t   otherwise                  write vector
 *   S_t = (I - b_t b_t^T) Diag(alpha_t) S_{t-1} + b_t w_t^T   S_t in R^{dk x dv}, fp32
 *   o_t = S_t^T q_t                                           output (no 1/sqrt(d) scale)
 *
 * Sources of each part:
 *   - DeltaNet page (robocikowo.com "DeltaNet"), numbered steps 1-6: per-token
 *     q, k, v and a learning rate beta in (0, 1]; read the state with the key,
 *     error beta (v - read), rank-1 write, output read from the updated
 *     state.  That page writes the state transposed (dv x dk); here S is
 *     dk x dv and reads are S^T x.
 *   - FG2-GDN page (gist.science), section 1: Gated DeltaNet's scalar forget
 *     factor alpha_t and KDA's channel-wise alpha_t in R^{dk}.
 *   - FG2-GDN page, section 2 "Kerninnovation": channel-wise beta_t in R^{dk},
 *     k~ = sqrt(beta) (.) k, v~ = sqrt(beta) (.) v and the update
 *     S_t = (I - k~ k~^T) Diag(alpha_t) S_{t-1} + k~ v~^T.
 *   - FG2-GDN page, section 2 "Erweiterung: FG2-GDN+": decoupled erase
 *     strength beta^k and write strength beta^v (write vector beta^v (.) v).
 *   - DeltaNet page, step 7 and the remarks on Householder-product
 *     representations: training/prefill runs chunkwise over the sequence with
 *     the WY/UT form on tensor cores; inference uses the recurrent form.
 *
 * Layouts (row-major, contiguous, caller-owned device memory):
 *   q, k : [B, T, H, dk]  in io_dtype       v : [B, T, H, dv]  in io_dtype
 *   o    : [B, T, H, dv]  in io_dtype
 *   alpha  : NULL (alpha = 1), [B, T, H] (DR_SCALAR) or [B, T, H, dk] (DR_CHANNEL), fp32
 *   beta_k : [B, T, H] (DR_SCALAR) or [B, T, H, dk] (DR_CHANNEL), fp32
 *   beta_v : NULL (symmetric write, sqrt(beta_k) (.) v), [B, T, H] or [B, T, H, dv], fp32
 *   S0, S_T, S : [B, H, dk, dv] fp32.  S0 == NULL means a zero initial state.
 * The symmetric channel-wise form (beta_v == NULL, beta_k channel-wise) needs dk == dv.
 * Every pointer must be 16-byte aligned.
 *
 * Supported sizes: dk, dv in {64, 128}; chunk in {16, 32, 64}; T >= 0 (a
 * partial last chunk is handled); B, H >= 1; for the prefill B, H <= 65535
 * (they index a launch grid's y and z), and for the decode B * H < 2^31.
 *
 * Ownership and threading: the caller owns every buffer; the library
 * allocates no device memory and keeps no state between calls.  All work is
 * enqueued on the caller's stream (a cudaStream_t passed as void*, NULL = the
 * legacy default stream); no call synchronises.  S_T may alias S0.
 *
 * Errors: argument checks run on the host before anything is enqueued and
 * return DR_ERR_INVALID_ARG / DR_ERR_UNSUPPORTED / DR_ERR_ALIGNMENT /
 * DR_ERR_WORKSPACE; a failed launch returns DR_ERR_CUDA.  Conditions found on
 * the device (a chunk whose cumulative decay leaves the representable range,
 * or a bounded wait that expired) are recorded in the workspace status word
 * and read back with dr_workspace_status() after the caller's stream has
 * been synchronised.
 */
#ifndef DELTARULE_H
#define DELTARULE_H

#include <stddef.h>
#include <stdint.h>

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

typedef enum {
  DR_OK = 0,
  DR_ERR_INVALID_ARG = 1,   /* NULL required pointer, negative size, mode/shape mismatch */
  DR_ERR_UNSUPPORTED = 2,   /* valid but not implemented: sizes outside the lists above */
  DR_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
  DR_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than the entry point needs (see its comment) */
  DR_ERR_RANGE = 5,         /* device: cumulative decay inside a chunk below the factorised range */
  DR_ERR_TIMEOUT = 6,       /* device: a bounded wait expired; outputs are invalid */
  DR_ERR_CUDA = 7           /* a CUDA runtime call or kernel launch failed */
} dr_status;

typedef enum { DR_F32 = 0, DR_BF16 = 1 } dr_dtype;

typedef enum { DR_ABSENT = 0, DR_SCALAR = 1, DR_CHANNEL = 2 } dr_mode;

typedef struct {
  int B, T, H;          /* batch, sequence length (tokens), heads */
  int dk, dv;           /* key and value head dimensions */
  int chunk;            /* chunk length C of the WY/UT form (prefill only) */
  dr_dtype io_dtype;    /* dtype of q, k, v, o */
  dr_mode alpha_mode;   /* DR_ABSENT, DR_SCALAR or DR_CHANNEL (per key channel) */
  dr_mode beta_k_mode;  /* DR_SCALAR or DR_CHANNEL (per key channel) */
  dr_mode beta_v_mode;  /* DR_ABSENT, DR_SCALAR or DR_CHANNEL (per value channel) */
} dr_problem;

/*
 * Bytes of device workspace dr_chunk_fwd needs for problem p: the status word
 * (256 bytes), plus, when the library runs the four-CTA prefill (bf16, dk =
 * dv = 128, chunk 64, and no more heads B*H than clusters of four CTAs the
 * GPU holds at once), 266,240 bytes per (b, h) where it stages each chunk's
 * factor block.  0 if p is invalid.
 */
DR_API size_t dr_chunk_fwd_workspace(const dr_problem *p);

/*
 * Chunkwise prefill: all T tokens of every (b, h), starting from S0, writing
 * o_t for every token and the final state S_T.  Computed with the chunkwise
 * WY/UT (Householder-product) form: per chunk of C tokens the cumulative
 * gate, the UT transform T = (I + strictly-lower(B^ A^T))^-1, the serial
 * inter-chunk state pass in fp32 and the intra-chunk output (DeltaNet page,
 * step 7; FG2-GDN page, section 2, DPLR/WY remark).
 * workspace: device memory of at least dr_chunk_fwd_workspace(p) bytes,
 * reused across calls on the same stream; its status word is reset at the
 * start of every call.  A workspace that holds the status word but not the
 * four-CTA prefill's staging runs the two-CTA prefill instead (the same
 * operation; slower on batches with few heads).
 */
DR_API dr_status dr_chunk_fwd(const dr_problem *p,
                       const void *q, const void *k, const void *v,
                       const float *alpha, const float *beta_k, const float *beta_v,
                       const float *S0, void *o, float *S_T,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * One recurrent decode step for every (b, h) (DeltaNet page, steps 3-6 and
 * "inference uses the recurrent form"): reads S, writes the updated state
 * back into S in place and the output o.  p->T must be 1; p->chunk is
 * ignored.  q, k, v, o use the [B, 1, H, d] layouts above.
 */
DR_API dr_status dr_decode_step(const dr_problem *p,
                         const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta_k, const float *beta_v,
                         float *S, void *o, void *stream);

/*
 * OSDN per-feature write-side key scaling (OSDN summary page, "Method": the
 * diagonal preconditioner scales the key of the write while the read keeps
 * the erase key).  Same as dr_chunk_fwd / dr_decode_step, with the
 * transition S_t = (I - a_t b_t^T) Diag(alpha_t) S_{t-1} + a_t w_t^T, i.e.
 *   u_t = w_t - (Diag(alpha_t) S_{t-1})^T b_t,   S_t = Diag(alpha_t) S_{t-1} + a_t u_t^T,
 * where b_t = sqrt(beta_k_t) (.) k_t is the erase (read) key and
 * a_t = s_t (.) b_t the write key.
 *   s : [B, T, H, dk] fp32 (decode: [B, 1, H, dk]), 16-byte aligned, caller
 *       owned, read only.  NULL gives a = b, the same result as
 *       dr_chunk_fwd / dr_decode_step.
 * The preconditioner's own update rule is not part of the operation: s is
 * an input.  Every other argument, layout, the workspace and the errors are
 * those of dr_chunk_fwd / dr_decode_step.  With s, a bf16 prefill with
 * dk = dv = 128 and chunk 64 runs the tensor-core ring kernel whatever
 * DR_PREFILL_KERNEL says; other shapes run the CUDA-core kernel.
 */
DR_API dr_status dr_chunk_fwd_osdn(const dr_problem *p,
                                   const void *q, const void *k, const void *v,
                                   const float *alpha, const float *beta_k, const float *beta_v,
                                   const float *s, const float *S0, void *o, float *S_T,
                                   void *workspace, size_t workspace_bytes, void *stream);
DR_API dr_status dr_decode_step_osdn(const dr_problem *p,
                                     const void *q, const void *k, const void *v,
                                     const float *alpha, const float *beta_k, const float *beta_v,
                                     const float *s, float *S, void *o, void *stream);

/*
 * Packed variable-length batch: the chunkwise prefill of several sequences of
 * different lengths laid end to end, each an independent recurrence from its
 * own initial state.  The DeltaNet page's deployment setting (a chunkwise pass
 * over each prompt, then constant-state recurrent steps) in serving form: after
 * this call, dr_decode_step / dr_decode_step_osdn with B = number of sequences
 * continue every sequence from its row of S_T.
 *   p->B        number of sequences N;  p->T  total tokens Ttot of the packed arrays
 *   cu_seqlens  device int32 [N + 1], 4-byte aligned, cu[0] = 0, non-decreasing,
 *               cu[N] = Ttot: sequence n is tokens cu[n] .. cu[n+1]-1.  Empty
 *               sequences are allowed (their S_T is their S0).  Offsets are
 *               clamped to [0, Ttot] on the device, so malformed ones give wrong
 *               results but never an out-of-range access.
 *   q, k, o     [1, Ttot, H, dk|dv] (the dense layout with B = 1); v likewise
 *   alpha, beta_k, beta_v, s   [1, Ttot, H] or [1, Ttot, H, d] as in dr_chunk_fwd
 *               (s: the OSDN write-side key scale, or NULL)
 *   S0, S_T     [N, H, dk, dv] fp32, one state per sequence (S0 NULL: zero)
 * Workspace, stream, dtypes, chunk sizes and errors are those of dr_chunk_fwd;
 * cu_seqlens NULL returns DR_ERR_INVALID_ARG.  bf16 with dk = dv = 128 and
 * chunk 64 runs the tensor-core ring kernel, other shapes the CUDA-core kernel.
 */
DR_API dr_status dr_chunk_fwd_varlen(const dr_problem *p, const int *cu_seqlens,
                                     const void *q, const void *k, const void *v,
                                     const float *alpha, const float *beta_k, const float *beta_v,
                                     const float *s, const float *S0, void *o, float *S_T,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * Affine state maps, for a sequence split into consecutive segments (the
 * chunkwise form's linearity in the state, DeltaNet page step 7 / FG2-GDN
 * page section 2).  A segment maps its initial state to
 * its final state as S_out = M S_in + N: N is the segment's final state from a
 * zero initial state (dr_chunk_fwd with S0 = NULL), and M (dk x dk) its final
 * state when the write vectors are zero and S0 = I (dr_chunk_fwd with v = 0,
 * beta_v = NULL and dv = dk).  This call applies such maps to n independent
 * heads:  out_h = M_h S_h + N_h.
 *   M   [n, dk, dk] fp32;  S [n, dk, dv] fp32 or NULL (zero);  N, out [n, dk, dv] fp32
 *   dk in {64, 128}, dv a multiple of 32, n <= 65535; all 16-byte aligned device
 *   pointers; out may be N but not S.  Asynchronous on `stream`.
 */
DR_API dr_status dr_state_map_apply(int n, int dk, int dv, const float *M, const float *S, const float *N,
                                    float *out, void *stream);

/*
 * Backward pass: the gradients of
 *   L = sum(dout (.) o) + sum(dS_T (.) S_T)
 * with respect to every input of dr_chunk_fwd / dr_chunk_fwd_osdn, for the
 * forward defined by the recurrence (DeltaNet page steps 3-6; FG2-GDN page
 * section 2; OSDN summary "Method").  Reverse mode through
 *   X = Diag(alpha_t) S_{t-1},  u = w_t - X^T b_t,  S_t = X + a_t u^T,  o_t = S_t^T q_t.
 * The pass recomputes the forward itself (it keeps the state every 16 tokens in
 * the workspace and re-derives the states in between), so it takes the
 * forward's inputs, not its outputs.
 *   inputs   as dr_chunk_fwd_osdn (s may be NULL); p->chunk is ignored
 *   dout     [B,T,H,dv] in the I/O dtype;  dS_T [B,H,dk,dv] fp32 or NULL (zero)
 *   outputs  fp32, caller owned, overwritten:
 *            dq, dk [B,T,H,dk];  dv [B,T,H,dv];
 *            dalpha, dbeta_k, dbeta_v, ds in the shape of alpha, beta_k, beta_v, s
 *            (each non-NULL exactly when its input is given; dbeta_k always);
 *            dS0 [B,H,dk,dv] or NULL (not wanted).  A gate's gradient at beta = 0
 *            is reported as 0 (the square root has no derivative there).
 *   workspace >= dr_backward_workspace(p) bytes, 16-byte aligned, device memory
 *            (fp32 state checkpoints and per-head recomputation scratch; for
 *            the chunkwise kernel, also the four-CTA prefill's factor staging
 *            when its first pass runs on that kernel).
 * dk, dv in {64, 128}; fp32 or bf16 I/O.  Asynchronous on `stream`.  Errors as
 * dr_chunk_fwd, plus DR_ERR_INVALID_ARG for a missing or extra gradient buffer.
 */
DR_API size_t dr_backward_workspace(const dr_problem *p);
DR_API dr_status dr_backward(const dr_problem *p,
                             const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta_k, const float *beta_v,
                             const float *s, const float *S0, const void *dout, const float *dS_T,
                             float *dq, float *dk, float *dv, float *dalpha, float *dbeta_k,
                             float *dbeta_v, float *ds, float *dS0,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * dr_chunk_fwd for callers that cannot allocate device memory.  (The pages
 * have no counterpart; this is a deployment variant of dr_chunk_fwd.)  Some
 * hosts pre-plan every byte of device memory and give a kernel no workspace
 * hook -- plugin interfaces of inference runtimes, memory-budgeted serving
 * loops -- and some loops cannot afford cudaMalloc/cudaFree at all, since
 * cudaFree synchronises the device and cudaMalloc may.  This entry point
 * takes the same inputs and outputs as dr_chunk_fwd but no workspace: the
 * scratch dr_chunk_fwd would keep in the workspace (its device status word)
 * lives in a file-scope device array of 4096 bytes inside the library, which
 * every GPU that loads the library holds until the process exits.  Where
 * dr_chunk_fwd would pick the four-CTA prefill, whose factor staging does not
 * fit in that array, this call runs the two-CTA prefill, which needs the
 * status word only; it computes the same operation.  The call allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).
 * Device and set-up: the GPU used is the current device, which must be the
 * device of `stream` and the device that holds q; a q on another device is
 * refused with DR_ERR_INVALID_ARG.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) and caches it for the
 * life of the process; make that first call before any stream capture, and
 * after the last cudaDeviceReset of that device (a reset reloads the library's
 * device code, and the cached address would then be stale).
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents; each call clears the status word on its own stream before
 * its kernel runs.  Calls whose work overlaps on the GPU (several streams, or
 * several host threads) race on that word, so its device-side status is only
 * meaningful for calls that do not overlap.  Read it with dr_noalloc_status().
 */
DR_API dr_status dr_chunk_fwd_noalloc(const dr_problem *p,
                                      const void *q, const void *k, const void *v,
                                      const float *alpha, const float *beta_k, const float *beta_v,
                                      const float *S0, void *o, float *S_T, void *stream);

/*
 * Device status of the last dr_chunk_fwd_noalloc call on the current device
 * (the pages have no counterpart): synchronises `stream`, then reads the
 * status word from the library's static array and returns DR_OK,
 * DR_ERR_RANGE (a chunk's cumulative decay left the factorised range) or
 * DR_ERR_TIMEOUT (a bounded device wait expired).  Allocates nothing.
 * Returns DR_ERR_INVALID_ARG if dr_chunk_fwd_noalloc has not run on the
 * current device yet, DR_ERR_CUDA if the copy fails.  Like the entry point,
 * it reports the last call only when calls do not overlap on the GPU.
 */
DR_API dr_status dr_noalloc_status(void *stream);

/*
 * Synchronises `stream`, then reads the status word a previous dr_chunk_fwd
 * left in `workspace` (DR_OK, DR_ERR_RANGE or DR_ERR_TIMEOUT).  Returns
 * DR_ERR_CUDA if the copy fails.
 */
DR_API dr_status dr_workspace_status(const void *workspace, void *stream);

/* Static, human-readable name of a status code. */
DR_API const char *dr_status_string(dr_status s);

/* Library ABI version (major * 100 + minor). */
DR_API int dr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DELTARULE_H */
