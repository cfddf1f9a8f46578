// decode.cuh -- K5: one recurrent decode step of the gated delta rule, in place.
//
// For every head (b, h), with D = Diag(alpha):
//   r = (D S)^T b,  p = (D S)^T q          two reductions over the key dimension
//   u = w - r                              error of the read against the write vector
//   o = p + u (a . q)                      = S_new^T q
//   S <- D S + a u^T                       = (I - a b^T) D S + a w^T
// with the write key a = b, or a = s (.) b under OSDN's per-feature write-side key scaling
// (OSDN summary page, "Method").
// DeltaNet page, steps 3-6 (read, error, rank-1 write, output from the
// updated state); FG2-GDN page, section 2 (decay first, sqrt(beta) scaling,
// decoupled beta^v for FG2-GDN+).
//
// Memory-bound: each head's fp32 state (dk*dv*4 bytes) is read once and
// written once with coalesced accesses held in registers; the two reductions
// go through shared memory.  One CTA of 256 threads per head and slice of
// DVF/NSL value columns (NSL > 1 spreads a small batch over more SMs; a value
// column's reductions, error and update involve that column alone, so the
// slices are independent and compute exactly what one CTA would): warp w owns
// rows w, w+8, ...; lane l owns DVF/(32 NSL) consecutive columns of the slice.
#pragma once
#include "common.cuh"

namespace dr {

template <int CPL> struct VecF;
template <> struct VecF<4> { using T = float4; };
template <> struct VecF<2> { using T = float2; };
template <> struct VecF<1> { using T = float; };

template <typename IO, int DK, int DVF, int NSL = 1>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                   const float *__restrict__ alpha, int alpha_mode, const float *__restrict__ beta_k,
                   int beta_k_mode, const float *__restrict__ beta_v, int beta_v_mode,
                   const float *__restrict__ s_scale, float *__restrict__ S, IO *__restrict__ o) {
  constexpr int NW = 8;
  constexpr int RPW = DK / NW;
  constexpr int DV = DVF / NSL;  // value columns of this CTA's slice
  constexpr int CPL = DV / 32;
  using V = typename VecF<CPL>::T;
  static_assert(DK % NW == 0 && DVF % NSL == 0 && DV % 32 == 0 && CPL <= 4, "unsupported head dims");

  __shared__ float s_al[DK], s_b[DK], s_a[DK], s_q[DK], s_w[DV], s_u[DV];
  __shared__ float s_red_r[NW][DV], s_red_p[NW][DV];
  __shared__ float s_bq;

  const size_t bh = blockIdx.x / NSL;  // token-head index b*H + h (T == 1)
  const int v0 = static_cast<int>(blockIdx.x % NSL) * DV;  // first value column of the slice
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float *Sh = S + bh * DK * DVF + v0;

  // 1. issue the state loads first so they are in flight while the factors are formed
  float s[RPW][CPL];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = warp + rr * NW;
    V x = __ldcs(reinterpret_cast<const V *>(Sh + i * DVF + lane * CPL));
    const float *xf = reinterpret_cast<const float *>(&x);
#pragma unroll
    for (int c = 0; c < CPL; ++c) s[rr][c] = xf[c];
  }

  // 2. per-row factors: decay, erase key b = sqrt(beta_k) k, write key a, query; write vector w
  if (tid < DK) {
    const float bk = gate_at(beta_k, beta_k_mode, bh, DK, tid);
    const float bt = sqrtf(bk) * to_f32(k[bh * DK + tid]);
    s_b[tid] = bt;
    s_a[tid] = s_scale ? s_scale[bh * DK + tid] * bt : bt;
    s_q[tid] = to_f32(q[bh * DK + tid]);
    s_al[tid] = gate_at(alpha, alpha_mode, bh, DK, tid);
  }
  if (tid >= 128 && tid - 128 < DV) {
    const int j = tid - 128, jg = v0 + j;
    const float vj = to_f32(v[bh * DVF + jg]);
    const float ws = (beta_v_mode != MODE_ABSENT) ? gate_at(beta_v, beta_v_mode, bh, DVF, jg)
                                                  : sqrtf(gate_at(beta_k, beta_k_mode, bh, DK, jg));
    s_w[j] = ws * vj;
  }
  __syncthreads();
  if (warp == 0) {
    float acc = 0.f;
    for (int i = lane; i < DK; i += 32) acc += s_a[i] * s_q[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) s_bq = acc;
  }

  // 3. decay in registers and the two partial reductions over this warp's rows
  float r[CPL], p[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) r[c] = p[c] = 0.f;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = warp + rr * NW;
    const float al = s_al[i], bi = s_b[i], qi = s_q[i];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      s[rr][c] *= al;
      r[c] = fmaf(s[rr][c], bi, r[c]);
      p[c] = fmaf(s[rr][c], qi, p[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    s_red_r[warp][lane * CPL + c] = r[c];
    s_red_p[warp][lane * CPL + c] = p[c];
  }
  __syncthreads();

  // 4. finish the reductions; error u and output o per value column
  if (tid < DV) {
    float rs = 0.f, ps = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      rs += s_red_r[w][tid];
      ps += s_red_p[w][tid];
    }
    const float u = s_w[tid] - rs;
    s_u[tid] = u;
    o[bh * DVF + v0 + tid] = from_f32<IO>(fmaf(u, s_bq, ps));
  }
  __syncthreads();

  // 5. rank-1 write and in-place store of the new state
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = warp + rr * NW;
    const float ai = s_a[i];
    V x;
    float *xf = reinterpret_cast<float *>(&x);
#pragma unroll
    for (int c = 0; c < CPL; ++c) xf[c] = fmaf(ai, s_u[lane * CPL + c], s[rr][c]);
    __stcs(reinterpret_cast<V *>(Sh + i * DVF + lane * CPL), x);
  }
}

}  // namespace dr
