// state_map.cuh -- apply affine state maps: S_out = M S_in + N for independent heads.
//
// The chunkwise recurrence is linear in the state: a stretch of tokens maps its initial state to
// its final state as S_out = M S_in + N, with M the product of the stretch's transitions (dk x dk)
// and N its final state from S_in = 0 (dk x dv).  Composing these maps over consecutive segments of
// a long sequence gives every segment its initial state, the exchange step of a sequence-parallel
// prefill.  This kernel applies one map per head, in fp32 FFMA (the work is a few MFLOP per head).
//
// Grid: (dv / 32, n); 256 threads.  The CTA stages a dk x 32 block of S_in in shared memory; thread
// t owns column t % 32 and rows t / 32 + 8 r.
#pragma once
#include "common.cuh"

namespace dr {

template <int DK>
__global__ void __launch_bounds__(256)
state_map_apply_kernel(int dv, const float *__restrict__ M, const float *__restrict__ S,
                       const float *__restrict__ N, float *__restrict__ out) {
  constexpr int RPT = DK / 8;  // rows per thread
  __shared__ float sS[DK][32];
  const int tid = threadIdx.x, j = tid & 31, i0 = tid >> 5;
  const int col = blockIdx.x * 32 + j;
  const size_t head = blockIdx.y;
  const float *Mh = M + head * DK * DK;
  const size_t sbase = head * static_cast<size_t>(DK) * dv;
  for (int m = i0; m < DK; m += 8) sS[m][j] = S ? S[sbase + static_cast<size_t>(m) * dv + col] : 0.f;
  __syncthreads();
  float acc[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) acc[r] = 0.f;
  if (S) {
#pragma unroll 4
    for (int m = 0; m < DK; ++m) {
      const float sm = sS[m][j];
#pragma unroll
      for (int r = 0; r < RPT; ++r) acc[r] = fmaf(Mh[(i0 + 8 * r) * DK + m], sm, acc[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const size_t e = sbase + static_cast<size_t>(i0 + 8 * r) * dv + col;
    out[e] = acc[r] + N[e];
  }
}

}  // namespace dr
