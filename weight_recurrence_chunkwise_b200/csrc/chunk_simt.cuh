// chunk_simt.cuh -- chunkwise WY/UT prefill on CUDA cores, fp32 arithmetic.
//
// The fp32 path: with fp32 inputs the output must match to ~1e-4 of its RMS,
// which bf16 tensor-core operands cannot give, so every product here is an
// fp32 FFMA.  Same algebra as the tensor-core kernel (DeltaNet page, step 7;
// FG2-GDN page, section 2 WY remark).  For a chunk of L <= C tokens starting
// from state S (dk x VS slice of value columns):
//
//   gamma_r = prod_{j<=r} alpha_j             cumulative gate (K1)
//   Bh_r = gamma_r b_r,  Ac_r = a_r / gamma_r,  Qh_r = gamma_r q_r
//   (write key a = b, or a = s (.) b under OSDN's write-side key scaling)
//   A = strictly-lower(Bh Ac^T),  T = (I + A)^-1,  P = lower(Qh Ac^T)   (K2)
//   U = T (Wr - Bh S)                         (K2 + K3: rows u_r of the chunk)
//   O = Qh S + P U                            (K4)
//   S <- Diag(gamma_L) (S + Ac^T U)           (K3; Ac_r gamma_L = decayed key)
//
// Grid: (dv / VS, H, B); one CTA walks all chunks of one (b, h, value slice).
#pragma once
#include "common.cuh"

namespace dr {

template <int DK, int VS, int C>
struct SimtSmem {
  static constexpr int LDK = DK + 1, LC = C + 1, LV = VS + 1;
  static constexpr size_t floats = 3 * C * LDK     // Bh, Ac, Qh
                                   + 3 * C * LC    // A, T, P
                                   + 2 * C * LV    // Wr/U, X
                                   + DK * LV       // S slice
                                   + DK;           // gamma at chunk end
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename IO, int DK, int DV, int VS, int C>
__global__ void __launch_bounds__(256)
chunk_fwd_simt_kernel(int T, int H, const IO *__restrict__ q, const IO *__restrict__ k,
                      const IO *__restrict__ v, const float *__restrict__ alpha, int alpha_mode,
                      const float *__restrict__ beta_k, int beta_k_mode, const float *__restrict__ beta_v,
                      int beta_v_mode, const float *__restrict__ s_scale, const int *__restrict__ cu_seqlens,
                      const float *__restrict__ S0, IO *__restrict__ o, float *__restrict__ S_T,
                      uint32_t *__restrict__ status) {
  using L_ = SimtSmem<DK, VS, C>;
  constexpr int LDK = L_::LDK, LC = L_::LC, LV = L_::LV;
  extern __shared__ float sm[];
  float *Bh = sm;
  float *Ac = Bh + C * LDK;
  float *Qh = Ac + C * LDK;
  float *Am = Qh + C * LDK;
  float *Tm = Am + C * LC;
  float *Pm = Tm + C * LC;
  float *Wr = Pm + C * LC;   // write vectors, then U
  float *Xm = Wr + C * LV;
  float *Ss = Xm + C * LV;
  float *gL = Ss + DK * LV;

  const int tid = threadIdx.x;
  const int v0 = blockIdx.x * VS, h = blockIdx.y, b = blockIdx.z;
  // dense batch: tokens b*T ..; packed batch: sequence b is tokens cu[b] .. cu[b+1]-1 (clamped to
  // [0, Ttot] so that malformed offsets cannot address outside the arrays)
  size_t tok0 = static_cast<size_t>(b) * T;
  if (cu_seqlens) {
    const int cs = min(max(cu_seqlens[b], 0), T);
    tok0 = static_cast<size_t>(cs);
    T = min(max(cu_seqlens[b + 1], cs), T) - cs;
  }
  const size_t sbase = (static_cast<size_t>(b) * H + h) * DK * DV;

  for (int e = tid; e < DK * VS; e += blockDim.x) {
    const int i = e / VS, j = e % VS;
    Ss[i * LV + j] = S0 ? S0[sbase + static_cast<size_t>(i) * DV + v0 + j] : 0.f;
  }

  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = min(C, T - t0);
    __syncthreads();
    // ---- K1 + input scaling: one thread per key channel walks the chunk
    if (tid < DK) {
      float g = 1.f;
      for (int r = 0; r < C; ++r) {
        if (r < L) {
          const size_t th = (tok0 + t0 + r) * H + h;
          g *= gate_at(alpha, alpha_mode, th, DK, tid);
          const float bk = sqrtf(gate_at(beta_k, beta_k_mode, th, DK, tid)) * to_f32(k[th * DK + tid]);
          Bh[r * LDK + tid] = g * bk;
          const float ak = s_scale ? s_scale[th * DK + tid] * bk : bk;  // write key a
          Ac[r * LDK + tid] = ak / g;
          Qh[r * LDK + tid] = g * to_f32(q[th * DK + tid]);
        } else {
          Bh[r * LDK + tid] = 0.f;
          Ac[r * LDK + tid] = 0.f;
          Qh[r * LDK + tid] = 0.f;
        }
      }
      gL[tid] = g;
      if (!(g >= kMinChunkDecay)) raise_status(status, STATUS_RANGE);
    } else {
      for (int e = tid - DK; e < C * VS; e += blockDim.x - DK) {
        const int r = e / VS, j = e % VS;
        float w = 0.f;
        if (r < L) {
          const size_t th = (tok0 + t0 + r) * H + h;
          const float vj = to_f32(v[th * DV + v0 + j]);
          const float ws = (beta_v_mode != MODE_ABSENT) ? gate_at(beta_v, beta_v_mode, th, DV, v0 + j)
                                                        : sqrtf(gate_at(beta_k, beta_k_mode, th, DK, v0 + j));
          w = ws * vj;
        }
        Wr[r * LV + j] = w;
      }
    }
    __syncthreads();
    // ---- K2: A = strictly-lower(Bh Ac^T), P = lower(Qh Ac^T)
    for (int e = tid; e < C * C; e += blockDim.x) {
      const int r = e / C, i = e % C;
      float sa = 0.f, sp = 0.f;
      if (i <= r) {
        for (int c = 0; c < DK; ++c) {
          const float ac = Ac[i * LDK + c];
          sa = fmaf(Bh[r * LDK + c], ac, sa);
          sp = fmaf(Qh[r * LDK + c], ac, sp);
        }
      }
      Am[r * LC + i] = (i < r) ? sa : 0.f;
      Pm[r * LC + i] = sp;
    }
    __syncthreads();
    // ---- K2: T = (I + A)^-1, forward substitution, one column per thread
    if (tid < C) {
      const int j = tid;
      for (int r = 0; r < C; ++r) Tm[r * LC + j] = (r == j) ? 1.f : 0.f;
      for (int r = j + 1; r < L; ++r) {
        float acc = 0.f;
        for (int m = j; m < r; ++m) acc = fmaf(Am[r * LC + m], Tm[m * LC + j], acc);
        Tm[r * LC + j] = -acc;
      }
    }
    __syncthreads();
    // ---- X = Wr - Bh S and the inter-chunk part of the output, Qh S
    constexpr int PER = (C * VS) / 256;  // outputs per thread
    float o1[PER];
    {
      const int r = tid / (VS / PER), j0 = (tid % (VS / PER)) * PER;
      float xs[PER];
#pragma unroll
      for (int jj = 0; jj < PER; ++jj) xs[jj] = o1[jj] = 0.f;
      for (int c = 0; c < DK; ++c) {
        const float bh = Bh[r * LDK + c], qh = Qh[r * LDK + c];
#pragma unroll
        for (int jj = 0; jj < PER; ++jj) {
          const float s = Ss[c * LV + j0 + jj];
          xs[jj] = fmaf(bh, s, xs[jj]);
          o1[jj] = fmaf(qh, s, o1[jj]);
        }
      }
#pragma unroll
      for (int jj = 0; jj < PER; ++jj) Xm[r * LV + j0 + jj] = Wr[r * LV + j0 + jj] - xs[jj];
    }
    __syncthreads();
    // ---- U = T X  (stored over Wr)
    {
      const int r = tid / (VS / PER), j0 = (tid % (VS / PER)) * PER;
      float u[PER];
#pragma unroll
      for (int jj = 0; jj < PER; ++jj) u[jj] = 0.f;
      for (int m = 0; m <= r; ++m) {
        const float tv = Tm[r * LC + m];
#pragma unroll
        for (int jj = 0; jj < PER; ++jj) u[jj] = fmaf(tv, Xm[m * LV + j0 + jj], u[jj]);
      }
#pragma unroll
      for (int jj = 0; jj < PER; ++jj) Wr[r * LV + j0 + jj] = u[jj];
    }
    __syncthreads();
    // ---- K4: O = Qh S + P U
    {
      const int r = tid / (VS / PER), j0 = (tid % (VS / PER)) * PER;
      for (int m = 0; m <= r; ++m) {
        const float pv = Pm[r * LC + m];
#pragma unroll
        for (int jj = 0; jj < PER; ++jj) o1[jj] = fmaf(pv, Wr[m * LV + j0 + jj], o1[jj]);
      }
      if (r < L) {
        const size_t th = (tok0 + t0 + r) * H + h;
#pragma unroll
        for (int jj = 0; jj < PER; ++jj) o[th * DV + v0 + j0 + jj] = from_f32<IO>(o1[jj]);
      }
    }
    // ---- K3: S <- Diag(gamma_L) (S + Ac^T U)
    for (int e = tid; e < DK * VS; e += blockDim.x) {
      const int i = e / VS, j = e % VS;
      float acc = Ss[i * LV + j];
      for (int r = 0; r < L; ++r) acc = fmaf(Ac[r * LDK + i], Wr[r * LV + j], acc);
      Ss[i * LV + j] = gL[i] * acc;
    }
  }
  __syncthreads();
  if (S_T) {
    for (int e = tid; e < DK * VS; e += blockDim.x) {
      const int i = e / VS, j = e % VS;
      S_T[sbase + static_cast<size_t>(i) * DV + v0 + j] = Ss[i * LV + j];
    }
  }
}

}  // namespace dr
