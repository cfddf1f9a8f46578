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
//   A = strictly-lower(Bh Ac^T),  P = lower(Qh Ac^T)                     (K2)
//   U = (I + A)^-1 (Wr - Bh S)                (K2 + K3: forward substitution, rows u_r of the chunk)
//   O = Qh S + P U                            (K4)
//   S <- Diag(gamma_L) (S + Ac^T U)           (K3; Ac_r gamma_L = decayed key)
//
// Grid: (dv / VS, H, B); one CTA walks all chunks of one (b, h, value slice).  Every product is a
// register-tiled loop over shared-memory operands, so its loads overlap its FFMA chains.
#pragma once
#include "common.cuh"

namespace dr {

template <int DK, int VS, int C>
struct SimtSmem {
  static constexpr int LDK = DK + 1, LC = C + 1, LV = VS + 1;
  static constexpr size_t floats = 3 * C * LDK     // Bh, Ac, Qh
                                   + 2 * C * LC    // A, P
                                   + 3 * C * LV    // write vectors, X -> U, the output's Qh S part
                                   + DK * LV       // S slice
                                   + DK            // gamma at chunk end
                                   + C * LDK       // staged channel decays of the chunk
                                   + 2 * C;        // staged per-row decays and strengths
  static constexpr size_t bytes = floats * sizeof(float);
};

// acc[TR][TN] += sum_k a[i * ai + k * ak] b[k * bk + j * bj]: a thread's register tile of a product of two
// shared-memory operands, given as strided views from the tile's first row / column (the k loop's loads
// are independent of the accumulation chains)
template <int TR, int TN>
__device__ __forceinline__ void simt_tile_mm(float (&acc)[TR][TN], int K, const float *a, int ai, int ak,
                                             const float *b, int bk, int bj) {
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float av[TR], bv[TN];
#pragma unroll
    for (int i = 0; i < TR; ++i) av[i] = a[i * ai + k * ak];
#pragma unroll
    for (int j = 0; j < TN; ++j) bv[j] = b[k * bk + j * bj];
#pragma unroll
    for (int i = 0; i < TR; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

template <typename IO, int DK, int DV, int VS, int C>
__global__ void __launch_bounds__(256, 2)  // launched with 256 threads
chunk_fwd_simt_kernel(int T, int H, const IO *__restrict__ q, const IO *__restrict__ k,
                      const IO *__restrict__ v, const float *__restrict__ alpha, int alpha_mode,
                      const float *__restrict__ beta_k, int beta_k_mode, const float *__restrict__ beta_v,
                      int beta_v_mode, const float *__restrict__ s_scale, const int *__restrict__ cu_seqlens,
                      const float *__restrict__ S0, IO *__restrict__ o, float *__restrict__ S_T,
                      uint32_t *__restrict__ status) {
  static_assert(VS == 32 && (C == 16 || C == 32 || C == 64) && (DK == 64 || DK == 128), "tile shapes");
  constexpr int kNT = 256;  // the launch's block size
  using L_ = SimtSmem<DK, VS, C>;
  constexpr int LDK = L_::LDK, LC = L_::LC, LV = L_::LV;
  extern __shared__ float sm[];
  float *Bh = sm;
  float *Ac = Bh + C * LDK;
  float *Qh = Ac + C * LDK;
  float *Am = Qh + C * LDK;
  float *Pm = Am + C * LC;
  float *Wr = Pm + C * LC;   // write vectors
  float *Xm = Wr + C * LV;   // X = Wr - Bh S, then U in place
  float *Om = Xm + C * LV;   // Qh S
  float *Ss = Om + C * LV;
  float *gL = Ss + DK * LV;
  float *sAl = gL + DK;         // [C][LDK] channel decays of the chunk
  float *sRow = sAl + C * LDK;  // [2][C] per-row decay and erase strength

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

#pragma unroll
  for (int e = tid; e < DK * VS; e += kNT) {
    const int i = e / VS, j = e % VS;
    Ss[i * LV + j] = S0 ? S0[sbase + static_cast<size_t>(i) * DV + v0 + j] : 0.f;
  }

  // thread tiles: [Bh; Qh] x (Ac^T | S) over 2C rows; the output over C rows; the state over DK rows
  constexpr int TR2 = C / 16, TNA = C / 8, TNV = 4;      // 32 row blocks x 8 column blocks
  constexpr int TRO = C == 16 ? 1 : C / 32, TNO = C == 16 ? 2 : 4, NCO = VS / TNO;  // output tile
  constexpr int TRS = DK / 32;                            // state tile: 32 row blocks x 8 column blocks
  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = min(C, T - t0);
    __syncthreads();
    // ---- stage the chunk: q, k, the gates (coalesced, all threads) and the write vectors; rows past
    // the chunk's end read as identity transitions (alpha 1, beta 0, zero vectors)
#pragma unroll
    for (int e = tid; e < C * DK; e += kNT) {  // all of a thread's loads in flight together
      const int r = e / DK, c = e % DK;
      const bool valid = r < L;
      const size_t th = (tok0 + t0 + min(r, L - 1)) * H + h;
      Qh[r * LDK + c] = valid ? to_f32(q[th * DK + c]) : 0.f;
      Bh[r * LDK + c] = valid ? to_f32(k[th * DK + c]) : 0.f;
      if (alpha_mode == MODE_CHANNEL) sAl[r * LDK + c] = valid ? __ldg(alpha + th * DK + c) : 1.f;
      if (beta_k_mode == MODE_CHANNEL) Ac[r * LDK + c] = valid ? __ldg(beta_k + th * DK + c) : 0.f;
    }
    for (int r = tid; r < C; r += kNT) {
      const bool valid = r < L;
      const size_t th = (tok0 + t0 + min(r, L - 1)) * H + h;
      sRow[r] = (valid && alpha_mode == MODE_SCALAR) ? __ldg(alpha + th) : 1.f;
      sRow[C + r] = (valid && beta_k_mode == MODE_SCALAR) ? __ldg(beta_k + th) : 0.f;
    }
#pragma unroll
    for (int e = tid; e < C * VS; e += kNT) {
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
    __syncthreads();
    // ---- K1 + input scaling: one thread per key channel walks the staged chunk
    if (tid < DK) {
      float g = 1.f;
#pragma unroll 8
      for (int r = 0; r < C; ++r) {
        const float a = alpha_mode == MODE_CHANNEL ? sAl[r * LDK + tid] : sRow[r];
        const float bt = beta_k_mode == MODE_CHANNEL ? Ac[r * LDK + tid] : sRow[C + r];
        g *= a;
        const float bk = sqrtf(bt) * Bh[r * LDK + tid];
        float ak = bk;  // write key a
        if (s_scale && r < L) ak *= s_scale[((tok0 + t0 + r) * H + h) * DK + tid];
        Bh[r * LDK + tid] = g * bk;
        Ac[r * LDK + tid] = ak / g;
        Qh[r * LDK + tid] *= g;
      }
      gL[tid] = g;
      if (!(g >= kMinChunkDecay)) raise_status(status, STATUS_RANGE);
    }
    __syncthreads();
    // ---- K2: [A; P] = [Bh; Qh] Ac^T (A strictly lower, P lower), and [X; Qh S] = [Wr; 0] - [Bh; -Qh] S
    {
      const int rb = tid >> 3, cb = tid & 7;
      // a thread's TR2 rows of [Bh; Qh] lie all in Bh or all in Qh (TR2 divides C)
      const float *xq = rb * TR2 < C ? Bh + rb * TR2 * LDK : Qh + (rb * TR2 - C) * LDK;
      {
        float acc[TR2][TNA] = {};
        simt_tile_mm(acc, DK, xq, LDK, 1, Ac + cb * TNA * LDK, 1, LDK);
#pragma unroll
        for (int i = 0; i < TR2; ++i) {
          const int r = rb * TR2 + i;
#pragma unroll
          for (int jn = 0; jn < TNA; ++jn) {
            const int n = cb * TNA + jn;
            if (r < C) Am[r * LC + n] = n < r ? acc[i][jn] : 0.f;
            else Pm[(r - C) * LC + n] = n <= r - C ? acc[i][jn] : 0.f;
          }
        }
      }
      {
        float acc[TR2][TNV] = {};
        simt_tile_mm(acc, DK, xq, LDK, 1, Ss + cb * TNV, LV, 1);
#pragma unroll
        for (int i = 0; i < TR2; ++i) {
          const int r = rb * TR2 + i;
#pragma unroll
          for (int jv = 0; jv < TNV; ++jv) {
            const int j = cb * TNV + jv;
            if (r < C) Xm[r * LV + j] = Wr[r * LV + j] - acc[i][jv];
            else Om[(r - C) * LV + j] = acc[i][jv];
          }
        }
      }
    }
    __syncthreads();
    // ---- K2 + K3: U = (I + A)^-1 X by forward substitution, in place over X.  Eight threads per value
    // column; thread qd keeps rows qd, qd + 8, ... of its column in registers and adds its share of
    // each row's sum, which a three-step butterfly completes.  Rows past the chunk's end have x = 0
    // and a zero row of A, so their u is 0.
    {
      const int j = tid >> 3, qd = tid & 7;
      float u[C / 8];
#pragma unroll
      for (int r = 0; r < C; ++r) {
        float acc0 = 0.f, acc1 = 0.f;  // two chains
#pragma unroll
        for (int i = 0; i < C / 8; ++i) {
          const int m = 8 * i + qd;
          if (8 * i < r && m < r) {
            if (i & 1) acc1 = fmaf(Am[r * LC + m], u[i], acc1);
            else acc0 = fmaf(Am[r * LC + m], u[i], acc0);
          }
        }
        float acc = acc0 + acc1;
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if ((r & 7) == qd) u[r >> 3] = Xm[r * LV + j] - acc;
      }
#pragma unroll
      for (int i = 0; i < C / 8; ++i) Xm[(8 * i + qd) * LV + j] = u[i];
    }
    __syncthreads();
    // ---- K4: O = Qh S + P U;  K3: S <- Diag(gamma_L) (S + Ac^T U)  (disjoint outputs, no barrier)
    {
      const int rb = tid / NCO, cb = tid % NCO;
      float acc[TRO][TNO];
#pragma unroll
      for (int i = 0; i < TRO; ++i)
#pragma unroll
        for (int jo = 0; jo < TNO; ++jo) acc[i][jo] = Om[(rb * TRO + i) * LV + cb * TNO + jo];
      simt_tile_mm(acc, C, Pm + rb * TRO * LC, LC, 1, Xm + cb * TNO, LV, 1);
#pragma unroll
      for (int i = 0; i < TRO; ++i) {
        const int r = rb * TRO + i;
        if (r < L) {
          const size_t th = (tok0 + t0 + r) * H + h;
#pragma unroll
          for (int jo = 0; jo < TNO; ++jo) o[th * DV + v0 + cb * TNO + jo] = from_f32<IO>(acc[i][jo]);
        }
      }
    }
    {
      const int rb = tid >> 3, cb = tid & 7;
      float acc[TRS][TNV];
#pragma unroll
      for (int i = 0; i < TRS; ++i)
#pragma unroll
        for (int jv = 0; jv < TNV; ++jv) acc[i][jv] = Ss[(rb * TRS + i) * LV + cb * TNV + jv];
      simt_tile_mm(acc, C, Ac + rb * TRS, 1, LDK, Xm + cb * TNV, LV, 1);
#pragma unroll
      for (int i = 0; i < TRS; ++i) {
        const int ii = rb * TRS + i;
        const float g = gL[ii];
#pragma unroll
        for (int jv = 0; jv < TNV; ++jv) Ss[ii * LV + cb * TNV + jv] = g * acc[i][jv];
      }
    }
  }
  __syncthreads();
  if (S_T) {
    for (int e = tid; e < DK * VS; e += kNT) {
      const int i = e / VS, j = e % VS;
      S_T[sbase + static_cast<size_t>(i) * DV + v0 + j] = Ss[i * LV + j];
    }
  }
}

}  // namespace dr
