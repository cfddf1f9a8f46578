// chunk_tc.cuh -- fused chunkwise WY/UT prefill on the 5th-generation tensor cores
// (tcgen05.mma, fp16 operands in shared memory, fp32 accumulators in TMEM).
//
// One CTA owns one (b, h, slice of VS = 64 value columns) and walks its chunks
// of C = 64 tokens in order, carrying the fp32 state slice S (dk x VS) in
// registers.  Per chunk (DeltaNet page, step 7 and the Householder-product
// remark; FG2-GDN page, section 2, sqrt(beta) keeps the rank-1 WY structure):
//
//  K1  gamma_r = prod_{j<=r} alpha_j (per key channel), its reverse
//      R_r = prod_{j>r} alpha_j and gamma_C; no exp/log needed:
//        exp(g_r) = gamma_r,  exp(g_C - g_r) = R_r,  exp(-g_r) = R_r / gamma_C.
//  a0  b = sqrt(beta_k) k,  w = beta_v v  or  sqrt(beta_k) v.
//      Operand tiles:  Qh = gamma q,  Bh = gamma b,  Ac = b R / gamma_C,  Kd = b R.
//  K2  D1 = [Qh; Bh] Ac^T                      (P raw | A raw)           MMA 128x64x128
//      P = lower(Qh Ac^T),  T = (I + strictly-lower(Bh Ac^T))^-1         (fp32, CUDA cores)
//      D2 = [T; P] Bh  -> W = T Bh (rows 0..63)                          MMA 128x128x64
//      D5 = [T; P] Wr  -> U0 = T Wr (rows 0..63)                         MMA 128x64x64
//  K3  D3 = [-W; Qh] S -> -W S (rows 0..63), Qh S (rows 64..127)         MMA 128x64x128
//      U = U0 - W S  (fp16 operand)
//      D4 = Kd^T U                                                       MMA 128x64x64
//      S <- Diag(gamma_C) S + D4   (fp32, registers)
//  K4  D3 += [T; P] U  -> O = Qh S + P U (rows 64..127)                  MMA 128x64x64
//
// All MMAs use M = 128: rows 0..63 and 64..127 of a 128-row A operand carry two
// different 64-row matrices, and rows that are not needed are ignored in TMEM.
// Thread layout: 8 warps; warp w reads TMEM lanes 32*(w%4).. and column half w/4.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace dr {
namespace tc {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dim
constexpr int VS = 64;    // value columns per CTA
constexpr int NT = 256;   // threads

// shared-memory map (bytes from a 1024-aligned base); fp16 tiles use the 128B swizzle
constexpr uint32_t OFF_QKB = 0;                          // [-W; Qh; Bh] 192 x 128
constexpr uint32_t OFF_AC = OFF_QKB + 192 * 256;         // Ac 64 x 128
constexpr uint32_t OFF_KD = OFF_AC + 64 * 256;           // Kd 64 x 128
constexpr uint32_t OFF_TP = OFF_KD + 64 * 256;           // [T; P] 128 x 64
constexpr uint32_t OFF_WR = OFF_TP + 128 * 128;          // write vectors 64 x VS
constexpr uint32_t OFF_S = OFF_WR + 64 * 128;            // state (fp16 copy) 128 x VS
constexpr uint32_t OFF_U = OFF_S + 128 * 128;            // U 64 x VS
constexpr uint32_t OFF_AF = OFF_U + 64 * 128;            // A, fp32 64 x 65
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4;        // T, fp32 64 x 65
constexpr uint32_t OFF_XF = OFF_TF + 64 * 65 * 4;        // block products, fp32 3 x 16 x 17
constexpr uint32_t OFF_GC = OFF_XF + 3 * 16 * 17 * 4;    // gamma_C, 128 fp32
constexpr uint32_t OFF_PX = OFF_GC + 128 * 4;            // half-chunk gate products, 2 x 128 fp32
constexpr uint32_t OFF_END = OFF_PX + 256 * 4;
constexpr size_t SMEM_BYTES = OFF_END + 1024;            // + alignment slack

// TMEM columns
constexpr uint32_t COL_D1 = 0;     // [P raw | A raw], later U0 (64 columns)
constexpr uint32_t COL_D2 = 64;    // W (128 columns)
constexpr uint32_t COL_D3 = 192;   // [-W S | Qh S + P U] (64 columns)
constexpr uint32_t COL_D4 = 256;   // Kd^T U (64 columns)
constexpr uint32_t TMEM_COLS = 512;

// Smallest cumulative decay over one chunk for which every fp16 operand stays
// finite: Ac = b exp(-g) grows like 1/gamma_C, so gamma_C >= 2^-14 keeps it
// below 2^15 |b|.  Operands that still leave the fp16 range raise STATUS_RANGE.
constexpr float kMinChunkDecayF16 = 6.103515625e-05f;
constexpr float kF16Max = 65000.f;

// Operand tiles hold fp16: bf16's 8-bit significand loses too much in the
// products (measured max error ~3% of the output RMS), fp16's 11 bits meet the
// tolerance with margin, and every operand fits its range once the chunk's
// cumulative decay stays above kMinChunkDecayF16.
__device__ __forceinline__ void st_h16x16(uint8_t *tile, int row, int col0, int R, const float (&v)[16]) {
  uint4 lo, hi;
  lo.x = pack_f16x2(v[0], v[1]);
  lo.y = pack_f16x2(v[2], v[3]);
  lo.z = pack_f16x2(v[4], v[5]);
  lo.w = pack_f16x2(v[6], v[7]);
  hi.x = pack_f16x2(v[8], v[9]);
  hi.y = pack_f16x2(v[10], v[11]);
  hi.z = pack_f16x2(v[12], v[13]);
  hi.w = pack_f16x2(v[14], v[15]);
  *reinterpret_cast<uint4 *>(tile + sw128_off16(row, col0 >> 3, R)) = lo;
  *reinterpret_cast<uint4 *>(tile + sw128_off16(row, (col0 >> 3) + 1, R)) = hi;
}

__device__ __forceinline__ void st_h16(uint8_t *tile, int row, int col, int R, float x) {
  *reinterpret_cast<__half *>(tile + sw128_off(row, col, R)) = __float2half_rn(x);
}

template <typename IO>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_tc_kernel(int T, int H, int DV, const IO *__restrict__ q, const IO *__restrict__ k,
                    const IO *__restrict__ v, const float *__restrict__ alpha, int alpha_mode,
                    const float *__restrict__ beta_k, int beta_k_mode, const float *__restrict__ beta_v,
                    int beta_v_mode, const float *__restrict__ S0, IO *__restrict__ o, float *__restrict__ S_T,
                    uint32_t *__restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *tQKB = sm + OFF_QKB;
  uint8_t *tAC = sm + OFF_AC;
  uint8_t *tKD = sm + OFF_KD;
  uint8_t *tTP = sm + OFF_TP;
  uint8_t *tWR = sm + OFF_WR;
  uint8_t *tS = sm + OFF_S;
  uint8_t *tU = sm + OFF_U;
  float *sA = reinterpret_cast<float *>(sm + OFF_AF);
  float *sT = reinterpret_cast<float *>(sm + OFF_TF);
  float *sX = reinterpret_cast<float *>(sm + OFF_XF);
  float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
  float *sPX = reinterpret_cast<float *>(sm + OFF_PX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int trow = quarter * 32 + lane;  // TMEM lane (accumulator row) this thread reads
  const int v0 = blockIdx.x * VS, h = blockIdx.y, b = blockIdx.z;
  const size_t sbase = (static_cast<size_t>(b) * H + h) * DK * DV;

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  uint32_t phase = 0;
  bool aborted = false;

  // MMA completion: one thread issued and committed; everyone waits (bounded).
  auto wait_mma = [&]() -> bool {
    const bool ok = mbar_wait(&mma_bar, phase & 1u, kWaitLimitNs);
    phase++;
    tc_fence_after();
    if (!ok && lane == 0) raise_status(status, STATUS_TIMEOUT);
    return __syncthreads_or(!ok) == 0;
  };

  // fp32 state slice in registers: row k = trow, columns half*32 .. half*32+31 of the slice
  float Sreg[32];
  {
    const float *src = S0 ? S0 + sbase + static_cast<size_t>(trow) * DV + v0 + half * 32 : nullptr;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      Sreg[j] = x.x;
      Sreg[j + 1] = x.y;
      Sreg[j + 2] = x.z;
      Sreg[j + 3] = x.w;
    }
#pragma unroll
    for (int j = 0; j < 32; j += 16) {
      float t16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t16[i] = Sreg[j + i];
      st_h16x16(tS, trow, half * 32 + j, 128, t16);
    }
  }

  const uint32_t a_base = smem_u32(sm);
  for (int t0 = 0; t0 < T && !aborted; t0 += C) {
    const int L = min(C, T - t0);

    // ------------------------------------------------------------ K1 + a0 (operand tiles)
    {
      const int kc = tid & 127, rh = tid >> 7;
      float al[32], pre[32];
      float p = 1.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int r = rh * 32 + j;
        float a = 1.f;
        if (r < L) a = gate_at(alpha, alpha_mode, (static_cast<size_t>(b) * T + t0 + r) * H + h, DK, kc);
        al[j] = a;
        p *= a;
        pre[j] = p;
      }
      sPX[rh * 128 + kc] = p;
      __syncthreads();
      const float other = sPX[(1 - rh) * 128 + kc];
      const float head = rh ? other : 1.f;  // product of the rows before my half
      const float tail = rh ? 1.f : other;  // product of the rows after my half
      const float gC = (rh ? other : 1.f) * p * (rh ? 1.f : other);
      const float inv_gC = 1.f / gC;
      if (rh == 0) {
        sGC[kc] = gC;
        if (!(gC >= kMinChunkDecayF16)) raise_status(status, STATUS_RANGE);
      }
      float suf = tail;  // product of rows strictly after row j
#pragma unroll
      for (int j = 31; j >= 0; --j) {
        const int r = rh * 32 + j;
        float bk = 0.f, qv = 0.f;
        if (r < L) {
          const size_t th = (static_cast<size_t>(b) * T + t0 + r) * H + h;
          bk = sqrtf(gate_at(beta_k, beta_k_mode, th, DK, kc)) * to_f32(k[th * DK + kc]);
          qv = to_f32(q[th * DK + kc]);
        }
        const float g = head * pre[j];
        st_h16(tQKB, 64 + r, kc, 192, g * qv);        // Qh
        st_h16(tQKB, 128 + r, kc, 192, g * bk);       // Bh
        const float ac = bk * suf * inv_gC;
        if (!(fabsf(ac) < kF16Max)) raise_status(status, STATUS_RANGE);
        st_h16(tAC, r, kc, 64, ac);                    // Ac = b exp(-g)
        st_h16(tKD, r, kc, 64, bk * suf);             // Kd = b exp(g_C - g)
        suf *= al[j];
      }
      // write vectors w (rows c, value columns of this slice)
      {
        const int c = tid >> 2, vg = (tid & 3) * 16;
        float w16[16];
        if (c < L) {
          const size_t th = (static_cast<size_t>(b) * T + t0 + c) * H + h;
          const IO *vp = v + th * DV + v0 + vg;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = v0 + vg + i;
            const float ws = (beta_v_mode != MODE_ABSENT) ? gate_at(beta_v, beta_v_mode, th, DV, col)
                                                          : sqrtf(gate_at(beta_k, beta_k_mode, th, DK, col));
            w16[i] = ws * to_f32(vp[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) w16[i] = 0.f;
        }
        st_h16x16(tWR, c, vg, 64, w16);
      }
    }
    fence_async_smem();
    __syncthreads();

    // ------------------------------------------------------------ m1: D1 = [Qh; Bh] Ac^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        umma_f16(tmem + COL_D1, desc_kmajor(a_base + OFF_QKB + 64 * 128, 192, kk),
                  desc_kmajor(a_base + OFF_AC, 64, kk), idesc, kk > 0);
      umma_commit(&mma_bar);
    }
    if (!wait_mma()) { aborted = true; break; }

    // ------------------------------------------------------------ E1: P (fp16 tile), A (fp32)
    {
      float x[32];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32), *reinterpret_cast<float(*)[16]>(x));
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32 + 16), *reinterpret_cast<float(*)[16]>(x + 16));
      tmem_ld_wait();
      if (quarter < 2) {  // rows 0..63: Qh Ac^T -> P (diagonal included)
        const int r = trow;
#pragma unroll
        for (int j = 0; j < 32; j += 16) {
          float t16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) t16[i] = (half * 32 + j + i <= r) ? x[j + i] : 0.f;
          st_h16x16(tTP, 64 + r, half * 32 + j, 128, t16);
        }
      } else {  // rows 64..127: Bh Ac^T -> strictly lower A
        const int r = trow - 64;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = half * 32 + i;
          sA[r * 65 + col] = (col < r) ? x[i] : 0.f;
        }
      }
    }
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ K2: T = (I + A)^-1, blocked 4 x 16
    if (tid < 64) {  // diagonal blocks: one column of one block per thread
      const int bb = tid >> 4, col = tid & 15, o16 = bb * 16;
      float xcol[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == col) ? 1.f : 0.f;
        if (r > col) {
#pragma unroll
          for (int m = 0; m < 16; ++m)
            if (m >= col && m < r) acc -= sA[(o16 + r) * 65 + o16 + m] * xcol[m];
        }
        xcol[r] = (r < col) ? 0.f : acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sT[(o16 + r) * 65 + o16 + col] = xcol[r];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      const int nblk = 4 - d;
      // X_ij = sum_{m in [j16, i16)} A[i16 + rr][m] T[m][j16 + cc],  i = j + d
      for (int e = tid; e < nblk * 256; e += NT) {
        const int jb = e >> 8, rr = (e >> 4) & 15, cc = e & 15, ib = jb + d;
        float acc = 0.f;
        for (int m = jb * 16; m < ib * 16; ++m) acc += sA[(ib * 16 + rr) * 65 + m] * sT[m * 65 + jb * 16 + cc];
        sX[(jb * 16 + rr) * 17 + cc] = acc;
      }
      __syncthreads();
      // T_ij = - T_ii X_ij
      for (int e = tid; e < nblk * 256; e += NT) {
        const int jb = e >> 8, rr = (e >> 4) & 15, cc = e & 15, ib = jb + d;
        float acc = 0.f;
        for (int m = 0; m <= rr; ++m) acc += sT[(ib * 16 + rr) * 65 + ib * 16 + m] * sX[(jb * 16 + m) * 17 + cc];
        sT[(ib * 16 + rr) * 65 + jb * 16 + cc] = -acc;
      }
      __syncthreads();
    }
    {  // T (lower, fp16) into rows 0..63 of [T; P]
      const int r = tid >> 2, c0 = (tid & 3) * 16;
      float t16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t16[i] = (c0 + i <= r) ? sT[r * 65 + c0 + i] : 0.f;
      st_h16x16(tTP, r, c0, 128, t16);
    }
    fence_async_smem();
    __syncthreads();

    // ------------------------------------------------------------ m2: D2 = [T;P] Bh,  m3: D1 = [T;P] Wr
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id2 = idesc_f16_f32(128, 128, false, true);
      const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_D2, desc_kmajor(a_base + OFF_TP, 128, kk),
                  desc_mnmajor(a_base + OFF_QKB + 128 * 128, 192, kk), id2, kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_D1, desc_kmajor(a_base + OFF_TP, 128, kk), desc_mnmajor(a_base + OFF_WR, 64, kk),
                  id3, kk > 0);
      umma_commit(&mma_bar);
    }
    if (!wait_mma()) { aborted = true; break; }

    // ------------------------------------------------------------ E2: -W (fp16) into rows 0..63 of [-W; Qh; Bh]
    if (quarter < 2) {
#pragma unroll
      for (int j = 0; j < 64; j += 16) {
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D2 + half * 64 + j), x);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = -x[i];
        st_h16x16(tQKB, trow, half * 64 + j, 192, x);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ K3: D3 = [-W; Qh] S
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_f16_f32(128, VS, false, true);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        umma_f16(tmem + COL_D3, desc_kmajor(a_base + OFF_QKB, 192, kk), desc_mnmajor(a_base + OFF_S, 128, kk), id,
                  kk > 0);
      umma_commit(&mma_bar);
    }
    if (!wait_mma()) { aborted = true; break; }

    // ------------------------------------------------------------ E3: U = U0 - W S (fp16)
    if (quarter < 2) {
#pragma unroll
      for (int j = 0; j < 32; j += 16) {
        float ws[16], u0[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D3 + half * 32 + j), ws);
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32 + j), u0);
        tmem_ld_wait();
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          u0[i] += ws[i];
          mx = fmaxf(mx, fabsf(u0[i]));
        }
        if (!(mx < kF16Max)) raise_status(status, STATUS_RANGE);
        st_h16x16(tU, trow, half * 32 + j, 64, u0);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ K3/K4: D4 = Kd^T U,  D3 += [T;P] U
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id4 = idesc_f16_f32(128, VS, true, true);
      const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_D4, desc_mnmajor(a_base + OFF_KD, 64, kk), desc_mnmajor(a_base + OFF_U, 64, kk), id4,
                  kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_D3, desc_kmajor(a_base + OFF_TP, 128, kk), desc_mnmajor(a_base + OFF_U, 64, kk), id3,
                  1u);
      umma_commit(&mma_bar);
    }
    if (!wait_mma()) { aborted = true; break; }

    // ------------------------------------------------------------ E4: S update (fp32 regs -> fp16 tile), outputs
    {
      const float gc = sGC[trow];
#pragma unroll
      for (int j = 0; j < 32; j += 16) {
        float ds[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D4 + half * 32 + j), ds);
        tmem_ld_wait();
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          Sreg[j + i] = fmaf(gc, Sreg[j + i], ds[i]);
          ds[i] = Sreg[j + i];
          mx = fmaxf(mx, fabsf(ds[i]));
        }
        if (!(mx < kF16Max)) raise_status(status, STATUS_RANGE);
        st_h16x16(tS, trow, half * 32 + j, 128, ds);
      }
      if (quarter >= 2) {
        const int r = trow - 64;
        float x[32];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D3 + half * 32), *reinterpret_cast<float(*)[16]>(x));
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D3 + half * 32 + 16), *reinterpret_cast<float(*)[16]>(x + 16));
        tmem_ld_wait();
        if (r < L) {
          const size_t th = (static_cast<size_t>(b) * T + t0 + r) * H + h;
          IO *dst = o + th * DV + v0 + half * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[i] = from_f32<IO>(x[i]);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted && S_T) {
    float *dst = S_T + sbase + static_cast<size_t>(trow) * DV + v0 + half * 32;
#pragma unroll
    for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(dst + j) = make_float4(Sreg[j], Sreg[j + 1], Sreg[j + 2], Sreg[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc
}  // namespace dr
