// chunk_tc.cuh -- fused chunkwise WY/UT prefill on the 5th-generation tensor cores
// (tcgen05.mma, fp16 operands in shared memory, fp32 accumulators in TMEM).
//
// One CTA owns one (b, h, slice of VS = 64 value columns) and walks its chunks
// of C = 64 tokens in order, carrying the fp32 state slice S (dk x VS) in
// registers.  Per chunk (DeltaNet page, step 7 and the Householder-product
// remark; FG2-GDN page, section 2, sqrt(beta) keeps the rank-1 WY structure):
//
//  K1  gamma_r = prod_{j<=r} alpha_j per key channel (= exp(g_r)); gamma_C = gamma_{C-1}.
//  a0  b = sqrt(beta_k) k,  w = beta_v v  or  sqrt(beta_k) v.
//      Operand tiles:  Qh = gamma q,  Bh = gamma b,  Ac = b / gamma   (= b exp(-g)).
//  K2  D1 = [Qh; Bh] Ac^T                      (P raw | A raw)           MMA 128x64x128
//      P = lower(Qh Ac^T),  T = (I + strictly-lower(Bh Ac^T))^-1         (fp32, CUDA cores)
//      D2 = [T; P] Bh  -> W = T Bh (rows 0..63)                          MMA 128x128x64
//      D1 = [T; P] Wr  -> U0 = T Wr (rows 0..63)                         MMA 128x64x64
//  K3  D3 = [-W; Qh] S -> -W S (rows 0..63), Qh S (rows 64..127)         MMA 128x64x128
//      U = U0 - W S  (fp16 operand)
//      D4 = Ac^T U                                                       MMA 128x64x64
//      S <- Diag(gamma_C) (S + D4)    since  Kd = Ac (.) gamma_C  (fp32, registers)
//  K4  D3 += [T; P] U  -> O = Qh S + P U (rows 64..127)                  MMA 128x64x64
//
// All MMAs use M = 128: rows 0..63 and 64..127 of a 128-row A operand carry two
// different 64-row matrices, and rows that are not needed are ignored in TMEM.
//
// Data movement: the raw q, k, v (and channel beta_v) tiles of chunk c+1 are
// fetched by TMA into a staging area as soon as chunk c has turned its raw
// tiles into operands, and the fp32 gates of chunk c+1 are prefetched into
// registers at the same point, so both loads overlap the rest of chunk c.
//
// Thread layout: 16 warps; warp w reads TMEM lanes 32*(w%4).. and column quarter w/4.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace dr {
namespace tc {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dim
constexpr int VS = 64;    // value columns per CTA
constexpr int NT = 512;   // threads
constexpr int RG = 16;    // rows of a chunk handled by one elementwise thread

// shared-memory map (bytes from a 1024-aligned base); fp16 operand tiles use the 128B swizzle
constexpr uint32_t OFF_QKB = 0;                          // [-W; Qh; Bh] 192 x 128 fp16
constexpr uint32_t OFF_AC = OFF_QKB + 192 * 256;         // Ac 64 x 128
constexpr uint32_t OFF_TP = OFF_AC + 64 * 256;           // [T; P] 128 x 64
constexpr uint32_t OFF_WR = OFF_TP + 128 * 128;          // write vectors 64 x VS
constexpr uint32_t OFF_S = OFF_WR + 64 * 128;            // state (fp16 copy) 128 x VS
constexpr uint32_t OFF_U = OFF_S + 128 * 128;            // U 64 x VS
constexpr uint32_t OFF_RQ = OFF_U + 64 * 128;            // raw q, bf16 64 x 128 (TMA, row-major)
constexpr uint32_t OFF_RK = OFF_RQ + 64 * 256;           // raw k
constexpr uint32_t OFF_RV = OFF_RK + 64 * 256;           // raw v slice, bf16 64 x VS
constexpr uint32_t OFF_RW = OFF_RV + 64 * VS * 2;        // write scale, fp32 64 x VS (TMA'd beta_v or sqrt(beta_k))
constexpr uint32_t OFF_AF = OFF_RW + 64 * VS * 4;        // A, fp32 64 x 65
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4;        // T, fp32 64 x 65
constexpr uint32_t OFF_XF = OFF_TF + 64 * 65 * 4;        // block products, fp32 3 x 16 x 17
constexpr uint32_t OFF_GC = OFF_XF + 3 * 16 * 17 * 4;    // gamma_C, 128 fp32
constexpr uint32_t OFF_PX = OFF_GC + 128 * 4;            // per-row-group gate products, 4 x 128 fp32
constexpr uint32_t OFF_END = OFF_PX + 4 * 128 * 4;
constexpr size_t SMEM_BYTES = OFF_END + 1024;            // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t COL_D1 = 0;     // [P raw | A raw], later U0 (64 columns)
constexpr uint32_t COL_D2 = 64;    // W (128 columns)
constexpr uint32_t COL_D3 = 192;   // [-W S | Qh S + P U] (64 columns)
constexpr uint32_t COL_D4 = 256;   // Ac^T U (64 columns)
constexpr uint32_t TMEM_COLS = 512;

// Operand tiles hold fp16: bf16's 8-bit significand loses too much in the
// products (measured max error ~3% of the output RMS), fp16's 11 bits meet the
// tolerance with margin.  Ac = b exp(-g) grows like 1/gamma_C, so the chunk's
// cumulative decay must stay >= 2^-14 (sum of log alpha >= -9.7 over a chunk);
// operands that still leave the fp16 range raise STATUS_RANGE.
constexpr float kMinChunkDecayF16 = 6.103515625e-05f;
constexpr float kF16Max = 65000.f;

struct Params {
  int T, H, DV;
  const float *alpha;
  int alpha_mode;
  const float *beta_k;
  int beta_k_mode;
  const float *beta_v;
  int beta_v_mode;
  const float *S0;
  void *o;
  float *S_T;
  uint32_t *status;
};

__device__ __forceinline__ void st_h16x8(uint8_t *tile, int row, int col0, int R, const float *v) {
  uint4 x;
  x.x = pack_f16x2(v[0], v[1]);
  x.y = pack_f16x2(v[2], v[3]);
  x.z = pack_f16x2(v[4], v[5]);
  x.w = pack_f16x2(v[6], v[7]);
  *reinterpret_cast<uint4 *>(tile + sw128_off16(row, col0 >> 3, R)) = x;
}
__device__ __forceinline__ void st_h16x16(uint8_t *tile, int row, int col0, int R, const float *v) {
  st_h16x8(tile, row, col0, R, v);
  st_h16x8(tile, row, col0 + 8, R, v + 8);
}
__device__ __forceinline__ void st_h16(uint8_t *tile, int row, int col, int R, float x) {
  *reinterpret_cast<__half *>(tile + sw128_off(row, col, R)) = __float2half_rn(x);
}
__device__ __forceinline__ float bf16_at(const uint8_t *base, int idx) {
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
}

template <typename IO>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bv,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar, raw_bar;
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *tQKB = sm + OFF_QKB;
  uint8_t *tAC = sm + OFF_AC;
  uint8_t *tTP = sm + OFF_TP;
  uint8_t *tWR = sm + OFF_WR;
  uint8_t *tS = sm + OFF_S;
  uint8_t *tU = sm + OFF_U;
  const uint8_t *rQ = sm + OFF_RQ;
  const uint8_t *rK = sm + OFF_RK;
  const uint8_t *rV = sm + OFF_RV;
  float *rW = reinterpret_cast<float *>(sm + OFF_RW);
  float *sA = reinterpret_cast<float *>(sm + OFF_AF);
  float *sT = reinterpret_cast<float *>(sm + OFF_TF);
  float *sX = reinterpret_cast<float *>(sm + OFF_XF);
  float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
  float *sPX = reinterpret_cast<float *>(sm + OFF_PX);

  const int T = p.T, H = p.H, DV = p.DV;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
  const int trow = quarter * 32 + lane;          // TMEM lane (accumulator row) this thread reads
  const int v0 = blockIdx.x * VS, h = blockIdx.y, b = blockIdx.z;
  const size_t sbase = (static_cast<size_t>(b) * H + h) * DK * DV;
  const bool bv_tma = p.beta_v_mode == MODE_CHANNEL;
  const bool sym_channel = p.beta_v_mode == MODE_ABSENT && p.beta_k_mode == MODE_CHANNEL;
  const uint32_t raw_bytes = 2 * 64 * 256 + 64 * VS * 2 + (bv_tma ? 64 * VS * 4 : 0);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    mbar_init(&raw_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (bv_tma) tma_prefetch_desc(&tm_bv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  uint32_t mphase = 0, rphase = 0;
  bool aborted = false;

  auto issue_raw = [&](int t0) {  // one thread: TMA of chunk [t0, t0 + C)
    mbar_arrive_expect_tx(&raw_bar, raw_bytes);
    tma_load_4d(sm + OFF_RQ, &tm_q, &raw_bar, 0, h, t0, b);
    tma_load_4d(sm + OFF_RK, &tm_k, &raw_bar, 0, h, t0, b);
    tma_load_4d(sm + OFF_RV, &tm_v, &raw_bar, v0, h, t0, b);
    if (bv_tma) tma_load_4d(sm + OFF_RW, &tm_bv, &raw_bar, v0, h, t0, b);
  };
  // Waits are bounded; the decision to stop is made uniformly by the whole CTA.
  auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
    const bool ok = mbar_wait(bar, ph & 1u, kWaitLimitNs);
    ph++;
    if (!ok && lane == 0) raise_status(p.status, STATUS_TIMEOUT);
    return __syncthreads_or(!ok) == 0;
  };
  auto wait_mma = [&]() -> bool {
    const bool ok = wait_bar(&mma_bar, mphase);
    tc_fence_after();
    return ok;
  };

  // gate prefetch: thread (kc, rg) holds alpha and beta_k of its 16 rows of the next chunk;
  // threads of the write-vector layout hold the scalar write scale of their row.
  const int kc = tid & 127, rg = tid >> 7;
  const int wc = tid >> 3, wj0 = (tid & 7) * 8;  // write-vector element block: row wc, columns wj0..wj0+7
  float pal[RG], pbe[RG], pws = 0.f;
  auto prefetch_gates = [&](int t0) {
    const int L = min(C, T - t0);
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      const int r = rg * RG + j;
      pal[j] = 1.f;
      pbe[j] = 0.f;
      if (r < L) {
        const size_t th = (static_cast<size_t>(b) * T + t0 + r) * H + h;
        pal[j] = gate_at(p.alpha, p.alpha_mode, th, DK, kc);
        pbe[j] = gate_at(p.beta_k, p.beta_k_mode, th, DK, kc);
      }
    }
    pws = 0.f;
    if (wc < L && !bv_tma && !sym_channel) {
      const size_t th = (static_cast<size_t>(b) * T + t0 + wc) * H + h;
      pws = (p.beta_v_mode == MODE_SCALAR) ? __ldg(p.beta_v + th) : sqrtf(__ldg(p.beta_k + th));
    }
  };

  // fp32 state slice in registers: row k = trow, columns cq*16 .. cq*16+15 of the slice
  float Sreg[16];
  {
    const float *src = p.S0 ? p.S0 + sbase + static_cast<size_t>(trow) * DV + v0 + cq * 16 : nullptr;
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
      float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      Sreg[j] = x.x;
      Sreg[j + 1] = x.y;
      Sreg[j + 2] = x.z;
      Sreg[j + 3] = x.w;
    }
    st_h16x16(tS, trow, cq * 16, 128, Sreg);
  }
  if (T > 0) {
    if (tid == 0) issue_raw(0);
    prefetch_gates(0);
  }

  const uint32_t a_base = smem_u32(sm);
  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = min(C, T - t0);
    if (!wait_bar(&raw_bar, rphase)) { aborted = true; break; }

    // ------------------------------------------------------------ K1 + a0 (operand tiles)
    {
      float pre[RG];
      float pr = 1.f;
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        pr *= pal[j];
        pre[j] = pr;
      }
      sPX[rg * 128 + kc] = pr;
      __syncthreads();
      float head = 1.f, gC = 1.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float x = sPX[g * 128 + kc];
        if (g < rg) head *= x;
        gC *= x;
      }
      if (rg == 0) {
        sGC[kc] = gC;
        if (!(gC >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
      }
      const bool own_w = sym_channel && kc >= v0 && kc < v0 + VS;
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const int r = rg * RG + j;
        const float sb = sqrtf(pbe[j]);
        const float bk = sb * bf16_at(rK, r * DK + kc);  // rows >= L: k = 0 (TMA fill), beta = 0
        const float qv = bf16_at(rQ, r * DK + kc);
        const float g = head * pre[j];
        const float ac = bk * __frcp_rn(g);
        amax = fmaxf(amax, fabsf(ac));
        st_h16(tQKB, 64 + r, kc, 192, g * qv);   // Qh
        st_h16(tQKB, 128 + r, kc, 192, g * bk);  // Bh
        st_h16(tAC, r, kc, 64, ac);              // Ac = b exp(-g)
        if (own_w) rW[r * VS + (kc - v0)] = sb;  // write scale sqrt(beta_k) of this value column
      }
      if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      if (sym_channel) __syncthreads();
      // write vectors w (rows c, value columns of this slice)
      {
        float w8[8];
        const bool valid = wc < L;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float vv = bf16_at(rV, wc * VS + wj0 + i);
          const float sc = (bv_tma || sym_channel) ? rW[wc * VS + wj0 + i] : pws;
          w8[i] = valid ? sc * vv : 0.f;
        }
        st_h16x8(tWR, wc, wj0, 64, w8);
      }
    }
    fence_async_smem();
    __syncthreads();
    // the raw staging area and the gate registers are free: fetch chunk c+1 now
    if (t0 + C < T) {
      if (tid == 0) issue_raw(t0 + C);
      prefetch_gates(t0 + C);
    }

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
      float x[16];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + cq * 16), x);
      tmem_ld_wait();
      if (quarter < 2) {  // rows 0..63: Qh Ac^T -> P (diagonal included)
        const int r = trow;
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (cq * 16 + i <= r) ? x[i] : 0.f;
        st_h16x16(tTP, 64 + r, cq * 16, 128, x);
      } else {  // rows 64..127: Bh Ac^T -> strictly lower A
        const int r = trow - 64;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int col = cq * 16 + i;
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
      const int r = tid >> 3, c0 = (tid & 7) * 8;
      float t8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t8[i] = (c0 + i <= r) ? sT[r * 65 + c0 + i] : 0.f;
      st_h16x8(tTP, r, c0, 128, t8);
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
      for (int j = 0; j < 32; j += 16) {
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D2 + cq * 32 + j), x);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = -x[i];
        st_h16x16(tQKB, trow, cq * 32 + j, 192, x);
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
      float ws[16], u0[16];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D3 + cq * 16), ws);
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + cq * 16), u0);
      tmem_ld_wait();
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        u0[i] += ws[i];
        mx = fmaxf(mx, fabsf(u0[i]));
      }
      if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
      st_h16x16(tU, trow, cq * 16, 64, u0);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ K3/K4: D4 = Ac^T U,  D3 += [T;P] U
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id4 = idesc_f16_f32(128, VS, true, true);
      const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_D4, desc_mnmajor(a_base + OFF_AC, 64, kk), desc_mnmajor(a_base + OFF_U, 64, kk), id4,
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
      float ds[16];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D4 + cq * 16), ds);
      tmem_ld_wait();
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        Sreg[i] = gc * (Sreg[i] + ds[i]);
        mx = fmaxf(mx, fabsf(Sreg[i]));
      }
      if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
      st_h16x16(tS, trow, cq * 16, 128, Sreg);
      if (quarter >= 2) {
        const int r = trow - 64;
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D3 + cq * 16), x);
        tmem_ld_wait();
        if (r < L) {
          const size_t th = (static_cast<size_t>(b) * T + t0 + r) * H + h;
          IO *dst = static_cast<IO *>(p.o) + th * DV + v0 + cq * 16;
          uint4 lo, hi;
          lo.x = pack_bf16x2(x[0], x[1]);
          lo.y = pack_bf16x2(x[2], x[3]);
          lo.z = pack_bf16x2(x[4], x[5]);
          lo.w = pack_bf16x2(x[6], x[7]);
          hi.x = pack_bf16x2(x[8], x[9]);
          hi.y = pack_bf16x2(x[10], x[11]);
          hi.z = pack_bf16x2(x[12], x[13]);
          hi.w = pack_bf16x2(x[14], x[15]);
          reinterpret_cast<uint4 *>(dst)[0] = lo;
          reinterpret_cast<uint4 *>(dst)[1] = hi;
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted && p.S_T) {
    float *dst = p.S_T + sbase + static_cast<size_t>(trow) * DV + v0 + cq * 16;
#pragma unroll
    for (int j = 0; j < 16; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(Sreg[j], Sreg[j + 1], Sreg[j + 2], Sreg[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc
}  // namespace dr
