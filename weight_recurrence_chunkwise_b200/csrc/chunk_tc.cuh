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
//      Operand tiles:  Qh = gamma q,  Bh = gamma b,  Ac = b R / gamma_C  (= b exp(-g)),
//      R_r = prod_{j>r} alpha_j (reverse products: no division per element).
//  K2  D1 = [Qh; Bh] Ac^T                      (P raw | A raw)           MMA 128x64x128
//      P = lower(Qh Ac^T),  T = (I + strictly-lower(Bh Ac^T))^-1         (warp MMAs, tri_inverse.cuh)
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
#include "tri_inverse.cuh"

namespace dr {
namespace tc {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dim
constexpr int VS = 64;    // value columns per CTA
constexpr int NT = 512;   // threads
constexpr int RG = 8;     // rows of a chunk handled by one elementwise thread (two columns each)

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
constexpr uint32_t OFF_AH = OFF_RW + 64 * VS * 4;        // A, fp16 64 x LD (inverse input)
constexpr uint32_t OFF_AHT = OFF_AH + 64 * tri::LD * 2;  // A^T
constexpr uint32_t OFF_THT = OFF_AHT + 64 * tri::LD * 2; // T^T (inverse scratch)
constexpr uint32_t OFF_GC = OFF_THT + 64 * tri::LD * 2;  // gamma_C, 128 fp32
constexpr uint32_t OFF_PX = OFF_GC + 128 * 4;            // per-row-group gate products, 8 x 128 fp32
constexpr uint32_t OFF_END = OFF_PX + 8 * 128 * 4;
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
  const float *s = nullptr;  // write-side key scale [B,T,H,dk] (a = s (.) b); only the ring kernel reads it
  const int *cu_seqlens = nullptr;  // packed batch: sequence b is tokens cu[b] .. cu[b+1]-1 (ring kernel only)
  // ring kernel, dense batch only: the state at the start of every chunk, [B, H, ceil(T/64), dk, dv] fp32
  // (for the chunkwise backward pass); NULL: not stored
  float *states = nullptr;
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

// Gate values of two adjacent key channels (c, c+1) of one token: scalar, channel or absent (= 1).
__device__ __forceinline__ float2 gate_pair(const float *g, int mode, size_t th, int c) {
  if (mode == MODE_ABSENT) return make_float2(1.f, 1.f);
  if (mode == MODE_SCALAR) {
    const float x = __ldg(g + th);
    return make_float2(x, x);
  }
  return __ldg(reinterpret_cast<const float2 *>(g + th * DK + c));
}
__device__ __forceinline__ float sqrt_fast(float x) { return x > 0.f ? x * rsqrtf(x) : 0.f; }

template <typename IO>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bv,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar, raw_bar;
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
  __half *sAh = reinterpret_cast<__half *>(sm + OFF_AH);
  __half *sAhT = reinterpret_cast<__half *>(sm + OFF_AHT);
  __half *sThT = reinterpret_cast<__half *>(sm + OFF_THT);
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
  // rows 0..63 of [T; P] hold the lower-triangular T; its upper blocks stay zero
  reinterpret_cast<uint4 *>(tTP)[tid] = make_uint4(0u, 0u, 0u, 0u);
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
  // Waits are bounded and the decision to stop is taken by the whole CTA at once.
  // TMA data: every thread waits on the barrier (each then sees the bytes).
  auto wait_raw = [&]() -> bool {
    const bool ok = mbar_wait(&raw_bar, rphase & 1u, kWaitLimitNs);
    rphase++;
    if (!ok && lane == 0) raise_status(p.status, STATUS_TIMEOUT);
    return __syncthreads_or(!ok) == 0;
  };
  // MMA completion: one thread waits, the CTA barrier releases the others.
  auto wait_mma = [&]() -> bool {
    bool ok = true;
    if (tid == 0) ok = mbar_wait(&mma_bar, mphase & 1u, kWaitLimitNs);
    mphase++;
    const bool fail = __syncthreads_or(!ok) != 0;
    tc_fence_after();
    if (fail && tid == 0) raise_status(p.status, STATUS_TIMEOUT);
    return !fail;
  };

  // Elementwise layout: thread (kp, rgp) owns key channels 2kp, 2kp+1 and rows 8rgp .. 8rgp+7.
  const int kp = tid & 63, rgp = tid >> 6, c0 = 2 * kp;
  const int wc = tid >> 3, wj0 = (tid & 7) * 8;  // write-vector block: row wc, columns wj0..wj0+7
  float pal[2 * RG], pbe[2 * RG], pws = 0.f;     // prefetched gates of the next chunk
#pragma unroll
  for (int i = 0; i < 2 * RG; ++i) pal[i] = pbe[i] = 1.f;
  // Loads only, issued one chunk ahead: every value lands directly in its register and is
  // masked or broadcast only when it is consumed, so nothing here waits for memory.
  // Rows past the end of the sequence load the last valid row (masked at use).
  auto prefetch_gates = [&](int t0) {
    const int L = min(C, T - t0);
    const size_t thb = (static_cast<size_t>(b) * T + t0) * H + h;
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      const size_t th = thb + static_cast<size_t>(min(rgp * RG + j, L - 1)) * H;
      if (p.alpha_mode == MODE_CHANNEL) {
        const float2 a = __ldg(reinterpret_cast<const float2 *>(p.alpha + th * DK + c0));
        pal[2 * j] = a.x;
        pal[2 * j + 1] = a.y;
      } else if (p.alpha_mode == MODE_SCALAR) {
        pal[2 * j] = __ldg(p.alpha + th);
      }
      if (p.beta_k_mode == MODE_CHANNEL) {
        const float2 bt = __ldg(reinterpret_cast<const float2 *>(p.beta_k + th * DK + c0));
        pbe[2 * j] = bt.x;
        pbe[2 * j + 1] = bt.y;
      } else {
        pbe[2 * j] = __ldg(p.beta_k + th);
      }
    }
    if (!bv_tma && !sym_channel)  // raw scalar strength of row wc (beta_v, or beta_k for the symmetric write)
      pws = __ldg((p.beta_v_mode == MODE_SCALAR ? p.beta_v : p.beta_k) + thb +
                  static_cast<size_t>(min(wc, L - 1)) * H);
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

  // shared-memory descriptors of the operand tiles (K steps are added per MMA)
  const uint32_t a_base = smem_u32(sm);
  const uint64_t dQB = sdesc_sw128(a_base + OFF_QKB + 64 * 128, 16, 1024);   // [Qh; Bh], K-major, R = 192
  const uint64_t dWQ = sdesc_sw128(a_base + OFF_QKB, 16, 1024);              // [-W; Qh], K-major, R = 192
  const uint64_t dBh = sdesc_sw128(a_base + OFF_QKB + 128 * 128, 192 * 128, 1024);  // Bh as MN-major B
  const uint64_t dAcK = sdesc_sw128(a_base + OFF_AC, 16, 1024);              // Ac, K-major B (N = 64)
  const uint64_t dAcM = sdesc_sw128(a_base + OFF_AC, 64 * 128, 1024);        // Ac^T as MN-major A (M = 128)
  const uint64_t dTP = sdesc_sw128(a_base + OFF_TP, 16, 1024);               // [T; P], K-major (K = 64)
  const uint64_t dWr = sdesc_sw128(a_base + OFF_WR, 64 * 128, 1024);         // Wr, MN-major B
  const uint64_t dS = sdesc_sw128(a_base + OFF_S, 128 * 128, 1024);          // S, MN-major B
  const uint64_t dU = sdesc_sw128(a_base + OFF_U, 64 * 128, 1024);           // U, MN-major B
  // K step kk of a K-major tile with R rows: +32 B inside a 64-column block, +R*128 B per block
  auto kstep = [](uint64_t d, int R, int kk) -> uint64_t {
    return d + static_cast<uint64_t>(((kk >> 2) * R * 128 + (kk & 3) * 32) >> 4);
  };
  // K step kk of an MN-major tile: 16 rows of 128 B
  auto mstep = [](uint64_t d, int kk) -> uint64_t { return d + static_cast<uint64_t>(kk * 128); };

  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = min(C, T - t0);
    if (!wait_raw()) { aborted = true; break; }

    // ------------------------------------------------------------ K1 + a0 (operand tiles)
    {
      // gates of this chunk: mask rows past the end (alpha = 1, beta = 0), broadcast scalars
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const bool valid = rgp * RG + j < L;
        if (p.alpha_mode != MODE_CHANNEL) pal[2 * j + 1] = pal[2 * j];
        if (p.alpha_mode == MODE_ABSENT || !valid) pal[2 * j] = pal[2 * j + 1] = 1.f;
        if (p.beta_k_mode != MODE_CHANNEL) pbe[2 * j + 1] = pbe[2 * j];
        if (!valid) pbe[2 * j] = pbe[2 * j + 1] = 0.f;
      }
      float pre[2 * RG];
      float p0 = 1.f, p1 = 1.f;
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        p0 *= pal[2 * j];
        p1 *= pal[2 * j + 1];
        pre[2 * j] = p0;
        pre[2 * j + 1] = p1;
      }
      *reinterpret_cast<float2 *>(sPX + rgp * 128 + c0) = make_float2(p0, p1);
      __syncthreads();
      // head: product of the row groups before mine; tail: after mine; gamma_C: all
      float h0 = 1.f, h1 = 1.f, t0a = 1.f, t1a = 1.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 x = *reinterpret_cast<const float2 *>(sPX + g * 128 + c0);
        if (g < rgp) {
          h0 *= x.x;
          h1 *= x.y;
        } else if (g > rgp) {
          t0a *= x.x;
          t1a *= x.y;
        }
      }
      const float g0 = h0 * p0 * t0a, g1 = h1 * p1 * t1a;
      if (rgp == 0) {
        *reinterpret_cast<float2 *>(sGC + c0) = make_float2(g0, g1);
        if (!(fminf(g0, g1) >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
      }
      const bool own_w = sym_channel && c0 >= v0 && c0 < v0 + VS;
      // swizzled byte offsets of (row, c0) inside the K-major tiles: row & 7 == j for row = 8 rgp + j (+64, +128)
      const uint32_t blk = static_cast<uint32_t>(kp >> 5), ch = static_cast<uint32_t>((kp & 31) >> 2);
      const uint32_t inb = static_cast<uint32_t>((kp & 3) * 4);
      uint8_t *pQ = tQKB + blk * 192 * 128 + (64 + rgp * RG) * 128 + inb;
      uint8_t *pB = tQKB + blk * 192 * 128 + (128 + rgp * RG) * 128 + inb;
      uint8_t *pA = tAC + blk * 64 * 128 + (rgp * RG) * 128 + inb;
      // exp(-g_r) = R_r / gamma_C with R_r = product of the gates after row r (no division per element)
      const float ig0 = __fdividef(1.f, g0), ig1 = __fdividef(1.f, g1);
      float suf0 = t0a * ig0, suf1 = t1a * ig1;  // R_r / gamma_C for the last row of my group
      const bool beta_scalar = p.beta_k_mode == MODE_SCALAR;
      float amax = 0.f;
#pragma unroll
      for (int j = RG - 1; j >= 0; --j) {
        const int r = rgp * RG + j;
        const uint32_t sw = ((ch ^ static_cast<uint32_t>(j)) << 4) + j * 128;
        const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(rK + (r * DK + c0) * 2);
        const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(rQ + (r * DK + c0) * 2);
        const float2 kf = __bfloat1622float2(k2), qf = __bfloat1622float2(q2);
        float s0, s1;
        if (beta_scalar) {  // one square root per row
          s0 = s1 = sqrt_fast(pbe[2 * j]);
        } else {
          s0 = sqrt_fast(pbe[2 * j]);
          s1 = sqrt_fast(pbe[2 * j + 1]);
        }
        const float b0 = s0 * kf.x, b1 = s1 * kf.y;  // rows >= L: k = 0 (TMA fill), beta = 0
        const float ga = h0 * pre[2 * j], gb = h1 * pre[2 * j + 1];
        const float a0 = b0 * suf0, a1 = b1 * suf1;
        suf0 *= pal[2 * j];
        suf1 *= pal[2 * j + 1];
        amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
        *reinterpret_cast<uint32_t *>(pQ + sw) = pack_f16x2(ga * qf.x, gb * qf.y);  // Qh
        *reinterpret_cast<uint32_t *>(pB + sw) = pack_f16x2(ga * b0, gb * b1);      // Bh
        *reinterpret_cast<uint32_t *>(pA + sw) = pack_f16x2(a0, a1);                // Ac = b exp(-g)
        if (own_w) *reinterpret_cast<float2 *>(rW + r * VS + (c0 - v0)) = make_float2(s0, s1);
      }
      if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      if (sym_channel) __syncthreads();
      // write vectors w (rows c, value columns of this slice)
      {
        const uint4 vraw = *reinterpret_cast<const uint4 *>(rV + (wc * VS + wj0) * 2);
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vraw);
        float sc[8];
        if (bv_tma || sym_channel) {
          const float4 s_lo = *reinterpret_cast<const float4 *>(rW + wc * VS + wj0);
          const float4 s_hi = *reinterpret_cast<const float4 *>(rW + wc * VS + wj0 + 4);
          sc[0] = s_lo.x; sc[1] = s_lo.y; sc[2] = s_lo.z; sc[3] = s_lo.w;
          sc[4] = s_hi.x; sc[5] = s_hi.y; sc[6] = s_hi.z; sc[7] = s_hi.w;
        } else {
          const float sc0 = (p.beta_v_mode == MODE_SCALAR) ? pws : sqrt_fast(pws);
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = sc0;
        }
        const bool valid = wc < L;
        float w8[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 vf = __bfloat1622float2(v2[i]);
          w8[2 * i] = valid ? sc[2 * i] * vf.x : 0.f;
          w8[2 * i + 1] = valid ? sc[2 * i + 1] * vf.y : 0.f;
        }
        st_h16x8(tWR, wc, wj0, 64, w8);
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
        umma_f16(tmem + COL_D1, kstep(dQB, 192, kk), kstep(dAcK, 64, kk), idesc, kk > 0);
      umma_commit(&mma_bar);
    }
    // the raw staging area and the gate registers are free: fetch chunk c+1 while m1 runs
    if (t0 + C < T) {
      if (tid == 0) issue_raw(t0 + C);
      prefetch_gates(t0 + C);
    }
    if (!wait_mma()) { aborted = true; break; }

    // ------------------------------------------------------------ E1: P (fp16 tile), A and A^T (fp16)
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
        for (int i = 0; i < 16; i += 2) {
          const int col = cq * 16 + i;
          const float x0 = (col < r) ? x[i] : 0.f, x1 = (col + 1 < r) ? x[i + 1] : 0.f;
          *reinterpret_cast<uint32_t *>(sAh + r * tri::LD + col) = pack_f16x2(x0, x1);
          sAhT[col * tri::LD + r] = __float2half_rn(x0);
          sAhT[(col + 1) * tri::LD + r] = __float2half_rn(x1);
        }
      }
    }
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ K2: T = (I + A)^-1 (warp MMAs)
    tri::inverse64(sAh, sAhT, sThT, warp, lane, [&](int bi, int bj, const tri::Frag &F, int ln) {
      const int r = ln >> 2, qq = ln & 3;
      const int row = 16 * bi + r, col = 16 * bj + 2 * qq;
      *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col, 128)) = pack_f16x2(F.v[0], F.v[1]);
      *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col, 128)) = pack_f16x2(F.v[2], F.v[3]);
      *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col + 8, 128)) = pack_f16x2(F.v[4], F.v[5]);
      *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col + 8, 128)) = pack_f16x2(F.v[6], F.v[7]);
    }, [] { __syncthreads(); });
    fence_async_smem();
    __syncthreads();

    // ------------------------------------------------------------ m2: D2 = [T;P] Bh,  m3: D1 = [T;P] Wr
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id2 = idesc_f16_f32(128, 128, false, true);
      const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D2, kstep(dTP, 128, kk), mstep(dBh, kk), id2, kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D1, kstep(dTP, 128, kk), mstep(dWr, kk), id3, kk > 0);
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
      for (int kk = 0; kk < DK / 16; ++kk) umma_f16(tmem + COL_D3, kstep(dWQ, 192, kk), mstep(dS, kk), id, kk > 0);
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
      for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D4, mstep(dAcM, kk), mstep(dU, kk), id4, kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D3, kstep(dTP, 128, kk), mstep(dU, kk), id3, 1u);
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
