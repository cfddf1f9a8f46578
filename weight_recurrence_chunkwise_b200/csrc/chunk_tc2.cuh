// chunk_tc2.cuh -- chunkwise WY/UT prefill on a cluster of two CTAs per (b, h).
//
// Same algebra as chunk_tc.cuh (DeltaNet page, step 7; FG2-GDN page, section 2):
//   chunk-local:  gamma, Qh = gamma q, Bh = gamma b, Ac = b exp(-g), P = lower(Qh Ac^T),
//                 T = (I + strictly-lower(Bh Ac^T))^-1, W = T Bh
//   state pass:   U0 = T Wr, U = U0 - W S, O = Qh S + P U, S <- Diag(gamma_C)(S + Ac^T U)
//
// The chunk-local factors do not depend on the value slice, so the two CTAs of
// a head (value columns 0..63 and 64..127) share them: CTA r computes them for
// the chunks c with c % 2 == r, writes them into its slot r, and copies the
// slot into the other CTA's slot r over DSMEM.  Each CTA runs two warp groups
// at once: warps 0..7 build its chunks' factors (local role), warps 8..15 run
// the serial state pass over every chunk for its value slice (chain role).  The
// local work of chunk c+1 therefore overlaps the state pass of chunk c, and
// each CTA does only half of the local work.
//
// Slots: the K-major stacked tile STK holds, in 320 rows,
//   [-W_0 (0..63); Qh_0 (64..127); Bh (128..191); Qh_1 (192..255); -W_1 (256..319)]
// so that [Qh_0; Bh], [Bh; Qh_1] (local MMA) and [-W_0; Qh_0], [Qh_1; -W_1]
// (state-pass MMA) are each 128 contiguous rows.  For slot 1 every 128-row
// product therefore has its two halves swapped; `tl` (rows of T, W, U0, -W S)
// and `pl` (rows of P, Qh S, O) give the TMEM lane base of each half.
//
// Synchronisation (every wait bounded):
//   full[s]   slot s is ready: local arrive (own slot) or the peer's remote
//             arrive.expect_tx + bulk-copy bytes (the peer's slot)
//   own_free  this CTA's state pass is done with its copy of slot `rank`
//   peer_free the peer's state pass is done with its copy of slot `rank`
#pragma once
#include "chunk_tc.cuh"

namespace dr {
namespace tc2 {

using tc::C;
using tc::DK;
using tc::VS;
using tc::kF16Max;
using tc::kMinChunkDecayF16;
using tc::Params;

constexpr int NT = 512;   // threads
constexpr int NL = 256;   // local role: threads 0..255
constexpr int BAR_LOCAL = 1, BAR_CHAIN = 2;
constexpr int RGL = 16;   // rows per local elementwise thread (two key channels each)

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t STK_ROWS = 320;
constexpr uint32_t OFF_STK = 0;                              // 2 column blocks x 320 rows x 128 B
constexpr uint32_t OFF_AC0 = OFF_STK + 2 * STK_ROWS * 128;   // Ac of slot 0 (64 x 128)
constexpr uint32_t OFF_AC1 = OFF_AC0 + 64 * 256;
constexpr uint32_t OFF_TP0 = OFF_AC1 + 64 * 256;             // [T; P] of slot 0 (128 x 64)
constexpr uint32_t OFF_TP1 = OFF_TP0 + 128 * 128;            // [P; T] of slot 1
constexpr uint32_t OFF_GC0 = OFF_TP1 + 128 * 128;            // gamma_C of slot 0 (128 fp32)
constexpr uint32_t OFF_GC1 = OFF_GC0 + 512;
constexpr uint32_t OFF_S = OFF_GC1 + 512;                    // state, fp16 copy (128 x VS)
constexpr uint32_t OFF_U = OFF_S + 128 * 128;                // U (64 x VS)
constexpr uint32_t OFF_WR = OFF_U + 64 * 128;                // write vectors (raw v lands here, swizzled)
constexpr uint32_t OFF_RB = OFF_WR + 64 * 128;               // write scales, fp32 64 x VS
constexpr uint32_t OFF_AH = OFF_RB + 64 * VS * 4;            // A (fp16, stride tri::LD); raw q staging
constexpr uint32_t OFF_THT = OFF_AH + 64 * tri::LD * 2;      // T^T (inverse scratch)
constexpr uint32_t OFF_PX = OFF_THT + 64 * tri::LD * 2;      // row-group gate products, 4 x 128 fp32
constexpr uint32_t OFF_END = OFF_PX + 4 * 128 * 4;
constexpr size_t SMEM_BYTES = OFF_END + 1024;
static_assert(OFF_S % 1024 == 0 && OFF_U % 1024 == 0 && OFF_WR % 1024 == 0 && OFF_AH % 1024 == 0,
              "tile alignment");
static_assert(OFF_THT + 64 * tri::LD * 2 >= OFF_AH + 64 * 256, "raw q staging fits in the inverse scratch");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
constexpr uint32_t SLOT_BYTES = 2 * 128 * 128 + 64 * 256 + 128 * 128 + 512;  // bytes copied to the peer

// TMEM columns
constexpr uint32_t COL_D1 = 0;     // local: [P raw | A raw] (64)
constexpr uint32_t COL_D2 = 64;    // local: W (128)
constexpr uint32_t COL_U0 = 192;   // chain: U0 (64)
constexpr uint32_t COL_D3 = 256;   // chain: [-W S | Qh S + P U] (64), even chunks
constexpr uint32_t COL_D4 = 320;   // chain: Ac^T U (64)
constexpr uint32_t COL_D3B = 384;  // chain: D3 of odd chunks (64)
constexpr uint32_t TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t col_d3(int c) { return (c & 1) ? COL_D3B : COL_D3; }

__host__ __device__ constexpr uint32_t off_ac(int s) { return s ? OFF_AC1 : OFF_AC0; }
__host__ __device__ constexpr uint32_t off_tp(int s) { return s ? OFF_TP1 : OFF_TP0; }
__host__ __device__ constexpr uint32_t off_gc(int s) { return s ? OFF_GC1 : OFF_GC0; }
__host__ __device__ constexpr int row_q(int s) { return s ? 192 : 64; }    // Qh rows in STK
__host__ __device__ constexpr int row_w(int s) { return s ? 256 : 0; }     // -W rows in STK
__host__ __device__ constexpr int row_chain(int s) { return s ? 192 : 0; } // state-pass A operand
__host__ __device__ constexpr int row_m1(int s) { return s ? 128 : 64; }   // local A operand [Qh; Bh] / [Bh; Qh]
__host__ __device__ constexpr int lane_t(int s) { return s ? 64 : 0; }     // T, W, U0, -W S
__host__ __device__ constexpr int lane_p(int s) { return s ? 0 : 64; }     // P, Qh S, O

template <typename IO>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_qk, bar_lmma, bar_cmma, bar_v, bar_full[2], bar_own_free, bar_peer_free;
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase_addr = smem_u32(sm);

  const int T = p.T, H = p.H, DV = p.DV;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster_ctarank());  // value slice; equals blockIdx.x
  const int peer = rank ^ 1;
  const int v0 = rank * VS, h = blockIdx.y, b = blockIdx.z;
  const int nchunks = (T + C - 1) / C;
  const bool bv_tma = p.beta_v_mode == MODE_CHANNEL;
  const bool sym_channel = p.beta_v_mode == MODE_ABSENT && p.beta_k_mode == MODE_CHANNEL;
  const bool scale_tma = bv_tma || sym_channel;  // per-column write scales come by TMA
  const uint32_t qk_bytes = 64 * 256 + 2 * 64 * 128;
  const uint32_t v_bytes = 64 * 128 + (scale_tma ? 64 * VS * 4 : 0);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_qk, 1);
    mbar_init(&bar_lmma, 1);
    mbar_init(&bar_cmma, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_own_free, 1);
    mbar_init(&bar_peer_free, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (scale_tma) tma_prefetch_desc(&tm_b);
  }
  // [T; P] tiles: the upper blocks of T are never written and stay zero
  for (int i = tid; i < 2 * 128 * 128 / 16; i += NT)
    reinterpret_cast<uint4 *>(sm + OFF_TP0)[i] = make_uint4(0u, 0u, 0u, 0u);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // descriptors (K steps added per MMA)
  auto kstep = [](uint64_t d, int R, int kk) -> uint64_t {
    return d + static_cast<uint64_t>(((kk >> 2) * R * 128 + (kk & 3) * 32) >> 4);
  };
  auto mstep = [](uint64_t d, int kk) -> uint64_t { return d + static_cast<uint64_t>(kk * 128); };

  if (tid < NL) {
    // ================================================================== local role
    const int ltid = tid;
    uint32_t ph_qk = 0, ph_mma = 0, ph_own = 0, ph_peer = 0;
    bool aborted = false;
    const int kp = ltid & 63, rgl = ltid >> 6, c0 = 2 * kp;
    const int quarter = warp & 3, half = warp >> 2;  // warps 0..7
    float pal[2 * RGL], pbe[2 * RGL];
#pragma unroll
    for (int i = 0; i < 2 * RGL; ++i) pal[i] = pbe[i] = 1.f;

    auto issue_qk = [&](int c) {
      const int t0 = c * C;
      mbar_arrive_expect_tx(&bar_qk, qk_bytes);
      tma_load_4d(sm + OFF_AH, &tm_q, &bar_qk, 0, h, t0, b);                          // raw q, row-major
      tma_load_4d(sm + OFF_STK + 128 * 128, &tm_k, &bar_qk, 0, h, t0, b);             // raw k -> Bh rows
      tma_load_4d(sm + OFF_STK + STK_ROWS * 128 + 128 * 128, &tm_k, &bar_qk, 64, h, t0, b);
    };
    // Scalar gates (alpha absent or per token, beta_k per token): warp 0 stages the 64 row gates
    // of the next chunk in shared memory by cp.async (lane l: rows 2l, 2l+1); everything else is
    // per element.
    const bool gates_scalar = p.alpha_mode != MODE_CHANNEL && p.beta_k_mode == MODE_SCALAR;
    float *sGate = reinterpret_cast<float *>(sm + OFF_PX) + 256;  // [0..63] alpha, [64..127] beta_k
    auto prefetch_gates = [&](int c) {  // loads only; masking and broadcast happen at use
      const int t0 = c * C, L = min(C, T - t0);
      const size_t thb = (static_cast<size_t>(b) * T + t0) * H + h;
      if (gates_scalar) {
        if (warp == 0) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const size_t th = thb + static_cast<size_t>(min(2 * lane + e, L - 1)) * H;
            if (p.alpha_mode == MODE_SCALAR) cp_async4(sGate + 2 * lane + e, p.alpha + th);
            cp_async4(sGate + 64 + 2 * lane + e, p.beta_k + th);
          }
          cp_async_commit();
        }
        return;
      }
#pragma unroll
      for (int j = 0; j < RGL; ++j) {
        const size_t th = thb + static_cast<size_t>(min(rgl * RGL + j, L - 1)) * H;
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
    };
    // TMA data: every thread waits; signals: one thread waits, the group barrier releases the others
    auto wait_all = [&](uint64_t *bar, uint32_t &ph) -> bool {
      const bool ok = mbar_wait(bar, ph & 1u, kWaitLimitNs);
      ph++;
      const bool fail = bar_or(BAR_LOCAL, NL, !ok);
      if (fail && ltid == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };
    auto wait_one = [&](uint64_t *bar, uint32_t &ph, bool cluster_scope) -> bool {
      bool ok = true;
      if (ltid == 0)
        ok = cluster_scope ? mbar_wait_cluster(bar, ph & 1u, kWaitLimitNs) : mbar_wait(bar, ph & 1u, kWaitLimitNs);
      ph++;
      const bool fail = bar_or(BAR_LOCAL, NL, !ok);
      tc_fence_after();
      if (fail && ltid == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };

    const int s = rank;  // this CTA always fills slot `rank`
    uint8_t *tQB = sm + OFF_STK;
    uint8_t *tAC = sm + off_ac(s);
    uint8_t *tTP = sm + off_tp(s);
    float *sGC = reinterpret_cast<float *>(sm + off_gc(s));
    float *sPX = reinterpret_cast<float *>(sm + OFF_PX);
    __half *sAh = reinterpret_cast<__half *>(sm + OFF_AH);
    __half *sThT = reinterpret_cast<__half *>(sm + OFF_THT);
    const uint8_t *rQ = sm + OFF_AH;
    const int tl = lane_t(s), pl = lane_p(s);

    const uint64_t dM1 = sdesc_sw128(sbase_addr + OFF_STK + row_m1(s) * 128, 16, 1024);
    const uint64_t dAcK = sdesc_sw128(sbase_addr + off_ac(s), 16, 1024);
    const uint64_t dTP = sdesc_sw128(sbase_addr + off_tp(s), 16, 1024);
    const uint64_t dBh = sdesc_sw128(sbase_addr + OFF_STK + 128 * 128, STK_ROWS * 128, 1024);

    if (rank < nchunks) {
      if (ltid == 0) issue_qk(rank);
      prefetch_gates(rank);
    }
    for (int c = rank; c < nchunks; c += 2) {
      const int t0 = c * C, L = min(C, T - t0);
      if (c >= 2) {
        if (!wait_one(&bar_own_free, ph_own, false)) { aborted = true; break; }
        if (!wait_one(&bar_peer_free, ph_peer, true)) { aborted = true; break; }
      }
      if (!wait_all(&bar_qk, ph_qk)) { aborted = true; break; }

      // -------------------------------------------------------------- K1 + a0: Qh, Bh (in place), Ac, gamma_C
      if (gates_scalar) {
        // row gates: gamma_r (inclusive product), 1/gamma_r, sqrt(beta_r); 64 rows over warp 0
        float *sRow = sPX;  // [0..63] gamma, [64..127] 1/gamma, [128..191] sqrt(beta)
        if (warp == 0) {
          cp_async_wait_all();  // this lane's own staged rows
          const float2 ga = *reinterpret_cast<const float2 *>(sGate + 2 * lane);
          const float2 gb = *reinterpret_cast<const float2 *>(sGate + 64 + 2 * lane);
          const bool asc = p.alpha_mode == MODE_SCALAR;
          const float a0 = (asc && 2 * lane < L) ? ga.x : 1.f, a1 = (asc && 2 * lane + 1 < L) ? ga.y : 1.f;
          const float b0 = (2 * lane < L) ? gb.x : 0.f, b1 = (2 * lane + 1 < L) ? gb.y : 0.f;
          float pr = a0 * a1, incl = pr;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl *= y;
          }
          const float up = __shfl_up_sync(0xffffffffu, incl, 1);
          const float ex = (lane == 0) ? 1.f : up;  // product of the rows before 2*lane
          const float g0 = ex * a0, g1 = g0 * a1;
          const float gC = __shfl_sync(0xffffffffu, incl, 31);
          sRow[2 * lane] = g0;
          sRow[2 * lane + 1] = g1;
          sRow[64 + 2 * lane] = __fdividef(1.f, g0);
          sRow[64 + 2 * lane + 1] = __fdividef(1.f, g1);
          sRow[128 + 2 * lane] = tc::sqrt_fast(b0);
          sRow[128 + 2 * lane + 1] = tc::sqrt_fast(b1);
          *reinterpret_cast<float4 *>(sGC + 4 * lane) = make_float4(gC, gC, gC, gC);
          if (lane == 0 && !(gC >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
        }
        bar_sync(BAR_LOCAL, NL);
        // elements: (row r, 8-column chunk j8), four per thread, 16-byte loads and stores
        const int j8 = ltid & 15;
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = (ltid >> 4) + 16 * i;
          const float g = sRow[r], gi = sRow[64 + r], sb = sRow[128 + r];
          const uint4 qraw = *reinterpret_cast<const uint4 *>(rQ + (r * DK + j8 * 8) * 2);
          uint4 *pk = reinterpret_cast<uint4 *>(tQB + sw128_off16(128 + r, j8, STK_ROWS));
          const uint4 kraw = *pk;
          const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qraw);
          const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw);
          uint32_t oq[4], ob[4], oa[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 qf = __bfloat1622float2(q2[e]), kf = __bfloat1622float2(k2[e]);
            const float b0 = sb * kf.x, b1 = sb * kf.y;
            const float x0 = b0 * gi, x1 = b1 * gi;
            amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
            oq[e] = pack_f16x2(g * qf.x, g * qf.y);
            ob[e] = pack_f16x2(g * b0, g * b1);
            oa[e] = pack_f16x2(x0, x1);
          }
          *reinterpret_cast<uint4 *>(tQB + sw128_off16(row_q(s) + r, j8, STK_ROWS)) = make_uint4(oq[0], oq[1], oq[2], oq[3]);
          *pk = make_uint4(ob[0], ob[1], ob[2], ob[3]);
          *reinterpret_cast<uint4 *>(tAC + sw128_off16(r, j8, 64)) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        }
        if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      } else {
#pragma unroll
        for (int j = 0; j < RGL; ++j) {
          const bool valid = rgl * RGL + j < L;
          if (p.alpha_mode != MODE_CHANNEL) pal[2 * j + 1] = pal[2 * j];
          if (p.alpha_mode == MODE_ABSENT || !valid) pal[2 * j] = pal[2 * j + 1] = 1.f;
          if (p.beta_k_mode != MODE_CHANNEL) pbe[2 * j + 1] = pbe[2 * j];
          if (!valid) pbe[2 * j] = pbe[2 * j + 1] = 0.f;
        }
        float pre[2 * RGL];
        float p0 = 1.f, p1 = 1.f;
#pragma unroll
        for (int j = 0; j < RGL; ++j) {
          p0 *= pal[2 * j];
          p1 *= pal[2 * j + 1];
          pre[2 * j] = p0;
          pre[2 * j + 1] = p1;
        }
        *reinterpret_cast<float2 *>(sPX + rgl * 128 + c0) = make_float2(p0, p1);
        bar_sync(BAR_LOCAL, NL);
        float h0 = 1.f, h1 = 1.f, t0a = 1.f, t1a = 1.f;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float2 x = *reinterpret_cast<const float2 *>(sPX + g * 128 + c0);
          if (g < rgl) {
            h0 *= x.x;
            h1 *= x.y;
          } else if (g > rgl) {
            t0a *= x.x;
            t1a *= x.y;
          }
        }
        const float g0 = h0 * p0 * t0a, g1 = h1 * p1 * t1a;
        if (rgl == 0) {
          *reinterpret_cast<float2 *>(sGC + c0) = make_float2(g0, g1);
          if (!(fminf(g0, g1) >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
        }
        const float ig0 = __fdividef(1.f, g0), ig1 = __fdividef(1.f, g1);
        float suf0 = t0a * ig0, suf1 = t1a * ig1;  // R_r / gamma_C for the last row of my group
        const bool beta_scalar = p.beta_k_mode == MODE_SCALAR;
        const uint32_t blk = static_cast<uint32_t>(kp >> 5), ch = static_cast<uint32_t>((kp & 31) >> 2);
        const uint32_t inb = static_cast<uint32_t>((kp & 3) * 4);
        uint8_t *pQ = tQB + blk * STK_ROWS * 128 + (row_q(s) + rgl * RGL) * 128 + inb;
        uint8_t *pB = tQB + blk * STK_ROWS * 128 + (128 + rgl * RGL) * 128 + inb;
        uint8_t *pA = tAC + blk * 64 * 128 + (rgl * RGL) * 128 + inb;
        float amax = 0.f;
#pragma unroll
        for (int j = RGL - 1; j >= 0; --j) {
          const int r = rgl * RGL + j;
          const uint32_t sw = ((ch ^ static_cast<uint32_t>(j & 7)) << 4) + j * 128;
          const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(pB + sw);  // raw k (swizzled)
          const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(rQ + (r * DK + c0) * 2);
          const float2 kf = __bfloat1622float2(k2), qf = __bfloat1622float2(q2);
          float s0, s1;
          if (beta_scalar) {
            s0 = s1 = tc::sqrt_fast(pbe[2 * j]);
          } else {
            s0 = tc::sqrt_fast(pbe[2 * j]);
            s1 = tc::sqrt_fast(pbe[2 * j + 1]);
          }
          const float b0 = s0 * kf.x, b1 = s1 * kf.y;
          const float ga = h0 * pre[2 * j], gb = h1 * pre[2 * j + 1];
          const float a0 = b0 * suf0, a1 = b1 * suf1;
          suf0 *= pal[2 * j];
          suf1 *= pal[2 * j + 1];
          amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
          *reinterpret_cast<uint32_t *>(pQ + sw) = pack_f16x2(ga * qf.x, gb * qf.y);  // Qh
          *reinterpret_cast<uint32_t *>(pB + sw) = pack_f16x2(ga * b0, gb * b1);      // Bh (in place of k)
          *reinterpret_cast<uint32_t *>(pA + sw) = pack_f16x2(a0, a1);                // Ac
        }
        if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      }
      fence_async_smem();
      bar_sync(BAR_LOCAL, NL);
      const uint32_t rbar = mapa_shared(smem_u32(&bar_full[s]), static_cast<uint32_t>(peer));
      auto copy_part = [&](uint32_t off, uint32_t bytes) {
        bulk_copy_to_peer(mapa_shared(sbase_addr + off, static_cast<uint32_t>(peer)), sm + off, bytes, rbar);
      };

      // -------------------------------------------------------------- m1: D1 = [Qh; Bh] Ac^T (halves swapped for slot 1)
      if (warp == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint32_t idesc = idesc_f16_f32(128, 64, false, false);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            umma_f16(tmem + COL_D1, kstep(dM1, STK_ROWS, kk), kstep(dAcK, 64, kk), idesc, kk > 0);
          umma_commit(&bar_lmma);
          // Qh, Ac and gamma_C of this chunk are final: start moving them into the peer's slot.  The
          // peer's full[s] phase completes on the copied bytes alone, so the arrive needs no release.
          mbar_expect_tx_remote_relaxed(rbar, SLOT_BYTES);
          copy_part(OFF_STK + row_q(s) * 128, 64 * 128);
          copy_part(OFF_STK + STK_ROWS * 128 + row_q(s) * 128, 64 * 128);
          copy_part(off_ac(s), 64 * 256);
          copy_part(off_gc(s), 512);
        }
        __syncwarp();
      }
      if (c + 2 < nchunks) prefetch_gates(c + 2);
      if (!wait_one(&bar_lmma, ph_mma, false)) { aborted = true; break; }

      // -------------------------------------------------------------- E1: P -> [T;P] tile, A -> fp16 scratch
      {
        float x[16];
        const int lane0 = quarter * 32;
        // D1 rows: slot 0 -> lanes 0..63 = P raw, 64..127 = A raw; slot 1 -> swapped
        const int p_lanes = s ? 64 : 0;
        const int trow = lane0 + lane;
        const bool is_p = (trow >= p_lanes) && (trow < p_lanes + 64);
        const int r = trow - (is_p ? p_lanes : (64 - p_lanes));
#pragma unroll
        for (int jh = 0; jh < 32; jh += 16) {
          tmem_ld16(tmem_addr(tmem, lane0, COL_D1 + half * 32 + jh), x);
          tmem_ld_wait();
          if (is_p) {
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = (half * 32 + jh + i <= r) ? x[i] : 0.f;
            tc::st_h16x16(tTP, pl + r, half * 32 + jh, 128, x);
          } else {
            const int col0 = half * 32 + jh;
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = (col0 + i < r) ? x[i] : 0.f;
            uint4 lo, hi;  // 16-byte stores: rows are 144 bytes apart, conflict-free per 8 lanes
            lo.x = pack_f16x2(x[0], x[1]);
            lo.y = pack_f16x2(x[2], x[3]);
            lo.z = pack_f16x2(x[4], x[5]);
            lo.w = pack_f16x2(x[6], x[7]);
            hi.x = pack_f16x2(x[8], x[9]);
            hi.y = pack_f16x2(x[10], x[11]);
            hi.z = pack_f16x2(x[12], x[13]);
            hi.w = pack_f16x2(x[14], x[15]);
            *reinterpret_cast<uint4 *>(sAh + r * tri::LD + col0) = lo;
            *reinterpret_cast<uint4 *>(sAh + r * tri::LD + col0 + 8) = hi;
          }
        }
      }
      tc_fence_before();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- K2: T = (I + A)^-1 (warp MMAs)
      tri::inverse64(sAh, nullptr, sThT, warp, lane, [&](int bi, int bj, const tri::Frag &F, int ln) {
        const int rr = ln >> 2, qq = ln & 3;
        const int row = tl + 16 * bi + rr, col = 16 * bj + 2 * qq;
        *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col, 128)) = pack_f16x2(F.v[0], F.v[1]);
        *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col, 128)) = pack_f16x2(F.v[2], F.v[3]);
        *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col + 8, 128)) = pack_f16x2(F.v[4], F.v[5]);
        *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col + 8, 128)) = pack_f16x2(F.v[6], F.v[7]);
      }, [] { bar_sync(BAR_LOCAL, NL); });
      fence_async_smem();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- m2: D2 = [T;P] Bh -> W at lanes tl
      if (warp == 0) {
        if (elect_one()) {
          copy_part(off_tp(s), 128 * 128);  // [T; P] is final
          tc_fence_after();
          const uint32_t id2 = idesc_f16_f32(128, 128, false, true);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            umma_f16(tmem + COL_D2, kstep(dTP, 128, kk), mstep(dBh, kk), id2, kk > 0);
          umma_commit(&bar_lmma);
        }
        __syncwarp();
      }
      if (!wait_one(&bar_lmma, ph_mma, false)) { aborted = true; break; }
      // Bh and the inverse scratch are free: fetch chunk c+2's raw q and k now
      if (ltid == 0 && c + 2 < nchunks) issue_qk(c + 2);

      // -------------------------------------------------------------- E2: -W -> STK rows of slot s
      if ((quarter * 32 >= tl) && (quarter * 32 < tl + 64)) {
        const int r = quarter * 32 + lane - tl;
#pragma unroll
        for (int j = 0; j < 64; j += 16) {
          float x[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D2 + half * 64 + j), x);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = -x[i];
          tc::st_h16x16(tQB, row_w(s) + r, half * 64 + j, STK_ROWS, x);
        }
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- hand the slot to both state passes
      if (ltid == 0) {
        copy_part(OFF_STK + row_w(s) * 128, 64 * 128);
        copy_part(OFF_STK + STK_ROWS * 128 + row_w(s) * 128, 64 * 128);
        mbar_arrive(&bar_full[s]);
      }
    }
    (void)aborted;
  } else {
    // ================================================================== chain role
    const int ct = tid - NL;
    const int cw = warp - 8;
    const int quarter = cw & 3, half = cw >> 2;
    const int trow = quarter * 32 + lane;
    uint32_t ph_v = 0, ph_mma = 0, ph_full[2] = {0u, 0u};
    bool aborted = false;
    const size_t sbase = (static_cast<size_t>(b) * H + h) * DK * DV;
    uint8_t *tS = sm + OFF_S;
    uint8_t *tU = sm + OFF_U;
    uint8_t *tWR = sm + OFF_WR;
    const float *rB = reinterpret_cast<const float *>(sm + OFF_RB);
    const int wc = ct >> 2, wjb = (ct & 3) * 2;  // write-vector row and its two 8-column chunks

    auto issue_v = [&](int c) {
      const int t0 = c * C;
      mbar_arrive_expect_tx(&bar_v, v_bytes);
      tma_load_4d(tWR, &tm_v, &bar_v, v0, h, t0, b);
      if (scale_tma) tma_load_4d(sm + OFF_RB, &tm_b, &bar_v, v0, h, t0, b);
    };
    float pws = 0.f;  // scalar write strength of row wc (raw; square root at use if symmetric)
    auto prefetch_ws = [&](int c) {
      if (scale_tma) return;
      const int t0 = c * C, L = min(C, T - t0);
      const size_t th = (static_cast<size_t>(b) * T + t0 + min(wc, L - 1)) * H + h;
      pws = __ldg((p.beta_v_mode == MODE_SCALAR ? p.beta_v : p.beta_k) + th);
    };
    auto wait_all = [&](uint64_t *bar, uint32_t &ph, bool cluster_scope) -> bool {
      const bool ok = cluster_scope ? mbar_wait_cluster(bar, ph & 1u, kWaitLimitNs) : mbar_wait(bar, ph & 1u, kWaitLimitNs);
      ph++;
      const bool fail = bar_or(BAR_CHAIN, NT - NL, !ok);
      if (fail && ct == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };
    auto wait_mma = [&]() -> bool {
      bool ok = true;
      if (ct == 0) ok = mbar_wait(&bar_cmma, ph_mma & 1u, kWaitLimitNs);
      ph_mma++;
      const bool fail = bar_or(BAR_CHAIN, NT - NL, !ok);
      tc_fence_after();
      if (fail && ct == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };

    // fp32 state slice: row trow, columns half*32 .. half*32+31 of this CTA's value slice
    float Sreg[32];
    {
      const float *src = p.S0 ? p.S0 + sbase + static_cast<size_t>(trow) * DV + v0 + half * 32 : nullptr;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        Sreg[j] = x.x;
        Sreg[j + 1] = x.y;
        Sreg[j + 2] = x.z;
        Sreg[j + 3] = x.w;
      }
      tc::st_h16x16(tS, trow, half * 32, 128, Sreg);
      tc::st_h16x16(tS, trow, half * 32 + 16, 128, Sreg + 16);
    }
    const uint64_t dS = sdesc_sw128(sbase_addr + OFF_S, 128 * 128, 1024);
    const uint64_t dU = sdesc_sw128(sbase_addr + OFF_U, 64 * 128, 1024);
    const uint64_t dWr = sdesc_sw128(sbase_addr + OFF_WR, 64 * 128, 1024);

    // write vectors of the chunk whose raw v sits in Wr, in place (after bar_v)
    auto convert_wr = [&]() {
      float sc[16];
      if (scale_tma) {
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 x = *reinterpret_cast<const float4 *>(rB + wc * VS + wjb * 8 + i);
          sc[i] = x.x;
          sc[i + 1] = x.y;
          sc[i + 2] = x.z;
          sc[i + 3] = x.w;
        }
        if (sym_channel) {
#pragma unroll
          for (int i = 0; i < 16; ++i) sc[i] = tc::sqrt_fast(sc[i]);
        }
      } else {
        const float s0 = (p.beta_v_mode == MODE_SCALAR) ? pws : tc::sqrt_fast(pws);
#pragma unroll
        for (int i = 0; i < 16; ++i) sc[i] = s0;
      }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        uint4 *ptr = reinterpret_cast<uint4 *>(tWR + sw128_off16(wc, wjb + jj, 64));
        const uint4 raw = *ptr;
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
        float w8[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 vf = __bfloat1622float2(v2[i]);
          w8[2 * i] = sc[jj * 8 + 2 * i] * vf.x;  // rows >= L: v = 0 (TMA fill)
          w8[2 * i + 1] = sc[jj * 8 + 2 * i + 1] * vf.y;
        }
        uint4 out;
        out.x = pack_f16x2(w8[0], w8[1]);
        out.y = pack_f16x2(w8[2], w8[3]);
        out.z = pack_f16x2(w8[4], w8[5]);
        out.w = pack_f16x2(w8[6], w8[7]);
        *ptr = out;
      }
    };
    // outputs of chunk c: its D3 columns at lanes pl hold Qh S + P U
    auto store_o = [&](int c) {
      const int pl = lane_p(c & 1), t0 = c * C, L = min(C, T - t0);
      if ((quarter * 32 >= pl) && (quarter * 32 < pl + 64)) {
        const int r = trow - pl;
#pragma unroll
        for (int j = 0; j < 32; j += 16) {
          float x[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, col_d3(c) + half * 32 + j), x);
          tmem_ld_wait();
          if (r < L) {
            const size_t th = (static_cast<size_t>(b) * T + t0 + r) * H + h;
            IO *dst = static_cast<IO *>(p.o) + th * DV + v0 + half * 32 + j;
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
    };

    // Software pipeline: the write vectors of chunk c+1 are built while the second MMA group of
    // chunk c runs, and the outputs of chunk c are stored while the first MMA group of chunk c+1
    // runs (D3 alternates between two column sets), so the serial path per chunk is
    // MMA group 1 -> U -> MMA group 2 -> S.
    if (nchunks > 0) {
      if (ct == 0) issue_v(0);
      prefetch_ws(0);
      if (wait_all(&bar_v, ph_v, false)) {
        convert_wr();
        if (nchunks > 1) prefetch_ws(1);
      } else {
        aborted = true;
      }
      fence_async_smem();
      bar_sync(BAR_CHAIN, NT - NL);
    }
    for (int c = 0; c < nchunks && !aborted; ++c) {
      const int s = c & 1;
      const int tl = lane_t(s);
      const uint32_t cD3 = col_d3(c);
      if (!wait_all(&bar_full[s], ph_full[s], true)) { aborted = true; break; }
      const float gc = reinterpret_cast<const float *>(sm + off_gc(s))[trow];

      // -------------------------------------------------------------- U0 = [T;P] Wr,  D3 = STK(s) S
      if (cw == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint64_t dTP = sdesc_sw128(sbase_addr + off_tp(s), 16, 1024);
          const uint64_t dCh = sdesc_sw128(sbase_addr + OFF_STK + row_chain(s) * 128, 16, 1024);
          const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_U0, kstep(dTP, 128, kk), mstep(dWr, kk), id3, kk > 0);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) umma_f16(tmem + cD3, kstep(dCh, STK_ROWS, kk), mstep(dS, kk), id3, kk > 0);
          umma_commit(&bar_cmma);
        }
        __syncwarp();
      }
      if (c > 0) store_o(c - 1);
      if (!wait_mma()) { aborted = true; break; }
      if (ct == 0 && c + 1 < nchunks) issue_v(c + 1);  // Wr and the scale staging are free

      // -------------------------------------------------------------- E3: U = U0 - W S (rows at lanes tl)
      if ((quarter * 32 >= tl) && (quarter * 32 < tl + 64)) {
        const int r = trow - tl;
#pragma unroll
        for (int j = 0; j < 32; j += 16) {
          float ws[16], u0[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, cD3 + half * 32 + j), ws);
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_U0 + half * 32 + j), u0);
          tmem_ld_wait();
          float mx = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            u0[i] += ws[i];
            mx = fmaxf(mx, fabsf(u0[i]));
          }
          if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
          tc::st_h16x16(tU, r, half * 32 + j, 64, u0);
        }
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_CHAIN, NT - NL);

      // -------------------------------------------------------------- D4 = Ac^T U,  D3 += [T;P] U
      if (cw == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint64_t dAcM = sdesc_sw128(sbase_addr + off_ac(s), 64 * 128, 1024);
          const uint64_t dTP = sdesc_sw128(sbase_addr + off_tp(s), 16, 1024);
          const uint32_t id4 = idesc_f16_f32(128, VS, true, true);
          const uint32_t id3 = idesc_f16_f32(128, VS, false, true);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D4, mstep(dAcM, kk), mstep(dU, kk), id4, kk > 0);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + cD3, kstep(dTP, 128, kk), mstep(dU, kk), id3, 1u);
          umma_commit(&bar_cmma);
        }
        __syncwarp();
      }
      // write vectors of the next chunk while these MMAs run
      if (c + 1 < nchunks) {
        if (!wait_all(&bar_v, ph_v, false)) { aborted = true; break; }
        convert_wr();
        if (c + 2 < nchunks) prefetch_ws(c + 2);
        fence_async_smem();
      }
      if (!wait_mma()) { aborted = true; break; }
      // this CTA's copy of slot s is no longer read
      if (ct == 0) {
        if (s == rank) mbar_arrive(&bar_own_free);
        else mbar_arrive_remote(mapa_shared(smem_u32(&bar_peer_free), static_cast<uint32_t>(peer)));
      }

      // -------------------------------------------------------------- E4: S <- Diag(gamma_C) (S + Ac^T U)
      {
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < 32; j += 16) {
          float ds[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D4 + half * 32 + j), ds);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            Sreg[j + i] = gc * (Sreg[j + i] + ds[i]);
            mx = fmaxf(mx, fabsf(Sreg[j + i]));
          }
          tc::st_h16x16(tS, trow, half * 32 + j, 128, Sreg + j);
        }
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_CHAIN, NT - NL);
    }
    if (!aborted && nchunks > 0) store_o(nchunks - 1);
    if (!aborted && p.S_T) {
      float *dst = p.S_T + sbase + static_cast<size_t>(trow) * DV + v0 + half * 32;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = make_float4(Sreg[j], Sreg[j + 1], Sreg[j + 2], Sreg[j + 3]);
    }
  }

  // both roles done; keep this CTA's shared memory alive until the peer is done with it
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc2
}  // namespace dr
