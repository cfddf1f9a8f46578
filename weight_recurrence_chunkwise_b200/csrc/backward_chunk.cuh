// backward_chunk.cuh -- the backward pass in the chunkwise (WY/UT) form on the tensor cores
// (tcgen05.mma, fp16 operands in 128-byte-swizzled shared memory, fp32 accumulators in TMEM), for
// bf16 I/O, dk = dv = 128 and chunks of 64 tokens.
//
// Algebra (DeltaNet page, step 7; FG2-GDN page, section 2), per chunk with initial state S (stored
// by the forward ring kernel) and dS = the gradient of the chunk's final state, rows r of the chunk,
// gamma_r = prod_{j<=r} alpha_j per key channel, b = sqrt(beta_k) (.) k, a = s (.) b (or b), w the
// write vector:
//   Qh = gamma q, Bh = gamma b, Ac = a / gamma, A = strictly-lower(Bh Ac^T), P = lower(Qh Ac^T),
//   T = (I + A)^-1, Y = W - Bh S, U = T Y, M = S + Ac^T U, dM = Diag(gamma_C) dS
//   dU = P^T dO + Ac dM,  dV = T^T dU,  dS_prev = Qh^T dO + dM - Bh^T dV   (the chain between chunks)
//   dP = lower(dO U^T), dA = strictly-lower(-dV U^T)
//   dQh^T = S dO^T + Ac^T dP^T,  dBh^T = -S dV^T + Ac^T dA^T,  dAc^T = Bh^T dA + Qh^T dP + dM U^T
//   dgamma_r = q (.) dQh + b (.) dBh - Ac (.) dAc / gamma  (+ rowsum(dS (.) M) on the last row)
//   dalpha_j = sum_{r>=j} dgamma_r gamma_r / alpha_j,  dq = gamma dQh,  db = gamma dBh,  da = dAc / gamma
// then the chain rule through b, a and w.  The products that carry the gradients per key channel
// (dQh, dBh, dAc) are formed transposed -- TMEM lane = key channel -- so that the per-channel
// gate arithmetic (the running product gamma, the reverse cumulative sum of dalpha) is local to a
// thread.
//
// One CTA of 256 threads per (b, h) walks its chunks from the last to the first; the fp32 gradient
// of the state is carried in TMEM (lane = key row i), where the step of every chunk accumulates onto it.  Every product uses
// M = 128; where only 64 rows are meaningful, the other 64 rows read neighbouring tiles and are
// ignored in TMEM.
#pragma once
#include "chunk_tc.cuh"

namespace dr {
namespace bwc {

using tc::C;
using tc::DK;
using tc::kF16Max;
using tc::kMinChunkDecayF16;
constexpr int DV = 128;
constexpr int NT = 256;

// shared memory (bytes from a 1024-aligned base); 64-column blocks of R rows x 128 bytes
constexpr uint32_t SX = 0;                        // [Bh; Qh]   128 x 128 (raw k, q land here)
constexpr uint32_t SX_CB = 128 * 128;
constexpr uint32_t SAC = 2 * SX_CB;               // Ac         64 x 128
constexpr uint32_t SAC_CB = 64 * 128;
constexpr uint32_t STP = SAC + 2 * SAC_CB;        // K1's gate products; [A -> T; T^T scratch -> P]  128 x 64; raw q
constexpr uint32_t SSS = STP + 128 * 128;         // S (fp16)   128 (dk) x 128 (dv)
constexpr uint32_t SWY = SSS + 2 * 128 * 128;     // W -> Y -> dU   64 x 128; raw k at the end
constexpr uint32_t SWY_CB = 64 * 128;
constexpr uint32_t SUU = SWY + 2 * SWY_CB;        // U          64 x 128
constexpr uint32_t SDM = SUU + 2 * SWY_CB;        // dM         128 x 128
constexpr uint32_t SDO = SDM + 2 * 128 * 128;     // [dO; -dV]  128 x 128
// the chunk's fp32 state lands in [SWY, SDO) (free at the chunk's start): four 128-row boxes of 32 columns
constexpr uint32_t SST = SWY;
constexpr uint32_t SST_B = 128 * 128;
static_assert(SST + 4 * SST_B == SDO, "state staging spans the write-vector, U and dM tiles");
constexpr uint32_t SDPA = SDO + 2 * 128 * 128;    // raw v (64 x 128), then [dP; dA]   128 x 64
constexpr uint32_t SGC = SDPA + 128 * 128;        // gamma_C, 128 fp32
constexpr uint32_t SROW = SGC + 512;              // scalar gates: gamma_r, 1/gamma_r, sqrt(beta_r), alpha_r
constexpr uint32_t SRT = SROW + 1024;             // last-row term partials, [2][128] fp32
constexpr uint32_t SXC = SRT + 1024;              // per-channel exchange between the row halves, [2][128]
constexpr uint32_t SRED = SXC + 1024;             // per-row sums over channels: [64 rows][4 warps][2] fp32
constexpr uint32_t SRV = SRED + 64 * 4 * 2 * 4;   // per-row sums over value columns: [64 rows][4 warps] fp32
constexpr uint32_t SEND = SRV + 64 * 4 * 4;
constexpr size_t SMEM_BYTES = SEND + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t COL_D1 = 0;     // [A | P] raw (64); later [dP | dA] raw
constexpr uint32_t COL_BS = 64;    // [Bh S | .] (128); later Ac^T U, dU, then [dQh^T | dBh^T]
constexpr uint32_t COL_U = 192;    // [U | .] (128); later dV, then dAc^T (64)
constexpr uint32_t COL_AU = 320;   // the state gradient (128), across chunks
constexpr uint32_t TMEM_COLS = 512;

// Sums of v[k] over the 32 lanes of a warp for k = 0 .. N-1 (N = 8 or 32); lane l returns the sum of entry
// l % N.  Butterfly steps over the lane bits above log2 N add whole arrays; each later step on lane bit b
// keeps the half of the entries whose index bit b equals the lane's bit and adds the partner's copy of
// it, so 31 shuffles serve 32 entries.
template <int N>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[N], int lane) {
#pragma unroll
  for (int off = 16; off >= N; off >>= 1)
#pragma unroll
    for (int k = 0; k < N; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], off);
#pragma unroll
  for (int off = N / 2; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < off; ++k) {
      const float send = up ? v[k] : v[k + off];
      const float keep = up ? v[k + off] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

struct BwdChunkParams {
  int T, H, nchunks;
  const float *alpha;
  int alpha_mode;
  const float *beta_k;
  int beta_k_mode;
  const float *beta_v;
  int beta_v_mode;
  const float *s;            // write-side key scale or nullptr
  const __nv_bfloat16 *q, *k, *v;
  const float *states;       // [B, H, nchunks, dk, dv]: the state at the start of every chunk
  const float *dS_T;         // [B, H, dk, dv] or nullptr
  float *dq, *dk, *dv, *dalpha, *dbeta_k, *dbeta_v, *ds, *dS0;
  uint32_t *status;
};

template <bool kChanGates, bool kScaled>
__global__ void __launch_bounds__(NT, 1)
chunk_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_st, const BwdChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_ld, bar_mma;
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int h = blockIdx.x, b = blockIdx.y, H = p.H, T = p.T, NC = p.nchunks;
  const size_t head = static_cast<size_t>(b) * H + h;
  const bool sym_write = p.beta_v_mode == MODE_ABSENT;  // w = sqrt(beta_k) (.) v
  // the kernel's global inputs and outputs never overlap
  const float *__restrict__ g_alpha = p.alpha;
  const float *__restrict__ g_beta_k = p.beta_k;
  const float *__restrict__ g_beta_v = p.beta_v;
  const float *__restrict__ g_s = p.s;
  float *__restrict__ g_dq = p.dq;
  float *__restrict__ g_dk = p.dk;
  float *__restrict__ g_dv = p.dv;
  float *__restrict__ g_dalpha = p.dalpha;
  float *__restrict__ g_dbeta_k = p.dbeta_k;
  float *__restrict__ g_dbeta_v = p.dbeta_v;
  float *__restrict__ g_ds = p.ds;

  uint8_t *X = sm + SX, *tAC = sm + SAC, *tTP = sm + STP, *tSS = sm + SSS, *tWY = sm + SWY, *tUU = sm + SUU;
  uint8_t *tDM = sm + SDM, *tDO = sm + SDO, *tDPA = sm + SDPA;
  float *sGC = reinterpret_cast<float *>(sm + SGC);
  float *sRow = reinterpret_cast<float *>(sm + SROW);
  float *sRT = reinterpret_cast<float *>(sm + SRT);
  float *sXC = reinterpret_cast<float *>(sm + SXC);
  float *sRed = reinterpret_cast<float *>(sm + SRED);
  float *sRV = reinterpret_cast<float *>(sm + SRV);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_ld, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_st);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  uint32_t ph_ld = 0, ph_mma = 0;
  bool ok = true;

  // bounded waits; a failure in any thread stops every thread at the same point
  auto wait_mma = [&]() -> bool {
    bool w = true;
    if (tid == 0) w = mbar_wait(&bar_mma, ph_mma & 1u, kWaitLimitNs);
    ph_mma++;
    const bool fail = bar_or(1, NT, !w);
    tc_fence_after();
    if (fail && tid == 0) raise_status(p.status, STATUS_TIMEOUT);
    return !fail;
  };
  auto wait_ld = [&]() -> bool {
    const bool w = mbar_wait(&bar_ld, ph_ld & 1u, kWaitLimitNs);
    ph_ld++;
    const bool fail = bar_or(1, NT, !w);
    if (fail && tid == 0) raise_status(p.status, STATUS_TIMEOUT);
    return !fail;
  };
  // single-thread MMA issue: nk K-steps of 16 into column `col`; desc(kk) give the operands
  auto issue = [&](uint32_t col, int nk, uint32_t idesc, bool acc, auto adesc, auto bdesc) {
    for (int kk = 0; kk < nk; ++kk) umma_f16(tmem + col, adesc(kk), bdesc(kk), idesc, (acc || kk > 0) ? 1u : 0u);
  };
  auto kmaj = [](uint32_t saddr, int R) {  // K-major tile of R rows: descriptor of K-step kk
    return [saddr, R](int kk) {
      return sdesc_sw128(saddr + static_cast<uint32_t>((kk >> 2) * R * 128 + (kk & 3) * 32), 16, 1024);
    };
  };
  auto mnmaj = [](uint32_t saddr, int R) {  // MN-major tile (rows = K) whose column blocks are R rows apart
    return [saddr, R](int kk) {
      return sdesc_sw128(saddr + static_cast<uint32_t>(kk) * 2048u, static_cast<uint32_t>(R) * 128u, 1024);
    };
  };

  // the gradient of the state: row i = 32 quarter + lane, value columns 64 half .. 64 half + 63
  const int srow = quarter * 32 + lane;
  // Between chunks it lives in TMEM columns COL_AU .. COL_AU + 127 (lane = key row): the state step's
  // product accumulates onto it there, and registers hold it only where a stage reads it.
  auto ld_au = [&](float (&x)[64]) {  // my row half of the 128 columns at COL_AU
#pragma unroll
    for (int j = 0; j < 64; j += 16)
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), *reinterpret_cast<float(*)[16]>(x + j));
    tmem_ld_wait();
  };
  {
    float x[64];
    const float *src = p.dS_T ? p.dS_T + head * DK * DV + static_cast<size_t>(srow) * DV + half * 64 : nullptr;
#pragma unroll
    for (int j = 0; j < 64; j += 4) {
      const float4 y = src ? __ldg(reinterpret_cast<const float4 *>(src + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
      x[j] = y.x;
      x[j + 1] = y.y;
      x[j + 2] = y.z;
      x[j + 3] = y.w;
    }
#pragma unroll
    for (int j = 0; j < 64; j += 16)
      tmem_st16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), *reinterpret_cast<const float(*)[16]>(x + j));
    tmem_st_wait();
  }

  // element helpers for a thread's row of a 128-row, 128-column tile (two 64-column blocks)
  auto st_row64 = [](uint8_t *tile, int R, int row, int col0, const float *v) {  // 64 values from col0
#pragma unroll
    for (int j = 0; j < 64; j += 16) tc::st_h16x16(tile, row, col0 + j, R, v + j);
  };

  // write scale of value columns col .. col + 3 of chunk row r (token index th): beta_v, or sqrt(beta_k)
  // when the write is symmetric (dk = dv)
  auto wscale4 = [&](int r, size_t th, int col) -> float4 {
    if (p.beta_v_mode == MODE_CHANNEL) return __ldg(reinterpret_cast<const float4 *>(g_beta_v + th * DV + col));
    if (p.beta_v_mode == MODE_SCALAR) {
      const float y = __ldg(g_beta_v + th);
      return make_float4(y, y, y, y);
    }
    if (p.beta_k_mode == MODE_CHANNEL) {
      const float4 y = __ldg(reinterpret_cast<const float4 *>(g_beta_k + th * DK + col));
      return make_float4(tc::sqrt_fast(y.x), tc::sqrt_fast(y.y), tc::sqrt_fast(y.z), tc::sqrt_fast(y.w));
    }
    float y;
    if constexpr (kChanGates) y = tc::sqrt_fast(__ldg(g_beta_k + th));
    else y = sRow[128 + r];  // the scan's sqrt(beta_k) of the row (0 past the end of the sequence)
    return make_float4(y, y, y, y);
  };

#pragma unroll 1
  for (int c = NC - 1; c >= 0 && ok; --c) {
    const int t0 = c * C, L = min(C, T - t0);
    const size_t tok0 = static_cast<size_t>(b) * T + t0;  // first token of the chunk (dense batch)

    // ------------------------------------------------------------------ loads: q, k, v, dO and the fp32 state (TMA)
    if (tid == 0) {
      const int srow0 = (static_cast<int>(head) * NC + c) * DK;  // the state's first row in the states map
      mbar_arrive_expect_tx(&bar_ld, 8 * 64 * 128 + 4 * 128 * 128);
      tma_load_4d(X + 64 * 128, &tm_q, &bar_ld, 0, h, t0, b);
      tma_load_4d(X + SX_CB + 64 * 128, &tm_q, &bar_ld, 64, h, t0, b);
      tma_load_4d(X, &tm_k, &bar_ld, 0, h, t0, b);
      tma_load_4d(X + SX_CB, &tm_k, &bar_ld, 64, h, t0, b);
      tma_load_4d(tDPA, &tm_v, &bar_ld, 0, h, t0, b);
      tma_load_4d(tDPA + 64 * 128, &tm_v, &bar_ld, 64, h, t0, b);
      tma_load_4d(tDO, &tm_do, &bar_ld, 0, h, t0, b);
      tma_load_4d(tDO + 128 * 128, &tm_do, &bar_ld, 64, h, t0, b);
#pragma unroll
      for (int j = 0; j < 4; ++j) tma_load_2d(sm + SST + j * SST_B, &tm_st, &bar_ld, 32 * j, srow0);
      if (c > 0) {
        for (int x = 0; x < 128; x += 64) {
          tma_prefetch_l2_4d(&tm_q, x, h, t0 - C, b);
          tma_prefetch_l2_4d(&tm_k, x, h, t0 - C, b);
          tma_prefetch_l2_4d(&tm_v, x, h, t0 - C, b);
          tma_prefetch_l2_4d(&tm_do, x, h, t0 - C, b);
        }
        for (int j = 0; j < 4; ++j) tma_prefetch_l2_2d(&tm_st, 32 * j, srow0 - DK);
      }
    }
    if (c > 0) {  // the previous chunk's gates into L2: thread = (row tid / 4, 128-byte line tid % 4)
      const int pr = tid >> 2, pl = tid & 3;
      const size_t tp = (tok0 - C + pr) * H + h;
      if (p.alpha_mode == MODE_CHANNEL) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_alpha + tp * DK + 32 * pl));
      else if (p.alpha_mode == MODE_SCALAR && pl == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_alpha + tp));
      if (p.beta_k_mode == MODE_CHANNEL) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_beta_k + tp * DK + 32 * pl));
      else if (pl == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_beta_k + tp));
      if (p.beta_v_mode == MODE_CHANNEL) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_beta_v + tp * DV + 32 * pl));
      if (kScaled) asm volatile("prefetch.global.L2 [%0];" ::"l"(g_s + tp * DK + 32 * pl));
    }
    // gates
    float pal[4 * 8], pbe[4 * 8];  // channel gates: rows 8 rg .. 8 rg + 7, channels c0 .. c0 + 3
    const int rg = tid >> 5, c0 = 4 * (tid & 31);
    if constexpr (kChanGates) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const size_t th = (tok0 + min(rg * 8 + j, L - 1)) * H + h;
        if (p.alpha_mode == MODE_CHANNEL) {
          const float4 a = __ldg(reinterpret_cast<const float4 *>(p.alpha + th * DK + c0));
          pal[4 * j] = a.x; pal[4 * j + 1] = a.y; pal[4 * j + 2] = a.z; pal[4 * j + 3] = a.w;
        } else {
          const float a = p.alpha_mode == MODE_SCALAR ? __ldg(p.alpha + th) : 1.f;
          pal[4 * j] = pal[4 * j + 1] = pal[4 * j + 2] = pal[4 * j + 3] = a;
        }
        if (p.beta_k_mode == MODE_CHANNEL) {
          const float4 x = __ldg(reinterpret_cast<const float4 *>(p.beta_k + th * DK + c0));
          pbe[4 * j] = x.x; pbe[4 * j + 1] = x.y; pbe[4 * j + 2] = x.z; pbe[4 * j + 3] = x.w;
        } else {
          const float x = __ldg(p.beta_k + th);
          pbe[4 * j] = pbe[4 * j + 1] = pbe[4 * j + 2] = pbe[4 * j + 3] = x;
        }
        if (rg * 8 + j >= L) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pal[4 * j + e] = 1.f;
            pbe[4 * j + e] = 0.f;
          }
        }
      }
    } else if (warp == 0) {  // scalar gates: warp 0 scans the row gates (lane: rows 2 lane, 2 lane + 1)
      float al[2], be[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 2 * lane + e;
        const size_t th = (tok0 + min(r, L - 1)) * H + h;
        al[e] = (p.alpha_mode == MODE_SCALAR && r < L) ? __ldg(p.alpha + th) : 1.f;
        be[e] = r < L ? __ldg(p.beta_k + th) : 0.f;
      }
      float incl = al[0] * al[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl *= y;
      }
      const float up = __shfl_up_sync(0xffffffffu, incl, 1);
      const float g0 = (lane == 0 ? 1.f : up) * al[0], g1 = g0 * al[1];
      sRow[2 * lane] = g0;
      sRow[2 * lane + 1] = g1;
      sRow[64 + 2 * lane] = __fdividef(1.f, g0);
      sRow[64 + 2 * lane + 1] = __fdividef(1.f, g1);
      sRow[128 + 2 * lane] = tc::sqrt_fast(be[0]);
      sRow[128 + 2 * lane + 1] = tc::sqrt_fast(be[1]);
      sRow[192 + 2 * lane] = al[0];
      sRow[192 + 2 * lane + 1] = al[1];
      const float gC = __shfl_sync(0xffffffffu, incl, 31);
#pragma unroll
      for (int e = 0; e < 4; ++e) sGC[4 * lane + e] = gC;
      if (lane == 0 && !(gC >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
    }
    // wait for the tiles
    if (!wait_ld()) { ok = false; break; }
    // S of this chunk: the fp16 operand tile, and the state part of the last-row term sum_v dS S.  The
    // staged fp32 rows are 128-byte-swizzled boxes of 32 columns.
    float rt = 0.f;
#pragma unroll 1
    for (int j = 0; j < 64; j += 16) {
      float x[16], d[16];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), d);
      const uint8_t *box = sm + SST + ((half * 64 + j) >> 5) * SST_B + srow * 128;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ch = (((half * 64 + j) & 31) >> 2) + e;  // 16-byte chunk of the row within the box
        const float4 y = *reinterpret_cast<const float4 *>(box + ((ch ^ (srow & 7)) << 4));
        x[4 * e] = y.x;
        x[4 * e + 1] = y.y;
        x[4 * e + 2] = y.z;
        x[4 * e + 3] = y.w;
      }
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) rt += d[e] * x[e];
      tc::st_h16x16(tSS, srow, half * 64 + j, 128, x);
    }

    // ------------------------------------------------------------------ K1: Qh, Bh, Ac; write vectors; dO -> fp16
    float amax = 0.f;
    if constexpr (kChanGates) {
      float *sPX = reinterpret_cast<float *>(tTP);  // row-group gate products, 8 x 128 fp32 (T comes later)
      float pg[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) pg[e] *= pal[4 * j + e];
      *reinterpret_cast<float4 *>(sPX + rg * 128 + c0) = make_float4(pg[0], pg[1], pg[2], pg[3]);
      __syncthreads();
      float gr[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        if (g < rg) {
          const float4 x = *reinterpret_cast<const float4 *>(sPX + g * 128 + c0);
          gr[0] *= x.x; gr[1] *= x.y; gr[2] *= x.z; gr[3] *= x.w;
        }
      }
      if (rg == 7) {
        const float4 gC = make_float4(gr[0] * pg[0], gr[1] * pg[1], gr[2] * pg[2], gr[3] * pg[3]);
        *reinterpret_cast<float4 *>(sGC + c0) = gC;
        if (!(fminf(fminf(gC.x, gC.y), fminf(gC.z, gC.w)) >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
      }
      const uint32_t blk = static_cast<uint32_t>(c0 >> 6), grp = static_cast<uint32_t>((c0 & 63) >> 3);
      const uint32_t inb = static_cast<uint32_t>((c0 & 7) * 2);
      uint8_t *pQ = X + blk * SX_CB + (64 + rg * 8) * 128 + inb;
      uint8_t *pB = X + blk * SX_CB + (rg * 8) * 128 + inb;
      uint8_t *pA = tAC + blk * SAC_CB + (rg * 8) * 128 + inb;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t sw = ((grp ^ static_cast<uint32_t>(jj)) << 4) + jj * 128;
        const uint2 kraw = *reinterpret_cast<const uint2 *>(pB + sw), qraw = *reinterpret_cast<const uint2 *>(pQ + sw);
        const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw);
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qraw);
        const float2 k01 = __bfloat1622float2(k2[0]), k23 = __bfloat1622float2(k2[1]);
        const float2 q01 = __bfloat1622float2(q2[0]), q23 = __bfloat1622float2(q2[1]);
        const float kf[4] = {k01.x, k01.y, k23.x, k23.y}, qf[4] = {q01.x, q01.y, q23.x, q23.y};
        float sc[4] = {1.f, 1.f, 1.f, 1.f};
        if constexpr (kScaled) {
          const size_t th = (tok0 + min(rg * 8 + jj, L - 1)) * H + h;
          const float4 x = __ldg(reinterpret_cast<const float4 *>(p.s + th * DK + c0));
          sc[0] = x.x; sc[1] = x.y; sc[2] = x.z; sc[3] = x.w;
        }
        float oq[4], ob[4], oa[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          gr[e] *= pal[4 * jj + e];
          const float bv = tc::sqrt_fast(pbe[4 * jj + e]) * kf[e];
          float av = bv * __fdividef(1.f, gr[e]);
          if constexpr (kScaled) av *= sc[e];
          amax = fmaxf(amax, fabsf(av));
          oq[e] = gr[e] * qf[e];
          ob[e] = gr[e] * bv;
          oa[e] = av;
        }
        *reinterpret_cast<uint2 *>(pQ + sw) = make_uint2(pack_f16x2(oq[0], oq[1]), pack_f16x2(oq[2], oq[3]));
        *reinterpret_cast<uint2 *>(pB + sw) = make_uint2(pack_f16x2(ob[0], ob[1]), pack_f16x2(ob[2], ob[3]));
        *reinterpret_cast<uint2 *>(pA + sw) = make_uint2(pack_f16x2(oa[0], oa[1]), pack_f16x2(oa[2], oa[3]));
      }
    } else {
      __syncthreads();  // the row gates of warp 0
      const int j8 = tid & 15;
#pragma unroll 1
      for (int i = 0; i < 4; ++i) {
        const int r = (tid >> 4) + 16 * i;
        const float g = sRow[r], gi = sRow[64 + r], sbt = sRow[128 + r];
        float ssc[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
        if constexpr (kScaled) {
          const float4 *src = reinterpret_cast<const float4 *>(p.s + ((tok0 + min(r, L - 1)) * H + h) * DK + j8 * 8);
          const float4 lo = __ldg(src), hi = __ldg(src + 1);
          ssc[0] = lo.x; ssc[1] = lo.y; ssc[2] = lo.z; ssc[3] = lo.w;
          ssc[4] = hi.x; ssc[5] = hi.y; ssc[6] = hi.z; ssc[7] = hi.w;
        }
        uint4 *pq = reinterpret_cast<uint4 *>(X + sw128_off16(64 + r, j8, 128));
        uint4 *pk = reinterpret_cast<uint4 *>(X + sw128_off16(r, j8, 128));
        const uint4 qraw = *pq, kraw = *pk;
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qraw);
        const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw);
        uint32_t oq[4], ob[4], oa[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 qf = __bfloat1622float2(q2[e]), kf = __bfloat1622float2(k2[e]);
          const float b0 = sbt * kf.x, b1 = sbt * kf.y;
          float x0 = b0 * gi, x1 = b1 * gi;
          if constexpr (kScaled) {
            x0 *= ssc[2 * e];
            x1 *= ssc[2 * e + 1];
          }
          amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
          oq[e] = pack_f16x2(g * qf.x, g * qf.y);
          ob[e] = pack_f16x2(g * b0, g * b1);
          oa[e] = pack_f16x2(x0, x1);
        }
        *pq = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        *pk = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        *reinterpret_cast<uint4 *>(tAC + sw128_off16(r, j8, 64)) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
      }
    }
    if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
    // write vectors W = wsc (.) v (raw v waits in the dP/dA tile), and dO as fp16 in place: thread row
    // tid >> 2, 8-column groups (tid & 3) + 4 g of 16 (four lanes cover 32 adjacent columns)
    {
      const int r = tid >> 2;
      const bool valid = r < L;
      const size_t th = (tok0 + min(r, L - 1)) * H + h;
      float4 wq[8];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = 8 * ((tid & 3) + 4 * g);
        wq[2 * g] = wscale4(r, th, col);
        wq[2 * g + 1] = wscale4(r, th, col + 4);
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int c8 = (tid & 3) + 4 * g;  // 8-column group (0..15)
        const float wsc[8] = {wq[2 * g].x,     wq[2 * g].y,     wq[2 * g].z,     wq[2 * g].w,
                              wq[2 * g + 1].x, wq[2 * g + 1].y, wq[2 * g + 1].z, wq[2 * g + 1].w};
        uint4 *pd = reinterpret_cast<uint4 *>(tDO + sw128_off16(r, c8, 128));
        const uint4 vraw = *reinterpret_cast<const uint4 *>(tDPA + sw128_off16(r, c8, 64)), draw = *pd;
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vraw);
        const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&draw);
        uint32_t ow[4], od[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 vf = __bfloat1622float2(v2[e]), df = __bfloat1622float2(d2[e]);
          ow[e] = pack_f16x2(valid ? wsc[2 * e] * vf.x : 0.f, valid ? wsc[2 * e + 1] * vf.y : 0.f);
          od[e] = pack_f16x2(valid ? df.x : 0.f, valid ? df.y : 0.f);
        }
        *reinterpret_cast<uint4 *>(tWY + sw128_off16(r, c8, 64)) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        *pd = make_uint4(od[0], od[1], od[2], od[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ m1: [A | P] = [Bh; Qh] Ac^T;  Bh S
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_D1, DK / 16, idesc_f16_f32(128, 64, false, false), false, kmaj(sb + SX, 128), kmaj(sb + SAC, 64));
        issue(COL_BS, DK / 16, idesc_f16_f32(128, 128, false, true), false, kmaj(sb + SX, 128),
              mnmaj(sb + SSS, 128));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    if (!wait_mma()) { ok = false; break; }
    // E1a: A (strictly lower) -> TP rows 0..63
    if (quarter < 2) {
      float x[32];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32), *reinterpret_cast<float(*)[16]>(x));
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32 + 16), *reinterpret_cast<float(*)[16]>(x + 16));
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = (half * 32 + i < srow) ? x[i] : 0.f;
      tc::st_h16x16(tTP, srow, half * 32, 128, x);
      tc::st_h16x16(tTP, srow, half * 32 + 16, 128, x + 16);
    }
    tc_fence_before();
    __syncthreads();
    // T = (I + A)^-1 (warps 0..3)
    if (warp < 4) {
      tri::Frag Trow[4];
      tri::inverse64_rows<tri::Sw128Layout>(tTP, tTP + 64 * 128, warp, lane, Trow, [] { bar_sync(2, 128); });
      const int rr = lane >> 2, qq = lane & 3;
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        if (d <= warp) {
          const tri::Frag &F = Trow[d];
          const int row = 16 * warp + rr, col = 16 * (warp - d) + 2 * qq;
          *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col, 128)) = pack_f16x2(F.v[0], F.v[1]);
          *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col, 128)) = pack_f16x2(F.v[2], F.v[3]);
          *reinterpret_cast<uint32_t *>(tTP + sw128_off(row, col + 8, 128)) = pack_f16x2(F.v[4], F.v[5]);
          *reinterpret_cast<uint32_t *>(tTP + sw128_off(row + 8, col + 8, 128)) = pack_f16x2(F.v[6], F.v[7]);
        }
      }
    }
    __syncthreads();
    // E1b: P (lower with diagonal) -> TP rows 64..127 (after the inverse's scratch use);  Y = W - Bh S
    if (quarter >= 2) {
      const int r = srow - 64;
      float x[32];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32), *reinterpret_cast<float(*)[16]>(x));
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32 + 16), *reinterpret_cast<float(*)[16]>(x + 16));
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = (half * 32 + i <= r) ? x[i] : 0.f;
      tc::st_h16x16(tTP, srow, half * 32, 128, x);
      tc::st_h16x16(tTP, srow, half * 32 + 16, 128, x + 16);
    } else {
      // rows 0..63 of Bh S: Y = W - Bh S into the write-vector tile, in place
#pragma unroll 1
      for (int j = 0; j < 64; j += 16) {
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_BS + half * 64 + j), x);
        tmem_ld_wait();
        float y[16];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int c8 = (half * 64 + j) / 8 + g;
          const uint4 wraw = *reinterpret_cast<const uint4 *>(tWY + sw128_off16(srow, c8, 64));
          const __half2 *w2 = reinterpret_cast<const __half2 *>(&wraw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 wf = __half22float2(w2[e]);
            y[8 * g + 2 * e] = wf.x - x[8 * g + 2 * e];
            y[8 * g + 2 * e + 1] = wf.y - x[8 * g + 2 * e + 1];
          }
        }
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(y[e]));
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
        tc::st_h16x16(tWY, srow, half * 64 + j, 64, y);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ U = [T; P] Y
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_U, C / 16, idesc_f16_f32(128, 128, false, true), false, kmaj(sb + STP, 128), mnmaj(sb + SWY, 64));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    if (!wait_mma()) { ok = false; break; }
    if (quarter < 2) {
#pragma unroll 1
      for (int j = 0; j < 64; j += 16) {
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_U + half * 64 + j), x);
        tmem_ld_wait();
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(x[e]));
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
        tc::st_h16x16(tUU, srow, half * 64 + j, 64, x);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ Ac^T U (into the spent Bh S columns);  dM = Diag(gamma_C) dS
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_BS, C / 16, idesc_f16_f32(128, 128, true, true), false, mnmaj(sb + SAC, 64), mnmaj(sb + SUU, 64));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    const float gci = sGC[srow];
    {  // dM as the fp16 operand while the product runs
      float mx = 0.f;
#pragma unroll 1
      for (int j = 0; j < 64; j += 16) {
        float d[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), d);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          d[e] *= gci;
          mx = fmaxf(mx, fabsf(d[e]));
        }
        tc::st_h16x16(tDM, srow, half * 64 + j, 128, d);
      }
      if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
    }
    if (!wait_mma()) { ok = false; break; }
    // last-row term: sum_v dS (S + Ac^T U), per key row; the two value halves meet in shared memory.  Then
    // dM in fp32 replaces dS in TMEM: the state step accumulates onto it.
#pragma unroll 1
    for (int j = 0; j < 64; j += 16) {
      float d[16], a[16];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), d);
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_BS + half * 64 + j), a);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        rt += d[e] * a[e];
        d[e] *= gci;
      }
      tmem_st16(tmem_addr(tmem, quarter * 32, COL_AU + half * 64 + j), d);
    }
    tmem_st_wait();
    sRT[half * 128 + srow] = rt;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ dU = P^T dO + Ac dM
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_BS, C / 16, idesc_f16_f32(128, 128, true, true), false, mnmaj(sb + STP + 64 * 128, 128),
              mnmaj(sb + SDO, 128));
        issue(COL_BS, DK / 16, idesc_f16_f32(128, 128, false, true), true, kmaj(sb + SAC, 64), mnmaj(sb + SDM, 128));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    if (!wait_mma()) { ok = false; break; }
    if (quarter < 2) {  // dU -> the write-vector tile (Y is no longer read)
#pragma unroll 1
      for (int j = 0; j < 64; j += 16) {
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_BS + half * 64 + j), x);
        tmem_ld_wait();
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(x[e]));
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
        tc::st_h16x16(tWY, srow, half * 64 + j, 64, x);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ dV^T = dU^T T -> -dV, dv, write strengths
    // formed transposed (TMEM lane = value column) so that every global access below is a whole 128-byte
    // line per warp and all eight warps share the epilogue
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_U, C / 16, idesc_f16_f32(128, 64, true, true), false, mnmaj(sb + SWY, 64), mnmaj(sb + STP, 128));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    {
      // thread: value column vc = srow, rows 32 half .. 32 half + 31 in blocks of 8 whose write scales load
      // one block ahead
      const int vc = srow, r0 = 32 * half;
      const bool row_sums = p.beta_v_mode == MODE_SCALAR || (p.beta_v_mode == MODE_ABSENT && p.beta_k_mode != MODE_CHANNEL);
      // the block's raw write-scale sources, loaded one block ahead and transformed at use (a square
      // root applied here would make the thread wait for the loads at once): beta_v (per channel or per
      // row), or for a symmetric write beta_k (per channel or per row), or the scan's sqrt(beta_k)
      const bool w_scan = !kChanGates && p.beta_v_mode == MODE_ABSENT;
      const bool w_sqrt = kChanGates && p.beta_v_mode == MODE_ABSENT;
      const float *w_src = p.beta_v_mode != MODE_ABSENT ? g_beta_v : g_beta_k;
      const bool w_chan = p.beta_v_mode == MODE_CHANNEL || (p.beta_v_mode == MODE_ABSENT && p.beta_k_mode == MODE_CHANNEL);
      auto ld_w = [&](int jb, float (&w)[8]) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int r = r0 + jb + e;
          if (w_scan) {
            w[e] = sRow[128 + r];
          } else {
            const size_t th = (tok0 + min(r, L - 1)) * H + h;
            w[e] = __ldg(w_chan ? w_src + th * DV + vc : w_src + th);
          }
        }
      };
      float cw[8];
      ld_w(0, cw);
      if (!wait_mma()) { ok = false; break; }
#pragma unroll 1
      for (int jb = 0; jb < 32; jb += 8) {
        float nw[8];
        if (jb < 24) ld_w(jb + 8, nw);
        float x[8], xr[8], vf[8];  // dV of the block's rows; raw v; v dV
        tmem_ld8(tmem_addr(tmem, quarter * 32, COL_U + r0 + jb), x);
        // the block's raw v before any store of the block (the loads need not wait behind them)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          vf[e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tDPA + sw128_off(r0 + jb + e, vc, 64)));
        tmem_ld_wait();
        // global rows of the block: one 64-bit base, then 32-bit strides of H x DV floats
        const size_t rbase = ((tok0 + r0 + jb) * H + h) * DV + vc;
        const int rstride = H * DV;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int r = r0 + jb + e;
          *reinterpret_cast<__half *>(tDO + sw128_off(64 + r, vc, 128)) = __float2half_rn(-x[e]);
          xr[e] = vf[e] * x[e];
          if (r < L) {
            const float w = w_sqrt ? tc::sqrt_fast(cw[e]) : cw[e];
            const size_t o = rbase + static_cast<size_t>(e * rstride);
            g_dv[o] = w * x[e];
            if (p.beta_v_mode == MODE_CHANNEL) {
              g_dbeta_v[o] = xr[e];
            } else if (p.beta_v_mode == MODE_ABSENT && p.beta_k_mode == MODE_CHANNEL) {
              // symmetric channel write (dk = dv): d beta_k += 0.5 v dV / sqrt(beta_k), stored now, added to below
              g_dbeta_k[o] = w > 0.f ? 0.5f * __fdividef(xr[e], w) : 0.f;
            }
          }
        }
        if (row_sums) {  // rows r0 + jb + (lane & 7), summed over my warp's 32 value columns
          const float v = warp_transpose_sum<8>(xr, lane);
          if (lane < 8) sRV[(r0 + jb + lane) * 4 + quarter] = v;
        }
        if (jb < 24) {
#pragma unroll
          for (int e = 0; e < 8; ++e) cw[e] = nw[e];
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < 64 && tid < L) {  // scalar write strength: one value per row
      const int r = tid;
      const size_t th = (tok0 + r) * H + h;
      const float rs = sRV[4 * r] + sRV[4 * r + 1] + sRV[4 * r + 2] + sRV[4 * r + 3];
      if (p.beta_v_mode == MODE_SCALAR) g_dbeta_v[th] = rs;
      else if (p.beta_k_mode == MODE_SCALAR) sRV[4 * r] = rs;  // symmetric scalar write: folded in below
    }

    // ------------------------------------------------------------------ dS_prev = Qh^T dO - Bh^T dV + dM;  [dP | dA]
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        const uint32_t id = idesc_f16_f32(128, 128, true, true);
        issue(COL_AU, C / 16, id, true, mnmaj(sb + SX + 64 * 128, 128), mnmaj(sb + SDO, 128));
        issue(COL_AU, C / 16, id, true, mnmaj(sb + SX, 128), mnmaj(sb + SDO + 64 * 128, 128));
        issue(COL_D1, DV / 16, idesc_f16_f32(128, 64, false, false), false, kmaj(sb + SDO, 128), kmaj(sb + SUU, 64));
        umma_commit(&bar_mma);
      }
      __syncwarp();
    }
    if (!wait_mma()) { ok = false; break; }
    {  // dP (lower with diagonal, lanes 0..63) and dA (strictly lower, lanes 64..127)
      const int r = srow & 63;
      float x[32];
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32), *reinterpret_cast<float(*)[16]>(x));
      tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + half * 32 + 16), *reinterpret_cast<float(*)[16]>(x + 16));
      tmem_ld_wait();
      const bool strict = quarter >= 2;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int col = half * 32 + i;
        x[i] = (strict ? col < r : col <= r) ? x[i] : 0.f;
      }
      tc::st_h16x16(tDPA, srow, half * 32, 128, x);
      tc::st_h16x16(tDPA, srow, half * 32 + 16, 128, x + 16);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------------ [dQh^T | dBh^T] and dAc^T, lanes = key channels
    if (warp == 0) {
      if (elect_one()) {
        tc_fence_after();
        issue(COL_BS, DV / 16, idesc_f16_f32(128, 128, false, false), false, kmaj(sb + SSS, 128), kmaj(sb + SDO, 128));
        issue(COL_BS, C / 16, idesc_f16_f32(128, 128, true, false), true, mnmaj(sb + SAC, 64), kmaj(sb + SDPA, 128));
        const uint32_t id = idesc_f16_f32(128, 64, true, true);
        issue(COL_U, C / 16, id, false, mnmaj(sb + SX, 128), mnmaj(sb + SDPA + 64 * 128, 128));
        issue(COL_U, C / 16, id, true, mnmaj(sb + SX + 64 * 128, 128), mnmaj(sb + SDPA, 128));
        issue(COL_U, DV / 16, idesc_f16_f32(128, 64, false, false), true, kmaj(sb + SDM, 128), kmaj(sb + SUU, 64));
        umma_commit(&bar_mma);
        // the chunk's raw q and k for the per-channel stage, into the tiles T and dU have left
        mbar_arrive_expect_tx(&bar_ld, 4 * 64 * 128);
        tma_load_4d(tTP, &tm_q, &bar_ld, 0, h, t0, b);
        tma_load_4d(tTP + 64 * 128, &tm_q, &bar_ld, 64, h, t0, b);
        tma_load_4d(tWY, &tm_k, &bar_ld, 0, h, t0, b);
        tma_load_4d(tWY + SWY_CB, &tm_k, &bar_ld, 64, h, t0, b);
      }
      __syncwarp();
    }
    // the per-channel stage's decays (channel i = srow, rows 32 half ..), requested while the products run
    float s12a[kChanGates ? 32 : 1];
    if constexpr (kChanGates) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int r = 32 * half + j;
        const size_t th = (tok0 + min(r, L - 1)) * H + h;
        s12a[j] = 1.f;
        if (r < L) {
          if (p.alpha_mode == MODE_CHANNEL) s12a[j] = __ldg(g_alpha + th * DK + srow);
          else if (p.alpha_mode == MODE_SCALAR) s12a[j] = __ldg(g_alpha + th);
        }
      }
    }
    if (!wait_mma()) { ok = false; break; }

    // ------------------------------------------------------------------ per key channel: gate gradients and outputs
    // thread: key channel i = srow, rows 32 half .. 32 half + 31 of the chunk; q and k are read raw from the
    // tiles just loaded
    {
      const int i = srow, r0 = 32 * half;
      const float rowterm = sRT[i] + sRT[128 + i];
      auto raw_at = [&](const uint8_t *tile, int r) {  // bf16 (r, channel i) of a 64-row swizzled tile
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + sw128_off(r, i, 64)));
      };
      if (!wait_ld()) { ok = false; break; }
      if constexpr (kChanGates) {
        // shared scratch [32 rows][256 threads] in tiles the products above have released
        float *sAl = reinterpret_cast<float *>(X);     // alpha of my rows
        float *sGam = reinterpret_cast<float *>(tDM);  // gamma of my rows
        float *sSuf = reinterpret_cast<float *>(tSS);  // the lower half's suffix sums
        // gamma of my rows: forward products (the lower half passes its product to the upper half)
        float prod = 1.f;
        {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            sAl[j * NT + tid] = s12a[j];
            prod *= s12a[j];
          }
        }
        if (half == 0) sXC[i] = prod;
        __syncthreads();
        {
          float g = half == 0 ? 1.f : sXC[i];
#pragma unroll 4
          for (int j = 0; j < 32; ++j) {
            g *= sAl[j * NT + tid];
            sGam[j * NT + tid] = g;
          }
        }
        // reverse over my rows in blocks of 8 whose gate loads run one block ahead: dgamma, the local
        // suffix sums of dgamma gamma, and the outputs
        float acc = 0.f;
        float cb[8], cs[8], cp[8];  // beta_k, s and the stored write-side d beta_k of the block's rows
        auto load_blk = [&](int jb, float (&bk)[8], float (&sc)[8], float (&pv)[8]) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int r = r0 + jb + e;
            const size_t th = (tok0 + min(r, L - 1)) * H + h;
            bk[e] = p.beta_k_mode == MODE_CHANNEL ? __ldg(g_beta_k + th * DK + i) : __ldg(g_beta_k + th);
            sc[e] = kScaled ? __ldg(g_s + th * DK + i) : 1.f;
            pv[e] = (sym_write && p.beta_k_mode == MODE_CHANNEL) ? g_dbeta_k[th * DK + i] : 0.f;
          }
        };
        load_blk(24, cb, cs, cp);
#pragma unroll 1
        for (int jb = 24; jb >= 0; jb -= 8) {
          float nb[8], ns[8], np[8];
          if (jb > 0) load_blk(jb - 8, nb, ns, np);
          float dq[8], db[8], da[8];
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_BS + r0 + jb), dq);
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_BS + 64 + r0 + jb), db);
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_U + r0 + jb), da);
          // the block's shared-memory operands before any store of the block
          float gmv[8], qvv[8], kvv[8], alv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            gmv[e] = sGam[(jb + e) * NT + tid];
            alv[e] = sAl[(jb + e) * NT + tid];
            qvv[e] = raw_at(tTP, r0 + jb + e);
            kvv[e] = raw_at(tWY, r0 + jb + e);
          }
          tmem_ld_wait();
          const size_t obase = ((tok0 + r0 + jb) * H + h) * DK + i;  // row r0 + jb; rows H x DK floats apart
          const int ostride = H * DK;
          float xg[8], xb[8];  // dgamma gamma and d beta_k per row, for gates that are scalar per row
#pragma unroll
          for (int e = 7; e >= 0; --e) {
            const int j = jb + e, r = r0 + j;
            const bool valid = r < L;
            const float gm = gmv[e], ginv = __fdividef(1.f, gm);
            const float qv = qvv[e], kv = kvv[e];
            const float sbt = valid ? tc::sqrt_fast(cb[e]) : 0.f;
            const float scv = kScaled ? (valid ? cs[e] : 0.f) : 1.f;
            const float bv = sbt * kv, av = scv * bv, dav = da[e] * ginv;
            float dg = qv * dq[e] + bv * db[e] - av * dav * ginv;
            if (r == C - 1) dg += rowterm;
            acc += dg * gm;
            if (half == 0) sSuf[j * NT + tid] = acc;
            xg[e] = dg * gm;
            const float dbt = gm * db[e] + scv * dav;  // through b = sqrt(beta) k and a = s b
            const float dbk = sbt > 0.f ? 0.5f * kv * __fdividef(dbt, sbt) : 0.f;
            xb[e] = dbk;
            if (valid) {
              const size_t o = obase + static_cast<size_t>(e * ostride);
              g_dq[o] = gm * dq[e];
              g_dk[o] = sbt * dbt;
              if constexpr (kScaled) g_ds[o] = bv * dav;
              if (p.beta_k_mode == MODE_CHANNEL) g_dbeta_k[o] = cp[e] + dbk;
              if (p.alpha_mode == MODE_CHANNEL && half == 1) g_dalpha[o] = __fdividef(acc, alv[e]);
            }
          }
          if (p.beta_k_mode != MODE_CHANNEL) {  // summed over channels: rows r0 + jb + (lane & 7)
            const float v = warp_transpose_sum<8>(xb, lane);
            if (lane < 8) sRed[((r0 + jb + lane) * 4 + quarter) * 2] = v;
          }
          if (p.alpha_mode == MODE_SCALAR) {
            const float v = warp_transpose_sum<8>(xg, lane);
            if (lane < 8) sRed[((r0 + jb + lane) * 4 + quarter) * 2 + 1] = v;
          }
          if (jb > 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              cb[e] = nb[e];
              cs[e] = ns[e];
              cp[e] = np[e];
            }
          }
        }
        // the upper half's total flows into the lower half's suffix sums
        if (half == 1) sXC[128 + i] = acc;
        __syncthreads();
        if (half == 0 && p.alpha_mode == MODE_CHANNEL) {
          const float off = sXC[128 + i];
#pragma unroll 4
          for (int j = 0; j < 32; ++j)
            if (j < L) g_dalpha[((tok0 + j) * H + h) * DK + i] = __fdividef(sSuf[j * NT + tid] + off, sAl[j * NT + tid]);
        }
      } else {
        // gates scalar per row (the scan's gamma, 1/gamma, sqrt(beta_k) in shared memory); the per-row
        // terms are summed over channels block by block
        float cs[8];
        auto load_s = [&](int jb, float (&sc)[8]) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            sc[e] = kScaled ? __ldg(g_s + ((tok0 + min(r0 + jb + e, L - 1)) * H + h) * DK + i) : 1.f;
        };
        load_s(0, cs);
#pragma unroll 1
        for (int jb = 0; jb < 32; jb += 8) {
          float ns[8];
          if (jb < 24) load_s(jb + 8, ns);
          float dq[8], db[8], da[8];
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_BS + r0 + jb), dq);
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_BS + 64 + r0 + jb), db);
          tmem_ld8(tmem_addr(tmem, quarter * 32, COL_U + r0 + jb), da);
          float qvv[8], kvv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            qvv[e] = raw_at(tTP, r0 + jb + e);
            kvv[e] = raw_at(tWY, r0 + jb + e);
          }
          tmem_ld_wait();
          const size_t obase = ((tok0 + r0 + jb) * H + h) * DK + i;  // row r0 + jb; rows H x DK floats apart
          const int ostride = H * DK;
          float xg[8], xb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int r = r0 + jb + e;
            const bool valid = r < L;
            const float gm = sRow[r], ginv = sRow[64 + r], sbt = sRow[128 + r];
            const float qv = qvv[e], kv = kvv[e];
            const float scv = kScaled ? (valid ? cs[e] : 0.f) : 1.f;
            const float bv = sbt * kv, av = scv * bv, dav = da[e] * ginv;
            float dg = qv * dq[e] + bv * db[e] - av * dav * ginv;
            if (r == C - 1) dg += rowterm;
            xg[e] = dg * gm;
            const float dbt = gm * db[e] + scv * dav;
            xb[e] = sbt > 0.f ? 0.5f * kv * __fdividef(dbt, sbt) : 0.f;
            if (valid) {
              const size_t o = obase + static_cast<size_t>(e * ostride);
              g_dq[o] = gm * dq[e];
              g_dk[o] = sbt * dbt;
              if constexpr (kScaled) g_ds[o] = bv * dav;
            }
          }
          // sums over my warp's 32 channels: rows r0 + jb + (lane & 7)
          const float sbk = warp_transpose_sum<8>(xb, lane);
          if (lane < 8) sRed[((r0 + jb + lane) * 4 + quarter) * 2] = sbk;
          if (p.alpha_mode == MODE_SCALAR) {
            const float sg = warp_transpose_sum<8>(xg, lane);
            if (lane < 8) sRed[((r0 + jb + lane) * 4 + quarter) * 2 + 1] = sg;
          }
          if (jb < 24) {
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[e] = ns[e];
          }
        }
      }
      __syncthreads();
      // scalar gates: per-row sums over the four channel quarters; the decay's gradient is then a suffix
      // sum over the rows, divided by the row's alpha (warp 0: rows 2 lane, 2 lane + 1)
      if (warp == 0 && (p.alpha_mode == MODE_SCALAR || p.beta_k_mode == MODE_SCALAR)) {
        float gs[2], bs[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = 2 * lane + e;
          gs[e] = sRed[(r * 4) * 2 + 1] + sRed[(r * 4 + 1) * 2 + 1] + sRed[(r * 4 + 2) * 2 + 1] + sRed[(r * 4 + 3) * 2 + 1];
          bs[e] = sRed[(r * 4) * 2] + sRed[(r * 4 + 1) * 2] + sRed[(r * 4 + 2) * 2] + sRed[(r * 4 + 3) * 2];
        }
        if (p.alpha_mode == MODE_SCALAR) {
          float sfx = gs[0] + gs[1];  // becomes the sum over rows >= 2 lane
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, sfx, off);
            if (lane + off < 32) sfx += y;
          }
          const float after = __shfl_down_sync(0xffffffffu, sfx, 1);
          const float s1 = gs[1] + (lane < 31 ? after : 0.f), s0 = gs[0] + s1;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 2 * lane + e;
            if (r < L) {
              const size_t th = (tok0 + r) * H + h;
              const float a = kChanGates ? __ldg(g_alpha + th) : sRow[192 + r];
              g_dalpha[th] = (e ? s1 : s0) / a;
            }
          }
        }
        if (p.beta_k_mode == MODE_SCALAR) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 2 * lane + e;
            if (r < L) {
              const size_t th = (tok0 + r) * H + h;
              float v = bs[e];
              if (sym_write) {  // w = sqrt(beta_k) v as well: 0.5 / sqrt(beta_k) sum_v v dV
                const float sbt = kChanGates ? tc::sqrt_fast(__ldg(g_beta_k + th)) : sRow[128 + r];
                v += sbt > 0.f ? 0.5f * sRV[4 * r] / sbt : 0.f;
              }
              g_dbeta_k[th] = v;
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (ok && p.dS0) {
    float dS[64];
    ld_au(dS);
    float *dst = p.dS0 + head * DK * DV + static_cast<size_t>(srow) * DV + half * 64;
#pragma unroll
    for (int j = 0; j < 64; j += 4) *reinterpret_cast<float4 *>(dst + j) = make_float4(dS[j], dS[j + 1], dS[j + 2], dS[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace bwc
}  // namespace dr
