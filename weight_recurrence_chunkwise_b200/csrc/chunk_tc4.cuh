// chunk_tc4.cuh -- chunkwise WY/UT prefill on a cluster of four CTAs per (b, h), for batches with
// few heads (dk = dv = 128, bf16 I/O).
//
// Algebra (DeltaNet page, step 7; FG2-GDN page, section 2), per chunk of C = 64 tokens, with the
// erase key b = sqrt(beta_k) (.) k and the write key a = b, or a = s (.) b under OSDN's per-feature
// write-side key scaling (OSDN summary page, "Method"; kernel flag kScaled):
//   chunk-local:  gamma, Qh = gamma q, Bh = gamma b, Ac = a / gamma, P = lower(Qh Ac^T),
//                 T = (I + strictly-lower(Bh Ac^T))^-1, W = T Bh
//   state pass:   U0 = T Wr, U = U0 - W S, O = Qh S + P U, S <- Diag(gamma_C)(S + Ac^T U)
//
// Work split: CTA r of the cluster runs the state pass for value columns 32r..32r+31 over every
// chunk (chain role, warps 8..15), and builds the chunk-local factors of the chunks c with
// c % 4 == r (local role, warps 0..7).
//
// The local role works in a private area of its shared memory and hands a finished chunk over
// through global memory: one bulk store of the factor block (66,048 bytes: -W, Qh, Ac, [T; P],
// gamma_C) into this head's staging entry for producer r, then a release arrive on ready[r] of all
// four CTAs.  Each chain role loads the block back (one bulk load per chunk, from L2) into one of
// its two factor slots once the slot is free and the chunk is ready.  Unlike a hand-off through
// the peers' slots, the local work of a chunk never holds a slot of a state pass, so four
// producers can each spend up to four chunk periods on a chunk.
//
// Synchronisation (every wait bounded):
//   ready[r]  (in every CTA) producer r's staging entry holds its next chunk (release/acquire,
//             one phase per chunk of that producer)
//   gfree     (in the producing CTA) all four state passes have loaded its last chunk, so the
//             staging entry may be overwritten (one phase per chunk of that producer)
//   full[j]   slot j of this CTA holds its chunk (bulk-load bytes)
// Ordering of the staging memory: the producer's bulk store completes (wait_group 0) and is fenced
// against the generic proxy, then one release fence precedes the (relaxed) arrives; a consumer
// fences after its acquire before its bulk load.
#pragma once
#include "chunk_tc.cuh"

namespace dr {
namespace tc4 {

using tc::C;
using tc::DK;
using tc::kF16Max;
using tc::kMinChunkDecayF16;
using tc::Params;

constexpr int NCTA = 4;  // CTAs per (b, h)
constexpr int VQ = 32;   // value columns per CTA
constexpr int NT = 512;  // threads
constexpr int NL = 256;  // local role: threads 0..255
constexpr int BAR_LOCAL = 1, BAR_CHAIN = 2, BAR_INV = 3;  // BAR_INV: warps 0..3 in the UT inverse
constexpr int RGL = 8;   // channel-gate K1: rows per local thread (8 row groups x 32 groups of 4 channels)
constexpr int NSLOT = 2;

// factor block layout (bytes from its base; the same in the working area, the slots and the
// staging entries); every tile 1024-aligned
constexpr uint32_t SX = 0;             // X, two column blocks of 128 rows x 128 B
constexpr uint32_t SX_CB = 128 * 128;  // column-block stride of X
constexpr uint32_t SAC = 2 * SX_CB;    // Ac, two column blocks of 64 rows x 128 B
constexpr uint32_t STP = SAC + 64 * 256;  // [T; P], one column block of 128 rows x 128 B
constexpr uint32_t SGC = STP + 128 * 128; // gamma_C, 128 fp32
constexpr uint32_t FAC_BYTES = SGC + 512;  // 66,048: the block handed over
constexpr uint32_t BLK_STRIDE = 65 * 1024;  // 66,560
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_WK = 0;                       // the local role's working area
constexpr uint32_t OFF_SL = BLK_STRIDE;              // the chain's factor slots
constexpr uint32_t OFF_S = OFF_SL + NSLOT * BLK_STRIDE;  // state, fp16 copy (128 rows x 128 B; columns 0..31 used)
constexpr uint32_t OFF_WR = OFF_S + 128 * 128;       // write vectors (raw v lands here, swizzled)
constexpr uint32_t OFF_GS = OFF_WR + 64 * 128;       // scalar gates of the next own chunk (alpha, beta_k)
constexpr uint32_t OFF_ROW = OFF_GS + 128 * 4;       // its row gates: gamma, 1/gamma, sqrt(beta_k), gamma_C
constexpr uint32_t OFF_END = OFF_ROW + 256 * 4;
constexpr size_t SMEM_BYTES = OFF_END + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_SL % 1024 == 0 && OFF_S % 1024 == 0 && OFF_WR % 1024 == 0, "tile alignment");
// global staging: per (b, h), one entry of BLK_STRIDE bytes per producer
constexpr size_t STAGE_BYTES_PER_HEAD = static_cast<size_t>(NCTA) * BLK_STRIDE;

// TMEM columns
constexpr uint32_t COL_D1 = 0;     // local: [A raw | P raw] (64)
constexpr uint32_t COL_D2 = 64;    // local: W (128)
constexpr uint32_t COL_U0 = 192;   // chain: U0 (32)
constexpr uint32_t COL_D3 = 256;   // chain: [-W S | Qh S + P U] (32), even chunks
constexpr uint32_t COL_D4 = 320;   // chain: Ac^T U (32)
constexpr uint32_t COL_D3B = 384;  // chain: D3 of odd chunks (32)
constexpr uint32_t TMEM_COLS = 512;

__host__ __device__ constexpr uint32_t slot_off(int j) { return OFF_SL + static_cast<uint32_t>(j) * BLK_STRIDE; }
__host__ __device__ constexpr uint32_t col_d3(int c) { return (c & 1) ? COL_D3B : COL_D3; }

__device__ __forceinline__ bool mbar_test_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bulk copies between global and this CTA's shared memory (both addresses 16-byte aligned, size a
// multiple of 16).  The store belongs to this thread's bulk group; the load completes on `bar`.
__device__ __forceinline__ void bulk_store_global(void *dst, const void *src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src_smem)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_store_commit_wait() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_load_global(void *dst_smem, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst_smem)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Orders this thread's async-proxy accesses to global memory (bulk copies) with its generic-proxy ones.
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// Release-acquire fence at cluster scope: with it, the relaxed arrives that follow publish this
// thread's earlier writes like release arrives, for one fence instead of one per arrive.
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// kChanGates: the gates vary per key channel (alpha per channel, or beta_k per channel); else
// they are one value per row (alpha absent or per token, beta_k per token).
// kScaled: a write-side key scale s [B,T,H,dk] is given (Params::s).
// stage: STAGE_BYTES_PER_HEAD bytes per (b, h) of global memory, 16-byte aligned.
template <typename IO, bool kChanGates, bool kScaled>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_quad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                      const Params p, uint8_t *stage) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_qk, bar_lmma, bar_cmma, bar_out, bar_v, bar_gfree;
  __shared__ uint64_t bar_full[NSLOT], bar_ready[NCTA];
  __shared__ uint32_t tmem_base_sh;
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase_addr = smem_u32(sm);

  const int H = p.H, DV = p.DV;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster_ctarank());  // value slice; equals blockIdx.x
  const int v0 = rank * VQ, h = blockIdx.y, b = blockIdx.z;  // b: batch row, or sequence of a packed batch
  uint8_t *stage_head = stage + (static_cast<size_t>(b) * H + h) * STAGE_BYTES_PER_HEAD;
  // Token range of this sequence.  Dense batch: tokens b*T .. b*T+T-1 of the [B,T,H,.] arrays, TMA
  // coordinates (t, b).  Packed batch (cu_seqlens): tokens cu[b] .. cu[b+1]-1 of the [1,Ttot,H,.]
  // arrays, TMA coordinates (cu[b] + t, 0).  Rows past the sequence end inside a chunk may hold the
  // next sequence's tokens; they act as identity transitions like the padded rows of a dense batch.
  // The offsets are clamped to [0, Ttot], so malformed ones cannot address outside the arrays.
  const int *cu = p.cu_seqlens;
  const int cs = cu ? min(max(cu[b], 0), p.T) : 0;
  const int T = cu ? min(max(cu[b + 1], cs), p.T) - cs : p.T;
  const size_t tok0 = cu ? static_cast<size_t>(cs) : static_cast<size_t>(b) * p.T;
  const int tt0 = cs, tb = cu ? 0 : b;
  const int nchunks = (T + C - 1) / C;
  const bool sym_channel = p.beta_v_mode == MODE_ABSENT && p.beta_k_mode == MODE_CHANNEL;
  const bool scale_col = p.beta_v_mode == MODE_CHANNEL || sym_channel;  // per-column write scales

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_qk, 1);
    mbar_init(&bar_lmma, 1);
    mbar_init(&bar_cmma, 1);
    mbar_init(&bar_out, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_gfree, NCTA);  // every state pass
    for (int j = 0; j < NSLOT; ++j) mbar_init(&bar_full[j], 1);
    for (int r = 0; r < NCTA; ++r) mbar_init(&bar_ready[r], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_a);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every CTA's barriers exist before any remote arrive
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
    uint32_t ph_qk = 0, ph_mma = 0;
    // Single-thread work is spread over two warps: warp 0 issues the MMAs; ltid 128 (warp 4) issues
    // the TMA loads, L2 prefetches and DSMEM copies and tracks the free[] phases.
    constexpr int kIo = 128;
    uint32_t ph_gfree = 0;  // parity of the next wait on gfree (ltid kIo only)
    const int rgl = ltid >> 5, c0 = 4 * (ltid & 31);  // channel-gate K1: rows 8 rgl.., channels c0..c0+3
    const int quarter = warp & 3, half = warp >> 2;  // warps 0..7
    constexpr bool gates_scalar = !kChanGates;
    float *sGate = reinterpret_cast<float *>(sm + OFF_GS);  // [0..63] alpha, [64..127] beta_k
    float pal[4 * RGL], pbe[4 * RGL];                        // channel-gate K1: this thread's gates
#pragma unroll
    for (int i = 0; i < 4 * RGL; ++i) pal[i] = pbe[i] = 1.f;

    // channel-wise decays arrive by TMA with q and k, into the slot's Ac and [T; P] tiles (free until
    // K1 writes them): four 128-byte-swizzled boxes of 32 channels x 64 rows, fp32
    const bool a_tma = kChanGates && p.alpha_mode == MODE_CHANNEL;
    auto issue_qk = [&](int c) {  // raw q and k of chunk c, in place into the working area
      const int t0 = c * C;
      uint8_t *X = sm + OFF_WK;
      mbar_arrive_expect_tx(&bar_qk, 4 * 64 * 128 + (a_tma ? 4 * 64 * 128 : 0));
      if (a_tma) {
#pragma unroll
        for (int i = 0; i < 4; ++i) tma_load_4d(X + SAC + i * 64 * 128, &tm_a, &bar_qk, 32 * i, h, tt0 + t0, tb);
      }
      tma_load_4d(X + 64 * 128, &tm_q, &bar_qk, 0, h, tt0 + t0, tb);
      tma_load_4d(X + SX_CB + 64 * 128, &tm_q, &bar_qk, 64, h, tt0 + t0, tb);
      tma_load_4d(X, &tm_k, &bar_qk, 0, h, tt0 + t0, tb);
      tma_load_4d(X + SX_CB, &tm_k, &bar_qk, 64, h, tt0 + t0, tb);
    };
    // gates of chunk c.  Scalar: staged by cp.async (warp 0, lane l: rows 2l, 2l+1), one own chunk
    // ahead.  Channel: L2 prefetch one own chunk ahead (prefetch_gates), then loaded into registers
    // at the top of the chunk's iteration (load_gates), so they are live only until K1.
    // Loads only; masking and broadcast happen at use.
    auto prefetch_gates = [&](int c) {
      const int t0 = c * C, L = min(C, T - t0);
      const size_t thb = (tok0 + t0) * H + h;
      if constexpr (kScaled) {  // thread ltid: 128-byte line (ltid & 3) of row (ltid >> 2) of s
        const size_t th = thb + static_cast<size_t>(min(ltid >> 2, L - 1)) * H;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.s + th * DK + (ltid & 3) * 32));
      }
      if constexpr (gates_scalar) {
        if (warp == 0) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const size_t th = thb + static_cast<size_t>(min(2 * lane + e, L - 1)) * H;
            if (p.alpha_mode == MODE_SCALAR) cp_async4(sGate + 2 * lane + e, p.alpha + th);
            cp_async4(sGate + 64 + 2 * lane + e, p.beta_k + th);
          }
          cp_async_commit();
        }
      } else {
        // thread ltid: 128-byte line (ltid & 3) of row (ltid >> 2) of each channel-wise gate
        const size_t th = thb + static_cast<size_t>(min(ltid >> 2, L - 1)) * H;
        const size_t off = th * DK + (ltid & 3) * 32;
        // channel alpha: the TMA L2 prefetch two own chunks ahead covers it
        if (p.beta_k_mode == MODE_CHANNEL) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.beta_k + off));
      }
    };
    auto load_gates = [&](int c) {  // channel-gate K1 only
      const int t0 = c * C, L = min(C, T - t0);
      const size_t thb = (tok0 + t0) * H + h;
#pragma unroll
      for (int j = 0; j < RGL; ++j) {  // 16-byte loads: four channels of a row per request
        const size_t th = thb + static_cast<size_t>(min(rgl * RGL + j, L - 1)) * H;
        if (p.alpha_mode == MODE_CHANNEL) {
          // by TMA (read in K1)
        } else if (p.alpha_mode == MODE_SCALAR) {
          pal[4 * j] = __ldg(p.alpha + th);
        }
        if (p.beta_k_mode == MODE_CHANNEL) {
          const float4 bt = __ldg(reinterpret_cast<const float4 *>(p.beta_k + th * DK + c0));
          pbe[4 * j] = bt.x;
          pbe[4 * j + 1] = bt.y;
          pbe[4 * j + 2] = bt.z;
          pbe[4 * j + 3] = bt.w;
        } else {
          pbe[4 * j] = __ldg(p.beta_k + th);
        }
      }
    };
    // Scalar gates, warp 0: the row gates of own chunk c from its staged alpha, beta_k -- gamma_r
    // (inclusive product), 1/gamma_r, sqrt(beta_r) and gamma_C -- done one own chunk ahead, so that
    // K1 starts on the elements at once.
    float *sRow = reinterpret_cast<float *>(sm + OFF_ROW);
    auto scan_gates = [&](int c) {
      const int L = min(C, T - c * C);
      cp_async_wait_all();  // this lane's own staged rows
      const float2 ga = *reinterpret_cast<const float2 *>(sGate + 2 * lane);
      const float2 gb = *reinterpret_cast<const float2 *>(sGate + 64 + 2 * lane);
      const bool asc = p.alpha_mode == MODE_SCALAR;
      const float a0 = (asc && 2 * lane < L) ? ga.x : 1.f, a1 = (asc && 2 * lane + 1 < L) ? ga.y : 1.f;
      const float b0 = (2 * lane < L) ? gb.x : 0.f, b1 = (2 * lane + 1 < L) ? gb.y : 0.f;
      float incl = a0 * a1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl *= y;
      }
      const float up = __shfl_up_sync(0xffffffffu, incl, 1);
      const float ex = (lane == 0) ? 1.f : up;  // product of the rows before 2*lane
      const float g0 = ex * a0, g1 = g0 * a1;
      *reinterpret_cast<float2 *>(sRow + 2 * lane) = make_float2(g0, g1);
      *reinterpret_cast<float2 *>(sRow + 64 + 2 * lane) = make_float2(__fdividef(1.f, g0), __fdividef(1.f, g1));
      *reinterpret_cast<float2 *>(sRow + 128 + 2 * lane) = make_float2(tc::sqrt_fast(b0), tc::sqrt_fast(b1));
      if (lane == 31) sRow[192] = incl;
    };
    // TMA data: every thread waits; signals: one thread waits, the group barrier releases the others
    auto wait_all = [&](uint64_t *bar, uint32_t &ph) -> bool {
      const bool ok = mbar_wait(bar, ph & 1u, kWaitLimitNs);
      ph++;
      const bool fail = bar_or(BAR_LOCAL, NL, !ok);
      if (fail && ltid == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };
    auto wait_one = [&](uint64_t *bar, uint32_t &ph) -> bool {
      bool ok = true;
      if (ltid == 0) ok = mbar_wait(bar, ph & 1u, kWaitLimitNs);
      ph++;
      const bool fail = bar_or(BAR_LOCAL, NL, !ok);
      tc_fence_after();
      if (fail && ltid == 0) raise_status(p.status, STATUS_TIMEOUT);
      return !fail;
    };

    auto prefetch_qk_l2 = [&](int c) {
      for (int x = 0; x < DK; x += 64) {
        tma_prefetch_l2_4d(&tm_q, x, h, tt0 + c * C, tb);
        tma_prefetch_l2_4d(&tm_k, x, h, tt0 + c * C, tb);
      }
      if (a_tma)
        for (int x = 0; x < DK; x += 32) tma_prefetch_l2_4d(&tm_a, x, h, tt0 + c * C, tb);
    };
    if (rank < nchunks) {
      if (ltid == kIo) {
        issue_qk(rank);
        if (rank + NCTA < nchunks) prefetch_qk_l2(rank + NCTA);
      }
      prefetch_gates(rank);
      if constexpr (gates_scalar) {
        if (warp == 0) scan_gates(rank);
      }
    }
    for (int c = rank; c < nchunks; c += NCTA) {
      const int t0 = c * C, L = min(C, T - t0);
      uint8_t *X = sm + OFF_WK;
      uint8_t *tAC = X + SAC;
      uint8_t *tTP = X + STP;
      float *sGC = reinterpret_cast<float *>(X + SGC);
      const uint32_t xaddr = sbase_addr + OFF_WK;
      if (ltid == kIo && c + 2 * NCTA < nchunks) prefetch_qk_l2(c + 2 * NCTA);
      if constexpr (!gates_scalar) load_gates(c);
      if (!wait_all(&bar_qk, ph_qk)) break;

      // -------------------------------------------------------------- K1: Qh, Bh (in place), Ac, gamma_C
      if constexpr (gates_scalar) {
        // row gates: computed by scan_gates at the end of the previous own chunk (or before the loop)
        if (warp == 0) {
          const float gC = sRow[192];
          *reinterpret_cast<float4 *>(sGC + 4 * lane) = make_float4(gC, gC, gC, gC);
          if (lane == 0 && !(gC >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
        }
        // elements: (row r, 8-column group j8), four per thread, 16-byte loads and stores
        const int j8 = ltid & 15;
        float amax = 0.f;
        float ssc[kScaled ? 4 : 1][kScaled ? 8 : 1];  // write-side key scales of my four rows
        if constexpr (kScaled) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = min((ltid >> 4) + 16 * i, L - 1);
            const float4 *src = reinterpret_cast<const float4 *>(
                p.s + ((tok0 + t0 + r) * H + h) * DK + j8 * 8);
            const float4 lo = __ldg(src), hi = __ldg(src + 1);
            ssc[i][0] = lo.x; ssc[i][1] = lo.y; ssc[i][2] = lo.z; ssc[i][3] = lo.w;
            ssc[i][4] = hi.x; ssc[i][5] = hi.y; ssc[i][6] = hi.z; ssc[i][7] = hi.w;
          }
        }
#pragma unroll(kScaled ? 4 : 1)
        for (int i = 0; i < 4; ++i) {
          const int r = (ltid >> 4) + 16 * i;
          const float g = sRow[r], gi = sRow[64 + r], sb = sRow[128 + r];
          uint4 *pq = reinterpret_cast<uint4 *>(X + sw128_off16(64 + r, j8, 128));
          uint4 *pk = reinterpret_cast<uint4 *>(X + sw128_off16(r, j8, 128));
          const uint4 qraw = *pq, kraw = *pk;
          const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qraw);
          const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw);
          uint32_t oq[4], ob[4], oa[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 qf = __bfloat1622float2(q2[e]), kf = __bfloat1622float2(k2[e]);
            const float b0 = sb * kf.x, b1 = sb * kf.y;
            float x0 = b0 * gi, x1 = b1 * gi;
            if constexpr (kScaled) {
              x0 *= ssc[i][2 * e];
              x1 *= ssc[i][2 * e + 1];
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
        if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      } else {
        float *sPX = reinterpret_cast<float *>(tTP);  // row-group gate products, 8 x 128 fp32
        if (a_tma) {  // my rows' decays from the TMA boxes (box c0 / 32, 16-byte chunk of 4 channels)
          const uint8_t *abox = X + SAC + (c0 >> 5) * (64 * 128);
          const uint32_t ach = static_cast<uint32_t>((c0 & 31) >> 2);
#pragma unroll
          for (int jj = 0; jj < RGL; ++jj) {
            const int row = rgl * RGL + jj;
            const float4 a = *reinterpret_cast<const float4 *>(abox + row * 128 + ((ach ^ static_cast<uint32_t>(row & 7)) << 4));
            pal[4 * jj] = a.x;
            pal[4 * jj + 1] = a.y;
            pal[4 * jj + 2] = a.z;
            pal[4 * jj + 3] = a.w;
          }
          bar_sync(BAR_LOCAL, NL);  // every thread has read its decays before sPX and Ac overwrite them
        }
#pragma unroll
        for (int jj = 0; jj < RGL; ++jj) {
          const bool valid = rgl * RGL + jj < L;
#pragma unroll
          for (int e = 1; e < 4; ++e) {
            if (p.alpha_mode != MODE_CHANNEL) pal[4 * jj + e] = pal[4 * jj];
            if (p.beta_k_mode != MODE_CHANNEL) pbe[4 * jj + e] = pbe[4 * jj];
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (p.alpha_mode == MODE_ABSENT || !valid) pal[4 * jj + e] = 1.f;
            if (!valid) pbe[4 * jj + e] = 0.f;
          }
        }
        float pg[4] = {1.f, 1.f, 1.f, 1.f};  // gate product of my row group
#pragma unroll
        for (int jj = 0; jj < RGL; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) pg[e] *= pal[4 * jj + e];
        *reinterpret_cast<float4 *>(sPX + rgl * 128 + c0) = make_float4(pg[0], pg[1], pg[2], pg[3]);
        bar_sync(BAR_LOCAL, NL);
        float gr[4] = {1.f, 1.f, 1.f, 1.f};  // gamma_r of the current row: starts at the groups before mine
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          if (g < rgl) {
            const float4 x = *reinterpret_cast<const float4 *>(sPX + g * 128 + c0);
            gr[0] *= x.x;
            gr[1] *= x.y;
            gr[2] *= x.z;
            gr[3] *= x.w;
          }
        }
        if (rgl == 7) {  // the last group: gamma_C = (groups before) x (my group)
          const float4 gC = make_float4(gr[0] * pg[0], gr[1] * pg[1], gr[2] * pg[2], gr[3] * pg[3]);
          *reinterpret_cast<float4 *>(sGC + c0) = gC;
          if (!(fminf(fminf(gC.x, gC.y), fminf(gC.z, gC.w)) >= kMinChunkDecayF16)) raise_status(p.status, STATUS_RANGE);
        }
        const bool beta_scalar = p.beta_k_mode == MODE_SCALAR;
        // element (row, c0..c0+3): 8 bytes inside one 16-byte group of the swizzled row; rows of my
        // group are 8 rgl + jj, so the swizzle of row jj is (group ^ jj)
        const uint32_t blk = static_cast<uint32_t>(c0 >> 6), grp = static_cast<uint32_t>((c0 & 63) >> 3);
        const uint32_t inb = static_cast<uint32_t>((c0 & 7) * 2);
        uint8_t *pQ = X + blk * SX_CB + (64 + rgl * RGL) * 128 + inb;
        uint8_t *pB = X + blk * SX_CB + (rgl * RGL) * 128 + inb;
        uint8_t *pA = tAC + blk * 64 * 128 + (rgl * RGL) * 128 + inb;
        float amax = 0.f;
        // rows in batches of RB: a batch's raw k and q are read before any of its results are
        // written back in place, so their shared-memory loads overlap
        constexpr int RB = kScaled ? 1 : 4;  // the scaled variant has no registers to spare
#pragma unroll
        for (int j0 = 0; j0 < RGL; j0 += RB) {
          uint2 kraw[RB], qraw[RB];
#pragma unroll
          for (int jb = 0; jb < RB; ++jb) {
            const int jj = j0 + jb;
            const uint32_t sw = ((grp ^ static_cast<uint32_t>(jj & 7)) << 4) + jj * 128;
            kraw[jb] = *reinterpret_cast<const uint2 *>(pB + sw);  // raw k
            qraw[jb] = *reinterpret_cast<const uint2 *>(pQ + sw);  // raw q
          }
#pragma unroll
          for (int jb = 0; jb < RB; ++jb) {
            const int jj = j0 + jb;
            const uint32_t sw = ((grp ^ static_cast<uint32_t>(jj & 7)) << 4) + jj * 128;
            const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw[jb]);
            const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qraw[jb]);
            float kf[4], qf[4];
            {
              const float2 k01 = __bfloat1622float2(k2[0]), k23 = __bfloat1622float2(k2[1]);
              const float2 q01 = __bfloat1622float2(q2[0]), q23 = __bfloat1622float2(q2[1]);
              kf[0] = k01.x; kf[1] = k01.y; kf[2] = k23.x; kf[3] = k23.y;
              qf[0] = q01.x; qf[1] = q01.y; qf[2] = q23.x; qf[3] = q23.y;
            }
            float sc[4] = {1.f, 1.f, 1.f, 1.f};
            if constexpr (kScaled) {
              const size_t th = (tok0 + t0 + min(rgl * RGL + jj, L - 1)) * H + h;
              const float4 x = __ldg(reinterpret_cast<const float4 *>(p.s + th * DK + c0));
              sc[0] = x.x; sc[1] = x.y; sc[2] = x.z; sc[3] = x.w;
            }
            float sb[4];
            if (beta_scalar) {
              sb[0] = sb[1] = sb[2] = sb[3] = tc::sqrt_fast(pbe[4 * jj]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) sb[e] = tc::sqrt_fast(pbe[4 * jj + e]);
            }
            float oq[4], ob[4], oa[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              gr[e] *= pal[4 * jj + e];
              const float bv = sb[e] * kf[e];
              float av = bv * __fdividef(1.f, gr[e]);  // a / gamma_r
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
        }
        if (!(amax < kF16Max)) raise_status(p.status, STATUS_RANGE);
      }
      fence_async_smem();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- m1: D1 = [Bh; Qh] Ac^T
      if (warp == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint64_t dX = sdesc_sw128(xaddr + SX, 16, 1024);
          const uint64_t dAcK = sdesc_sw128(xaddr + SAC, 16, 1024);
          const uint32_t idesc = idesc_f16_f32(128, 64, false, false);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            umma_f16(tmem + COL_D1, kstep(dX, 128, kk), kstep(dAcK, 64, kk), idesc, kk > 0);
          umma_commit(&bar_lmma);
        }
        __syncwarp();
      }
      if (gates_scalar && c + NCTA < nchunks) prefetch_gates(c + NCTA);
      if (!wait_one(&bar_lmma, ph_mma)) break;

      // -------------------------------------------------------------- E1a: A -> TP rows 0..63 (inverse input)
      if (quarter < 2) {
        const int r = quarter * 32 + lane;
#pragma unroll 1
        for (int jh = 0; jh < 32; jh += 16) {
          float x[16];
          const int col0 = half * 32 + jh;
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + col0), x);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = (col0 + i < r) ? x[i] : 0.f;
          tc::st_h16x16(tTP, r, col0, 128, x);
        }
      }
      tc_fence_before();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- K2: T = (I + A)^-1 (warp MMAs)
      {
        if (warp < 4) {
          tri::Frag Trow[4];
          tri::inverse64_rows<tri::Sw128Layout>(tTP, tTP + 64 * 128, warp, lane, Trow,
                                                [] { bar_sync(BAR_INV, 128); });
          // every read of A is done: T replaces it
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
      }
      fence_async_smem();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- m2: D2 = [T; .] Bh -> W at lanes 0..63
      if (warp == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint64_t dTP = sdesc_sw128(xaddr + STP, 16, 1024);
          const uint64_t dBh = sdesc_sw128(xaddr + SX, SX_CB, 1024);
          const uint32_t id2 = idesc_f16_f32(128, 128, false, true);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            umma_f16(tmem + COL_D2, kstep(dTP, 128, kk), mstep(dBh, kk), id2, kk > 0);
          umma_commit(&bar_lmma);
        }
        __syncwarp();
      }
      if (!gates_scalar && c + NCTA < nchunks) prefetch_gates(c + NCTA);
      if (!wait_one(&bar_lmma, ph_mma)) break;

      // -------------------------------------------------------------- E2: -W -> X rows 0..63;  E1b: P -> TP rows 64..127
      if (quarter < 2) {
        const int r = quarter * 32 + lane;
#pragma unroll 1
        for (int jw = 0; jw < 64; jw += 16) {
          float x[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D2 + half * 64 + jw), x);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = -x[i];
          tc::st_h16x16(X, r, half * 64 + jw, 128, x);
        }
      } else {
        const int r = (quarter - 2) * 32 + lane;
#pragma unroll 1
        for (int jh = 0; jh < 32; jh += 16) {
          float x[16];
          const int col0 = half * 32 + jh;
          tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D1 + col0), x);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = (col0 + i <= r) ? x[i] : 0.f;
          tc::st_h16x16(tTP, 64 + r, col0, 128, x);
        }
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_LOCAL, NL);

      // -------------------------------------------------------------- hand the block to the four state passes
      // (through this producer's staging entry, once every state pass has loaded its previous chunk
      // from there); then the working area takes the raw q/k of the next own chunk
      if (ltid == kIo) {
        bool ok = true;
        if (c >= NCTA) {
          ok = mbar_wait_cluster(&bar_gfree, ph_gfree & 1u, kWaitLimitNs);
          ph_gfree ^= 1u;
        }
        if (ok) {
          uint8_t *dst = stage_head + static_cast<size_t>(rank) * BLK_STRIDE;
          bulk_store_global(dst, X, 32768);
          bulk_store_global(dst + 32768, X + 32768, 32768);
          bulk_store_global(dst + 65536, X + 65536, FAC_BYTES - 65536);
          bulk_store_commit_wait();
          if (c + NCTA < nchunks) issue_qk(c + NCTA);  // the store has read the working area
          // the block is in global memory: one release fence orders it before all four arrives
          fence_proxy_async_all();
          fence_acq_rel_cluster();
#pragma unroll 1
          for (int r = 0; r < NCTA; ++r)
            mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bar_ready[rank]), static_cast<uint32_t>(r)));
        } else {
          raise_status(p.status, STATUS_TIMEOUT);  // the next wait for raw q/k then fails for all
        }
      }
      if constexpr (gates_scalar) {
        if (warp == 0 && c + NCTA < nchunks) scan_gates(c + NCTA);
      }
    }
  } else {
    // ================================================================== chain role
    const int ct = tid - NL;
    const int cw = warp - 8;
    const int quarter = cw & 3, half = cw >> 2;
    const int trow = quarter * 32 + lane;
    const int hc = half * 16;  // this thread's 16 columns of the slice
    uint32_t ph_v = 0, ph_mma = 0, ph_out = 0;
    int u0_ready = -1;      // elected issuing thread: the chunk whose U0 is already issued
    uint32_t ph_full = 0;   // bit j: parity of the next wait on full[j]
    uint32_t ph_ready = 0;  // ct == 128: bit r, parity of the next wait on ready[r]
    int n_loaded = 0;       // ct == 128: chunks whose factor block has been requested (in order)
    bool aborted = false;
    const size_t sbase = (static_cast<size_t>(b) * H + h) * DK * DV;
    uint8_t *tS = sm + OFF_S;
    uint8_t *tWR = sm + OFF_WR;
    const int vbox = v0 & ~63;                // v arrives in 64-column boxes
    const int vgrp = (v0 & 63) >> 3;          // the slice's first 16-byte group inside the box
    const int wc = ct >> 2, wjb = ct & 3;     // write-vector row and its 8-column group of the slice

    // factor block of chunk c from its producer's staging entry into slot c % 2 (ct == 128; the
    // slot is free and the producer's ready phase for c has completed)
    auto issue_fac = [&](int c) {
      const int r = c & (NCTA - 1);
      ph_ready ^= 1u << r;
      fence_proxy_async_all();
      uint64_t *fb = &bar_full[c % NSLOT];
      uint8_t *dst = sm + slot_off(c % NSLOT);
      const uint8_t *src = stage_head + static_cast<size_t>(r) * BLK_STRIDE;
      mbar_arrive_expect_tx(fb, FAC_BYTES);
      bulk_load_global(dst, src, 32768, fb);
      bulk_load_global(dst + 32768, src + 32768, 32768, fb);
      bulk_load_global(dst + 65536, src + 65536, FAC_BYTES - 65536, fb);
      ++n_loaded;
    };
    // request, in order, every ready block up to chunk `last` whose slot is free (ct == 128)
    auto pump = [&](int last) {
#pragma unroll 1
      while (n_loaded <= last && n_loaded < nchunks) {
        const int r = n_loaded & (NCTA - 1);
        if (!mbar_test_cluster(&bar_ready[r], (ph_ready >> r) & 1u)) break;
        issue_fac(n_loaded);
      }
    };

    auto issue_v = [&](int c) {
      mbar_arrive_expect_tx(&bar_v, 64 * 128);
      tma_load_4d(tWR, &tm_v, &bar_v, vbox, h, tt0 + c * C, tb);
    };
    // write scales of row wc of chunk c: one scalar (raw; square root at use if symmetric), or 8
    // per-column values (beta_v, or beta_k of the same channels when the write is symmetric)
    float pws = 0.f;
    float psc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) psc[i] = 0.f;
    auto prefetch_ws = [&](int c) {
      const int t0 = c * C, L = min(C, T - t0);
      const size_t th = (tok0 + t0 + min(wc, L - 1)) * H + h;
      if (scale_col) {
        const float *src = (p.beta_v_mode == MODE_CHANNEL ? p.beta_v + th * DV : p.beta_k + th * DK) + v0 + wjb * 8;
        const float4 x = __ldg(reinterpret_cast<const float4 *>(src));
        const float4 y = __ldg(reinterpret_cast<const float4 *>(src + 4));
        psc[0] = x.x; psc[1] = x.y; psc[2] = x.z; psc[3] = x.w;
        psc[4] = y.x; psc[5] = y.y; psc[6] = y.z; psc[7] = y.w;
      } else {
        pws = __ldg((p.beta_v_mode == MODE_SCALAR ? p.beta_v : p.beta_k) + th);
      }
    };
    // separate write strengths beta_v of chunk c into L2, ahead of prefetch_ws: this CTA's 32 value
    // columns of each row (one 128-byte line), or one value per row if scalar.  (Symmetric writes
    // read beta_k, whose rows the local roles already bring into L2.)
    auto prefetch_ws_l2 = [&](int c) {
      if (p.beta_v_mode == MODE_ABSENT) return;
      const int t0 = c * C, L = min(C, T - t0);
      if (ct < C) {
        const size_t th = (tok0 + t0 + min(ct, L - 1)) * H + h;
        const float *a = p.beta_v_mode == MODE_CHANNEL ? p.beta_v + th * DV + v0 : p.beta_v + th;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
      }
    };
    // write vectors of the chunk whose raw v sits in Wr (after bar_v): the slice's 16-byte group
    // vgrp + wjb of row wc becomes group wjb.  No thread reads the groups written here unless it
    // writes its own (vgrp == 0), so the conversion is race-free in place.
    auto convert_wr = [&](int wL) {  // wL: valid rows of the chunk
      float sc[8];
      if (scale_col) {
#pragma unroll
        for (int i = 0; i < 8; ++i) sc[i] = sym_channel ? tc::sqrt_fast(psc[i]) : psc[i];
      } else {
        const float s0 = (p.beta_v_mode == MODE_SCALAR) ? pws : tc::sqrt_fast(pws);
#pragma unroll
        for (int i = 0; i < 8; ++i) sc[i] = s0;
      }
      const uint4 raw = *reinterpret_cast<const uint4 *>(tWR + sw128_off16(wc, vgrp + wjb, 64));
      const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
      float w8[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 vf = __bfloat1622float2(v2[i]);
        w8[2 * i] = sc[2 * i] * vf.x;
        w8[2 * i + 1] = sc[2 * i + 1] * vf.y;
      }
      if (wc >= wL) {  // past the sequence end: TMA zero fill, or the next packed sequence's v
#pragma unroll
        for (int i = 0; i < 8; ++i) w8[i] = 0.f;
      }
      uint4 out;
      out.x = pack_f16x2(w8[0], w8[1]);
      out.y = pack_f16x2(w8[2], w8[3]);
      out.z = pack_f16x2(w8[4], w8[5]);
      out.w = pack_f16x2(w8[6], w8[7]);
      *reinterpret_cast<uint4 *>(tWR + sw128_off16(wc, wjb, 64)) = out;
    };
    // outputs of chunk c: lanes 64..127 of its D3 columns hold Qh S + P U
    auto store_o = [&](int c) {
      const int t0 = c * C, L = min(C, T - t0);
      if (quarter >= 2) {
        const int r = trow - 64;
        float x[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, col_d3(c) + hc), x);
        tmem_ld_wait();
        if (r < L && p.o) {
          const size_t th = (tok0 + t0 + r) * H + h;
          IO *dst = static_cast<IO *>(p.o) + th * DV + v0 + hc;
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
    };

    // fp32 state slice: row trow, columns hc .. hc+15 of this CTA's value slice
    float Sreg[16];
    {
      const float *src = p.S0 ? p.S0 + sbase + static_cast<size_t>(trow) * DV + v0 + hc : nullptr;
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        Sreg[j] = x.x;
        Sreg[j + 1] = x.y;
        Sreg[j + 2] = x.z;
        Sreg[j + 3] = x.w;
      }
      tc::st_h16x16(tS, trow, hc, 128, Sreg);
    }
    const uint64_t dS = sdesc_sw128(sbase_addr + OFF_S, 128 * 128, 1024);
    const uint64_t dWr = sdesc_sw128(sbase_addr + OFF_WR, 64 * 128, 1024);
    constexpr uint32_t id_n = idesc_f16_f32(128, VQ, false, true);   // A K-major, B MN-major
    constexpr uint32_t id_t = idesc_f16_f32(128, VQ, true, true);    // A MN-major (Ac^T), B MN-major
    // U0 = [T; P] Wr of the chunk in the slot at `slot_addr` (elected issuing thread only)
    auto issue_u0 = [&](uint32_t slot_addr) {
      const uint64_t dTP = sdesc_sw128(slot_addr + STP, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        umma_f16(tmem + COL_U0, kstep(dTP, 128, kk), mstep(dWr, kk), id_n, kk > 0);
    };

    // Software pipeline as in the two-CTA ring: the write vectors of chunk c+1 are built while the
    // second MMA group of chunk c runs, and the outputs of chunk c are stored while the first MMA
    // group of chunk c+1 runs (D3 alternates between two column sets).
    if (nchunks > 0) {
      if (ct == 128) pump(NSLOT - 1);
      if (ct == 0) {
        issue_v(0);
        for (int c = 1; c < 3 && c < nchunks; ++c) tma_prefetch_l2_4d(&tm_v, vbox, h, tt0 + c * C, tb);
      }
      for (int c = 1; c < 3 && c < nchunks; ++c) prefetch_ws_l2(c);
      prefetch_ws(0);
      const bool ok_v = mbar_wait(&bar_v, ph_v & 1u, kWaitLimitNs);
      ph_v ^= 1u;
      if (ok_v) convert_wr(min(C, T));
      fence_async_smem();
      if (bar_or(BAR_CHAIN, NT - NL, !ok_v)) {
        if (ct == 0) raise_status(p.status, STATUS_TIMEOUT);
        aborted = true;
      }
    }
    // iteration c builds the write vectors of chunk c+1 and runs the state pass of chunk c; the
    // extra last iteration only stores the outputs of the final chunk
    for (int c = 0; c <= nchunks && !aborted; ++c) {
      const bool run = c < nchunks;
      const int j = c % NSLOT;
      const uint32_t xaddr = sbase_addr + slot_off(j);
      const uint32_t cD3 = col_d3(c);
      float gc = 0.f;
      if (run) {
        // this chunk's block: requested now if it was not ready before
        bool ok_f = true;
        if (ct == 128 && n_loaded == c) {
          const int r = c & (NCTA - 1);
          ok_f = mbar_wait_cluster(&bar_ready[r], (ph_ready >> r) & 1u, kWaitLimitNs);
          if (ok_f) issue_fac(c);
        }
        ok_f = mbar_wait(&bar_full[j], (ph_full >> j) & 1u, kWaitLimitNs) && ok_f;
        ph_full ^= 1u << j;
        if (bar_or(BAR_CHAIN, NT - NL, !ok_f)) {
          if (ct == 0) raise_status(p.status, STATUS_TIMEOUT);
          aborted = true;
          break;
        }
        // this CTA has read the producer's staging entry; the block carries no data back
        if (ct == 128)
          mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bar_gfree), static_cast<uint32_t>(c & (NCTA - 1))));
        gc = reinterpret_cast<const float *>(sm + slot_off(j) + SGC)[trow];

        // ------------------------------------------------------------ U0 = [T;P] Wr,  D3 = [-W; Qh] S
        if (cw == 0) {
          if (elect_one()) {
            tc_fence_after();
            const uint64_t dX = sdesc_sw128(xaddr + SX, 16, 1024);
            if (u0_ready != c) issue_u0(xaddr);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
              umma_f16(tmem + cD3, kstep(dX, 128, kk), mstep(dS, kk), id_n, kk > 0);
            umma_commit(&bar_cmma);
          }
          __syncwarp();
        }
      }
      // the previous chunk's second MMA group (its outputs, and the last reads of its slot): waited
      // for here, where the first group of this chunk runs, by the threads that store the outputs
      // and by the one that requests blocks, which refills the slot with chunk c+1
      bool ok_out = true;
      if (c > 0) {
        if (quarter >= 2 || ct == 128) ok_out = mbar_wait(&bar_out, ph_out & 1u, kWaitLimitNs);
        ph_out ^= 1u;
        tc_fence_after();
        if (!ok_out) raise_status(p.status, STATUS_TIMEOUT);
        if (ok_out && ct == 128) pump(c + 1);
        if (ok_out) store_o(c - 1);  // overlaps the MMAs above
      }
      if (!run) break;
      if (p.states) {  // this chunk's initial state, for the backward pass (dense batches only)
        float *dst = p.states + ((sbase / (static_cast<size_t>(DK) * DV)) * nchunks + c) * DK * DV +
                     static_cast<size_t>(trow) * DV + v0 + hc;
#pragma unroll
        for (int jj = 0; jj < 16; jj += 4)
          *reinterpret_cast<float4 *>(dst + jj) = make_float4(Sreg[jj], Sreg[jj + 1], Sreg[jj + 2], Sreg[jj + 3]);
      }
      // MMA group 1 done
      {
        bool ok = ok_out;
        if (ct == 0) ok = mbar_wait(&bar_cmma, ph_mma & 1u, kWaitLimitNs) && ok;
        ph_mma ^= 1u;
        const bool fail = bar_or(BAR_CHAIN, NT - NL, !ok);
        tc_fence_after();
        if (fail) {
          if (ct == 0) raise_status(p.status, STATUS_TIMEOUT);
          aborted = true;
          break;
        }
      }
      if (ct == 128) {
        if (c + 1 < nchunks) issue_v(c + 1);  // Wr is free
        if (c + 3 < nchunks) tma_prefetch_l2_4d(&tm_v, vbox, h, tt0 + (c + 3) * C, tb);
      }
      if (c + 3 < nchunks) prefetch_ws_l2(c + 3);
      if (c + 1 < nchunks) prefetch_ws(c + 1);

      // -------------------------------------------------------------- E3: U = U0 - W S -> X rows 0..63
      uint8_t *tU = sm + slot_off(j) + SX;
      if (quarter < 2) {
        float ws[16], u0[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, cD3 + hc), ws);
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_U0 + hc), u0);
        tmem_ld_wait();
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          u0[i] += ws[i];
          mx = fmaxf(mx, fabsf(u0[i]));
        }
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
        tc::st_h16x16(tU, trow, hc, 128, u0);
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_CHAIN, NT - NL);

      // -------------------------------------------------------------- D4 = Ac^T U,  D3 += [T;P] U
      if (cw == 0) {
        if (elect_one()) {
          tc_fence_after();
          const uint64_t dAcM = sdesc_sw128(xaddr + SAC, 64 * 128, 1024);
          const uint64_t dTP = sdesc_sw128(xaddr + STP, 16, 1024);
          const uint64_t dU = sdesc_sw128(xaddr + SX, 128 * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + COL_D4, mstep(dAcM, kk), mstep(dU, kk), id_t, kk > 0);
          umma_commit(&bar_cmma);  // the state update waits for Ac^T U alone
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) umma_f16(tmem + cD3, kstep(dTP, 128, kk), mstep(dU, kk), id_n, 1u);
          umma_commit(&bar_out);   // the outputs and the slot's reuse wait for this (next iteration)
        }
        __syncwarp();
      }
      // the slot of chunk c+1 has been free since chunk c-1 was done: request its block if ready
      if (ct == 128) pump(c + 1);
      // while group 2 runs: v of chunk c+1 (TMA data: every thread waits) into write vectors, in
      // place in Wr; then group 2's completion.  One group barrier decides both waits.
      {
        bool ok = true;
        if (c + 1 < nchunks) {
          ok = mbar_wait(&bar_v, ph_v & 1u, kWaitLimitNs);
          ph_v ^= 1u;
          if (ok) convert_wr(min(C, T - (c + 1) * C));
          fence_async_smem();
        }
        if (ct == 0) ok = mbar_wait(&bar_cmma, ph_mma & 1u, kWaitLimitNs) && ok;
        ph_mma ^= 1u;
        const bool fail = bar_or(BAR_CHAIN, NT - NL, !ok);
        tc_fence_after();
        if (fail) {
          if (ct == 0) raise_status(p.status, STATUS_TIMEOUT);
          aborted = true;
          break;
        }
      }
      // U0 of the next chunk, if its block has landed (its write vectors were just built)
      if (cw == 0 && c + 1 < nchunks) {
        if (elect_one()) {
          const int j1 = (c + 1) % NSLOT;
          if (mbar_test_cluster(&bar_full[j1], (ph_full >> j1) & 1u)) {
            tc_fence_after();
            issue_u0(sbase_addr + slot_off(j1));
            u0_ready = c + 1;
          }
        }
        __syncwarp();
      }
      // -------------------------------------------------------------- E4: S <- Diag(gamma_C) (S + Ac^T U)
      {
        float mx = 0.f;
        float ds[16];
        tmem_ld16(tmem_addr(tmem, quarter * 32, COL_D4 + hc), ds);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          Sreg[i] = gc * (Sreg[i] + ds[i]);
          mx = fmaxf(mx, fabsf(Sreg[i]));
        }
        tc::st_h16x16(tS, trow, hc, 128, Sreg);
        if (!(mx < kF16Max)) raise_status(p.status, STATUS_RANGE);
      }
      fence_async_smem();
      tc_fence_before();
      bar_sync(BAR_CHAIN, NT - NL);  // S (fp16) complete for the next chunk's first MMA group
      tc_fence_after();
    }
    if (!aborted && p.S_T) {
      float *dst = p.S_T + sbase + static_cast<size_t>(trow) * DV + v0 + hc;
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = make_float4(Sreg[j], Sreg[j + 1], Sreg[j + 2], Sreg[j + 3]);
    }
  }

  // both roles done; keep this CTA's barriers alive until no other CTA of the cluster can arrive on them
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc4
}  // namespace dr
