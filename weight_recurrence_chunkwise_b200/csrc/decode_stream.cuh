// decode_stream.cuh -- K5 for dk = dv = 128 on many heads: the decode step of decode.cuh as a
// persistent kernel that prefetches the next head's state while it updates the current one.
//
// Arithmetic, per head (DeltaNet page, steps 3-6; FG2-GDN page, section 2; OSDN summary,
// "Method"), identical to decode_step_kernel operation by operation, so the two give the same bits:
//   r = (D S)^T b,  p = (D S)^T q,  u = w - r,  o = p + u (a . q),  S <- D S + a u^T
//
// The step moves 128 KiB of fp32 state per head (read, then written in place) and does about one
// flop per byte, so it is bound by HBM.  decode_step_kernel (one CTA per head, two per SM) has a
// head's loads in flight only while that CTA waits on them, and none while it reduces and stores.
// Here two CTAs per SM each walk heads blockIdx.x, blockIdx.x + gridDim.x, ...: once the CTA has
// moved the current head from shared memory into registers (the first block barrier of the step
// orders those reads before any overwrite), every thread copies its 16 x 4 tile of the CTA's next
// head into the same place with 16-byte asynchronous copies (cp.async, one commit group per head),
// so that load is in flight while the current head is reduced, updated and stored from registers.
// A thread reads back only the tile it copied itself, so its wait_group is all the landing needs;
// the next head's per-row factors are loaded into registers during the current head and published
// at its end.  One 64 KiB stage per CTA keeps two CTAs (16 warps) on each SM; a deeper ring with
// one CTA per SM was slower (its single CTA serialises every head's reduce-update chain).  Tile
// layout as in decode_step_kernel: warp w owns rows w, w+8, ...; lane l owns columns 4l..4l+3.
#pragma once
#include "common.cuh"

namespace dr {

__device__ __forceinline__ void cp_async16_cg(void *dst_smem, const void *src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kDecodeStages = 1;  // per CTA; two CTAs per SM
constexpr size_t kDecodeStreamSmem = size_t(kDecodeStages) * 128 * 128 * sizeof(float);

template <typename IO>
__global__ void __launch_bounds__(256, 2)
decode_stream_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                     const float *__restrict__ alpha, int alpha_mode, const float *__restrict__ beta_k,
                     int beta_k_mode, const float *__restrict__ beta_v, int beta_v_mode,
                     const float *__restrict__ s_scale, float *__restrict__ S, IO *__restrict__ o,
                     long long nheads) {
  constexpr int DK = 128, DV = 128, NW = 8, RPW = DK / NW, CPL = 4, NST = kDecodeStages;
  extern __shared__ float4 stage_mem[];  // NST x [DK][DV] fp32
  float *stages = reinterpret_cast<float *>(stage_mem);
  __shared__ float s_al[2][DK], s_b[2][DK], s_a[2][DK], s_q[2][DK], s_w[2][DV];
  __shared__ float s_u[DV];
  __shared__ float s_red_r[NW][DV], s_red_p[NW][DV];
  __shared__ float s_bq;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long G = gridDim.x, h0 = blockIdx.x;

  auto issue_state = [&](long long bh, int stg) {
    const float *src = S + bh * (DK * DV);
    float *dst = stages + stg * (DK * DV);
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int off = (warp + rr * NW) * DV + lane * CPL;
      cp_async16_cg(dst + off, src + off);
    }
  };
  // raw per-row (threads 0..127) or per-column (threads 128..255) inputs of one head
  struct Raw {
    float kk, bk, sc, qq, al, vv, ws;
  };
  auto load_raw = [&](long long bh, Raw &f) {
    if (tid < DK) {
      f.bk = gate_at(beta_k, beta_k_mode, bh, DK, tid);
      f.kk = to_f32(k[bh * DK + tid]);
      f.sc = s_scale ? s_scale[bh * DK + tid] : 1.f;
      f.qq = to_f32(q[bh * DK + tid]);
      f.al = gate_at(alpha, alpha_mode, bh, DK, tid);
    } else {
      const int j = tid - 128;
      f.vv = to_f32(v[bh * DV + j]);
      f.ws = (beta_v_mode != MODE_ABSENT) ? gate_at(beta_v, beta_v_mode, bh, DV, j)
                                          : sqrtf(gate_at(beta_k, beta_k_mode, bh, DK, j));
    }
  };
  auto publish = [&](const Raw &f, int buf) {
    if (tid < DK) {
      const float bt = sqrtf(f.bk) * f.kk;
      s_b[buf][tid] = bt;
      s_a[buf][tid] = s_scale ? f.sc * bt : bt;
      s_q[buf][tid] = f.qq;
      s_al[buf][tid] = f.al;
    } else {
      s_w[buf][tid - 128] = f.ws * f.vv;
    }
  };

  // prologue: the states of this CTA's first NST heads in flight; the first head's factors
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    const long long bh = h0 + j * G;
    if (bh < nheads) issue_state(bh, j);
    cp_async_commit_group();
  }
  if (h0 < nheads) {
    Raw f;
    load_raw(h0, f);
    publish(f, 0);
  }
  __syncthreads();

  for (long long it = 0;; ++it) {
    const long long bh = h0 + it * G;
    if (bh >= nheads) break;
    const int buf = static_cast<int>(it & 1), stg = static_cast<int>(it % NST);
    // the next head's factors, consumed at the end of this iteration
    const long long bh_next = bh + G;
    Raw fn;
    if (bh_next < nheads) load_raw(bh_next, fn);
    // this thread's tile of the current head has landed: into registers (the stage takes the head
    // NST ahead once the block barrier below has ordered these reads before the copies)
    cp_async_wait_group<NST - 1>();
    float s[RPW][CPL];
    {
      const float *src = stages + stg * (DK * DV);
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const float4 x = *reinterpret_cast<const float4 *>(src + (warp + rr * NW) * DV + lane * CPL);
        s[rr][0] = x.x, s[rr][1] = x.y, s[rr][2] = x.z, s[rr][3] = x.w;
      }
    }
    if (warp == 0) {
      float acc = 0.f;
      for (int i = lane; i < DK; i += 32) acc += s_a[buf][i] * s_q[buf][i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) s_bq = acc;
    }
    // decay in registers and the two partial reductions over this warp's rows
    float r[CPL], p[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) r[c] = p[c] = 0.f;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int i = warp + rr * NW;
      const float al = s_al[buf][i], bi = s_b[buf][i], qi = s_q[buf][i];
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
    // every thread's reads of the stage are complete: copy in the head NST ahead (one commit group
    // per iteration, empty past the last head)
    const long long bh_ahead = bh + NST * G;
    if (bh_ahead < nheads) issue_state(bh_ahead, stg);
    cp_async_commit_group();
    // finish the reductions; error u and output o per value column
    if (tid < DV) {
      float rs = 0.f, ps = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        rs += s_red_r[w][tid];
        ps += s_red_p[w][tid];
      }
      const float u = s_w[buf][tid] - rs;
      s_u[tid] = u;
      o[bh * DV + tid] = from_f32<IO>(fmaf(u, s_bq, ps));
    }
    __syncthreads();
    // rank-1 write and in-place store of the new state
    float *Sh = S + bh * (DK * DV);
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int i = warp + rr * NW;
      const float ai = s_a[buf][i];
      float4 x;
      x.x = fmaf(ai, s_u[lane * CPL + 0], s[rr][0]);
      x.y = fmaf(ai, s_u[lane * CPL + 1], s[rr][1]);
      x.z = fmaf(ai, s_u[lane * CPL + 2], s[rr][2]);
      x.w = fmaf(ai, s_u[lane * CPL + 3], s[rr][3]);
      __stcs(reinterpret_cast<float4 *>(Sh + i * DV + lane * CPL), x);
    }
    if (bh_next < nheads) publish(fn, buf ^ 1);
    __syncthreads();  // the next head's factors are visible; s_u, s_red and s_bq are free
  }
  cp_async_wait_group<0>();
}

}  // namespace dr
