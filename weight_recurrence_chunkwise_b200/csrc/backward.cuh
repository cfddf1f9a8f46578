// backward.cuh -- backward pass of the gated delta-rule recurrence, by recomputation.
//
// Forward (DeltaNet page, steps 3-6; FG2-GDN page, section 2 and "Erweiterung: FG2-GDN+"; OSDN
// summary, "Method"), per token t with D = Diag(alpha_t), erase key b, write key a = s (.) b
// (a = b without OSDN's scale) and write vector w:
//   X = D S_{t-1},   u = w - X^T b,   S_t = X + a u^T,   o_t = S_t^T q_t
// Reverse mode, with G the adjoint of S_t (G starts as dS_T):
//   G += q_t do_t^T                       (o_t = S_t^T q_t)
//   dq_t = S_t do_t = X do_t + a (u . do_t)
//   du = G^T a,   da = G u,   db = -X du,   dX = G - b du^T
//   dalpha_t[i] = sum_j dX[i][j] S_{t-1}[i][j],   G <- D dX  (the adjoint of S_{t-1})
// then the chain rule through b = sqrt(beta_k) (.) k, a = s (.) b and
// w = beta_v (.) v or sqrt(beta_k) (.) v.
//
// The value columns of S never mix, forward or backward (u_j, S[:, j] and G[:, j] involve column j
// only), so one CTA of 256 threads walks one (b, h) and one slice of VSB value columns.  It needs
// S_{t-1} at every step, so it keeps the forward's state every CK tokens (checkpoints, in the
// workspace) and, for each span of CK tokens from the last, recomputes the span's states into a
// per-(head, slice) scratch and walks the span backwards.  State, adjoint and scratch are fp32;
// each step is two cross-row reductions through shared memory and four row reductions over the
// lanes of a warp.  Thread layout as in the decode step: warp w owns rows w, w+8, ...; lane l owns
// VSB/32 consecutive columns of the slice.  Per-row gradients (dq, dk, ds, dalpha, dbeta_k) sum
// over the value columns, so each slice adds its part with atomics into outputs zeroed first;
// per-column gradients (dv, dbeta_v) are written by their slice.
//
// A correct, memory- and latency-bound implementation: two sequential passes over T per
// (head, slice), with 2*CK*dk*VSB*4 bytes of scratch traffic per span.
#pragma once
#include "common.cuh"

namespace dr {

struct BwdParams {
  int T, H;
  const void *q, *k, *v, *dout;
  const float *alpha;
  int alpha_mode;
  const float *beta_k;
  int beta_k_mode;
  const float *beta_v;
  int beta_v_mode;
  const float *s;       // OSDN write-side key scale [B,T,H,dk] or nullptr
  const float *S0;      // [B,H,dk,dv] or nullptr
  const float *dS_T;    // [B,H,dk,dv] or nullptr
  float *dq, *dk, *dv;  // [B,T,H,d] fp32
  float *dalpha, *dbeta_k, *dbeta_v, *ds;  // gate shapes, fp32 (nullptr where the input is absent)
  float *dS0;           // [B,H,dk,dv] fp32 or nullptr
  float *ckpt;          // [B*H][DVf/VSB][ceil(T/CK)][dk*VSB]
  float *scratch;       // [B*H][DVf/VSB][CK][dk*VSB]
};

// DV: the slice width handled by one CTA (VSB); DVF: the full value width.
template <typename IO, int DK, int DVF, int DV, int CK>
__global__ void __launch_bounds__(256) delta_rule_bwd_kernel(const BwdParams p) {
  constexpr int NW = 8, RPW = DK / NW, CPL = DV / 32, NSL = DVF / DV;
  static_assert(DK % NW == 0 && DV % 32 == 0 && DVF % DV == 0, "unsupported head dims");
  __shared__ float s_al[DK], s_b[DK], s_ab[DK], s_a[DK], s_q[DK], s_k[DK], s_sc[DK], s_sb[DK];
  __shared__ float s_w[DV], s_do[DV], s_u[DV], s_du[DV], s_v[DV], s_wsc[DV], s_pv[DV];
  __shared__ float s_xdo[DK], s_da[DK], s_db[DK], s_dal[DK];
  __shared__ float s_red[NW][DV];
  __shared__ float s_udo;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, H = p.H;
  const size_t bh = blockIdx.x;  // b * H + h
  const int slice = blockIdx.y, v0 = slice * DV;
  const size_t b = bh / H, h = bh % H;
  const int nck = (T + CK - 1) / CK;
  const size_t hs = bh * NSL + slice;  // (head, slice)
  float *ck = p.ckpt + hs * static_cast<size_t>(nck) * DK * DV;
  float *scr = p.scratch + hs * static_cast<size_t>(CK) * DK * DV;
  const bool sym = p.beta_v_mode == MODE_ABSENT;  // w = sqrt(beta_k) (.) v

  // per-token factors into shared memory (with_back: also q, do, v, k for the gradients)
  auto load_token = [&](int t, bool with_back) {
    const size_t th = (b * T + t) * H + h;
    if (tid < DK) {
      const float bk = gate_at(p.beta_k, p.beta_k_mode, th, DK, tid);
      const float sb = sqrtf(bk);
      const float kk = to_f32(static_cast<const IO *>(p.k)[th * DK + tid]);
      const float bt = sb * kk;
      const float sc = p.s ? p.s[th * DK + tid] : 1.f;
      s_sb[tid] = sb;
      s_b[tid] = bt;
      s_sc[tid] = sc;
      s_a[tid] = sc * bt;
      const float al = gate_at(p.alpha, p.alpha_mode, th, DK, tid);
      s_al[tid] = al;
      s_ab[tid] = al * bt;  // (D^T b)_i: X^T b = S^T (D b)
      if (with_back) {
        s_q[tid] = to_f32(static_cast<const IO *>(p.q)[th * DK + tid]);
        s_k[tid] = kk;
      }
    } else if (tid - 128 < DV && tid >= 128) {
      const int j = tid - 128, jg = v0 + j;  // local and full column index
      const float vj = to_f32(static_cast<const IO *>(p.v)[th * DVF + jg]);
      const float ws = sym ? sqrtf(gate_at(p.beta_k, p.beta_k_mode, th, DK, jg))
                           : gate_at(p.beta_v, p.beta_v_mode, th, DVF, jg);
      s_wsc[j] = ws;
      s_w[j] = ws * vj;
      if (with_back) {
        s_v[j] = vj;
        s_do[j] = to_f32(static_cast<const IO *>(p.dout)[th * DVF + jg]);
      }
    }
  };
  // cross-row reduction: out[j] = sum_i M[i][j] * f[i] over all rows (each warp's rows first)
  auto colsum = [&](const float (&M)[RPW][CPL], const float *f, float *out) {
    float part[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) part[c] = 0.f;
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float fi = f[warp + r * NW];
#pragma unroll
      for (int c = 0; c < CPL; ++c) part[c] = fmaf(M[r][c], fi, part[c]);
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) s_red[warp][lane * CPL + c] = part[c];
    __syncthreads();
    if (tid < DV) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) acc += s_red[w][tid];
      out[tid] = acc;
    }
    __syncthreads();
  };
  auto warp_sum = [](float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
  };
  // one forward step in registers: S <- D S + a (w - (D S)^T b)^T
  auto forward_step = [&](float (&S)[RPW][CPL]) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float al = s_al[warp + r * NW];
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[r][c] *= al;
    }
    colsum(S, s_b, s_u);  // s_u = X^T b
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float ai = s_a[warp + r * NW];
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[r][c] = fmaf(ai, s_w[lane * CPL + c] - s_u[lane * CPL + c], S[r][c]);
    }
  };
  // ld: row stride of the array (DV for the slice's checkpoints and scratch, DVF for S0, dS_T, dS0)
  auto store_state = [&](float *dst, int ld, const float (&S)[RPW][CPL]) {
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int c = 0; c < CPL; ++c) dst[(warp + r * NW) * ld + lane * CPL + c] = S[r][c];
  };
  auto load_state = [&](const float *src, int ld, float (&S)[RPW][CPL]) {
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[r][c] = src ? src[(warp + r * NW) * ld + lane * CPL + c] : 0.f;
  };

  float S[RPW][CPL];
  const size_t sbase = bh * static_cast<size_t>(DK) * DVF + v0;  // this slice of the full-width state
  // ---- pass 1: the forward, keeping the state before every CK-th token
  load_state(p.S0 ? p.S0 + sbase : nullptr, DVF, S);
  for (int t = 0; t < T; ++t) {
    if (t % CK == 0) store_state(ck + static_cast<size_t>(t / CK) * DK * DV, DV, S);
    __syncthreads();
    load_token(t, false);
    __syncthreads();
    forward_step(S);
  }

  // ---- pass 2: spans of CK tokens from the last, each recomputed then walked backwards
  float G[RPW][CPL];
  load_state(p.dS_T ? p.dS_T + sbase : nullptr, DVF, G);
  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * CK, L = min(CK, T - t0);
    __syncthreads();  // the previous span's scratch reads are done
    load_state(ck + static_cast<size_t>(c) * DK * DV, DV, S);
    for (int i = 0; i < L; ++i) {
      store_state(scr + static_cast<size_t>(i) * DK * DV, DV, S);  // state before token t0 + i
      if (i + 1 == L) break;
      __syncthreads();
      load_token(t0 + i, false);
      __syncthreads();
      forward_step(S);
    }
    for (int i = L - 1; i >= 0; --i) {
      const int t = t0 + i;
      const size_t th = (b * T + t) * H + h;
      __syncthreads();
      load_token(t, true);
      __syncthreads();  // also orders the scratch stores above before the loads below
      float Sp[RPW][CPL];  // S_{t-1}; X = D S_{t-1} is applied row by row where it is used
      load_state(scr + static_cast<size_t>(i) * DK * DV, DV, Sp);
      colsum(Sp, s_ab, s_u);  // s_u = X^T b
      if (tid < DV) s_u[tid] = s_w[tid] - s_u[tid];  // u = w - X^T b
      __syncthreads();
      if (warp == 0) {
        float acc = 0.f;
        for (int j = lane; j < DV; j += 32) acc += s_u[j] * s_do[j];
        acc = warp_sum(acc);
        if (lane == 0) s_udo = acc;
      }
      // G += q do^T
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const float qi = s_q[warp + r * NW];
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) G[r][cc] = fmaf(qi, s_do[lane * CPL + cc], G[r][cc]);
      }
      colsum(G, s_a, s_du);  // du = G^T a
      // row reductions: X do, G u, X du; then dX, dalpha, G <- D dX
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const int row = warp + r * NW;
        float sdo = 0.f, gu = 0.f, sdu = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          const int j = lane * CPL + cc;
          sdo = fmaf(Sp[r][cc], s_do[j], sdo);
          gu = fmaf(G[r][cc], s_u[j], gu);
          sdu = fmaf(Sp[r][cc], s_du[j], sdu);
        }
        const float bi = s_b[row], al = s_al[row];
        const float xdo = al * warp_sum(sdo);  // (X do)_i
        gu = warp_sum(gu);
        const float xdu = al * warp_sum(sdu);  // (X du)_i
        float dal = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          const float dX = G[r][cc] - bi * s_du[lane * CPL + cc];
          dal = fmaf(dX, Sp[r][cc], dal);
          G[r][cc] = al * dX;
        }
        dal = warp_sum(dal);
        if (lane == 0) {
          s_xdo[row] = xdo;
          s_da[row] = gu;
          s_db[row] = -xdu;
          s_dal[row] = dal;
        }
      }
      __syncthreads();
      // per-token gradients.  Per-row ones sum over all value columns: each slice adds its part
      // (outputs are zeroed before the launch); per-column ones belong to this slice alone.
      const float udo = s_udo;
      if (tid < DK) {
        const int i = tid;
        const float ai = s_a[i], sc = s_sc[i], sb = s_sb[i];
        const float dbt = s_db[i] + sc * s_da[i];  // through b, directly and through a = s (.) b
        atomicAdd(&p.dq[th * DK + i], s_xdo[i] + ai * udo);
        atomicAdd(&p.dk[th * DK + i], sb * dbt);
        if (p.ds) atomicAdd(&p.ds[th * DK + i], s_b[i] * s_da[i]);
        const float dbeta = sb > 0.f ? 0.5f * s_k[i] * dbt / sb : 0.f;  // d sqrt(beta) / d beta
        if (p.beta_k_mode == MODE_CHANNEL) atomicAdd(&p.dbeta_k[th * DK + i], dbeta);
        if (p.alpha_mode == MODE_CHANNEL) atomicAdd(&p.dalpha[th * DK + i], s_dal[i]);
        s_k[i] = dbeta;  // scalar-mode partials, summed below
      } else if (tid >= 128 && tid - 128 < DV) {
        const int j = tid - 128, jg = v0 + j;
        const float du = s_du[j];
        p.dv[th * DVF + jg] = s_wsc[j] * du;
        if (!sym && p.beta_v_mode == MODE_CHANNEL) p.dbeta_v[th * DVF + jg] = s_v[j] * du;
        // symmetric channel write w = sqrt(beta_k) (.) v (dk == dv): column jg is key channel jg
        if (sym && p.beta_k_mode == MODE_CHANNEL && s_sb[jg] > 0.f)
          atomicAdd(&p.dbeta_k[th * DK + jg], 0.5f * s_v[j] * du / s_sb[jg]);
        s_pv[j] = s_v[j] * du;  // scalar-mode partials
      }
      __syncthreads();
      if (warp == 0) {  // scalar gates: sums over the channels (this slice's part of the columns)
        float sa = 0.f, sbk = 0.f, svv = 0.f;
        for (int i = lane; i < DK; i += 32) {
          sa += s_dal[i];
          sbk += s_k[i];
        }
        for (int j = lane; j < DV; j += 32) svv += s_pv[j];
        sa = warp_sum(sa);
        sbk = warp_sum(sbk);
        svv = warp_sum(svv);
        if (lane == 0) {
          if (p.alpha_mode == MODE_SCALAR) atomicAdd(&p.dalpha[th], sa);
          if (p.beta_k_mode == MODE_SCALAR) {
            const float sb0 = s_sb[0];  // + through w = sqrt(beta) v
            atomicAdd(&p.dbeta_k[th], sbk + ((sym && sb0 > 0.f) ? 0.5f * svv / sb0 : 0.f));
          }
          if (!sym && p.beta_v_mode == MODE_SCALAR) atomicAdd(&p.dbeta_v[th], svv);
        }
      }
    }
  }
  if (p.dS0) store_state(p.dS0 + sbase, DVF, G);
}

}  // namespace dr
