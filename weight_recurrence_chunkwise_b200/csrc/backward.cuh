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
// only), so one CTA of 256 threads walks one (b, h) and one slice of 32 value columns.  Warp w owns
// rows [w DK/8, (w+1) DK/8); within it lane l holds a tile of R = DK/32 consecutive rows (row group
// l / 8) by 4 consecutive columns (column group l % 8).  It needs S_{t-1} at every step, so it keeps
// the forward's state every CK tokens (checkpoints, in the workspace) and, for each span of CK
// tokens from the last, recomputes the span's states into a per-(head, slice) scratch and walks the
// span backwards.  A thread reads back only the state elements it wrote, so the scratch needs no
// barrier.  State, adjoint and scratch are fp32.
//
// Latency is what bounds this kernel, so each span's token factors (gates, keys, values, output
// gradients; with sqrt(beta) and the products b, a already formed) are staged in shared memory by
// all threads at once, with the next span's lines prefetched into L2 meanwhile, and the previous
// token's recomputed state is loaded one step ahead.  The tile layout keeps the instruction count
// per step low (this kernel issues far more than it moves): row factors and state rows move as
// vectors, cross-row sums are R in-thread terms plus two butterfly stages and one barrier, and the
// four per-row sums (X do, G u, X du, G . S) over a row's 32 columns are 4 in-thread terms plus
// three stages in which every lane sends half of its remaining values and keeps the other half.
// A backward step has two block barriers: one for the cross-row sums u = w - X^T b and du = G^T a,
// taken together, one to publish them.  Per-row gradients (dq, dk, ds, dalpha, dbeta_k) sum over
// all value columns, so each
// slice adds its part with atomics into outputs zeroed before the launch; per-column gradients
// (dv, dbeta_v) are written by their slice.
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
  float *ckpt;          // [B*H][dv/32][ceil(T/CK)][dk*32]
  float *scratch;       // [B*H][dv/32][CK][dk*32]
};

constexpr int kBwdCols = 32;  // value columns per CTA

// Dynamic shared memory of the backward kernel: the span's staged token factors.
template <int DK, int CK>
constexpr int bwd_smem_bytes() {
  return (7 * CK * DK + 4 * CK * kBwdCols) * static_cast<int>(sizeof(float));
}

__device__ __forceinline__ void prefetch_l2(const void *ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// Butterfly sum of N values over the lanes whose index differs in the bits HI, HI/2, ..., LO: at
// each stage a lane sends half of its remaining values and keeps the other half, the lane with the
// stage's bit set keeping the upper half.  Afterwards x[k], k < N / 2^stages, holds the full sum of
// value n = k + sum over stages j of bit_j * N / 2^j.
template <int N, int HI, int LO>
__device__ __forceinline__ void butterfly_sum(float (&x)[N], int lane) {
#pragma unroll
  for (int o = HI, m = N; o >= LO; o >>= 1, m >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int k = 0; k < m / 2; ++k) {
      const float send = up ? x[k] : x[k + m / 2];
      const float keep = up ? x[k + m / 2] : x[k];
      x[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// R consecutive floats from 4R-byte-aligned shared memory, as one vector access.
template <int R>
__device__ __forceinline__ void lds_vec(const float *src, float (&x)[R]) {
  if constexpr (R == 4) {
    const float4 v = *reinterpret_cast<const float4 *>(src);
    x[0] = v.x, x[1] = v.y, x[2] = v.z, x[3] = v.w;
  } else {
    static_assert(R == 2, "R: 2 or 4");
    const float2 v = *reinterpret_cast<const float2 *>(src);
    x[0] = v.x, x[1] = v.y;
  }
}

template <typename IO, int DK, int DVF, int CK>
__global__ void __launch_bounds__(256, 2) delta_rule_bwd_kernel(const BwdParams p) {
  constexpr int DV = kBwdCols, NW = 8, RPW = DK / NW, NSL = DVF / DV;
  constexpr int R = RPW / 4, NQ = 4 * R;  // rows per thread; per-row sums per thread
  static_assert(DV == 32 && DVF % DV == 0 && (R == 2 || R == 4), "unsupported head dims");
  // span stage: per token, rows (key channels) then columns (this slice's value columns)
  extern __shared__ float4 smem_dyn[];
  float *f_al = reinterpret_cast<float *>(smem_dyn);
  float *f_b = f_al + CK * DK, *f_a = f_b + CK * DK, *f_q = f_a + CK * DK, *f_k = f_q + CK * DK;
  float *f_sb = f_k + CK * DK, *f_sc = f_sb + CK * DK;
  float *c_w = f_sc + CK * DK, *c_wsc = c_w + CK * DV, *c_v = c_wsc + CK * DV, *c_do = c_v + CK * DV;
  __shared__ float s_red[2][NW][DV];
  __shared__ __align__(16) float s_u[DV];
  __shared__ __align__(16) float s_du[DV];
  __shared__ __align__(16) float s_rows[NW][4][NQ];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = lane & 7, rg = lane >> 3;            // column group, row group
  const int c0 = 4 * cg, r0 = RPW * warp + R * rg;    // this thread's tile origin
  const int b3 = (lane >> 3) & 1, b4 = (lane >> 4) & 1;
  const int T = p.T, H = p.H;
  const size_t bh = blockIdx.x;  // b * H + h
  const int slice = blockIdx.y, v0 = slice * DV;
  const size_t b = bh / H, h = bh % H;
  const int nck = (T + CK - 1) / CK;
  const size_t hs = bh * NSL + slice;  // (head, slice)
  float *ck = p.ckpt + hs * static_cast<size_t>(nck) * DK * DV;
  float *scr = p.scratch + hs * static_cast<size_t>(CK) * DK * DV;
  const bool sym = p.beta_v_mode == MODE_ABSENT;  // w = sqrt(beta_k) (.) v
  const IO *gq = static_cast<const IO *>(p.q), *gk = static_cast<const IO *>(p.k);
  const IO *gv = static_cast<const IO *>(p.v), *gdo = static_cast<const IO *>(p.dout);
  auto tok = [&](int t) { return (b * T + t) * H + h; };

  // Stage the factors of tokens [t0, t0 + L) (back: also what the gradients need).
  auto load_span = [&](int t0, int L, bool back) {
    constexpr int RI = CK * DK / 256, CI = (CK * DV + 255) / 256;
#pragma unroll
    for (int r = 0; r < RI; ++r) {
      const int e = tid + r * 256, i = e / DK, ch = e % DK;
      if (i < L) {
        const size_t th = tok(t0 + i);
        const float kk = to_f32(gk[th * DK + ch]);
        const float sb = sqrtf(gate_at(p.beta_k, p.beta_k_mode, th, DK, ch));
        const float sc = p.s ? __ldg(p.s + th * DK + ch) : 1.f;
        const float bt = sb * kk;
        f_al[e] = gate_at(p.alpha, p.alpha_mode, th, DK, ch);
        f_b[e] = bt;
        f_a[e] = sc * bt;
        if (back) {
          f_q[e] = to_f32(gq[th * DK + ch]);
          f_k[e] = kk;
          f_sb[e] = sb;
          f_sc[e] = sc;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < CI; ++r) {
      const int e = tid + r * 256, i = e / DV, j = e % DV, jg = v0 + j;
      if (e < CK * DV && i < L) {
        const size_t th = tok(t0 + i);
        const float vj = to_f32(gv[th * DVF + jg]);
        const float ws = sym ? sqrtf(gate_at(p.beta_k, p.beta_k_mode, th, DK, jg))
                             : gate_at(p.beta_v, p.beta_v_mode, th, DVF, jg);
        c_w[e] = ws * vj;
        if (back) {
          c_wsc[e] = ws;
          c_v[e] = vj;
          c_do[e] = to_f32(gdo[th * DVF + jg]);
        }
      }
    }
  };
  // Pull the 128-byte lines of tokens [t0, t0 + L) into L2 (one thread per line).
  auto prefetch_span = [&](int t0, int L, bool back) {
    if (L <= 0) return;
    constexpr int KL = DK * sizeof(IO) / 128, GL = DK * 4 / 128;  // lines per key row / gate row
    const int per = KL * (back ? 2 : 1) + 1 + (back ? 1 : 0) + GL * 3;
    for (int e = tid; e < L * per; e += 256) {
      const int i = e / per, r = e % per;
      const size_t th = tok(t0 + i);
      const char *a = nullptr;
      if (r < KL) {
        a = reinterpret_cast<const char *>(gk + th * DK) + r * 128;
      } else if (back && r < 2 * KL) {
        a = reinterpret_cast<const char *>(gq + th * DK) + (r - KL) * 128;
      } else {
        const int r2 = r - KL * (back ? 2 : 1);
        if (r2 == 0) {
          a = reinterpret_cast<const char *>(gv + th * DVF + v0);
        } else if (back && r2 == 1) {
          a = reinterpret_cast<const char *>(gdo + th * DVF + v0);
        } else {
          const int g = r2 - 1 - (back ? 1 : 0), which = g / GL, line = g % GL;
          const float *gp = which == 0 ? p.alpha : which == 1 ? p.beta_k : p.s;
          const int mode = which == 0 ? p.alpha_mode : which == 1 ? p.beta_k_mode : (p.s ? MODE_CHANNEL : MODE_ABSENT);
          if (mode == MODE_CHANNEL) a = reinterpret_cast<const char *>(gp + th * DK) + line * 128;
          else if (mode == MODE_SCALAR && line == 0) a = reinterpret_cast<const char *>(gp + th);
        }
      }
      if (a) prefetch_l2(a);
    }
  };
  // the thread's R x 4 tile of a row-major state with row stride ld (16-byte aligned rows)
  auto store_state = [&](float *dst, int ld, const float (&S)[R][4]) {
#pragma unroll
    for (int r = 0; r < R; ++r)
      *reinterpret_cast<float4 *>(dst + (r0 + r) * ld + c0) = make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
  };
  auto load_state = [&](const float *src, int ld, float (&S)[R][4]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 v = src ? *reinterpret_cast<const float4 *>(src + (r0 + r) * ld + c0) : make_float4(0, 0, 0, 0);
      S[r][0] = v.x, S[r][1] = v.y, S[r][2] = v.z, S[r][3] = v.w;
    }
  };
  auto warp_sum = [](float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
  };
  // one forward step on staged token i: S <- D S + a (w - (D S)^T b)^T
  auto forward_step = [&](float (&S)[R][4], int i) {
    float al[R], bb[R], aa[R];
    lds_vec<R>(f_al + i * DK + r0, al);
    lds_vec<R>(f_b + i * DK + r0, bb);
    lds_vec<R>(f_a + i * DK + r0, aa);
    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        S[r][c] *= al[r];
        x[c] = fmaf(S[r][c], bb[r], x[c]);
      }
    butterfly_sum<4, 16, 8>(x, lane);  // column c0 + 2 b4 + b3, over the warp's rows
    s_red[0][warp][c0 + 2 * b4 + b3] = x[0];
    __syncthreads();
    if (tid < DV) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) acc += s_red[0][w][tid];
      s_u[tid] = c_w[i * DV + tid] - acc;
    }
    __syncthreads();
    float u[4];
    lds_vec<4>(s_u + c0, u);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) S[r][c] = fmaf(aa[r], u[c], S[r][c]);
  };

  float S[R][4];
  const size_t sbase = bh * static_cast<size_t>(DK) * DVF + v0;  // this slice of the full-width state
  // ---- pass 1: the forward, keeping the state before every CK-th token
  load_state(p.S0 ? p.S0 + sbase : nullptr, DVF, S);
  for (int c = 0; c < nck; ++c) {
    const int t0 = c * CK, L = min(CK, T - t0);
    store_state(ck + static_cast<size_t>(c) * DK * DV, DV, S);
    __syncthreads();  // the previous span's stage is no longer read
    load_span(t0, L, false);
    prefetch_span(t0 + CK, min(CK, T - t0 - CK), false);
    __syncthreads();
    for (int i = 0; i < L; ++i) forward_step(S, i);
  }
  if (nck > 0) prefetch_span((nck - 1) * CK, T - (nck - 1) * CK, true);

  // ---- pass 2: spans of CK tokens from the last, each recomputed then walked backwards
  float G[R][4];
  load_state(p.dS_T ? p.dS_T + sbase : nullptr, DVF, G);
  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * CK, L = min(CK, T - t0);
    load_state(ck + static_cast<size_t>(c) * DK * DV, DV, S);
    __syncthreads();
    load_span(t0, L, true);
    if (c > 0) prefetch_span(t0 - CK, CK, true);
    __syncthreads();
    for (int i = 0; i + 1 < L; ++i) {
      store_state(scr + static_cast<size_t>(i) * DK * DV, DV, S);  // state before token t0 + i
      forward_step(S, i);
    }
    // S now holds the state before token t0 + L - 1
    for (int i = L - 1; i >= 0; --i) {
      const size_t th = tok(t0 + i);
      float Sn[R][4];  // the state before token i - 1, loaded one step ahead
      if (i > 0) load_state(scr + static_cast<size_t>(i - 1) * DK * DV, DV, Sn);
      float al[R], bb[R], aa[R], qq[R], dO[4];
      lds_vec<R>(f_al + i * DK + r0, al);
      lds_vec<R>(f_b + i * DK + r0, bb);
      lds_vec<R>(f_a + i * DK + r0, aa);
      lds_vec<R>(f_q + i * DK + r0, qq);
      lds_vec<4>(c_do + i * DV + c0, dO);
      // G += q do^T; partial column sums of X^T b = S^T (D b) (values 0-3) and du = G^T a (4-7)
      float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float ab = al[r] * bb[r];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          G[r][c] = fmaf(qq[r], dO[c], G[r][c]);
          x[c] = fmaf(S[r][c], ab, x[c]);
          x[4 + c] = fmaf(G[r][c], aa[r], x[4 + c]);
        }
      }
      butterfly_sum<8, 16, 8>(x, lane);  // sum b4 (0: X^T b, 1: du) of columns c0 + 2 b3 + k
      s_red[b4][warp][c0 + 2 * b3] = x[0];
      s_red[b4][warp][c0 + 2 * b3 + 1] = x[1];
      __syncthreads();
      if (tid < 2 * DV) {
        const int j = tid & (DV - 1), which = tid >> 5;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) acc += s_red[which][w][j];
        if (which == 0) s_u[j] = c_w[i * DV + j] - acc;  // u = w - X^T b
        else s_du[j] = acc;
      }
      __syncthreads();
      float u[4], du[4];
      lds_vec<4>(s_u + c0, u);
      lds_vec<4>(s_du + c0, du);
      float udo = 0.f;  // u . do over the slice
#pragma unroll
      for (int c = 0; c < 4; ++c) udo = fmaf(u[c], dO[c], udo);
      udo += __shfl_xor_sync(0xffffffffu, udo, 1);
      udo += __shfl_xor_sync(0xffffffffu, udo, 2);
      udo += __shfl_xor_sync(0xffffffffu, udo, 4);
      // per-row sums over the tile's columns: S do, G u, S du, G . S; then G <- D (G - b du^T)
      float y[NQ];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float sdo = 0.f, gu = 0.f, sdu = 0.f, gs = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sdo = fmaf(S[r][c], dO[c], sdo);
          gu = fmaf(G[r][c], u[c], gu);
          sdu = fmaf(S[r][c], du[c], sdu);
          gs = fmaf(G[r][c], S[r][c], gs);
          G[r][c] = al[r] * fmaf(-bb[r], du[c], G[r][c]);
        }
        y[4 * r] = sdo, y[4 * r + 1] = gu, y[4 * r + 2] = sdu, y[4 * r + 3] = gs;
      }
      butterfly_sum<NQ, 4, 1>(y, lane);  // values (NQ/8) cg + k, summed over the row's 8 lanes
#pragma unroll
      for (int k = 0; k < NQ / 8; ++k) s_rows[warp][rg][(NQ / 8) * cg + k] = y[k];
      __syncwarp();
      float dal = 0.f, dbeta = 0.f;
      if (cg < R) {  // lane (rg, cg) finishes row r0 + cg
        const int row = r0 + cg, e = i * DK + row;
        float z[4];
        lds_vec<4>(&s_rows[warp][rg][4 * cg], z);
        const float sdo = z[0], gu = z[1], sdu = z[2];
        const float alr = f_al[e], br = f_b[e], sb = f_sb[e], sc = f_sc[e];
        dal = z[3] - br * sdu;                    // sum_j (G - b du^T)_j S_j
        const float dbt = -alr * sdu + sc * gu;   // through b, directly and through a = s (.) b
        dbeta = sb > 0.f ? 0.5f * f_k[e] * dbt / sb : 0.f;  // d sqrt(beta) / d beta
        atomicAdd(&p.dq[th * DK + row], alr * sdo + f_a[e] * udo);
        atomicAdd(&p.dk[th * DK + row], sb * dbt);
        if (p.ds) atomicAdd(&p.ds[th * DK + row], br * gu);
        if (p.beta_k_mode == MODE_CHANNEL) atomicAdd(&p.dbeta_k[th * DK + row], dbeta);
        if (p.alpha_mode == MODE_CHANNEL) atomicAdd(&p.dalpha[th * DK + row], dal);
      }
      __syncwarp();  // s_rows is rewritten next step
      // scalar gates: sums over the channels, one atomic per warp
      if (p.alpha_mode == MODE_SCALAR) {
        dal = warp_sum(dal);
        if (lane == 0) atomicAdd(&p.dalpha[th], dal);
      }
      if (p.beta_k_mode == MODE_SCALAR || warp == 0) {
        // warp 0 also owns the per-column terms of the slice (lane = column)
        float extra = 0.f;
        if (warp == 0) {
          const int jg = v0 + lane;
          const float duj = s_du[lane], wsc = c_wsc[i * DV + lane];
          const float pv = c_v[i * DV + lane] * duj;
          p.dv[th * DVF + jg] = wsc * duj;
          if (!sym && p.beta_v_mode == MODE_CHANNEL) p.dbeta_v[th * DVF + jg] = pv;
          // symmetric channel write w = sqrt(beta_k) (.) v (dk == dv): column jg is key channel jg
          if (sym && p.beta_k_mode == MODE_CHANNEL && wsc > 0.f)
            atomicAdd(&p.dbeta_k[th * DK + jg], 0.5f * pv / wsc);
          if (!sym && p.beta_v_mode == MODE_SCALAR) {
            const float svv = warp_sum(pv);
            if (lane == 0) atomicAdd(&p.dbeta_v[th], svv);
          }
          if (sym && p.beta_k_mode == MODE_SCALAR && wsc > 0.f) extra = 0.5f * pv / wsc;  // through w
        }
        if (p.beta_k_mode == MODE_SCALAR) {
          const float sbk = warp_sum(dbeta + extra);
          if (lane == 0) atomicAdd(&p.dbeta_k[th], sbk);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) S[r][c] = Sn[r][c];
    }
  }
  if (p.dS0) store_state(p.dS0 + sbase, DVF, G);
}

}  // namespace dr
