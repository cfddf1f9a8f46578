// tri_inverse.cuh -- T = (I + A)^-1 for a strictly lower-triangular 64 x 64 A
// (the UT transform of the chunkwise WY form), on warp-level tensor-core MMAs.
//
// The 64 x 64 matrix is split into 4 x 4 blocks of 16 x 16.  Every block
// product is two m16n8k16 MMAs (fp16 operands, fp32 accumulation), issued by
// one warp on register fragments, which suits these tiny dependent products
// far better than a round trip through tensor memory.
//
//  * Diagonal blocks (one warp each): for N = A_bb strictly lower (N^16 = 0),
//    (I + N)^-1 = (I - N)(I + N^2)(I + N^4)(I + N^8).
//  * Off-diagonal blocks, by distance d = i - j = 1, 2, 3 (warp i computes
//    block (i, j)):  T_ij = -T_ii * sum_{m=j}^{i-1} A_im T_mj.
//
// Fragment trick: a 16 x 16 matrix X is held as its accumulator fragment
// F(X) (8 floats per lane).  F(X) repacks directly into the A operand of an
// MMA; the B operand for "times Y" is the repacked F(Y^T).  Every matrix is
// therefore carried together with its transpose, and every product X Y is
// computed with its transpose Y^T X^T, so no lane shuffles are needed.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

namespace dr {
namespace tri {

constexpr int LD = 72;  // row stride (halves) of the padded 64 x 64 fp16 arrays: conflict-free fragment loads

struct Frag {
  float v[8];  // X[r][2q], X[r][2q+1], X[r+8][2q], X[r+8][2q+1], X[r][2q+8], X[r][2q+9], X[r+8][2q+8], X[r+8][2q+9]
};

__device__ __forceinline__ uint32_t h2u(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += X * Y, where Zt = F(Y^T).
__device__ __forceinline__ void mul_acc(Frag &D, const Frag &X, const Frag &Zt) {
  const uint32_t a[4] = {h2u(X.v[0], X.v[1]), h2u(X.v[2], X.v[3]), h2u(X.v[4], X.v[5]), h2u(X.v[6], X.v[7])};
  float dl[4] = {D.v[0], D.v[1], D.v[2], D.v[3]};
  float dr[4] = {D.v[4], D.v[5], D.v[6], D.v[7]};
  mma16816(dl, a, h2u(Zt.v[0], Zt.v[1]), h2u(Zt.v[4], Zt.v[5]));  // output columns 0..7
  mma16816(dr, a, h2u(Zt.v[2], Zt.v[3]), h2u(Zt.v[6], Zt.v[7]));  // output columns 8..15
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    D.v[i] = dl[i];
    D.v[4 + i] = dr[i];
  }
}
__device__ __forceinline__ Frag mul(const Frag &X, const Frag &Zt) {
  Frag D;
#pragma unroll
  for (int i = 0; i < 8; ++i) D.v[i] = 0.f;
  mul_acc(D, X, Zt);
  return D;
}
// I + s X (s = +1 or -1)
__device__ __forceinline__ Frag eye_plus(const Frag &X, float s, int lane) {
  const int r = lane >> 2, q = lane & 3;
  Frag D;
#pragma unroll
  for (int i = 0; i < 8; ++i) D.v[i] = s * X.v[i];
  D.v[0] += (r == 2 * q) ? 1.f : 0.f;
  D.v[1] += (r == 2 * q + 1) ? 1.f : 0.f;
  D.v[6] += (r == 2 * q) ? 1.f : 0.f;
  D.v[7] += (r == 2 * q + 1) ? 1.f : 0.f;
  return D;
}
__device__ __forceinline__ void negate(Frag &X) {
#pragma unroll
  for (int i = 0; i < 8; ++i) X.v[i] = -X.v[i];
}

// Block (bi, bj) of a row-major fp16 64 x 64 array with row stride LD.
__device__ __forceinline__ Frag load_frag(const __half *M, int bi, int bj, int lane) {
  const int r = lane >> 2, q = lane & 3;
  const __half *base = M + (16 * bi + r) * LD + 16 * bj + 2 * q;
  Frag F;
  const float2 x0 = __half22float2(*reinterpret_cast<const __half2 *>(base));
  const float2 x1 = __half22float2(*reinterpret_cast<const __half2 *>(base + 8 * LD));
  const float2 x2 = __half22float2(*reinterpret_cast<const __half2 *>(base + 8));
  const float2 x3 = __half22float2(*reinterpret_cast<const __half2 *>(base + 8 * LD + 8));
  F.v[0] = x0.x;
  F.v[1] = x0.y;
  F.v[2] = x1.x;
  F.v[3] = x1.y;
  F.v[4] = x2.x;
  F.v[5] = x2.y;
  F.v[6] = x3.x;
  F.v[7] = x3.y;
  return F;
}
__device__ __forceinline__ void store_frag(__half *M, int bi, int bj, const Frag &F, int lane) {
  const int r = lane >> 2, q = lane & 3;
  __half *base = M + (16 * bi + r) * LD + 16 * bj + 2 * q;
  *reinterpret_cast<uint32_t *>(base) = h2u(F.v[0], F.v[1]);
  *reinterpret_cast<uint32_t *>(base + 8 * LD) = h2u(F.v[2], F.v[3]);
  *reinterpret_cast<uint32_t *>(base + 8) = h2u(F.v[4], F.v[5]);
  *reinterpret_cast<uint32_t *>(base + 8 * LD + 8) = h2u(F.v[6], F.v[7]);
}

// Block (bi, bj) of the transpose of a row-major fp16 array: F(X^T) for X = M[bi][bj].
__device__ __forceinline__ Frag load_frag_t(const __half *M, int bi, int bj, int lane) {
  const int r = lane >> 2, q = lane & 3;
  const __half *base = M + (16 * bi + 2 * q) * LD + 16 * bj + r;
  Frag F;
  F.v[0] = __half2float(base[0]);
  F.v[1] = __half2float(base[LD]);
  F.v[2] = __half2float(base[8]);
  F.v[3] = __half2float(base[LD + 8]);
  F.v[4] = __half2float(base[8 * LD]);
  F.v[5] = __half2float(base[9 * LD]);
  F.v[6] = __half2float(base[8 * LD + 8]);
  F.v[7] = __half2float(base[9 * LD + 8]);
  return F;
}

// Called by every thread of the participating group (contains `sync()` barriers); warps 0..3 work.
// Ah: A (fp16, row stride LD, zero on and above A's diagonal); AhT: A^T, or nullptr to read
// the transposes from Ah.  ThT: scratch for T^T (fp16, row stride LD).
// put(bi, bj, F, lane): receives each lower block T_ij (i >= j) of the result.
template <typename Put, typename Sync>
__device__ __forceinline__ void inverse64(const __half *Ah, const __half *AhT, __half *ThT, int warp, int lane,
                                          Put put, Sync sync) {
  Frag Tii;  // diagonal block of this warp, kept for the off-diagonal levels
  if (warp < 4) {
    const int b = warp;
    const Frag N = load_frag(Ah, b, b, lane);
    const Frag Nt = AhT ? load_frag(AhT, b, b, lane) : load_frag_t(Ah, b, b, lane);
    const Frag N2 = mul(N, Nt), N2t = mul(Nt, N);
    const Frag N4 = mul(N2, N2t), N4t = mul(N2t, N2);
    const Frag N8t = mul(N4t, N4);
    const Frag X1 = eye_plus(N, -1.f, lane);
    const Frag Y1t = eye_plus(N2t, 1.f, lane);
    const Frag P1 = mul(X1, Y1t);
    const Frag Y2t = eye_plus(N4t, 1.f, lane);
    const Frag P2 = mul(P1, Y2t);
    const Frag Y3t = eye_plus(N8t, 1.f, lane);
    Tii = mul(P2, Y3t);
    const Frag Tt = mul(Y3t, P2);
    store_frag(ThT, b, b, Tt, lane);
    put(b, b, Tii, lane);
  }
  sync();
#pragma unroll 1
  for (int d = 1; d < 4; ++d) {
    if (warp >= d && warp < 4) {
      const int i = warp, j = warp - d;
      // Xt = X^T for X = sum_m A_im T_mj, accumulated as sum_m T_mj^T A_im^T
      Frag Xt;
#pragma unroll
      for (int e = 0; e < 8; ++e) Xt.v[e] = 0.f;
      for (int m = j; m < i; ++m) {
        const Frag Aim = load_frag(Ah, i, m, lane);
        const Frag Tmjt = load_frag(ThT, j, m, lane);  // (T_mj)^T
        mul_acc(Xt, Tmjt, Aim);
      }
      Frag Tij = mul(Tii, Xt);   // T_ii X
      Frag Tijt = mul(Xt, Tii);  // X^T T_ii^T
      negate(Tij);
      negate(Tijt);
      store_frag(ThT, j, i, Tijt, lane);
      put(i, j, Tij, lane);
    }
    sync();
  }
}

// ------------------------------------------------------------------ layout-generic variant
// Byte offset of element (r, c) of a 64 x 64 fp16 array.
struct Sw128Layout {  // 128-byte rows, 16-byte groups XOR-ed with (r & 7): a K-major MMA operand tile
  __device__ static uint32_t off(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + (c & 7) * 2);
  }
};
template <class Lay>
__device__ __forceinline__ Frag load_frag_l(const uint8_t *M, int bi, int bj, int lane) {
  const int r = 16 * bi + (lane >> 2), c = 16 * bj + 2 * (lane & 3);
  const float2 x0 = __half22float2(*reinterpret_cast<const __half2 *>(M + Lay::off(r, c)));
  const float2 x1 = __half22float2(*reinterpret_cast<const __half2 *>(M + Lay::off(r + 8, c)));
  const float2 x2 = __half22float2(*reinterpret_cast<const __half2 *>(M + Lay::off(r, c + 8)));
  const float2 x3 = __half22float2(*reinterpret_cast<const __half2 *>(M + Lay::off(r + 8, c + 8)));
  Frag F;
  F.v[0] = x0.x;
  F.v[1] = x0.y;
  F.v[2] = x1.x;
  F.v[3] = x1.y;
  F.v[4] = x2.x;
  F.v[5] = x2.y;
  F.v[6] = x3.x;
  F.v[7] = x3.y;
  return F;
}
template <class Lay>
__device__ __forceinline__ void store_frag_l(uint8_t *M, int bi, int bj, const Frag &F, int lane) {
  const int r = 16 * bi + (lane >> 2), c = 16 * bj + 2 * (lane & 3);
  *reinterpret_cast<uint32_t *>(M + Lay::off(r, c)) = h2u(F.v[0], F.v[1]);
  *reinterpret_cast<uint32_t *>(M + Lay::off(r + 8, c)) = h2u(F.v[2], F.v[3]);
  *reinterpret_cast<uint32_t *>(M + Lay::off(r, c + 8)) = h2u(F.v[4], F.v[5]);
  *reinterpret_cast<uint32_t *>(M + Lay::off(r + 8, c + 8)) = h2u(F.v[6], F.v[7]);
}
// F(X^T) for X = block (bi, bj)
template <class Lay>
__device__ __forceinline__ Frag load_frag_t_l(const uint8_t *M, int bi, int bj, int lane) {
  const int r0 = 16 * bi + 2 * (lane & 3), c0 = 16 * bj + (lane >> 2);
  auto at = [&](int r, int c) { return __half2float(*reinterpret_cast<const __half *>(M + Lay::off(r, c))); };
  Frag F;
  F.v[0] = at(r0, c0);
  F.v[1] = at(r0 + 1, c0);
  F.v[2] = at(r0, c0 + 8);
  F.v[3] = at(r0 + 1, c0 + 8);
  F.v[4] = at(r0 + 8, c0);
  F.v[5] = at(r0 + 9, c0);
  F.v[6] = at(r0 + 8, c0 + 8);
  F.v[7] = at(r0 + 9, c0 + 8);
  return F;
}

// inverse64 on arrays in layout Lay, keeping the result in registers: warp i < 4 ends with
// Trow[d] = T_{i, i-d} for d = 0..i.  Nothing is written to Ah, so the caller may overwrite it
// with T after the last `sync()`.  ThT (T^T scratch) must not overlap Ah.
template <class Lay, typename Sync>
__device__ __forceinline__ void inverse64_rows(const uint8_t *Ah, uint8_t *ThT, int warp, int lane, Frag (&Trow)[4],
                                               Sync sync) {
  if (warp < 4) {
    const int b = warp;
#pragma unroll
    for (int e = 0; e < 8; ++e) Trow[1].v[e] = Trow[2].v[e] = Trow[3].v[e] = 0.f;
    // (I + N)^-1 = (I - N)(I + N^2)(I + N^4)(I + N^8): P <- P (I + M), M <- M^2, as a loop
    Frag M = load_frag_l<Lay>(Ah, b, b, lane);
    Frag Mt = load_frag_t_l<Lay>(Ah, b, b, lane);
    Frag P = eye_plus(M, -1.f, lane), Yt;
#pragma unroll 1
    for (int k = 0; k < 3; ++k) {
      const Frag M2 = mul(M, Mt);
      Mt = mul(Mt, M);
      M = M2;
      Yt = eye_plus(Mt, 1.f, lane);
      if (k < 2) P = mul(P, Yt);
    }
    Trow[0] = mul(P, Yt);
    store_frag_l<Lay>(ThT, b, b, mul(Yt, P), lane);
  }
  sync();
  // one copy of the level code: the result goes to Trow[d] through a select, not an indexed store
#pragma unroll 1
  for (int d = 1; d < 4; ++d) {
    if (warp >= d && warp < 4) {
      const int i = warp, j = warp - d;
      Frag Xt;  // X^T for X = sum_m A_im T_mj
#pragma unroll
      for (int e = 0; e < 8; ++e) Xt.v[e] = 0.f;
#pragma unroll 1
      for (int m = j; m < i; ++m) mul_acc(Xt, load_frag_l<Lay>(ThT, j, m, lane), load_frag_l<Lay>(Ah, i, m, lane));
      Frag Tij = mul(Trow[0], Xt);
      Frag Tijt = mul(Xt, Trow[0]);
      negate(Tij);
      negate(Tijt);
      store_frag_l<Lay>(ThT, j, i, Tijt, lane);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        Trow[1].v[e] = (d == 1) ? Tij.v[e] : Trow[1].v[e];
        Trow[2].v[e] = (d == 2) ? Tij.v[e] : Trow[2].v[e];
        Trow[3].v[e] = (d == 3) ? Tij.v[e] : Trow[3].v[e];
      }
    }
    sync();
  }
}

}  // namespace tri
}  // namespace dr
