// umma_selftest.cuh -- diagnostic: one 128 x N x K bf16 or fp16 product through the exact
// tcgen05 building blocks the prefill kernel uses (128-byte swizzled shared
// tiles written by threads, K-major and MN-major smem descriptors, the kind::f16
// instruction descriptor, commit to an mbarrier, TMEM allocation and the
// 32x32b TMEM load).  The tests compare it with a host matmul so that a layout
// or descriptor mistake shows up in isolation.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "tri_inverse.cuh"

namespace dr {

// A, Bm: 16-bit elements, bf16 (bf16 != 0) or fp16.
template <int N, int K>
__global__ void __launch_bounds__(128)
umma_selftest_kernel(const uint16_t *__restrict__ A, const uint16_t *__restrict__ Bm,
                     float *__restrict__ D, int a_mn, int b_mn, int bf16, uint32_t *status) {
  constexpr int M = 128;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *sA = base;
  uint8_t *sB = base + M * K * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int e = tid; e < M * K; e += blockDim.x) {
    const int m = e / K, kk = e % K;
    const uint32_t off = a_mn ? sw128_off(kk, m, K) : sw128_off(m, kk, M);
    *reinterpret_cast<uint16_t *>(sA + off) = A[e];
  }
  for (int e = tid; e < K * N; e += blockDim.x) {
    const int kk = e / N, n = e % N;
    const uint32_t off = b_mn ? sw128_off(kk, n, K) : sw128_off(n, kk, N);
    *reinterpret_cast<uint16_t *>(sB + off) = Bm[e];
  }
  fence_async_smem();
  if (warp == 0) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base;
  if (tid == 0) {
    const uint32_t idesc = idesc_f16_f32(M, N, a_mn != 0, b_mn != 0, bf16 != 0);
#pragma unroll
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t ad = a_mn ? desc_mnmajor(smem_u32(sA), K, kk) : desc_kmajor(smem_u32(sA), M, kk);
      const uint64_t bd = b_mn ? desc_mnmajor(smem_u32(sB), K, kk) : desc_kmajor(smem_u32(sB), N, kk);
      umma_f16(tb, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    umma_commit(&bar);
  }
  const bool ok = mbar_wait(&bar, 0, kWaitLimitNs);
  tc_fence_after();
  if (!ok) {
    if (lane == 0) raise_status(status, STATUS_TIMEOUT);
  } else {
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 16) {
      float vals[16];
      tmem_ld16(tmem_addr(tb, 32 * warp, c0), vals);
      tmem_ld_wait();
      const int row = 32 * warp + lane;
#pragma unroll
      for (int i = 0; i < 16; ++i) D[row * N + c0 + i] = vals[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 128);
}

// T = (I + A)^-1 for the strictly lower part of a 64 x 64 fp32 matrix A (row-major),
// through the same warp-MMA routine the prefill kernel uses.  T (row-major fp32)
// must be zeroed by the caller: only its lower blocks are written.  128 threads.
// T = (I + A)^-1 of a 64 x 64 A by one of the prefill kernels' routines, for tests.
//   variant 0: the ring prefill's (inverse64_rows on the swizzled 128-byte-row tile layout);
//   variant 1: the one-CTA prefill's (inverse64 on padded row-major arrays).
// 128 threads; dynamic shared memory kTriSelftestSmem.
constexpr size_t kTriSelftestSmem =
    1024 + (3 * 64 * tri::LD * 2 > 128 * 128 ? 3 * 64 * tri::LD * 2 : 128 * 128);  // the larger variant
__global__ void __launch_bounds__(128) tri_selftest_kernel(int variant, const float *__restrict__ A,
                                                           float *__restrict__ Tout) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto put = [&](int bi, int bj, const tri::Frag &F, int ln) {
    const int row = 16 * bi + (ln >> 2), col = 16 * bj + 2 * (ln & 3);
    Tout[row * 64 + col] = F.v[0];
    Tout[row * 64 + col + 1] = F.v[1];
    Tout[(row + 8) * 64 + col] = F.v[2];
    Tout[(row + 8) * 64 + col + 1] = F.v[3];
    Tout[row * 64 + col + 8] = F.v[4];
    Tout[row * 64 + col + 9] = F.v[5];
    Tout[(row + 8) * 64 + col + 8] = F.v[6];
    Tout[(row + 8) * 64 + col + 9] = F.v[7];
  };
  if (variant == 1) {
    __half *Ah = reinterpret_cast<__half *>(sm), *AhT = Ah + 64 * tri::LD, *ThT = AhT + 64 * tri::LD;
    for (int e = tid; e < 64 * 64; e += blockDim.x) {
      const int r = e / 64, c = e % 64;
      const __half a = __float2half_rn(c < r ? A[e] : 0.f);
      Ah[r * tri::LD + c] = a;
      AhT[c * tri::LD + r] = a;
    }
    __syncthreads();
    tri::inverse64(Ah, AhT, ThT, warp, lane, put, [] { __syncthreads(); });
    return;
  }
  uint8_t *TP = sm;  // rows 0..63: A; rows 64..127: T^T scratch (one 128-row tile of 128-byte rows)
  for (int e = tid; e < 64 * 64; e += blockDim.x) {
    const int r = e / 64, c = e % 64;
    *reinterpret_cast<__half *>(TP + tri::Sw128Layout::off(r, c)) = __float2half_rn(c < r ? A[e] : 0.f);
  }
  __syncthreads();
  tri::Frag Trow[4];
  tri::inverse64_rows<tri::Sw128Layout>(TP, TP + 64 * 128, warp, lane, Trow, [] { __syncthreads(); });
#pragma unroll
  for (int d = 0; d < 4; ++d)
    if (d <= warp) put(warp, warp - d, Trow[d], lane);
}

}  // namespace dr
