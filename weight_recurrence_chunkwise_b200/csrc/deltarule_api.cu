// deltarule_api.cu -- the C ABI declared in include/deltarule.h: argument
// checks, workspace status word, and dispatch to the sm_100a kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/deltarule.h"
#include "../../include/deltarule_diag.h"
#include "chunk_simt.cuh"
#include "chunk_tc.cuh"
#include "chunk_tc3.cuh"
#include "chunk_tc4.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "decode_stream.cuh"
#include "state_map.cuh"
#include "backward.cuh"
#include "backward_chunk.cuh"
#include "umma_selftest.cuh"
#include "wait_selftest.cuh"

namespace {

constexpr size_t kWorkspaceBytes = 256;  // status word, padded to an allocation granule

// Prefill kernel variants (the library's choice is kDefault; the others are reachable only through
// dr_diag_chunk_fwd_variant, for comparisons).
enum PrefillVariant { kPrefillDefault = 0, kPrefillSingle = 1, kPrefillSimt = 2, kPrefillRing = 3, kPrefillQuad = 4 };
// Decode kernel variants, likewise (dr_diag_decode_step_variant).
enum DecodeVariant { kDecodeDefault = 0, kDecodePerHead = 1, kDecodeSplit4 = 2, kDecodeStream = 3 };

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dr_status check_common(const dr_problem *p, bool decode) {
  if (!p) return DR_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->T < 0 || p->dk <= 0 || p->dv <= 0) return DR_ERR_INVALID_ARG;
  if (decode && p->T != 1) return DR_ERR_INVALID_ARG;
  if (!decode && p->chunk <= 0) return DR_ERR_INVALID_ARG;
  if (p->io_dtype != DR_F32 && p->io_dtype != DR_BF16) return DR_ERR_INVALID_ARG;
  if (p->alpha_mode < DR_ABSENT || p->alpha_mode > DR_CHANNEL) return DR_ERR_INVALID_ARG;
  if (p->beta_k_mode != DR_SCALAR && p->beta_k_mode != DR_CHANNEL) return DR_ERR_INVALID_ARG;
  if (p->beta_v_mode < DR_ABSENT || p->beta_v_mode > DR_CHANNEL) return DR_ERR_INVALID_ARG;
  // sqrt(beta) (.) v with beta in R^{dk} only type-checks when dk == dv
  if (p->beta_v_mode == DR_ABSENT && p->beta_k_mode == DR_CHANNEL && p->dk != p->dv) return DR_ERR_INVALID_ARG;
  if ((p->dk != 64 && p->dk != 128) || (p->dv != 64 && p->dv != 128)) return DR_ERR_UNSUPPORTED;
  if (!decode && p->chunk != 16 && p->chunk != 32 && p->chunk != 64) return DR_ERR_UNSUPPORTED;
  if (!decode && (p->B > 65535 || p->H > 65535)) return DR_ERR_UNSUPPORTED;  // launch grid y and z
  const double elems = double(p->B) * p->T * p->H * (p->dk > p->dv ? p->dk : p->dv);
  if (elems > 9.0e15) return DR_ERR_INVALID_ARG;
  return DR_OK;
}

dr_status check_pointers(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                         const float *beta_k, const float *beta_v, const void *o) {
  const bool need_tokens = p->T > 0;
  if (need_tokens && (!q || !k || !v || !o || !beta_k)) return DR_ERR_INVALID_ARG;
  if (need_tokens && ((alpha == nullptr) != (p->alpha_mode == DR_ABSENT))) return DR_ERR_INVALID_ARG;
  if (need_tokens && ((beta_v == nullptr) != (p->beta_v_mode == DR_ABSENT))) return DR_ERR_INVALID_ARG;
  const void *ptrs[] = {q, k, v, alpha, beta_k, beta_v, o};
  for (const void *x : ptrs)
    if (x && !aligned16(x)) return DR_ERR_ALIGNMENT;
  return DR_OK;
}

dr_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

// ----------------------------------------------------------------- prefill, CUDA-core path
template <typename IO, int DK, int DV, int C>
dr_status simt_launch(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                      const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                      const float *S0, void *o, float *S_T, uint32_t *status, cudaStream_t st) {
  constexpr int VS = 32;
  auto kern = dr::chunk_fwd_simt_kernel<IO, DK, DV, VS, C>;
  constexpr size_t smem = dr::SimtSmem<DK, VS, C>::bytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return DR_ERR_CUDA;
  dim3 grid(DV / VS, p->H, p->B);
  kern<<<grid, 256, smem, st>>>(p->T, p->H, static_cast<const IO *>(q), static_cast<const IO *>(k),
                                static_cast<const IO *>(v), alpha, p->alpha_mode, beta_k, p->beta_k_mode,
                                beta_v, p->beta_v_mode, s_scale, cu, S0, static_cast<IO *>(o), S_T, status);
  return launch_status();
}

template <typename IO, int DK, int DV>
dr_status simt_by_chunk(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                        const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                        const float *S0, void *o, float *S_T, uint32_t *status, cudaStream_t st) {
  switch (p->chunk) {
    case 16:
      return simt_launch<IO, DK, DV, 16>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
    case 32:
      return simt_launch<IO, DK, DV, 32>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
    default:
      return simt_launch<IO, DK, DV, 64>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  }
}

template <typename IO>
dr_status simt_dispatch(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                        const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                        const float *S0, void *o, float *S_T, uint32_t *status, cudaStream_t st) {
  if (p->dk == 128 && p->dv == 128)
    return simt_by_chunk<IO, 128, 128>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  if (p->dk == 128 && p->dv == 64)
    return simt_by_chunk<IO, 128, 64>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  if (p->dk == 64 && p->dv == 128)
    return simt_by_chunk<IO, 64, 128>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  return simt_by_chunk<IO, 64, 64>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
}

// ----------------------------------------------------------------- prefill, tensor-core path (bf16 I/O)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 4-D map over a [B, T, H, D] row-major tensor (dims innermost first: D, H, T, B) with a box of
// `box_d` elements x 1 head x `box_t` tokens x 1 batch row; out-of-range rows read as zero.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, size_t esize, const void *base, int B, int T, int H, int D,
              int box_d, int box_t, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(D) * esize, cuuint64_t(D) * H * esize, cuuint64_t(D) * H * T * esize};
  const cuuint32_t box[4] = {cuuint32_t(box_d), 1u, cuuint32_t(box_t), 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return enc(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

dr_status tc_launch(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                    const float *beta_k, const float *beta_v, const float *S0, void *o, float *S_T,
                    uint32_t *status, cudaStream_t st) {
  using IO = __nv_bfloat16;
  namespace tc = dr::tc;
  alignas(64) CUtensorMap mq, mk, mv, mbv;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&mq, bf, 2, q, p->B, p->T, p->H, p->dk, tc::DK, tc::C) ||
      !make_map(&mk, bf, 2, k, p->B, p->T, p->H, p->dk, tc::DK, tc::C) ||
      !make_map(&mv, bf, 2, v, p->B, p->T, p->H, p->dv, tc::VS, tc::C))
    return DR_ERR_CUDA;
  if (p->beta_v_mode == DR_CHANNEL) {
    if (!make_map(&mbv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, beta_v, p->B, p->T, p->H, p->dv, tc::VS, tc::C))
      return DR_ERR_CUDA;
  } else {
    mbv = mv;  // unused by the kernel in this mode
  }
  tc::Params prm{p->T, p->H, p->dv, alpha, p->alpha_mode, beta_k, p->beta_k_mode, beta_v, p->beta_v_mode,
                 S0, o, S_T, status};
  auto kern = tc::chunk_fwd_tc_kernel<IO>;
  constexpr size_t smem = tc::SMEM_BYTES;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return DR_ERR_CUDA;
  dim3 grid(p->dv / tc::VS, p->H, p->B);
  kern<<<grid, tc::NT, smem, st>>>(mq, mk, mv, mbv, prm);
  return launch_status();
}

// states: NULL, or [B, H, ceil(T/64), dk, dv] fp32 receiving the state at the start of every chunk
// (dense batch only; the chunkwise backward's first pass, which passes o = NULL).
// Tensor maps of the cluster prefills: q, k and v in 64-column boxes of one chunk's rows; the
// channel-wise decays in 32-channel (128-byte) boxes (otherwise a copy of q's map, unused).
struct RingMaps {
  alignas(64) CUtensorMap q, k, v, a;
};
bool ring_maps(RingMaps &m, const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
               const float *alpha) {
  namespace tc = dr::tc;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  const int mB = cu ? 1 : p->B;  // a packed batch is one [1, Ttot, H, d] array
  if (!make_map(&m.q, bf, 2, q, mB, p->T, p->H, p->dk, 64, tc::C, sw) ||
      !make_map(&m.k, bf, 2, k, mB, p->T, p->H, p->dk, 64, tc::C, sw) ||
      !make_map(&m.v, bf, 2, v, mB, p->T, p->H, p->dv, tc::VS, tc::C, sw))
    return false;
  m.a = m.q;
  if (p->alpha_mode == DR_CHANNEL &&
      !make_map(&m.a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, alpha, mB, p->T, p->H, p->dk, 32, tc::C, sw))
    return false;
  return true;
}

dr_status tc_ring_launch(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                         const float *S0, void *o, float *S_T, uint32_t *status, cudaStream_t st,
                         float *states = nullptr) {
  using IO = __nv_bfloat16;
  namespace tc = dr::tc;
  namespace tc3 = dr::tc3;
  RingMaps m;
  if (!ring_maps(m, p, cu, q, k, v, alpha)) return DR_ERR_CUDA;
  tc::Params prm{p->T, p->H, p->dv, alpha, p->alpha_mode, beta_k, p->beta_k_mode, beta_v, p->beta_v_mode,
                 S0, o, S_T, status, s_scale, cu, states};
  const bool chan_gates = p->alpha_mode == DR_CHANNEL || p->beta_k_mode != DR_SCALAR;
  auto kern = s_scale ? (chan_gates ? tc3::chunk_fwd_ring_kernel<IO, true, true>
                                    : tc3::chunk_fwd_ring_kernel<IO, false, true>)
                      : (chan_gates ? tc3::chunk_fwd_ring_kernel<IO, true, false>
                                    : tc3::chunk_fwd_ring_kernel<IO, false, false>);
  constexpr size_t smem = tc3::SMEM_BYTES;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return DR_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, p->H, p->B);
  cfg.blockDim = dim3(tc3::NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, m.q, m.k, m.v, m.a, prm) != cudaSuccess) return DR_ERR_CUDA;
  return launch_status();
}

// The four-CTA prefill: one cluster of four CTAs per (b, h).
template <bool kChan, bool kScaled>
constexpr auto quad_kernel() {
  return dr::tc4::chunk_fwd_quad_kernel<__nv_bfloat16, kChan, kScaled>;
}
using QuadKernel = decltype(quad_kernel<false, false>());
QuadKernel pick_quad(bool chan, bool scaled) {
  return scaled ? (chan ? quad_kernel<true, true>() : quad_kernel<false, true>())
                : (chan ? quad_kernel<true, false>() : quad_kernel<false, false>());
}
cudaLaunchConfig_t quad_config(const dr_problem *p, cudaStream_t st, cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dr::tc4::NCTA, p->H, p->B);
  cfg.blockDim = dim3(dr::tc4::NT, 1, 1);
  cfg.dynamicSmemBytes = dr::tc4::SMEM_BYTES;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = dr::tc4::NCTA;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
// Clusters of the four-CTA prefill that the current device holds at once (0: unknown or none);
// computed once per device.
int quad_resident_clusters() {
  static std::mutex mu;
  static int cached[64];
  static bool known[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!known[dev]) {
    int n = 0;
    bool ok = true;
    for (int v = 0; v < 4 && ok; ++v) {
      ok = cudaFuncSetAttribute(pick_quad(v & 1, v & 2), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(dr::tc4::SMEM_BYTES)) == cudaSuccess;
    }
    if (ok) {
      dr_problem one{};
      one.B = 1;
      one.H = 1;
      cudaLaunchAttribute attr[1];
      cudaLaunchConfig_t cfg = quad_config(&one, nullptr, attr);
      if (cudaOccupancyMaxActiveClusters(&n, pick_quad(false, false), &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cached[dev] = n;
    known[dev] = true;
  }
  return cached[dev];
}
// Shapes the cluster prefills take: bf16 I/O, dk = dv = 128, chunk 64.
bool ring_problem(const dr_problem *p) {
  return p->io_dtype == DR_BF16 && p->dk == dr::tc::DK && p->chunk == dr::tc::C && p->dv == 2 * dr::tc::VS;
}
// The library's prefill choice for a problem the cluster kernels take: four CTAs per head when every
// head's cluster is resident at once (a second wave would double the time), else two.
bool quad_default(const dr_problem *p) {
  const long long heads = static_cast<long long>(p->B) * p->H;
  return heads <= quad_resident_clusters();
}
size_t quad_stage_bytes(const dr_problem *p) {
  return static_cast<size_t>(p->B) * p->H * dr::tc4::STAGE_BYTES_PER_HEAD;
}

// stage: quad_stage_bytes(p) bytes of device memory, 16-byte aligned.
dr_status tc_quad_launch(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                         const float *S0, void *o, float *S_T, uint32_t *status, uint8_t *stage, cudaStream_t st,
                         float *states = nullptr) {
  namespace tc = dr::tc;
  RingMaps m;
  if (!ring_maps(m, p, cu, q, k, v, alpha)) return DR_ERR_CUDA;
  tc::Params prm{p->T, p->H, p->dv, alpha, p->alpha_mode, beta_k, p->beta_k_mode, beta_v, p->beta_v_mode,
                 S0, o, S_T, status, s_scale, cu, states};
  const bool chan_gates = p->alpha_mode == DR_CHANNEL || p->beta_k_mode != DR_SCALAR;
  auto kern = pick_quad(chan_gates, s_scale != nullptr);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dr::tc4::SMEM_BYTES)) != cudaSuccess)
    return DR_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = quad_config(p, st, attr);
  if (cudaLaunchKernelEx(&cfg, kern, m.q, m.k, m.v, m.a, prm, stage) != cudaSuccess) return DR_ERR_CUDA;
  return launch_status();
}

// ----------------------------------------------------------------- decode
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <typename IO, int DK, int DV>
dr_status decode_launch(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                        const float *beta_k, const float *beta_v, const float *s_scale, float *S, void *o,
                        int variant, cudaStream_t st) {
  const long long heads = static_cast<long long>(p->B) * p->H;
  if (heads > 0x7fffffffLL) return DR_ERR_INVALID_ARG;
  // dk = dv = 128: four CTAs per head (32 value columns each) when there are no more heads than SMs,
  // else the persistent streaming kernel; other head sizes, one CTA per head
  if constexpr (DK == 128 && DV == 128) {
    const int sms = sm_count();
    if (variant == kDecodeDefault) variant = sms <= 0 ? kDecodePerHead : (heads <= sms ? kDecodeSplit4 : kDecodeStream);
    if (variant == kDecodeSplit4) {
      if (heads * 4 > 0x7fffffffLL) return DR_ERR_UNSUPPORTED;
      dr::decode_step_kernel<IO, DK, DV, 4><<<static_cast<unsigned>(heads * 4), 256, 0, st>>>(
          static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v), alpha, p->alpha_mode,
          beta_k, p->beta_k_mode, beta_v, p->beta_v_mode, s_scale, S, static_cast<IO *>(o));
      return launch_status();
    }
    if (variant == kDecodeStream) {
      if (sms <= 0) return DR_ERR_CUDA;
      auto kern = dr::decode_stream_kernel<IO>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(dr::kDecodeStreamSmem)) != cudaSuccess)
        return DR_ERR_CUDA;
      const long long grid = heads < 2LL * sms ? heads : 2LL * sms;  // two CTAs per SM
      kern<<<static_cast<unsigned>(grid), 256, dr::kDecodeStreamSmem, st>>>(
          static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v), alpha, p->alpha_mode,
          beta_k, p->beta_k_mode, beta_v, p->beta_v_mode, s_scale, S, static_cast<IO *>(o), heads);
      return launch_status();
    }
  } else {
    if (variant == kDecodeSplit4 || variant == kDecodeStream) return DR_ERR_UNSUPPORTED;
  }
  dr::decode_step_kernel<IO, DK, DV><<<static_cast<unsigned>(heads), 256, 0, st>>>(
      static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v), alpha, p->alpha_mode,
      beta_k, p->beta_k_mode, beta_v, p->beta_v_mode, s_scale, S, static_cast<IO *>(o));
  return launch_status();
}

template <typename IO>
dr_status decode_dispatch(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta_k, const float *beta_v, const float *s_scale, float *S, void *o,
                          int variant, cudaStream_t st) {
  if (p->dk == 128 && p->dv == 128)
    return decode_launch<IO, 128, 128>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
  if (p->dk == 128 && p->dv == 64)
    return decode_launch<IO, 128, 64>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
  if (p->dk == 64 && p->dv == 128)
    return decode_launch<IO, 64, 128>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
  return decode_launch<IO, 64, 64>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
}

// Prefill with an optional write-side key scale (NULL: a = b) and optional packed-sequence offsets
// (NULL: a dense [B, T, H, d] batch).
dr_status chunk_fwd_impl(const dr_problem *p, const int *cu, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta_k, const float *beta_v, const float *s_scale,
                         const float *S0, void *o, float *S_T, void *workspace, size_t workspace_bytes,
                         void *stream, int variant = kPrefillDefault) {
  dr_status s = check_common(p, false);
  if (s != DR_OK) return s;
  s = check_pointers(p, q, k, v, alpha, beta_k, beta_v, o);
  if (s != DR_OK) return s;
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)) || (s_scale && !aligned16(s_scale)))
    return DR_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < kWorkspaceBytes) return DR_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DR_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *status = static_cast<uint32_t *>(workspace);
  // a variant that cannot take the problem is refused before anything is enqueued
  const bool tc_shape = p->io_dtype == DR_BF16 && p->dk == dr::tc::DK && p->chunk == dr::tc::C;
  const bool ring_shape = ring_problem(p);
  const bool plain = !s_scale && !cu;  // the one-CTA-per-slice kernel takes neither extension
  if (variant == kPrefillSingle && !(plain && tc_shape && p->dv % dr::tc::VS == 0)) return DR_ERR_UNSUPPORTED;
  if ((variant == kPrefillRing || variant == kPrefillQuad) && !ring_shape) return DR_ERR_UNSUPPORTED;
  if (variant < kPrefillDefault || variant > kPrefillQuad) return DR_ERR_UNSUPPORTED;
  // The four-CTA kernel stages its factor blocks in the workspace, after the status word.  The
  // library's choice takes it only when the workspace holds that staging (dr_chunk_fwd_workspace
  // asks for it); a workspace with the status word alone runs the two-CTA kernel.
  const bool quad_fits = workspace_bytes >= kWorkspaceBytes + quad_stage_bytes(p);
  if (variant == kPrefillQuad && ring_shape && !quad_fits) return DR_ERR_WORKSPACE;
  const bool quad = ring_shape && (variant == kPrefillQuad || (variant == kPrefillDefault && quad_fits && quad_default(p)));
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DR_ERR_CUDA;
  const size_t state_bytes = sizeof(float) * size_t(p->B) * p->H * p->dk * p->dv;
  if (p->T == 0) {  // nothing to scan: the final state is the initial state
    if (!S_T) return DR_OK;
    const cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                          : cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, st))
                             : cudaMemsetAsync(S_T, 0, state_bytes, st);
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
  }
  if (p->io_dtype == DR_F32)
    return simt_dispatch<float>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  if (variant == kPrefillSimt)
    return simt_dispatch<__nv_bfloat16>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  if (quad)
    return tc_quad_launch(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status,
                          static_cast<uint8_t *>(workspace) + kWorkspaceBytes, st);
  if ((variant == kPrefillDefault || variant == kPrefillRing) && ring_shape)
    return tc_ring_launch(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
  if (plain && tc_shape && p->dv % dr::tc::VS == 0)
    return tc_launch(p, q, k, v, alpha, beta_k, beta_v, S0, o, S_T, status, st);
  return simt_dispatch<__nv_bfloat16>(p, cu, q, k, v, alpha, beta_k, beta_v, s_scale, S0, o, S_T, status, st);
}

dr_status decode_step_impl(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                           const float *beta_k, const float *beta_v, const float *s_scale, float *S, void *o,
                           void *stream, int variant = kDecodeDefault) {
  dr_status s = check_common(p, true);
  if (s != DR_OK) return s;
  s = check_pointers(p, q, k, v, alpha, beta_k, beta_v, o);
  if (s != DR_OK) return s;
  if (!S) return DR_ERR_INVALID_ARG;
  if (!aligned16(S) || (s_scale && !aligned16(s_scale))) return DR_ERR_ALIGNMENT;
  if (variant < kDecodeDefault || variant > kDecodeStream) return DR_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->io_dtype == DR_F32)
    return decode_dispatch<float>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
  return decode_dispatch<__nv_bfloat16>(p, q, k, v, alpha, beta_k, beta_v, s_scale, S, o, variant, st);
}

constexpr int kBwdSpan = 16;  // tokens between the backward pass's state checkpoints

size_t bwd_workspace_bytes(const dr_problem *p) {
  const size_t nck = (static_cast<size_t>(p->T) + kBwdSpan - 1) / kBwdSpan;
  return sizeof(float) * static_cast<size_t>(p->B) * p->H * (nck + kBwdSpan) * p->dk * p->dv;
}

template <typename IO, int DK, int DV>
dr_status bwd_launch(const dr::BwdParams &bp, int heads, cudaStream_t st) {
  auto kern = dr::delta_rule_bwd_kernel<IO, DK, DV, kBwdSpan>;
  constexpr int smem = dr::bwd_smem_bytes<DK, kBwdSpan>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DR_ERR_CUDA;
  kern<<<dim3(heads, DV / dr::kBwdCols), 256, smem, st>>>(bp);
  return launch_status();
}

template <typename IO>
dr_status bwd_dispatch(const dr_problem *p, const dr::BwdParams &bp, cudaStream_t st) {
  const int heads = p->B * p->H;
  if (p->dk == 128 && p->dv == 128) return bwd_launch<IO, 128, 128>(bp, heads, st);
  if (p->dk == 128 && p->dv == 64) return bwd_launch<IO, 128, 64>(bp, heads, st);
  if (p->dk == 64 && p->dv == 128) return bwd_launch<IO, 64, 128>(bp, heads, st);
  return bwd_launch<IO, 64, 64>(bp, heads, st);
}

// ----------------------------------------------------------------- backward, chunkwise on the tensor cores
// bf16 I/O, dk = dv = 128: a forward pass of the ring prefill keeps the state at the start of every
// chunk, then one CTA per (b, h) walks the chunks from the last (backward_chunk.cuh).
enum BackwardVariant { kBwdDefault = 0, kBwdSequential = 1, kBwdChunk = 2 };

bool bwd_chunk_shape(const dr_problem *p) { return p->io_dtype == DR_BF16 && p->dk == 128 && p->dv == 128; }

// The chunkwise backward's workspace: the status word, the chunk-start states, and (when its
// first pass runs on the four-CTA prefill) that kernel's factor staging.
size_t bwd_chunk_states_bytes(const dr_problem *p) {
  const size_t nc = (static_cast<size_t>(p->T) + dr::tc::C - 1) / dr::tc::C;
  return sizeof(float) * static_cast<size_t>(p->B) * p->H * nc * p->dk * p->dv;
}
bool bwd_first_pass_quad(const dr_problem *p) {
  dr_problem pf = *p;
  pf.chunk = dr::tc::C;
  return ring_problem(&pf) && quad_default(&pf);
}
size_t bwd_chunk_workspace_bytes(const dr_problem *p) {
  return kWorkspaceBytes + bwd_chunk_states_bytes(p) + (bwd_first_pass_quad(p) ? quad_stage_bytes(p) : 0);
}

int resolve_bwd_variant(const dr_problem *p, int variant) {
  if (variant == kBwdDefault) return bwd_chunk_shape(p) ? kBwdChunk : kBwdSequential;
  return variant;
}

size_t bwd_variant_workspace_bytes(const dr_problem *p, int variant) {
  return resolve_bwd_variant(p, variant) == kBwdChunk ? bwd_chunk_workspace_bytes(p) : bwd_workspace_bytes(p);
}

dr_status bwd_chunk_launch(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                           const float *beta_k, const float *beta_v, const float *s, const float *S0,
                           const void *dout, const float *dS_T, float *dq, float *dk, float *dv, float *dalpha,
                           float *dbeta_k, float *dbeta_v, float *ds, float *dS0, void *workspace,
                           size_t workspace_bytes, cudaStream_t st) {
  namespace bwc = dr::bwc;
  uint32_t *status = static_cast<uint32_t *>(workspace);
  uint8_t *ws8 = static_cast<uint8_t *>(workspace);
  float *states = reinterpret_cast<float *>(ws8 + kWorkspaceBytes);
  uint8_t *stage = ws8 + kWorkspaceBytes + bwd_chunk_states_bytes(p);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DR_ERR_CUDA;
  dr_problem pf = *p;
  pf.chunk = dr::tc::C;
  // first pass: the prefill with every chunk's initial state stored (no outputs), on the kernel the
  // forward would use when the workspace holds its staging
  const bool quad = bwd_first_pass_quad(p) &&
                    workspace_bytes >= kWorkspaceBytes + bwd_chunk_states_bytes(p) + quad_stage_bytes(p);
  dr_status r = quad ? tc_quad_launch(&pf, nullptr, q, k, v, alpha, beta_k, beta_v, s, S0, nullptr, nullptr, status,
                                      stage, st, states)
                     : tc_ring_launch(&pf, nullptr, q, k, v, alpha, beta_k, beta_v, s, S0, nullptr, nullptr, status,
                                      st, states);
  if (r != DR_OK) return r;
  alignas(64) CUtensorMap mq, mk, mv, mdo;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_map(&mq, bf, 2, q, p->B, p->T, p->H, p->dk, 64, dr::tc::C, sw) ||
      !make_map(&mk, bf, 2, k, p->B, p->T, p->H, p->dk, 64, dr::tc::C, sw) ||
      !make_map(&mv, bf, 2, v, p->B, p->T, p->H, p->dv, 64, dr::tc::C, sw) ||
      !make_map(&mdo, bf, 2, dout, p->B, p->T, p->H, p->dv, 64, dr::tc::C, sw))
    return DR_ERR_CUDA;
  const int nc = (p->T + dr::tc::C - 1) / dr::tc::C;
  alignas(64) CUtensorMap mst;  // the chunk-start states as rows of dv fp32: 32-column x 128-row boxes
  {
    auto enc = tensor_map_encoder();
    const cuuint64_t dims[2] = {cuuint64_t(p->dv), cuuint64_t(p->B) * p->H * nc * p->dk};
    const cuuint64_t strides[1] = {cuuint64_t(p->dv) * sizeof(float)};
    const cuuint32_t box[2] = {32u, 128u}, estr[2] = {1u, 1u};
    if (!enc || enc(&mst, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, states, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return DR_ERR_CUDA;
  }
  bwc::BwdChunkParams bp{p->T, p->H, nc, alpha, p->alpha_mode, beta_k, p->beta_k_mode, beta_v, p->beta_v_mode, s,
                         static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                         static_cast<const __nv_bfloat16 *>(v), states, dS_T, dq, dk, dv, dalpha, dbeta_k, dbeta_v,
                         ds, dS0, status};
  const bool chan = p->alpha_mode == DR_CHANNEL || p->beta_k_mode != DR_SCALAR;
  auto kern = s ? (chan ? bwc::chunk_bwd_kernel<true, true> : bwc::chunk_bwd_kernel<false, true>)
                : (chan ? bwc::chunk_bwd_kernel<true, false> : bwc::chunk_bwd_kernel<false, false>);
  constexpr size_t smem = bwc::SMEM_BYTES;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return DR_ERR_CUDA;
  kern<<<dim3(p->H, p->B), bwc::NT, smem, st>>>(mq, mk, mv, mdo, mst, bp);
  return launch_status();
}

}  // namespace

extern "C" {

size_t dr_backward_workspace(const dr_problem *p) {
  return check_common(p, false) == DR_OK ? bwd_variant_workspace_bytes(p, kBwdDefault) : 0;
}

static dr_status backward_impl(int variant, const dr_problem *p, const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta_k, const float *beta_v, const float *s,
                               const float *S0, const void *dout, const float *dS_T, float *dq, float *dk,
                               float *dv, float *dalpha, float *dbeta_k, float *dbeta_v, float *ds, float *dS0,
                               void *workspace, size_t workspace_bytes, void *stream) {
  dr_status st = check_common(p, false);
  if (st != DR_OK) return st;
  if (variant < kBwdDefault || variant > kBwdChunk) return DR_ERR_UNSUPPORTED;
  if (variant == kBwdChunk && !bwd_chunk_shape(p)) return DR_ERR_UNSUPPORTED;
  st = check_pointers(p, q, k, v, alpha, beta_k, beta_v, dout);
  if (st != DR_OK) return st;
  const bool need = p->T > 0;
  if (need && (!dq || !dk || !dv || !dbeta_k)) return DR_ERR_INVALID_ARG;
  if (need && ((dalpha == nullptr) != (alpha == nullptr))) return DR_ERR_INVALID_ARG;
  if (need && ((dbeta_v == nullptr) != (beta_v == nullptr))) return DR_ERR_INVALID_ARG;
  if (need && ((ds == nullptr) != (s == nullptr))) return DR_ERR_INVALID_ARG;
  const void *ptrs[] = {s, S0, dS_T, dq, dk, dv, dalpha, dbeta_k, dbeta_v, ds, dS0, workspace};
  for (const void *x : ptrs)
    if (x && !aligned16(x)) return DR_ERR_ALIGNMENT;
  if (static_cast<long long>(p->B) * p->H > 0x7fffffffLL) return DR_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t state_bytes = sizeof(float) * size_t(p->B) * p->H * p->dk * p->dv;
  if (p->T == 0) {  // nothing to differentiate but the identity S_T = S0
    if (!dS0) return DR_OK;
    const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, cs)
                               : cudaMemsetAsync(dS0, 0, state_bytes, cs);
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
  }
  if (!workspace || workspace_bytes < bwd_variant_workspace_bytes(p, variant)) return DR_ERR_WORKSPACE;
  if (resolve_bwd_variant(p, variant) == kBwdChunk)
    return bwd_chunk_launch(p, q, k, v, alpha, beta_k, beta_v, s, S0, dout, dS_T, dq, dk, dv, dalpha, dbeta_k,
                            dbeta_v, ds, dS0, workspace, workspace_bytes, cs);
  float *ws = static_cast<float *>(workspace);
  {  // the per-key-channel gradients are sums over value-column slices, accumulated in place
    const size_t tok = static_cast<size_t>(p->B) * p->T * p->H;
    const size_t gk = tok * p->dk * sizeof(float);
    auto gate_bytes = [&](int mode) { return mode == DR_CHANNEL ? gk : tok * sizeof(float); };
    struct Z { void *ptr; size_t bytes; } zs[] = {
        {dq, gk}, {dk, gk}, {ds, gk}, {dalpha, dalpha ? gate_bytes(p->alpha_mode) : 0},
        {dbeta_k, gate_bytes(p->beta_k_mode)}, {dbeta_v, dbeta_v ? gate_bytes(p->beta_v_mode) : 0}};
    for (const Z &z : zs)
      if (z.ptr && cudaMemsetAsync(z.ptr, 0, z.bytes, cs) != cudaSuccess) return DR_ERR_CUDA;
  }
  const size_t nck = (static_cast<size_t>(p->T) + kBwdSpan - 1) / kBwdSpan;
  dr::BwdParams bp{p->T, p->H, q, k, v, dout, alpha, p->alpha_mode, beta_k, p->beta_k_mode, beta_v,
                   p->beta_v_mode, s, S0, dS_T, dq, dk, dv, dalpha, dbeta_k, dbeta_v, ds, dS0, ws,
                   ws + static_cast<size_t>(p->B) * p->H * nck * p->dk * p->dv};
  if (p->io_dtype == DR_F32) return bwd_dispatch<float>(p, bp, cs);
  return bwd_dispatch<__nv_bfloat16>(p, bp, cs);
}

dr_status dr_backward(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                      const float *beta_k, const float *beta_v, const float *s, const float *S0, const void *dout,
                      const float *dS_T, float *dq, float *dk, float *dv, float *dalpha, float *dbeta_k,
                      float *dbeta_v, float *ds, float *dS0, void *workspace, size_t workspace_bytes,
                      void *stream) {
  return backward_impl(kBwdDefault, p, q, k, v, alpha, beta_k, beta_v, s, S0, dout, dS_T, dq, dk, dv, dalpha,
                       dbeta_k, dbeta_v, ds, dS0, workspace, workspace_bytes, stream);
}

int dr_version(void) { return 100; }

const char *dr_status_string(dr_status s) {
  switch (s) {
    case DR_OK: return "DR_OK";
    case DR_ERR_INVALID_ARG: return "DR_ERR_INVALID_ARG: invalid argument";
    case DR_ERR_UNSUPPORTED: return "DR_ERR_UNSUPPORTED: size or mode not supported";
    case DR_ERR_ALIGNMENT: return "DR_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case DR_ERR_WORKSPACE: return "DR_ERR_WORKSPACE: workspace missing or too small";
    case DR_ERR_RANGE: return "DR_ERR_RANGE: cumulative decay in a chunk below the supported range";
    case DR_ERR_TIMEOUT: return "DR_ERR_TIMEOUT: a bounded device wait expired";
    case DR_ERR_CUDA: return "DR_ERR_CUDA: CUDA call or launch failed";
  }
  return "unknown dr_status";
}

size_t dr_chunk_fwd_workspace(const dr_problem *p) {
  if (check_common(p, false) != DR_OK) return 0;
  return kWorkspaceBytes + (ring_problem(p) && quad_default(p) ? quad_stage_bytes(p) : 0);
}

dr_status dr_chunk_fwd(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                       const float *beta_k, const float *beta_v, const float *S0, void *o, float *S_T,
                       void *workspace, size_t workspace_bytes, void *stream) {
  return chunk_fwd_impl(p, nullptr, q, k, v, alpha, beta_k, beta_v, nullptr, S0, o, S_T, workspace, workspace_bytes,
                        stream);
}

dr_status dr_chunk_fwd_osdn(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                            const float *beta_k, const float *beta_v, const float *s, const float *S0, void *o,
                            float *S_T, void *workspace, size_t workspace_bytes, void *stream) {
  return chunk_fwd_impl(p, nullptr, q, k, v, alpha, beta_k, beta_v, s, S0, o, S_T, workspace, workspace_bytes,
                        stream);
}

dr_status dr_state_map_apply(int n, int dk, int dv, const float *M, const float *S, const float *N, float *out,
                             void *stream) {
  if (n < 0 || (dk != 64 && dk != 128) || dv <= 0 || dv % 32 != 0) return DR_ERR_INVALID_ARG;
  if (n == 0) return DR_OK;
  if (!M || !N || !out) return DR_ERR_INVALID_ARG;
  if (S && S == out) return DR_ERR_INVALID_ARG;  // S is read by other threads while out is written
  if (!aligned16(M) || !aligned16(N) || !aligned16(out) || (S && !aligned16(S))) return DR_ERR_ALIGNMENT;
  if (n > 65535) return DR_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(dv / 32, n);
  if (dk == 128)
    dr::state_map_apply_kernel<128><<<grid, 256, 0, st>>>(dv, M, S, N, out);
  else
    dr::state_map_apply_kernel<64><<<grid, 256, 0, st>>>(dv, M, S, N, out);
  return launch_status();
}

dr_status dr_chunk_fwd_varlen(const dr_problem *p, const int *cu_seqlens, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta_k, const float *beta_v,
                              const float *s, const float *S0, void *o, float *S_T, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (!cu_seqlens) return DR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return DR_ERR_ALIGNMENT;
  return chunk_fwd_impl(p, cu_seqlens, q, k, v, alpha, beta_k, beta_v, s, S0, o, S_T, workspace,
                        workspace_bytes, stream);
}

dr_status dr_decode_step(const dr_problem *p, const void *q, const void *k, const void *v, const float *alpha,
                         const float *beta_k, const float *beta_v, float *S, void *o, void *stream) {
  return decode_step_impl(p, q, k, v, alpha, beta_k, beta_v, nullptr, S, o, stream);
}

dr_status dr_decode_step_osdn(const dr_problem *p, const void *q, const void *k, const void *v,
                              const float *alpha, const float *beta_k, const float *beta_v, const float *s, float *S,
                              void *o, void *stream) {
  return decode_step_impl(p, q, k, v, alpha, beta_k, beta_v, s, S, o, stream);
}

// ----------------------------------------------------------------- prefill without allocation
// Scratch of dr_chunk_fwd_noalloc: a file-scope device array (every GPU that
// loads this library holds it until the process exits).  Host code must not
// pass the symbol itself to a kernel -- on the host it is only a stand-in --
// so its device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and cached.
constexpr size_t kStaticScratchBytes = 4096;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_addr[kMaxDevices] = {};
}  // namespace

dr_status dr_chunk_fwd_noalloc(const dr_problem *p, const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta_k, const float *beta_v, const float *S0,
                               void *o, float *S_T, void *stream) {
  const dr_status s = check_common(p, false);
  if (s != DR_OK) return s;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DR_ERR_UNSUPPORTED;
  if (q) {  // the array used is the current device's: the data must live there too
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, q) != cudaSuccess) {
      cudaGetLastError();
      return DR_ERR_INVALID_ARG;
    }
    if (a.type == cudaMemoryTypeDevice && a.device != dev) return DR_ERR_INVALID_ARG;
  }
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_addr[dev]) {
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_static_scratch) != cudaSuccess || !addr) return DR_ERR_CUDA;
      g_static_addr[dev] = addr;
    }
    scratch = g_static_addr[dev];
  }
  // The status word fits the array; the four-CTA prefill's staging does not, so such problems run
  // the two-CTA prefill (the library's choice for a workspace of that size).  The call clears the
  // status word at its start, on `stream`.
  static_assert(kWorkspaceBytes <= kStaticScratchBytes, "status word");
  return dr_chunk_fwd(p, q, k, v, alpha, beta_k, beta_v, S0, o, S_T, scratch, kStaticScratchBytes, stream);
}

dr_status dr_noalloc_status(void *stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DR_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    scratch = g_static_addr[dev];
  }
  if (!scratch) return DR_ERR_INVALID_ARG;  // no no-alloc call on this device yet
  return dr_workspace_status(scratch, stream);
}

dr_status dr_workspace_status(const void *workspace, void *stream) {
  if (!workspace) return DR_ERR_WORKSPACE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DR_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return DR_ERR_CUDA;
  if (w & dr::STATUS_TIMEOUT) return DR_ERR_TIMEOUT;
  if (w & dr::STATUS_RANGE) return DR_ERR_RANGE;
  return DR_OK;
}

size_t dr_diag_chunk_fwd_workspace(int variant, const dr_problem *p) {
  if (check_common(p, false) != DR_OK) return 0;
  if (variant == kPrefillQuad) return ring_problem(p) ? kWorkspaceBytes + quad_stage_bytes(p) : 0;
  return variant == kPrefillDefault ? dr_chunk_fwd_workspace(p) : kWorkspaceBytes;
}

int dr_diag_chunk_fwd_variant(int variant, const dr_problem *p, const void *q, const void *k, const void *v,
                              const float *alpha, const float *beta_k, const float *beta_v, const float *S0, void *o,
                              float *S_T, void *workspace, size_t workspace_bytes, void *stream) {
  return chunk_fwd_impl(p, nullptr, q, k, v, alpha, beta_k, beta_v, nullptr, S0, o, S_T, workspace, workspace_bytes,
                        stream, variant);
}

int dr_diag_decode_step_variant(int variant, const dr_problem *p, const void *q, const void *k, const void *v,
                                const float *alpha, const float *beta_k, const float *beta_v, const float *s,
                                float *S, void *o, void *stream) {
  return decode_step_impl(p, q, k, v, alpha, beta_k, beta_v, s, S, o, stream, variant);
}

size_t dr_diag_backward_workspace(int variant, const dr_problem *p) {
  if (check_common(p, false) != DR_OK || variant < kBwdDefault || variant > kBwdChunk) return 0;
  if (variant == kBwdChunk && !bwd_chunk_shape(p)) return 0;
  return bwd_variant_workspace_bytes(p, variant);
}

int dr_diag_backward_variant(int variant, const dr_problem *p, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta_k, const float *beta_v, const float *s,
                             const float *S0, const void *dout, const float *dS_T, float *dq, float *dk, float *dv,
                             float *dalpha, float *dbeta_k, float *dbeta_v, float *ds, float *dS0, void *workspace,
                             size_t workspace_bytes, void *stream) {
  return backward_impl(variant, p, q, k, v, alpha, beta_k, beta_v, s, S0, dout, dS_T, dq, dk, dv, dalpha, dbeta_k,
                       dbeta_v, ds, dS0, workspace, workspace_bytes, stream);
}

int dr_diag_umma_selftest(int N, int K, int a_mn, int b_mn, int bf16, const void *A, const void *B, float *D,
                          void *workspace, void *stream) {
  if (!A || !B || !D || !workspace) return DR_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *status = static_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DR_ERR_CUDA;
  const size_t smem = 1024 + size_t(128) * K * 2 + size_t(K) * N * 2;
  const auto *a = static_cast<const uint16_t *>(A);
  const auto *b = static_cast<const uint16_t *>(B);
#define DR_SELFTEST_CASE(NN, KK)                                                                      \
  if (N == NN && K == KK) {                                                                           \
    auto kern = dr::umma_selftest_kernel<NN, KK>;                                                     \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) \
      return DR_ERR_CUDA;                                                                             \
    kern<<<1, 128, smem, st>>>(a, b, D, a_mn, b_mn, bf16, status);                                          \
    return launch_status();                                                                           \
  }
  DR_SELFTEST_CASE(64, 64)
  DR_SELFTEST_CASE(64, 128)
  DR_SELFTEST_CASE(128, 64)
  DR_SELFTEST_CASE(128, 128)
#undef DR_SELFTEST_CASE
  return DR_ERR_UNSUPPORTED;
}

int dr_diag_wait_timeout(int cluster_scope, unsigned long long limit_ns, void *workspace,
                         unsigned long long *waited_ns, void *stream) {
  if (!workspace || limit_ns == 0 || limit_ns > 1000000000ull) return DR_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *status = static_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DR_ERR_CUDA;
  const int sc = cluster_scope ? 1 : 0;
  if (!sc) {
    dr::wait_selftest_kernel<<<1, 32, 0, st>>>(0, limit_ns, status, waited_ns);
    return launch_status();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(32, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dr::wait_selftest_kernel, sc, limit_ns, status, waited_ns) != cudaSuccess)
    return DR_ERR_CUDA;
  return launch_status();
}

int dr_diag_tri_inverse(int variant, const float *A, float *T, void *stream) {
  if (!A || !T || variant < 0 || variant > 1) return DR_ERR_INVALID_ARG;
  if (cudaFuncSetAttribute(dr::tri_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dr::kTriSelftestSmem)) != cudaSuccess)
    return DR_ERR_CUDA;
  dr::tri_selftest_kernel<<<1, 128, dr::kTriSelftestSmem, static_cast<cudaStream_t>(stream)>>>(variant, A, T);
  return launch_status();
}

}  // extern "C"
