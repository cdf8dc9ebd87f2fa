// a1: quantise main-KV rows to FP4 (E2M1 codes + one E4M3 scale per 16 channels, no
// global scale) and append them to the cache; optionally copy the indexer-K row too.
// Format: aprilzz.com "DeepSeek V4.1 Flash 发布…", section "FP4 KV 与部署层的几个改动";
// gkm0120.cn "技术调研报告" §2.2.1.
#include <cuda_fp8.h>

#include "common.cuh"
#include "fp4_quant.cuh"

namespace csa2 {
namespace {

// kE4M3K: the indexer-K row goes to an E4M3 cache (one byte per element, RNE, saturating),
// else it is copied as bf16.
template <bool kE4M3K>
__global__ void __launch_bounds__(256) quant_append_kernel(
    const float* __restrict__ x, int rows, int D, const int64_t* __restrict__ dst_row,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int64_t cap,
    const uint16_t* __restrict__ kin, void* __restrict__ kout, int d_I, int* status) {
  pdl_trigger();
  pdl_wait();
  const int gpr = D >> 4;                      // channel groups per row
  const int cpr = kin ? (d_I >> 3) : 0;        // 16-byte chunks of indexer K per row
  const int64_t n_q = (int64_t)rows * gpr;
  const int64_t n_c = (int64_t)rows * cpr;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;

  if (gid < n_q) {
    const int r = (int)(gid / gpr), g = (int)(gid % gpr);
    const int64_t dst = dst_row[r];
    if (dst < 0 || dst >= cap) {
      report(status, CSA2_ERR_CAPACITY);
    } else {
      const float4* src = reinterpret_cast<const float4*>(x + (int64_t)r * D + g * 16);
      float v[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(src + i);
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
      }
      uint32_t packed[2];
      const uint32_t sc = quantize16(v, packed);
      uint2* dc = reinterpret_cast<uint2*>(codes + dst * (int64_t)(D >> 1) + g * 8);
      *dc = make_uint2(packed[0], packed[1]);
      scales[dst * (int64_t)gpr + g] = (uint8_t)sc;
    }
  }
  if (gid < n_c) {
    const int r = (int)(gid / cpr), c = (int)(gid % cpr);
    const int64_t dst = dst_row[r];
    if (dst >= 0 && dst < cap) {
      const uint4 t = __ldg(reinterpret_cast<const uint4*>(kin + (int64_t)r * d_I) + c);
      if constexpr (kE4M3K) {
        // 8 bf16 -> 8 E4M3 bytes (bf16 -> fp32 is exact)
        const uint32_t wv[4] = {t.x, t.y, t.z, t.w};
        uint32_t outw[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t bits = (wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
          const uint32_t b = (uint32_t)__nv_cvt_float_to_fp8(__uint_as_float(bits << 16),
                                                             __NV_SATFINITE, __NV_E4M3);
          outw[e >> 2] |= b << (8 * (e & 3));
        }
        reinterpret_cast<uint2*>(static_cast<uint8_t*>(kout) + dst * (int64_t)d_I)[c] =
            make_uint2(outw[0], outw[1]);
      } else {
        reinterpret_cast<uint4*>(static_cast<uint16_t*>(kout) + dst * (int64_t)d_I)[c] = t;
      }
    } else {
      report(status, CSA2_ERR_CAPACITY);
    }
  }
}

// bf16 -> E4M3 (RNE, saturating to +-448), 8 elements per thread
__global__ void __launch_bounds__(256) e4m3_from_bf16_kernel(const uint16_t* __restrict__ in,
                                                             uint8_t* __restrict__ out, int64_t n) {
  pdl_trigger();
  pdl_wait();
  const int64_t i8 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  for (int e = 0; e < 8; ++e) {
    const int64_t i = i8 + e;
    if (i < n)
      out[i] = (uint8_t)__nv_cvt_float_to_fp8(__uint_as_float((uint32_t)__ldg(in + i) << 16),
                                              __NV_SATFINITE, __NV_E4M3);
  }
}

template <bool kE4M3K>
csa2_status_t append_impl(const float* x, int32_t rows, int32_t D, const int64_t* dst_row,
                          uint8_t* kv_codes, uint8_t* kv_scales, int64_t cap_rows,
                          const uint16_t* idx_k_in, void* idx_k, int32_t d_I, void* workspace,
                          size_t ws_bytes, void* stream) {
  if (rows < 0 || D < 32 || D > 4096 || (D % 32) != 0 || cap_rows <= 0) return CSA2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < CSA2_STATUS_BYTES) return CSA2_ERR_CAPACITY;
  if (rows == 0) return CSA2_OK;
  if (!x || !dst_row || !kv_codes || !kv_scales) return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(kv_codes) & 7))
    return CSA2_ERR_INVALID_ARG;
  if (idx_k_in) {
    if (!idx_k || d_I < 8 || (d_I % 8) != 0) return CSA2_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(idx_k_in) & 15) ||
        (reinterpret_cast<uintptr_t>(idx_k) & (kE4M3K ? 7 : 15)))
      return CSA2_ERR_INVALID_ARG;
  }
  const int64_t nq = (int64_t)rows * (D / 16);
  const int64_t nc = idx_k_in ? (int64_t)rows * (d_I / 8) : 0;
  const int64_t n = nq > nc ? nq : nc;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  if (blocks > 0x7FFFFFFF) return CSA2_ERR_UNSUPPORTED;
  const cudaError_t e = launch_pdl(
      quant_append_kernel<kE4M3K>, dim3((unsigned)blocks), dim3(threads), 0, (cudaStream_t)stream,
      x, rows, D, dst_row, kv_codes, kv_scales, cap_rows, idx_k_in, idx_k, idx_k_in ? d_I : 0,
      static_cast<int*>(workspace));
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // namespace
}  // namespace csa2

extern "C" size_t csa2_quant_append_workspace(void) { return CSA2_STATUS_BYTES; }

extern "C" csa2_status_t csa2_quant_append_e4m3k(const float* x, int32_t rows, int32_t D,
                                                 const int64_t* dst_row, uint8_t* kv_codes,
                                                 uint8_t* kv_scales, int64_t cap_rows,
                                                 const uint16_t* idx_k_in, uint8_t* idx_k,
                                                 int32_t d_I, void* workspace, size_t ws_bytes,
                                                 void* stream) {
  return csa2::append_impl<true>(x, rows, D, dst_row, kv_codes, kv_scales, cap_rows, idx_k_in, idx_k,
                                 d_I, workspace, ws_bytes, stream);
}

extern "C" csa2_status_t csa2_e4m3_from_bf16(const uint16_t* in, uint8_t* out, int64_t n,
                                             void* stream) {
  if (n < 0) return CSA2_ERR_INVALID_ARG;
  if (n == 0) return CSA2_OK;
  if (!in || !out) return CSA2_ERR_INVALID_ARG;
  const int64_t blocks = (n + 8 * 256 - 1) / (8 * 256);
  if (blocks > 0x7FFFFFFF) return CSA2_ERR_UNSUPPORTED;
  return csa2::launch_pdl(csa2::e4m3_from_bf16_kernel, dim3((unsigned)blocks), dim3(256), 0,
                          (cudaStream_t)stream, in, out, n) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

extern "C" csa2_status_t csa2_quant_append(const float* x, int32_t rows, int32_t D,
                                           const int64_t* dst_row, uint8_t* kv_codes,
                                           uint8_t* kv_scales, int64_t cap_rows,
                                           const uint16_t* idx_k_in, uint16_t* idx_k,
                                           int32_t d_I, void* workspace, size_t ws_bytes,
                                           void* stream) {
  return csa2::append_impl<false>(x, rows, D, dst_row, kv_codes, kv_scales, cap_rows, idx_k_in,
                                  idx_k, d_I, workspace, ws_bytes, stream);
}
