// One 16-channel group of the FP4 main-KV format: E2M1 codes with one E4M3 scale, no global
// scale (aprilzz.com "DeepSeek V4.1 Flash 发布…", section "FP4 KV 与部署层的几个改动").
// Shared by the append kernel and the compressor's epilogue, so both quantise alike.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace csa2 {

// E2M1 magnitude code of q >= 0: nearest of {0,.5,1,1.5,2,3,4,6}, exact midpoints to the
// even code, saturating at 6.  Each comparison is one threshold of the grid.
__device__ __forceinline__ uint32_t e2m1_magnitude(float q) {
  return (uint32_t)(q > 0.25f) + (uint32_t)(q >= 0.75f) + (uint32_t)(q > 1.25f) +
         (uint32_t)(q >= 1.75f) + (uint32_t)(q > 2.5f) + (uint32_t)(q >= 3.5f) +
         (uint32_t)(q > 5.0f);
}

// value of a non-negative E4M3 code (bias 7; exponent field 0 is subnormal m * 2^-9)
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return (float)m * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Quantise 16 values: scale = E4M3(amax / 6) (fp32 divide, round to nearest even,
// saturating), code_i = E2M1(|v_i| / dec(scale)) with v_i's sign bit (a zero scale gives
// signed zeros).  codes[k] holds code 8k .. 8k+7, code i in bits [4i, 4i+4).
__device__ __forceinline__ uint32_t quantize16(const float* v, uint32_t* codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const __nv_fp8_storage_t sc = __nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
  const float s = e4m3_value((uint32_t)sc & 0x7Fu);
  codes[0] = codes[1] = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t sign = __float_as_uint(v[i]) >> 31;
    const uint32_t mag = (s != 0.0f) ? e2m1_magnitude(__fdiv_rn(fabsf(v[i]), s)) : 0u;
    codes[i >> 3] |= ((sign << 3) | mag) << (4 * (i & 7));
  }
  return (uint32_t)sc;
}

}  // namespace csa2
