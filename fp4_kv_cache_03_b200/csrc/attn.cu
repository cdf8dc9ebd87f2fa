// a7: sparse attention over the selected FP4 entries joined with the layer's own
// sliding window, one softmax over both sets.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", sections "把 prefill 砍掉一半" (every layer
// keeps a 128-token window) and "CSA2：在层的维度上共享缓存" (each layer keeps its own main
// Q and window KV; Reuse layers attend with the latest indices);
// "FP4 KV 与部署层的几个改动" (E2M1 + per-16-channel E4M3, dequantised for the product).
//
// Split over key slots: CTA (split, q) gathers 64 slots of the list
// [indices[q][0..topk) ; window positions], dequantises FP4 rows in registers to bf16
// (exact: a 2-bit-mantissa value times a 4-bit-mantissa scale), and computes
// S = scale * Q K^T, a partial softmax (m, l) and O = P V for all heads; a second kernel
// merges the splits by log-sum-exp.
#include <cuda_bf16.h>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kSlots = 64;          // key slots per CTA
constexpr int kAttnThreads = 256;

struct AttnArgs {
  const uint16_t* q;
  int num_q, H, D;
  const uint8_t* codes;
  const uint8_t* scales;
  int64_t cap_rows;
  const int64_t* seq_start;
  const int32_t* seq_len;
  int q_per_seq;
  const int32_t* indices;
  int topk;
  const uint16_t* swa;
  int64_t swa_rows;
  const int64_t* swa_start;
  const int64_t* q_pos;
  int window;
  float scale;
  int nsplit;
  float* part_o;   // [num_q][nsplit][H][D]
  float* part_ml;  // [num_q][nsplit][H][2]
  float* out;
  float* lse;
  int* status;
};

__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = m < 4 ? 0.5f * (float)m : (m == 4 ? 2.0f : (m == 5 ? 3.0f : (m == 6 ? 4.0f : 6.0f)));
  return (c & 8u) ? -mag : mag;
}
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (b & 0x80u) ? -v : v;
}

__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int split = blockIdx.x, q = blockIdx.y, tid = threadIdx.x;
  const int H = a.H, D = a.D, KD = D + 8;  // padded key rows
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sK = sQ + (size_t)H * D;
  float* sS = reinterpret_cast<float*>(sK + (size_t)kSlots * KD);   // [H][kSlots]
  float* sM = sS + (size_t)H * kSlots;                                // [H]
  int* sValid = reinterpret_cast<int*>(sM + H);                       // [kSlots]

  const int seq = q / a.q_per_seq;
  const int64_t t = a.q_pos[q];
  const int64_t w0 = t - a.window + 1 > 0 ? t - a.window + 1 : 0;
  const int n_win = (int)(t + 1 - w0 < 0 ? 0 : t + 1 - w0);

  // Q -> shared
  const uint4* gq = reinterpret_cast<const uint4*>(a.q + (int64_t)q * H * D);
  for (int i = tid; i < H * D / 8; i += kAttnThreads) reinterpret_cast<uint4*>(sQ)[i] = gq[i];

  // gather + dequantise this split's key slots (one 16-channel group per item)
  const int gpr = D / 16;
  for (int it = tid; it < kSlots * gpr; it += kAttnThreads) {
    const int j = it / gpr, g = it % gpr;
    const int slot = split * kSlots + j;
    __nv_bfloat16* dst = sK + (size_t)j * KD + g * 16;
    bool ok = false;
    if (slot < a.topk) {
      const int p = a.indices[(int64_t)q * a.topk + slot];
      if (p >= 0) {
        const int64_t row = a.seq_start[seq] + p;
        if (p >= a.seq_len[seq]) {
          report(a.status, CSA2_ERR_INVALID_ARG);
        } else if (row >= a.cap_rows) {
          report(a.status, CSA2_ERR_CAPACITY);
        } else {
          const uint2 c = __ldg(reinterpret_cast<const uint2*>(a.codes + row * (D / 2) + g * 8));
          const float s = e4m3_value(__ldg(a.scales + row * gpr + g));
          const uint32_t cw[2] = {c.x, c.y};
          __align__(16) __nv_bfloat16 v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            v[i] = __float2bfloat16_rn(e2m1_value((cw[i >> 3] >> (4 * (i & 7))) & 15u) * s);
          reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<uint4*>(v)[0];
          reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<uint4*>(v)[1];
          ok = true;
        }
      } else if (p < -1) {
        report(a.status, CSA2_ERR_INVALID_ARG);
      }
    } else if (slot - a.topk < n_win) {
      const int64_t row = a.swa_start[seq] + w0 + (slot - a.topk);
      if (row < 0 || row >= a.swa_rows) {
        report(a.status, CSA2_ERR_CAPACITY);
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(a.swa + row * D + g * 16);
        reinterpret_cast<uint4*>(dst)[0] = __ldg(src);
        reinterpret_cast<uint4*>(dst)[1] = __ldg(src + 1);
        ok = true;
      }
    }
    if (!ok) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(0, 0, 0, 0);
    }
    if (g == 0) sValid[j] = ok ? 1 : 0;
  }
  __syncthreads();

  // S[h][j] = scale * Q[h] . K[j]
  {
    const int j = tid & (kSlots - 1), hg = tid >> 6;   // 4 head groups
    float acc[32];
    const int nh = H / 4;                              // heads per thread (<= 32)
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
    const __nv_bfloat16* kr = sK + (size_t)j * KD;
    for (int d = 0; d < D; d += 8) {
      const uint4 kv = *reinterpret_cast<const uint4*>(kr + d);
      const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv);
      float kf[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(k2[i]);
        kf[2 * i] = f.x; kf[2 * i + 1] = f.y;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (i < nh) {
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + (size_t)(hg + 4 * i) * D + d);
          const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(q2[u]);
            acc[i] = fmaf(f.x, kf[2 * u], acc[i]);
            acc[i] = fmaf(f.y, kf[2 * u + 1], acc[i]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nh) sS[(size_t)(hg + 4 * i) * kSlots + j] = sValid[j] ? acc[i] * a.scale : -INFINITY;
  }
  __syncthreads();

  // partial softmax per head: p = exp(s - m), m = max, l = sum p
  float* ml = a.part_ml + (((int64_t)q * a.nsplit + split) * H) * 2;
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < H; h += kAttnThreads / 32) {
      float* row = sS + (size_t)h * kSlots;
      const float x0 = row[lane], x1 = row[lane + 32];
      float m = fmaxf(x0, x1);
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float p0 = (x0 == -INFINITY) ? 0.0f : expf(x0 - m);
      const float p1 = (x1 == -INFINITY) ? 0.0f : expf(x1 - m);
      row[lane] = p0;
      row[lane + 32] = p1;
      float l = p0 + p1;
      for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) { ml[2 * h] = m; ml[2 * h + 1] = l; }
    }
  }
  __syncthreads();

  // O[h][d] = sum_j p[h][j] K[j][d]  (two dims, 16 heads per pass)
  {
    const int half = D / 2;
    const int dp = tid % half, hgrp = tid / half, hstep = (kAttnThreads / half) * 16;
    float* po = a.part_o + (((int64_t)q * a.nsplit + split) * H) * D;
    for (int h0 = hgrp * 16; h0 < H; h0 += hstep) {
      float acc0[16], acc1[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) { acc0[i] = 0.0f; acc1[i] = 0.0f; }
      for (int j = 0; j < kSlots; ++j) {
        const float2 kv =
            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sK + (size_t)j * KD + 2 * dp));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p = sS[(size_t)(h0 + i) * kSlots + j];
          acc0[i] = fmaf(p, kv.x, acc0[i]);
          acc1[i] = fmaf(p, kv.y, acc1[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        *reinterpret_cast<float2*>(po + (size_t)(h0 + i) * D + 2 * dp) = make_float2(acc0[i], acc1[i]);
    }
  }
}

__global__ void __launch_bounds__(kAttnThreads) attn_merge_kernel(const AttnArgs a) {
  const int q = blockIdx.x;
  const int H = a.H, D = a.D;
  for (int h = 0; h < H; ++h) {
    const float* ml = a.part_ml + ((int64_t)q * a.nsplit * H + h) * 2;
    float M = -INFINITY;
    for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, ml[(int64_t)s * H * 2]);
    float L = 0.0f;
    for (int s = 0; s < a.nsplit; ++s) {
      const float m = ml[(int64_t)s * H * 2];
      if (m != -INFINITY) L += expf(m - M) * ml[(int64_t)s * H * 2 + 1];
    }
    float* o = a.out + ((int64_t)q * H + h) * D;
    for (int d = threadIdx.x; d < D; d += kAttnThreads) {
      float acc = 0.0f;
      for (int s = 0; s < a.nsplit; ++s) {
        const float m = ml[(int64_t)s * H * 2];
        if (m != -INFINITY)
          acc += expf(m - M) * a.part_o[(((int64_t)q * a.nsplit + s) * H + h) * D + d];
      }
      o[d] = L > 0.0f ? acc / L : 0.0f;
    }
    if (a.lse && threadIdx.x == 0) a.lse[(int64_t)q * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
  }
}

size_t attn_smem(int H, int D) {
  return (size_t)H * D * 2 + (size_t)kSlots * (D + 8) * 2 + (size_t)H * kSlots * 4 + H * 4 +
         kSlots * 4;
}

bool attn_shape_ok(int H, int D) {
  const bool d_ok = D == 32 || D == 64 || D == 128 || D == 256 || D == 512;
  return d_ok && H >= 16 && H <= 128 && (H % 16) == 0 && attn_smem(H, D) <= 200 * 1024;
}

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_sparse_attn_workspace(int32_t num_q, int32_t H, int32_t D, int32_t topk,
                                             int32_t window) {
  if (num_q < 0 || H < 1 || D < 1 || topk < 0 || window < 0) return 0;
  const int64_t nsplit = ((int64_t)topk + window + kSlots - 1) / kSlots;
  size_t off = CSA2_STATUS_BYTES;
  off = a256(off + (size_t)num_q * nsplit * H * D * 4);
  off = a256(off + (size_t)num_q * nsplit * H * 2 * 4);
  return off;
}

extern "C" csa2_status_t csa2_sparse_attn(const uint16_t* q, int32_t num_q, int32_t H, int32_t D,
                                          const uint8_t* kv_codes, const uint8_t* kv_scales,
                                          int64_t cap_rows, csa2_seqs_t seqs,
                                          const int32_t* indices, int32_t topk,
                                          const uint16_t* swa_kv, int64_t swa_rows,
                                          const int64_t* swa_start, const int64_t* q_pos,
                                          int32_t window, float softmax_scale, float* out,
                                          float* lse, void* workspace, size_t ws_bytes,
                                          void* stream) {
  if (num_q < 0 || topk < 0 || topk > 2048 || window < 0 || window > 1024) return CSA2_ERR_INVALID_ARG;
  if (!attn_shape_ok(H, D)) return CSA2_ERR_UNSUPPORTED;
  if (seqs.num_seqs < 1 || seqs.q_per_seq < 1 || (int64_t)seqs.num_seqs * seqs.q_per_seq != num_q)
    return CSA2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < csa2_sparse_attn_workspace(num_q, H, D, topk, window))
    return CSA2_ERR_CAPACITY;
  if (num_q == 0) return CSA2_OK;
  if (!q || !out || !q_pos || !seqs.seq_start || !seqs.seq_len) return CSA2_ERR_INVALID_ARG;
  if (topk > 0 && (!indices || !kv_codes || !kv_scales || cap_rows <= 0)) return CSA2_ERR_INVALID_ARG;
  if (window > 0 && (!swa_kv || !swa_start || swa_rows < 0)) return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kv_codes) & 7) ||
      (reinterpret_cast<uintptr_t>(swa_kv) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return CSA2_ERR_INVALID_ARG;
  AttnArgs a{};
  a.q = q; a.num_q = num_q; a.H = H; a.D = D;
  a.codes = kv_codes; a.scales = kv_scales; a.cap_rows = cap_rows;
  a.seq_start = seqs.seq_start; a.seq_len = seqs.seq_len; a.q_per_seq = seqs.q_per_seq;
  a.indices = indices; a.topk = topk;
  a.swa = swa_kv; a.swa_rows = swa_rows; a.swa_start = swa_start; a.q_pos = q_pos;
  a.window = window; a.scale = softmax_scale;
  a.nsplit = (topk + window + kSlots - 1) / kSlots;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  size_t off = CSA2_STATUS_BYTES;
  a.part_o = reinterpret_cast<float*>(ws + off);
  off = a256(off + (size_t)num_q * a.nsplit * H * D * 4);
  a.part_ml = reinterpret_cast<float*>(ws + off);
  a.out = out; a.lse = lse;
  cudaStream_t st = (cudaStream_t)stream;
  if (a.nsplit > 0) {
    const size_t smem = attn_smem(H, D);
    if (cudaFuncSetAttribute(attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return CSA2_ERR_CUDA;
    attn_split_kernel<<<dim3(a.nsplit, num_q), kAttnThreads, smem, st>>>(a);
  }
  attn_merge_kernel<<<num_q, kAttnThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
