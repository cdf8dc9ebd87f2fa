// The sequence-axis compressor: every m consecutive tokens become one compressed entry
// (gkm0120.cn "DeepSeek-V4.1-Flash 技术调研报告" §2.2.1 三个压缩维度, sequence dimension:
// "every m tokens compressed into 1 entry"; aprilzz.com "CSA2：在层的维度上共享缓存": the
// encoder groups run at ratio 2), as a linear map of the m token rows, fused with the a1
// quantise + append of the entry into the FP4 cache.
//
// entry_j[n] = sum_k xcat_j[k] * w_t[n][k], xcat_j = [x_{jm}; ...; x_{jm+m-1}] (K = m * D_in)
//
// One CTA takes 128 entries: warp 0 streams 64-wide K chunks of the token rows (A, 128 rows)
// and of the map (B, D rows) by TMA into a two-stage ring, warp 1 issues tcgen05.mma
// (M = 128 entries, N = 256 or D output channels, K = 16 per instruction) into a TMEM
// accumulator of D fp32 columns, and warps 2-5 read each entry's row back 16 channels at a
// time -- one scale group -- and quantise it straight into the cache row dst_row[j]: the
// compressed entry never goes through HBM in fp32.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "fp4_quant.cuh"

namespace csa2 {
namespace {

constexpr int kCThreads = 192;        // 6 warps
constexpr int kCTile = 128;           // entries per CTA (MMA M)
constexpr int kCStages = 2;

struct CompressArgs {
  int n_entries;
  int K;                              // m * D_in
  const int64_t* dst_row;
  uint8_t* codes;
  uint8_t* scales;
  int64_t cap;
  int* status;
  uint64_t wait_ns;
};

template <int D>
struct CGeo {
  static constexpr int kN = D < 256 ? D : 256;        // MMA N
  static constexpr int kNParts = D / kN;
  static constexpr uint32_t kA = kCTile * 128;         // [128 rows][64 bf16]
  static constexpr uint32_t kB = D * 128;              // [D rows][64 bf16]
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kSmem = 1024 + kCStages * kStage;
  static constexpr uint32_t kTmemCols = D;             // 128, 256 or 512
};

template <int D>
__global__ void __launch_bounds__(kCThreads, 1)
    compress_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const CompressArgs a) {
  using G = CGeo<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full[kCStages], empty[kCStages], tfull, drain;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int n_chunks = a.K / 64;
  volatile int* abort = &abort_flag;

  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kCStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(&tfull, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) { tmem_alloc(&tmem_base, G::kTmemCols); tmem_relinquish(); }
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t filled = 0, filled_parity = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % kCStages;
        const uint32_t ph = (uint32_t)(c / kCStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort, a.status, a.wait_ns)) break;
        uint8_t* sa = base + s * G::kStage;
        mbar_arrive_expect_tx(&full[s], G::kStage);
        tma_load_2d(sa, &tm_x, c * 64, tile * kCTile, &full[s]);
        for (int p = 0; p < G::kNParts; ++p)
          tma_load_2d(sa + G::kA + p * (G::kN * 128), &tm_w, c * 64, p * G::kN, &full[s]);
        filled |= 1u << s;
        filled_parity = (filled_parity & ~(1u << s)) | (ph << s);
      }
      // no load of this CTA may still be landing when it exits
      for (int s = 0; s < kCStages; ++s)
        if (filled & (1u << s)) mbar_drain(&full[s], (filled_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kCTile, G::kN);
      bool ok = true;
      for (int c = 0; c < n_chunks && ok; ++c) {
        const int s = c % kCStages;
        ok = mbar_wait(&full[s], (uint32_t)(c / kCStages) & 1u, abort, a.status, a.wait_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(base + s * G::kStage);
#pragma unroll
        for (int k = 0; k < 4; ++k) {                       // 16-element K-steps of the chunk
          const uint64_t ad = sdesc_sw128(sa + k * 32, 16, 1024);
#pragma unroll
          for (int p = 0; p < G::kNParts; ++p) {
            const uint64_t bd = sdesc_sw128(sa + G::kA + p * (G::kN * 128) + k * 32, 16, 1024);
            umma_bf16(tmem + p * G::kN, ad, bd, idesc, (c > 0 || k > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(&tfull);
      // every MMA this thread issued has completed before the CTA frees TMEM and exits
      umma_commit(&drain);
      mbar_drain(&drain, 0);
    }
  } else {
    // ------------------- epilogue (warps 2..5): quantise + append -------------------
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    const int j = tile * kCTile + row;
    int wok = 1;
    if (lane == 0) wok = mbar_wait(&tfull, 0, abort, a.status, a.wait_ns) ? 1 : 0;
    wok = __shfl_sync(0xffffffffu, wok, 0);
    if (wok) {
      tc_fence_after();
      int64_t dst = -1;
      if (j < a.n_entries) {
        dst = a.dst_row[j];
        if (dst < 0 || dst >= a.cap) {
          report(a.status, CSA2_ERR_CAPACITY);
          dst = -1;
        }
      }
      const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
#pragma unroll 1
      for (int g = 0; g < D / 16; ++g) {
        float v[16];
        tmem_ld16(tmem + lane_base + g * 16, v);            // whole warp
        if (dst >= 0) {
          uint32_t packed[2];
          const uint32_t sc = quantize16(v, packed);
          *reinterpret_cast<uint2*>(a.codes + dst * (int64_t)(D / 2) + g * 8) = make_uint2(packed[0], packed[1]);
          a.scales[dst * (int64_t)(D / 16) + g] = (uint8_t)sc;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 compress_encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// bf16 [rows][cols] map, boxes of 64 columns x box_rows rows, 128-byte swizzle, zero fill
bool compress_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
  auto fn = compress_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t compress_launch(const uint16_t* x, const uint16_t* w_t, const CompressArgs& a,
                            cudaStream_t st) {
  using G = CGeo<D>;
  CUtensorMap tm_x, tm_w;
  if (!compress_map(&tm_x, x, a.n_entries, a.K, kCTile)) return checked(cudaErrorInvalidValue);
  if (!compress_map(&tm_w, w_t, D, a.K, G::kN)) return checked(cudaErrorInvalidValue);
  cudaError_t e = checked(cudaFuncSetAttribute(compress_kernel<D>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem));
  if (e != cudaSuccess) return e;
  return launch_pdl(compress_kernel<D>, dim3((a.n_entries + kCTile - 1) / kCTile), dim3(kCThreads),
                    (size_t)G::kSmem, st, tm_x, tm_w, a);
}

}  // namespace
}  // namespace csa2

extern "C" csa2_status_t csa2_compress_append(const uint16_t* x, int32_t n_entries, int32_t m,
                                              int32_t D_in, const uint16_t* w_t, int32_t D,
                                              const int64_t* dst_row, uint8_t* kv_codes,
                                              uint8_t* kv_scales, int64_t cap_rows,
                                              void* workspace, size_t ws_bytes, void* stream) {
  using namespace csa2;
  if (n_entries < 0 || m < 1 || D_in < 1 || cap_rows <= 0) return CSA2_ERR_INVALID_ARG;
  if (D != 128 && D != 256 && D != 512) return CSA2_ERR_UNSUPPORTED;
  const int64_t K = (int64_t)m * D_in;
  if (K % 64 != 0 || K > (1 << 20)) return CSA2_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < CSA2_STATUS_BYTES) return CSA2_ERR_CAPACITY;
  if (n_entries == 0) return CSA2_OK;
  if (!x || !w_t || !dst_row || !kv_codes || !kv_scales) return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(w_t) & 15) ||
      (reinterpret_cast<uintptr_t>(kv_codes) & 7))
    return CSA2_ERR_INVALID_ARG;
  CompressArgs a{};
  a.n_entries = n_entries;
  a.K = (int)K;
  a.dst_row = dst_row;
  a.codes = kv_codes;
  a.scales = kv_scales;
  a.cap = cap_rows;
  a.status = static_cast<int*>(workspace);
  a.wait_ns = wait_limit_ns();
  cudaStream_t st = (cudaStream_t)stream;
  const cudaError_t e = D == 128   ? compress_launch<128>(x, w_t, a, st)
                        : D == 256 ? compress_launch<256>(x, w_t, a, st)
                                   : compress_launch<512>(x, w_t, a, st);
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
