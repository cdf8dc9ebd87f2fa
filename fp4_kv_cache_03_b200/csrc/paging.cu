// Paged-cache helpers: cache rows of (sequence, position) pairs, and row gathers / scatters
// for moving a sequence's cached entries out of the cache and back (export and import of
// the persistent global cache: aprilzz.com "DeepSeek V4.1 Flash 发布…", section "FP4 KV 与部署
// 层的几个改动").
#include "common.cuh"

namespace csa2 {
namespace {

__global__ void __launch_bounds__(256) cache_rows_kernel(csa2_seqs_t s, const int32_t* seq,
                                                         const int32_t* pos, int n, int64_t* rows) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= n) return;
  const int sq = seq[i];
  const int p = pos[i];
  rows[i] = (sq < 0 || sq >= s.num_seqs || p < 0 || (s.block_table && (p >> 7) >= s.max_pages))
                ? -1
                : entry_row(s.seq_start, s.block_table, s.max_pages, sq, p);
}

// one warp per row, 4-byte words (row_bytes a multiple of 4)
template <bool kGather>
__global__ void __launch_bounds__(256) move_rows_kernel(const uint8_t* src, uint8_t* dst,
                                                        int64_t cap, int row_bytes,
                                                        const int64_t* rows, int n) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= n) return;
  const int64_t r = rows[i];
  const bool ok = r >= 0 && r < cap;
  const int words = row_bytes >> 2;
  if (kGather) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src + (ok ? r : 0) * (int64_t)row_bytes);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst + (int64_t)i * row_bytes);
    for (int k = lane; k < words; k += 32) d[k] = ok ? s[k] : 0u;
  } else if (ok) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src + (int64_t)i * row_bytes);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst + r * (int64_t)row_bytes);
    for (int k = lane; k < words; k += 32) d[k] = s[k];
  }
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" csa2_status_t csa2_cache_rows(csa2_seqs_t seqs, const int32_t* seq, const int32_t* pos,
                                         int32_t n, int64_t* rows, void* stream) {
  if (n < 0 || seqs.num_seqs < 1 || (seqs.block_table && seqs.max_pages < 1)) return CSA2_ERR_INVALID_ARG;
  if (n == 0) return CSA2_OK;
  if (!seq || !pos || !rows || (!seqs.seq_start && !seqs.block_table)) return CSA2_ERR_INVALID_ARG;
  return launch_pdl(cache_rows_kernel, dim3((n + 255) / 256), dim3(256), 0, (cudaStream_t)stream,
                    seqs, seq, pos, n, rows) == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

extern "C" csa2_status_t csa2_gather_rows(const uint8_t* table, int64_t cap_rows, int32_t row_bytes,
                                          const int64_t* rows, int32_t n, uint8_t* dst,
                                          void* stream) {
  if (n < 0 || row_bytes < 4 || (row_bytes & 3) || cap_rows < 0) return CSA2_ERR_INVALID_ARG;
  if (n == 0) return CSA2_OK;
  if (!table || !rows || !dst || (reinterpret_cast<uintptr_t>(table) & 15) ||
      (reinterpret_cast<uintptr_t>(dst) & 15))
    return CSA2_ERR_INVALID_ARG;
  return launch_pdl(move_rows_kernel<true>, dim3((n + 7) / 8), dim3(256), 0, (cudaStream_t)stream,
                    table, dst, cap_rows, (int)row_bytes, rows, (int)n) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

extern "C" csa2_status_t csa2_scatter_rows(const uint8_t* src, int32_t row_bytes, const int64_t* rows,
                                           int32_t n, uint8_t* table, int64_t cap_rows,
                                           void* stream) {
  if (n < 0 || row_bytes < 4 || (row_bytes & 3) || cap_rows < 0) return CSA2_ERR_INVALID_ARG;
  if (n == 0) return CSA2_OK;
  if (!table || !rows || !src || (reinterpret_cast<uintptr_t>(table) & 15) ||
      (reinterpret_cast<uintptr_t>(src) & 15))
    return CSA2_ERR_INVALID_ARG;
  return launch_pdl(move_rows_kernel<false>, dim3((n + 7) / 8), dim3(256), 0, (cudaStream_t)stream,
                    src, table, cap_rows, (int)row_bytes, rows, (int)n) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}
