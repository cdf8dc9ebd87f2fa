// Status-word helpers and device queries of the CSA2 C ABI.
#include "common.cuh"

#include <atomic>

namespace csa2 {
namespace {
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
std::atomic<uint64_t> g_wait_ns{kWaitLimitNs};
}
void note_cuda_error(cudaError_t e) { g_last_cuda_error = e; }
uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
}  // namespace csa2

extern "C" uint64_t csa2_set_wait_limit_ns(uint64_t ns) {
  return csa2::g_wait_ns.exchange(ns == 0 ? csa2::kWaitLimitNs : ns, std::memory_order_relaxed);
}

extern "C" const char* csa2_last_cuda_error(void) {
  return cudaGetErrorString(csa2::g_last_cuda_error);
}

extern "C" csa2_status_t csa2_status_reset(void* workspace, void* stream) {
  if (!workspace) return CSA2_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(int), (cudaStream_t)stream) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

extern "C" csa2_status_t csa2_status_fetch(const void* workspace, void* stream) {
  if (!workspace) return CSA2_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream) !=
      cudaSuccess)
    return CSA2_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return CSA2_ERR_CUDA;
  return (v >= CSA2_OK && v <= CSA2_ERR_TIMEOUT) ? (csa2_status_t)v : CSA2_ERR_CUDA;
}

extern "C" const char* csa2_status_string(csa2_status_t s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "unsupported shape";
    case CSA2_ERR_CAPACITY: return "capacity exceeded (workspace or cache rows)";
    case CSA2_ERR_CUDA: return "CUDA runtime error";
    case CSA2_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

extern "C" int32_t csa2_device_sms(void) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

extern "C" csa2_status_t csa2_layer_step(csa2_mode_t mode, int32_t num_q, const uint8_t* kv_codes,
                                         const uint8_t* kv_scales, int64_t cap_rows,
                                         csa2_seqs_t seqs, int32_t topk, int32_t* indices,
                                         const csa2_indexer_t* ix, const csa2_attention_t* at,
                                         void* stream) {
  if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
    return CSA2_ERR_INVALID_ARG;
  if (!at || (mode != CSA2_MODE_REUSE && !ix)) return CSA2_ERR_INVALID_ARG;
  csa2_status_t st = CSA2_OK;
  if (mode != CSA2_MODE_REUSE && ix->e4m3 != 0 && ix->e4m3 != 1) return CSA2_ERR_INVALID_ARG;
  if (mode == CSA2_MODE_FULL && !ix->e4m3) {
    st = csa2_index_full(static_cast<const uint16_t*>(ix->qI), ix->w, num_q, ix->H_I, ix->d_I,
                         static_cast<const uint16_t*>(ix->idx_k), cap_rows, seqs, ix->q_visible,
                         ix->max_visible, topk, indices, ix->pool_blocks, ix->block, ix->pool,
                         ix->workspace, ix->ws_bytes, stream);
  } else if (mode == CSA2_MODE_FULL) {
    st = csa2_index_full_e4m3(static_cast<const uint8_t*>(ix->qI), ix->w, num_q, ix->H_I, ix->d_I,
                              static_cast<const uint8_t*>(ix->idx_k), cap_rows, seqs, ix->q_visible,
                              ix->max_visible, topk, indices, ix->pool_blocks, ix->block, ix->pool,
                              ix->workspace, ix->ws_bytes, stream);
  } else if (mode == CSA2_MODE_REINDEX && !ix->e4m3) {
    st = csa2_index_pool(static_cast<const uint16_t*>(ix->qI), ix->w, num_q, ix->H_I, ix->d_I,
                         static_cast<const uint16_t*>(ix->idx_k), cap_rows, seqs, ix->q_visible,
                         ix->pool, ix->pool_blocks, ix->block, topk, indices, ix->workspace,
                         ix->ws_bytes, stream);
  } else if (mode == CSA2_MODE_REINDEX) {
    st = csa2_index_pool_e4m3(static_cast<const uint8_t*>(ix->qI), ix->w, num_q, ix->H_I, ix->d_I,
                              static_cast<const uint8_t*>(ix->idx_k), cap_rows, seqs, ix->q_visible,
                              ix->pool, ix->pool_blocks, ix->block, topk, indices, ix->workspace,
                              ix->ws_bytes, stream);
  }
  if (st != CSA2_OK) return st;
  return csa2_sparse_attn(at->q, num_q, at->H, at->D, kv_codes, kv_scales, cap_rows, seqs,
                          indices, topk, at->swa_kv, at->swa_rows, at->swa_start, at->q_pos,
                          at->window, at->swa_ring, at->softmax_scale, at->out, at->lse, mode, at->kv_stash,
                          at->stash_bytes, at->workspace, at->ws_bytes, stream);
}
