// a2-a5: the CSA2 indexer on B200.
//   Full (csa2_index_full):   score every visible entry, Top-K positions, and (decoder's
//                             first Full layer) the candidate pool of top blocks.
//   Reindex (csa2_index_pool): score only the pool's positions with this layer's own
//                             indexer Q, Top-K of those.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", section "CSA2：在层的维度上共享缓存"
// (Full/Reindex/Reuse, Top-512, pool of <= 2048 blocks x 8); gkm0120.cn "技术调研报告"
// §2.2.2 (modes table) and §2.2.3 (hierarchical sparse indexer).
//
// Score kernel: persistent, warp-specialised.  Warp 0 streams 128-entry tiles of the
// bf16 indexer K with TMA (128-byte swizzle) into a ring of shared-memory stages, warp 1
// issues tcgen05.mma (M = 128 entries, N = padded indexer heads, K = d_I) into a
// double-buffered TMEM accumulator, warps 2-5 read it back (tcgen05.ld), apply
// ReLU * w, sum the heads, and write one 32-bit ordered key per entry (plus the block
// maximum for the pool).  Selection: exact multi-CTA radix select over the keys
// (11/11/10-bit digits, per-row histograms), then an order-preserving compaction that
// breaks ties by lowest position.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kTileRows = 128;       // entries per MMA tile (M)
constexpr int kScoreThreads = 192;   // 6 warps
constexpr int kSelThreads = 256;
constexpr int kSelChunk = 8192;      // keys per select CTA
constexpr int kHistBins = 2048;
constexpr int kPasses = 3;           // digits: bits 31..21, 20..10, 9..0

// ---------------------------------------------------------------------------------
// visibility
// ---------------------------------------------------------------------------------
struct Seqs {
  const int64_t* seq_start;
  const int32_t* seq_len;
  const int32_t* q_visible;
  int q_per_seq;
  int max_visible;
  int* status;
};

__device__ __forceinline__ int visible_of(const Seqs& s, int q) {
  const int seq = q / s.q_per_seq;
  const int len = s.seq_len[seq];
  int v = s.q_visible ? s.q_visible[q] : len;
  if (v < 0) { report(s.status, CSA2_ERR_INVALID_ARG); v = 0; }
  if (v > len) { report(s.status, CSA2_ERR_INVALID_ARG); v = len; }
  if (v > s.max_visible) { report(s.status, CSA2_ERR_CAPACITY); v = s.max_visible; }
  return v;
}

// ---------------------------------------------------------------------------------
// score kernel
// ---------------------------------------------------------------------------------
struct ScoreArgs {
  Seqs seqs;
  const float* w;
  int num_q, H_I, d_I, n_pad;      // n_pad: MMA N (multiple of 16)
  int tiles_per_q;                 // host bound on tiles of one query
  int stages;
  // Reindex: tiles are 16 pool blocks of 8 rows each
  const int32_t* pool;
  int pool_blocks;
  // outputs
  uint32_t* keys;
  int64_t key_stride;
  uint32_t* bkeys;                 // block-max keys (Full with pool) or null
  int64_t bkey_stride;
  int block;                       // block size for bkeys (power of two <= 32)
};

struct ScoreSmem {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort;
};

template <bool kGather>
__device__ __forceinline__ bool tile_active(const ScoreArgs& a, int q, int t, int vis) {
  if (kGather) {
    const int b0 = t * 16;
    return b0 < a.pool_blocks && a.pool[(int64_t)q * a.pool_blocks + b0] >= 0;
  }
  return t * kTileRows < vis;
}

template <bool kGather>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                 const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ ScoreSmem ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = a.seqs.status;

  const int halves = a.d_I >> 6;                          // 64-element K chunks
  const uint32_t a_bytes = (uint32_t)halves * kTileRows * 128;
  const uint32_t b_half = (uint32_t)a.n_pad * 128;
  const uint32_t stage_bytes = a_bytes + (uint32_t)halves * b_half;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int S = a.stages;
  const int n_items = a.num_q * a.tiles_per_q;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&ss.full[s], 1); mbar_init(&ss.empty[s], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&ss.tfull[i], 1); mbar_init(&ss.tempty[i], 4); }
    ss.abort = 0;
    fence_barrier_init();
  }
  // padding rows of the B operand (heads >= H_I) must read as zero; TMA never writes them
  for (int s = 0; s < S; ++s) {
    uint8_t* b = base + (size_t)s * stage_bytes + a_bytes;
    for (uint32_t i = threadIdx.x * 16; i < (uint32_t)halves * b_half; i += blockDim.x * 16)
      *reinterpret_cast<uint4*>(b + i) = make_uint4(0, 0, 0, 0);
  }
  if (warp == 1) { tmem_alloc(&ss.tmem_base, a.n_pad * 2 < 32 ? 32 : a.n_pad * 2); tmem_relinquish(); }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
      int stage = 0;
      uint32_t phase = 0;
      for (int it = blockIdx.x; it < n_items && !*abort; it += gridDim.x) {
        const int q = it / a.tiles_per_q, t = it % a.tiles_per_q;
        const int vis = visible_of(a.seqs, q);
        if (!tile_active<kGather>(a, q, t, vis)) continue;
        if (!mbar_wait(&ss.empty[stage], phase ^ 1, abort, status)) break;
        uint8_t* sa = base + (size_t)stage * stage_bytes;
        uint8_t* sb = sa + a_bytes;
        const int64_t row0 = a.seqs.seq_start[q / a.seqs.q_per_seq];
        uint32_t bytes = (uint32_t)halves * (uint32_t)a.H_I * 128;
        int32_t blk_row[16];
        if (kGather) {
          const int32_t* pb = a.pool + (int64_t)q * a.pool_blocks + t * 16;
          for (int i = 0; i < 16; ++i) {
            const int j = (t * 16 + i < a.pool_blocks) ? pb[i] : -1;
            blk_row[i] = (j >= 0) ? (int32_t)(row0 + 8 * (int64_t)j) : -1;
            if (j >= 0) bytes += (uint32_t)halves * 8 * 128;
          }
        } else {
          bytes += a_bytes;
        }
        mbar_arrive_expect_tx(&ss.full[stage], bytes);
        for (int h = 0; h < halves; ++h) {
          tma_load_2d(sb + h * b_half, &tm_q, h * 64, q * a.H_I, &ss.full[stage]);
          if (kGather) {
            for (int i = 0; i < 16; ++i)
              if (blk_row[i] >= 0)
                tma_load_2d(sa + h * (kTileRows * 128) + i * 1024, &tm_k, h * 64, blk_row[i],
                            &ss.full[stage]);
          } else {
            tma_load_2d(sa + h * (kTileRows * 128), &tm_k, h * 64,
                        (int32_t)(row0 + (int64_t)t * kTileRows), &ss.full[stage]);
          }
        }
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTileRows, a.n_pad);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int it = blockIdx.x; it < n_items && !*abort; it += gridDim.x) {
        const int q = it / a.tiles_per_q, t = it % a.tiles_per_q;
        const int vis = visible_of(a.seqs, q);
        if (!tile_active<kGather>(a, q, t, vis)) continue;
        if (!mbar_wait(&ss.tempty[acc], acc_phase ^ 1, abort, status)) break;
        if (!mbar_wait(&ss.full[stage], phase, abort, status)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
        const uint32_t sb = sa + a_bytes;
        const uint32_t d = tmem + (uint32_t)(acc * a.n_pad);
        for (int k = 0; k < (a.d_I >> 4); ++k) {
          const int h = k >> 2, sub = k & 3;
          const uint64_t ad = sdesc_sw128(sa + h * (kTileRows * 128) + sub * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sb + h * b_half + sub * 32, 16, 1024);
          umma_bf16(d, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&ss.empty[stage]);
        umma_commit(&ss.tfull[acc]);
        if (++stage == S) { stage = 0; phase ^= 1; }
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // ------------------------------ epilogue (warps 2..5) ------------------------------
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;          // entry (or slot) within the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = blockIdx.x; it < n_items && !*abort; it += gridDim.x) {
      const int q = it / a.tiles_per_q, t = it % a.tiles_per_q;
      const int vis = visible_of(a.seqs, q);
      const bool active = tile_active<kGather>(a, q, t, vis);
      const int e = t * kTileRows + row;       // position (Full) or slot (Reindex)
      if (!active) {
        if (kGather && e < a.pool_blocks * 8) a.keys[(int64_t)q * a.key_stride + e] = 0u;
        continue;
      }
      if (!mbar_wait(&ss.tfull[acc], acc_phase, abort, status)) break;
      tc_fence_after();
      float v[32];
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * a.n_pad);
      tmem_ld16(taddr, v);
      if (a.n_pad > 16) tmem_ld16(taddr + 16, v + 16);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ss.tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }

      const float* wq = a.w + (int64_t)q * a.H_I;
      float s = 0.0f;
      for (int h = 0; h < a.H_I; ++h) s = fmaf(__ldg(wq + h), fmaxf(v[h], 0.0f), s);
      uint32_t key = ordered_key(s);
      if (kGather) {
        if (e < a.pool_blocks * 8) {
          const int j = a.pool[(int64_t)q * a.pool_blocks + (e >> 3)];
          const int64_t pos = 8 * (int64_t)j + (e & 7);
          if (j < 0 || pos >= vis) key = 0u;
          a.keys[(int64_t)q * a.key_stride + e] = key;
        }
      } else {
        if (e >= vis) key = 0u;
        if (e < vis) a.keys[(int64_t)q * a.key_stride + e] = key;
        if (a.bkeys) {
          uint32_t m = key;
          for (int o = 1; o < a.block; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
          if ((e & (a.block - 1)) == 0 && e < vis)
            a.bkeys[(int64_t)q * a.bkey_stride + e / a.block] = m;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.n_pad * 2 < 32 ? 32 : a.n_pad * 2);
  }
}

// ---------------------------------------------------------------------------------
// exact Top-K selection over 32-bit keys (0 = not a candidate)
// ---------------------------------------------------------------------------------
struct SelProblem {
  const uint32_t* keys;
  int64_t stride;
  int num_rows;
  int k;
  int32_t* out;
  int64_t out_stride;
  int len_mode;       // 0: visible positions, 1: visible blocks, 2: fixed slot count
  int block;          // len_mode 1: block size
  int fixed_len;      // len_mode 2
  const int32_t* pool;  // len_mode 2: output = 8 * pool[slot / 8] + slot % 8
  int pool_blocks;
  uint32_t* hist;     // [num_rows][kPasses][kHistBins]
  uint32_t* ccnt;     // [num_rows][chunks][2]
  int chunks;
};
struct SelArgs {
  SelProblem p[2];
  Seqs seqs;
};

__device__ __forceinline__ int row_len(const SelProblem& p, const Seqs& s, int r) {
  if (p.len_mode == 2) return p.fixed_len;
  const int v = visible_of(s, r);
  return p.len_mode == 0 ? v : (v + p.block - 1) / p.block;
}

constexpr int pass_shift(int p) { return p == 0 ? 21 : (p == 1 ? 10 : 0); }
constexpr int pass_bins(int p) { return p == 2 ? 1024 : 2048; }

struct Resolved {
  uint32_t prefix;   // key bits fixed by the resolved digits
  int krem;          // how many still to take among keys matching the prefix
  int n_valid;       // candidate count of the row
  int take_all;      // n_valid <= k: every candidate is selected
};

// Block-wide: reconstruct the threshold digits of passes [0, npass) from the row's
// histograms.  All threads return the same value.
__device__ Resolved resolve(const uint32_t* hist_row, int k, int npass) {
  __shared__ uint32_t warp_sum[kSelThreads / 32];
  __shared__ Resolved res;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // total candidates = sum of the pass-0 histogram
  uint32_t local = 0;
  for (int b = tid; b < kHistBins; b += kSelThreads) local += hist_row[b];
  for (int o = 16; o; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (lane == 0) warp_sum[wid] = local;
  __syncthreads();
  if (tid == 0) {
    uint32_t n = 0;
    for (int i = 0; i < kSelThreads / 32; ++i) n += warp_sum[i];
    res.n_valid = (int)n;
    res.take_all = (int)(n <= (uint32_t)k);
    res.prefix = 0u;
    res.krem = k;
  }
  __syncthreads();
  if (res.take_all) return res;
  for (int p = 0; p < npass; ++p) {
    const int bins = pass_bins(p);
    const int per = bins / kSelThreads;          // 8 or 4 bins per thread, contiguous
    const uint32_t* h = hist_row + p * kHistBins;
    uint32_t c[8];
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) { c[i] = h[tid * per + i]; mine += c[i]; }
    // suffix sum over threads: S(t) = sum_{t' >= t} mine(t')
    uint32_t incl = mine;                        // inclusive scan from high lanes down
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    __syncthreads();
    if (lane == 0) warp_sum[wid] = incl;         // lane 0 holds the warp total
    __syncthreads();
    uint32_t above = 0;                          // totals of warps above this one
    for (int i = wid + 1; i < kSelThreads / 32; ++i) above += warp_sum[i];
    const uint32_t S = incl + above;             // candidates in bins >= my first bin
    const uint32_t krem = (uint32_t)res.krem;
    const uint32_t S_next = S - mine;            // candidates in bins above my range
    __syncthreads();
    if (S >= krem && S_next < krem) {
      uint32_t run = S_next;
      for (int i = per - 1; i >= 0; --i) {
        if (run + c[i] >= krem) {
          res.prefix |= (uint32_t)(tid * per + i) << pass_shift(p);
          res.krem = (int)(krem - run);
          break;
        }
        run += c[i];
      }
    }
    __syncthreads();
  }
  return res;
}

__device__ __forceinline__ bool matches(uint32_t key, uint32_t prefix, int npass) {
  if (npass == 0) return true;
  const uint32_t mask = ~((1u << pass_shift(npass - 1)) - 1u);
  return (key & mask) == prefix;
}

template <int kPass>
__global__ void __launch_bounds__(kSelThreads) sel_hist_kernel(const SelArgs a) {
  const SelProblem& p = a.p[blockIdx.z];
  const int r = blockIdx.y, c = blockIdx.x;
  if (r >= p.num_rows || c >= p.chunks) return;
  const int len = row_len(p, a.seqs, r);
  const int lo = c * kSelChunk, hi = min(len, lo + kSelChunk);
  if (lo >= hi) return;
  uint32_t* hist_row = p.hist + (int64_t)r * kPasses * kHistBins;
  uint32_t prefix = 0;
  if (kPass > 0) {
    const Resolved rs = resolve(hist_row, p.k, kPass);
    if (rs.take_all) return;
    prefix = rs.prefix;
  }
  __shared__ uint32_t h[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) h[i] = 0;
  __syncthreads();
  const uint32_t* keys = p.keys + (int64_t)r * p.stride;
  const uint32_t dmask = (uint32_t)pass_bins(kPass) - 1u;
  for (int i = lo + threadIdx.x; i < hi; i += kSelThreads) {
    const uint32_t key = keys[i];
    if (key == 0u || !matches(key, prefix, kPass)) continue;
    atomicAdd(&h[(key >> pass_shift(kPass)) & dmask], 1u);
  }
  __syncthreads();
  uint32_t* out = hist_row + kPass * kHistBins;
  for (int i = threadIdx.x; i < pass_bins(kPass); i += kSelThreads)
    if (h[i]) atomicAdd(out + i, h[i]);
}

// threshold key T and how many keys equal to T to take
__device__ __forceinline__ void threshold(const Resolved& rs, uint32_t& T, int& need_eq) {
  if (rs.take_all) { T = 0u; need_eq = 0; }   // every key > 0 is selected
  else { T = rs.prefix; need_eq = rs.krem; }
}

__global__ void __launch_bounds__(kSelThreads) sel_count_kernel(const SelArgs a) {
  const SelProblem& p = a.p[blockIdx.z];
  const int r = blockIdx.y, c = blockIdx.x;
  if (r >= p.num_rows || c >= p.chunks) return;
  const int len = row_len(p, a.seqs, r);
  const int lo = c * kSelChunk, hi = min(len, lo + kSelChunk);
  if (lo >= hi) return;
  const Resolved rs = resolve(p.hist + (int64_t)r * kPasses * kHistBins, p.k, kPasses);
  uint32_t T; int need_eq;
  threshold(rs, T, need_eq);
  const uint32_t* keys = p.keys + (int64_t)r * p.stride;
  uint32_t gt = 0, eq = 0;
  for (int i = lo + threadIdx.x; i < hi; i += kSelThreads) {
    const uint32_t key = keys[i];
    gt += (key > T);
    eq += (key == T && key != 0u);
  }
  __shared__ uint32_t sg[kSelThreads / 32], se[kSelThreads / 32];
  for (int o = 16; o; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if ((threadIdx.x & 31) == 0) { sg[threadIdx.x >> 5] = gt; se[threadIdx.x >> 5] = eq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t G = 0, E = 0;
    for (int i = 0; i < kSelThreads / 32; ++i) { G += sg[i]; E += se[i]; }
    uint32_t* cc = p.ccnt + ((int64_t)r * p.chunks + c) * 2;
    cc[0] = G;
    cc[1] = E;
  }
}

// exclusive block scan of one value per thread; returns the block total in *total
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* total) {
  __shared__ uint32_t ws[kSelThreads / 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) ws[wid] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
  for (int i = 0; i < kSelThreads / 32; ++i) {
    if (i < wid) before += ws[i];
    tot += ws[i];
  }
  *total = tot;
  return before + x - v;
}

__global__ void __launch_bounds__(kSelThreads) sel_write_kernel(const SelArgs a) {
  const SelProblem& p = a.p[blockIdx.z];
  const int r = blockIdx.y, c = blockIdx.x;
  if (r >= p.num_rows || c >= p.chunks) return;
  const int len = row_len(p, a.seqs, r);
  const int lo = c * kSelChunk, hi = min(len, lo + kSelChunk);
  int32_t* out = p.out + (int64_t)r * p.out_stride;
  if (lo >= hi && c != 0) return;
  const Resolved rs = resolve(p.hist + (int64_t)r * kPasses * kHistBins, p.k, kPasses);
  if (c == 0) {  // -1 padding after the selected entries
    const int n_sel = min(p.k, rs.n_valid);
    for (int i = n_sel + threadIdx.x; i < p.k; i += kSelThreads) out[i] = -1;
  }
  if (lo >= hi) return;
  uint32_t T; int need_eq;
  threshold(rs, T, need_eq);
  // selections of the chunks before this one
  uint32_t gt_before = 0, eq_before = 0;
  const uint32_t* cc = p.ccnt + (int64_t)r * p.chunks * 2;
  for (int i = 0; i < c; ++i) { gt_before += cc[2 * i]; eq_before += cc[2 * i + 1]; }
  const uint32_t eq_take_before = min(eq_before, (uint32_t)need_eq);
  const uint32_t take_eq = (uint32_t)need_eq - eq_take_before;   // still to take, in order
  // this thread's contiguous segment
  const int per = kSelChunk / kSelThreads;
  const int s0 = lo + threadIdx.x * per, s1 = min(hi, s0 + per);
  const uint32_t* keys = p.keys + (int64_t)r * p.stride;
  uint32_t my_gt = 0, my_eq = 0;
  for (int i = s0; i < s1; ++i) {
    const uint32_t key = keys[i];
    my_gt += (key > T);
    my_eq += (key == T && key != 0u);
  }
  uint32_t tot;
  const uint32_t eq_rank = block_excl_scan(my_eq, &tot);   // eq keys before my segment
  const uint32_t my_take_eq = eq_rank >= take_eq ? 0u : min(my_eq, take_eq - eq_rank);
  const uint32_t pos0 = block_excl_scan(my_gt + my_take_eq, &tot);
  uint32_t o = gt_before + eq_take_before + pos0, taken_eq = 0;
  for (int i = s0; i < s1; ++i) {
    const uint32_t key = keys[i];
    bool sel = key > T;
    if (!sel && key == T && key != 0u) { sel = taken_eq < my_take_eq; ++taken_eq; }
    if (sel) {
      int32_t v = i;
      if (p.len_mode == 2) v = 8 * p.pool[(int64_t)r * p.pool_blocks + (i >> 3)] + (i & 7);
      out[o++] = v;
    }
  }
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 map over a row-major [rows][cols] array, box = 64 columns x box_rows rows,
// 128-byte swizzle, out-of-bounds reads as zero.
bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t keys, bkeys, hist, ccnt, total;
  int64_t key_stride, bkey_stride;
  int chunks_pos, chunks_blk;
};

WsLayout layout_of(int num_q, int64_t row_len, int64_t brow_len) {
  WsLayout L{};
  L.key_stride = (row_len + 63) / 64 * 64;
  L.bkey_stride = (brow_len + 63) / 64 * 64;
  L.chunks_pos = (int)std::max<int64_t>(1, (row_len + kSelChunk - 1) / kSelChunk);
  L.chunks_blk = (int)std::max<int64_t>(1, (brow_len + kSelChunk - 1) / kSelChunk);
  size_t off = CSA2_STATUS_BYTES;
  L.keys = off;
  off = align256(off + (size_t)num_q * L.key_stride * 4);
  L.bkeys = off;
  off = align256(off + (size_t)num_q * L.bkey_stride * 4);
  L.hist = off;
  off = align256(off + (size_t)2 * num_q * kPasses * kHistBins * 4);
  L.ccnt = off;
  off = align256(off + (size_t)num_q * (L.chunks_pos + L.chunks_blk) * 2 * 4);
  L.total = off;
  return L;
}

bool pow2_le32(int b) { return b >= 1 && b <= 32 && (b & (b - 1)) == 0; }

// shared driver for Full (kGather = false) and Reindex (kGather = true)
template <bool kGather>
csa2_status_t run_index(const uint16_t* qI, const float* w, int num_q, int H_I, int d_I,
                        const uint16_t* idx_k, int64_t cap_rows, csa2_seqs_t seqs,
                        const int32_t* q_visible, int max_visible, int topk, int32_t* indices,
                        int pool_blocks, int block, int32_t* pool_out, const int32_t* pool_in,
                        void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int64_t row_len = kGather ? (int64_t)pool_blocks * 8 : max_visible;
  const int64_t brow_len = (!kGather && pool_blocks > 0) ? (max_visible + block - 1) / block : 0;
  const WsLayout L = layout_of(num_q, row_len, brow_len);
  if (ws_bytes < L.total) return CSA2_ERR_CAPACITY;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(wsb);

  Seqs sq{seqs.seq_start, seqs.seq_len, q_visible, seqs.q_per_seq, max_visible, status};

  // histograms start at zero
  if (cudaMemsetAsync(wsb + L.hist, 0, L.ccnt - L.hist, stream) != cudaSuccess) return CSA2_ERR_CUDA;

  // ---- scores ----
  CUtensorMap tm_k, tm_q;
  const int box_rows = kGather ? 8 : kTileRows;
  if (!make_map(&tm_k, idx_k, cap_rows, d_I, box_rows)) return CSA2_ERR_CUDA;
  if (!make_map(&tm_q, qI, (int64_t)num_q * H_I, d_I, H_I)) return CSA2_ERR_CUDA;
  ScoreArgs sa{};
  sa.seqs = sq;
  sa.w = w;
  sa.num_q = num_q;
  sa.H_I = H_I;
  sa.d_I = d_I;
  sa.n_pad = H_I <= 16 ? 16 : 32;
  sa.tiles_per_q = (int)((row_len + kTileRows - 1) / kTileRows);
  sa.pool = pool_in;
  sa.pool_blocks = pool_blocks;
  sa.keys = reinterpret_cast<uint32_t*>(wsb + L.keys);
  sa.key_stride = L.key_stride;
  sa.bkeys = brow_len > 0 ? reinterpret_cast<uint32_t*>(wsb + L.bkeys) : nullptr;
  sa.bkey_stride = L.bkey_stride;
  sa.block = block;
  const uint32_t stage_bytes = (uint32_t)(d_I / 64) * (kTileRows * 128 + sa.n_pad * 128);
  sa.stages = std::min<int>(8, (int)((200u * 1024u) / stage_bytes));
  const size_t smem = (size_t)sa.stages * stage_bytes + 1024;
  const int n_items = num_q * sa.tiles_per_q;
  if (n_items > 0) {
    const int sms = device_sms();
    if (sms <= 0) return CSA2_ERR_CUDA;
    const int grid = std::min(n_items, sms);
    auto kern = score_kernel<kGather>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return CSA2_ERR_CUDA;
    kern<<<grid, kScoreThreads, smem, stream>>>(tm_k, tm_q, sa);
    if (cudaGetLastError() != cudaSuccess) return CSA2_ERR_CUDA;
  }

  // ---- selection ----
  SelArgs sel{};
  sel.seqs = sq;
  SelProblem& P = sel.p[0];
  P.keys = sa.keys;
  P.stride = L.key_stride;
  P.num_rows = num_q;
  P.k = topk;
  P.out = indices;
  P.out_stride = topk;
  P.len_mode = kGather ? 2 : 0;
  P.fixed_len = (int)row_len;
  P.pool = pool_in;
  P.pool_blocks = pool_blocks;
  P.hist = reinterpret_cast<uint32_t*>(wsb + L.hist);
  P.ccnt = reinterpret_cast<uint32_t*>(wsb + L.ccnt);
  P.chunks = L.chunks_pos;
  int nprob = 1;
  if (brow_len > 0) {
    SelProblem& B = sel.p[1];
    B = P;
    B.keys = sa.bkeys;
    B.stride = L.bkey_stride;
    B.k = pool_blocks;
    B.out = pool_out;
    B.out_stride = pool_blocks;
    B.len_mode = 1;
    B.block = block;
    B.pool = nullptr;
    B.hist = P.hist + (size_t)num_q * kPasses * kHistBins;
    B.ccnt = P.ccnt + (size_t)num_q * L.chunks_pos * 2;
    B.chunks = L.chunks_blk;
    nprob = 2;
  }
  const dim3 grid(std::max(L.chunks_pos, nprob == 2 ? L.chunks_blk : 1), num_q, nprob);
  sel_hist_kernel<0><<<grid, kSelThreads, 0, stream>>>(sel);
  sel_hist_kernel<1><<<grid, kSelThreads, 0, stream>>>(sel);
  sel_hist_kernel<2><<<grid, kSelThreads, 0, stream>>>(sel);
  sel_count_kernel<<<grid, kSelThreads, 0, stream>>>(sel);
  sel_write_kernel<<<grid, kSelThreads, 0, stream>>>(sel);
  return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status_t check_common(const uint16_t* qI, const float* w, int num_q, int H_I, int d_I,
                           const uint16_t* idx_k, int64_t cap_rows, const csa2_seqs_t& seqs,
                           int topk, const int32_t* indices, const void* ws) {
  if (num_q < 0 || H_I < 1 || H_I > 32 || (d_I != 64 && d_I != 128)) return CSA2_ERR_UNSUPPORTED;
  if (topk < 1 || topk > 4096) return CSA2_ERR_UNSUPPORTED;
  if (cap_rows <= 0 || cap_rows > 0x7FFFFFFF) return CSA2_ERR_INVALID_ARG;
  if (seqs.num_seqs < 1 || seqs.q_per_seq < 1 ||
      (int64_t)seqs.num_seqs * seqs.q_per_seq != num_q)
    return CSA2_ERR_INVALID_ARG;
  if (num_q == 0) return CSA2_OK;
  if (!qI || !w || !idx_k || !indices || !seqs.seq_start || !seqs.seq_len || !ws)
    return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qI) & 15) || (reinterpret_cast<uintptr_t>(idx_k) & 15) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_index_full_workspace(int32_t num_q, int32_t max_visible, int32_t topk,
                                            int32_t pool_blocks, int32_t block) {
  (void)topk;
  if (num_q < 0 || max_visible < 0 || block < 1) return 0;
  const int64_t brow = pool_blocks > 0 ? ((int64_t)max_visible + block - 1) / block : 0;
  return layout_of(num_q, max_visible, brow).total;
}

extern "C" size_t csa2_index_pool_workspace(int32_t num_q, int32_t pool_blocks, int32_t block,
                                            int32_t topk) {
  (void)topk;
  if (num_q < 0 || pool_blocks < 0 || block < 1) return 0;
  return layout_of(num_q, (int64_t)pool_blocks * block, 0).total;
}

extern "C" csa2_status_t csa2_index_full(const uint16_t* qI, const float* w, int32_t num_q,
                                         int32_t H_I, int32_t d_I, const uint16_t* idx_k,
                                         int64_t cap_rows, csa2_seqs_t seqs,
                                         const int32_t* q_visible, int32_t max_visible,
                                         int32_t topk, int32_t* indices, int32_t pool_blocks,
                                         int32_t block, int32_t* pool, void* workspace,
                                         size_t ws_bytes, void* stream) {
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices,
                                  workspace);
  if (st != CSA2_OK || num_q == 0) return st;
  if (max_visible < 0) return CSA2_ERR_INVALID_ARG;
  if (pool_blocks < 0 || pool_blocks > 8192) return CSA2_ERR_UNSUPPORTED;
  if (pool_blocks > 0 && (!pool || !pow2_le32(block))) return CSA2_ERR_UNSUPPORTED;
  if (pool_blocks == 0) block = 8;
  return run_index<false>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, max_visible,
                          topk, indices, pool_blocks, block, pool, nullptr, workspace, ws_bytes,
                          (cudaStream_t)stream);
}

extern "C" csa2_status_t csa2_index_pool(const uint16_t* qI, const float* w, int32_t num_q,
                                         int32_t H_I, int32_t d_I, const uint16_t* idx_k,
                                         int64_t cap_rows, csa2_seqs_t seqs,
                                         const int32_t* q_visible, const int32_t* pool,
                                         int32_t pool_blocks, int32_t block, int32_t topk,
                                         int32_t* indices, void* workspace, size_t ws_bytes,
                                         void* stream) {
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices,
                                  workspace);
  if (st != CSA2_OK || num_q == 0) return st;
  if (block != 8 || pool_blocks < 1 || pool_blocks > 8192 || !pool) return CSA2_ERR_UNSUPPORTED;
  // visible positions inside the pool never exceed the pool's reach; the bound only
  // clamps q_visible values that are larger than the sequence
  return run_index<true>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, 0x7FFFFFFF,
                         topk, indices, pool_blocks, block, nullptr, pool, workspace, ws_bytes,
                         (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------------
// csa2_index_full_noalloc: the same computation with the library's own scratch array,
// for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------------
// Scratch of the no-allocation entry point.  Every GPU that loads the library holds it
// until exit.  In host code this name is only a stand-in for the device array: the kernels
// get its device address, looked up below with the device current.
static __device__ __align__(256) unsigned char csa2_index_scratch[CSA2_INDEX_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of csa2_index_scratch on the current device (looked up once per device).
void* index_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, csa2_index_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}
}  // namespace

extern "C" csa2_status_t csa2_index_full_noalloc(const uint16_t* qI, const float* w,
                                                 int32_t num_q, int32_t H_I, int32_t d_I,
                                                 const uint16_t* idx_k, int64_t cap_rows,
                                                 csa2_seqs_t seqs, const int32_t* q_visible,
                                                 int32_t max_visible, int32_t topk,
                                                 int32_t* indices, int32_t pool_blocks,
                                                 int32_t block, int32_t* pool, void* stream) {
  if (max_visible < 0) return CSA2_ERR_INVALID_ARG;
  if (pool_blocks < 0 || pool_blocks > 8192) return CSA2_ERR_UNSUPPORTED;
  const size_t need = csa2_index_full_workspace(num_q, max_visible, topk, pool_blocks,
                                                pool_blocks > 0 ? block : 8);
  if (need == 0 || need > (size_t)CSA2_INDEX_NOALLOC_SCRATCH_BYTES) return CSA2_ERR_CAPACITY;
  void* ws = index_scratch_address();
  if (!ws) return CSA2_ERR_CUDA;
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices, ws);
  if (st != CSA2_OK || num_q == 0) return st;
  if (pool_blocks > 0 && (!pool || !pow2_le32(block))) return CSA2_ERR_UNSUPPORTED;
  if (pool_blocks == 0) block = 8;
  // the status word starts clear on every call (the histograms are cleared by run_index)
  if (cudaMemsetAsync(ws, 0, CSA2_STATUS_BYTES, (cudaStream_t)stream) != cudaSuccess)
    return CSA2_ERR_CUDA;
  return run_index<false>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, max_visible,
                          topk, indices, pool_blocks, block, pool, nullptr, ws,
                          (size_t)CSA2_INDEX_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream);
}
