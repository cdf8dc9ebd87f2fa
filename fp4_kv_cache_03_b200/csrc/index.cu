// a2-a5: the CSA2 indexer on B200.
//   Full (csa2_index_full):   score every visible entry, Top-K positions, and (decoder's
//                             first Full layer) the candidate pool of top blocks.
//   Reindex (csa2_index_pool): score only the pool's positions with this layer's own
//                             indexer Q, Top-K of those.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", section "CSA2：在层的维度上共享缓存"
// (Full/Reindex/Reuse, Top-512, pool of <= 2048 blocks x 8); gkm0120.cn "技术调研报告"
// §2.2.2 (modes table) and §2.2.3 (hierarchical sparse indexer).
//
// Score kernel: persistent, warp-specialised; each CTA takes one contiguous, equal share
// of the active 128-entry tiles of all queries (exact balance for ragged batches and
// causal chunks).  Warp 0 streams tiles of the bf16 indexer K with TMA (128-byte swizzle)
// into a ring of shared-memory stages, warp 1 issues tcgen05.mma (M = 128 entries,
// N = indexer heads padded to 16/32, K = d_I) into a double-buffered TMEM accumulator,
// warps 2-5 read it back (tcgen05.ld), apply ReLU * w, sum the heads and write one 32-bit
// order-preserving key per entry (plus the block maximum for the pool).  The epilogue also
// builds the first radix digit's histogram of every row (bits 31..21 of the key).
// Select kernel: a CTA per 8192-key chunk reads its row's histogram, finds the bin holding
// the K-th key, and appends the chunk's candidates (keys in that bin or above) to a
// per-row list in position order; the last CTA of the row (counted with an atomic, no
// waiting) finishes an exact radix select over the candidates (bits 20..10, then 9..0)
// and writes the Top-K in ascending position order, lowest position first among ties.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kTileRows = 128;         // entries per MMA tile (M)
constexpr int kScoreThreads = 192;     // 6 warps
constexpr int kSelThreads = 512;
constexpr int kSelChunk = 8192;        // keys per select CTA
constexpr int kHistBins = 2048;        // first digit: key bits 31..21
static_assert(kHistBins / 4 == kSelThreads, "one 16-byte piece of a histogram per select thread");
constexpr int kMaxRowsPerLaunch = 4096;
constexpr int kMaxListChunks = 1024;   // rows longer than this many chunks stream their keys
constexpr int kSelSingle = 16384;      // rows up to this long are selected by one CTA

// ---------------------------------------------------------------------------------
// visibility
// ---------------------------------------------------------------------------------
struct Seqs {
  const int64_t* seq_start;
  const int32_t* seq_len;
  const int32_t* q_visible;
  const int32_t* q_seq;            // or null: q / q_per_seq
  int q_per_seq;
  int num_seqs;
  int max_visible;
  int* status;
  const int32_t* block_table;      // or null: linear rows from seq_start
  int max_pages;
};

// the sequence of query q, or -1 for an out-of-range q_seq value
__device__ __forceinline__ int seq_of(const Seqs& s, int q) {
  const int seq = s.q_seq ? s.q_seq[q] : q / s.q_per_seq;
  return (seq >= 0 && seq < s.num_seqs) ? seq : -1;
}

// cache row of position p of query q's sequence; -1 for an invalid sequence or page (the
// sequence then sees nothing, or the page's entries are skipped)
__device__ __forceinline__ int64_t row_of_pos(const Seqs& s, int q, int64_t p) {
  const int seq = seq_of(s, q);
  return seq >= 0 ? entry_row(s.seq_start, s.block_table, s.max_pages, seq, p) : -1;
}

__device__ __forceinline__ int visible_of(const Seqs& s, int q) {
  const int seq = seq_of(s, q);
  if (seq < 0) { report(s.status, CSA2_ERR_INVALID_ARG); return 0; }
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
  int q0, num_q;                   // queries [q0, q0 + num_q) of this launch
  int H_I, d_I, n_pad;             // n_pad: MMA N (16 or 32)
  int stages;
  const int32_t* pool;             // Reindex: tiles are 16 pool blocks of 8 rows each
  int pool_blocks;
  uint32_t* keys;                  // [q][key_stride]
  int64_t key_stride;
  uint32_t* bkeys;                 // block-max keys [q][bkey_stride] (Full with pool) or null
  int64_t bkey_stride;
  int block;                       // block size for bkeys (power of two <= 32)
  uint32_t* hist;                  // [q][kHistBins] first-digit histogram of keys
  uint32_t* bhist;                 // same for block keys (or null)
  uint64_t wait_ns;                // bound of every wait
};

struct ScoreSmem {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Full scan: tiles of query q's visible entries
__device__ __forceinline__ int full_tiles(const ScoreArgs& a, int q) {
  return (visible_of(a.seqs, q) + kTileRows - 1) / kTileRows;
}

// the row (query) of flat tile index i: the largest r with rowp[r] <= i
__device__ __forceinline__ int find_row(const uint32_t* rowp, int n, uint32_t i) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rowp[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// kESize: bytes per indexer element (2: bf16, 1: E4M3).  Either way an indexer row is moved
// as 128-byte column chunks (64 bf16 or 128 E4M3 values) in the 128-byte-swizzled layout, and
// one MMA K-step reads 32 bytes of it (16 bf16 with kind::f16, 32 E4M3 with kind::f8f6f4).
template <bool kGather, int kESize>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                 const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ ScoreSmem ss;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* status = a.seqs.status;

  const int halves = a.d_I * kESize / 128;                // 128-byte K chunks
  constexpr int kChunkElems = 128 / kESize;                 // elements per chunk
  const uint32_t a_bytes = (uint32_t)halves * kTileRows * 128;
  const uint32_t b_half = (uint32_t)a.n_pad * 128;
  const uint32_t stage_bytes = a_bytes + (uint32_t)halves * b_half;
  // 1024-byte aligned base, derived from the shared array itself so that the compiler keeps
  // the shared address space (and knows these buffers do not alias `ss`)
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = a.stages;
  uint32_t* rowp = reinterpret_cast<uint32_t*>(base + (size_t)S * stage_bytes);   // [num_q + 1]
  uint32_t* shist = rowp + ((a.num_q + 1 + 31) & ~31);                             // [kHistBins]
  uint32_t* sbhist = shist + kHistBins;                                            // [kHistBins]

  // set-up that reads no global memory (it overlaps the previous kernel's tail)
  pdl_trigger();
  for (int i = tid; i < 2 * kHistBins; i += kScoreThreads) shist[i] = 0;
  if (tid == 0) {
    rowp[0] = 0;
    for (int s = 0; s < S; ++s) { mbar_init(&ss.full[s], 1); mbar_init(&ss.empty[s], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&ss.tfull[i], 1); mbar_init(&ss.tempty[i], 4); }
    mbar_init(&ss.drain, 1);
    ss.abort = 0;
    fence_barrier_init();
  }
  // padding rows of the B operand (heads >= H_I) must read as zero; TMA never writes them
  if (a.H_I < a.n_pad) {
    const uint32_t pad = (uint32_t)(a.n_pad - a.H_I) * 128;
    for (int s = 0; s < S; ++s) {
      uint8_t* b = base + (size_t)s * stage_bytes + a_bytes;
      for (uint32_t i = tid * 16; i < (uint32_t)halves * pad; i += kScoreThreads * 16) {
        const uint32_t h = i / pad, o = i % pad;
        *reinterpret_cast<uint4*>(b + h * b_half + (uint32_t)a.H_I * 128 + o) = make_uint4(0, 0, 0, 0);
      }
    }
  }
  if (warp == 1) { tmem_alloc(&ss.tmem_base, a.n_pad * 2 < 32 ? 32 : a.n_pad * 2); tmem_relinquish(); }
  pdl_wait();

  // active tiles of every query, then their exclusive prefix.  Reindex: every query takes
  // all ceil(pool_blocks / 16) tiles (a pool holds valid blocks first; the slots of -1
  // blocks get no load and key 0), so the pool is not read here.
  if (kGather) {
    const uint32_t tiles = (uint32_t)((a.pool_blocks + 15) / 16);
    for (int i = tid; i < a.num_q; i += kScoreThreads) rowp[i + 1] = tiles;
  } else {
    for (int i = tid; i < a.num_q; i += kScoreThreads) rowp[i + 1] = full_tiles(a, a.q0 + i);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t carry = 0;
    for (int b0 = 0; b0 < a.num_q; b0 += 32) {
      const int i = b0 + lane;
      uint32_t v = i < a.num_q ? rowp[i + 1] : 0u;
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      if (i < a.num_q) rowp[i + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  volatile int* abort = &ss.abort;
  const uint32_t total = rowp[a.num_q];
  const uint32_t t_lo = (uint32_t)(((uint64_t)total * blockIdx.x) / gridDim.x);
  const uint32_t t_hi = (uint32_t)(((uint64_t)total * (blockIdx.x + 1)) / gridDim.x);

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (kGather && t_lo < t_hi) {
      // Reindex: lanes 0-15 each fetch one of the tile's 16 pool blocks (8 rows x 2 halves);
      // lane 0 waits for the stage, arms its barrier and loads the query
      if (lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
      }
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0;                     // stages holding a load (bit s), its parity below
      uint32_t filled_parity = 0;
      int r = find_row(rowp, a.num_q, t_lo);
      for (uint32_t i = t_lo; i < t_hi; ++i) {
        if (__shfl_sync(0xffffffffu, *abort, 0)) break;
        while (rowp[r + 1] <= i) ++r;
        const int q = a.q0 + r, t = (int)(i - rowp[r]);
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&ss.empty[stage], phase ^ 1, abort, status, a.wait_ns) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        uint8_t* sa = base + (size_t)stage * stage_bytes;
        uint8_t* sb = sa + a_bytes;
        int j = (lane < 16 && t * 16 + lane < a.pool_blocks)
                    ? __ldg(a.pool + (int64_t)q * a.pool_blocks + t * 16 + lane)
                    : -1;
        const int64_t brow = j >= 0 ? row_of_pos(a.seqs, q, 8 * (int64_t)j) : -1;
        if (brow < 0) j = -1;                  // (a block of a missing page loads nothing)
        const uint32_t nvalid = (uint32_t)__popc(__ballot_sync(0xffffffffu, j >= 0));
        if (lane == 0)
          mbar_arrive_expect_tx(&ss.full[stage],
                                (uint32_t)halves * ((uint32_t)a.H_I * 128 + nvalid * 8 * 128));
        __syncwarp();
        for (int h = 0; h < halves; ++h) {
          if (lane == 0)
            tma_load_2d(sb + h * b_half, &tm_q, h * kChunkElems, q * a.H_I, &ss.full[stage]);
          if (j >= 0)
            tma_load_2d(sa + h * (kTileRows * 128) + lane * 1024, &tm_k, h * kChunkElems,
                        (int32_t)brow, &ss.full[stage]);
        }
        filled |= 1u << stage;
        filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      // no load of this CTA may still be landing when it exits (after an abort the MMA warp
      // has not consumed every stage); a consumed stage's phase has completed already
      if (lane == 0)
        for (int st = 0; st < S; ++st)
          if (filled & (1u << st)) mbar_drain(&ss.full[st], (filled_parity >> st) & 1u);
    } else if (!kGather && lane == 0 && t_lo < t_hi) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, filled_parity = 0;  // as in the Reindex producer
      int r = find_row(rowp, a.num_q, t_lo);
      for (uint32_t i = t_lo; i < t_hi && !*abort; ++i) {
        while (rowp[r + 1] <= i) ++r;
        const int q = a.q0 + r, t = (int)(i - rowp[r]);
        if (!mbar_wait(&ss.empty[stage], phase ^ 1, abort, status, a.wait_ns)) break;
        uint8_t* sa = base + (size_t)stage * stage_bytes;
        uint8_t* sb = sa + a_bytes;
        uint32_t bytes = (uint32_t)halves * (uint32_t)a.H_I * 128;
        int32_t blk_row[16];
        int64_t trow = 0;
        if (kGather) {
          const int32_t* pb = a.pool + (int64_t)q * a.pool_blocks + t * 16;
          for (int k = 0; k < 16; ++k) {
            const int j = (t * 16 + k < a.pool_blocks) ? pb[k] : -1;
            const int64_t br = j >= 0 ? row_of_pos(a.seqs, q, 8 * (int64_t)j) : -1;
            blk_row[k] = (int32_t)br;
            if (br >= 0) bytes += (uint32_t)halves * 8 * 128;
          }
        } else {
          // one tile = one page; a missing page loads zeros (outside the map), its keys are
          // dropped by the epilogue
          trow = row_of_pos(a.seqs, q, (int64_t)t * kTileRows);
          if (trow < 0) trow = -(int64_t)(1 << 30);
          bytes += a_bytes;
        }
        mbar_arrive_expect_tx(&ss.full[stage], bytes);
        for (int h = 0; h < halves; ++h) {
          tma_load_2d(sb + h * b_half, &tm_q, h * kChunkElems, q * a.H_I, &ss.full[stage]);
          if (kGather) {
            for (int k = 0; k < 16; ++k)
              if (blk_row[k] >= 0)
                tma_load_2d(sa + h * (kTileRows * 128) + k * 1024, &tm_k, h * kChunkElems,
                            blk_row[k], &ss.full[stage]);
          } else {
            tma_load_2d(sa + h * (kTileRows * 128), &tm_k, h * kChunkElems, (int32_t)trow,
                        &ss.full[stage]);
          }
        }
        filled |= 1u << stage;
        filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      for (int st = 0; st < S; ++st)
        if (filled & (1u << st)) mbar_drain(&ss.full[st], (filled_parity >> st) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0 && t_lo < t_hi) {
      const uint32_t idesc = kESize == 2 ? idesc_bf16(kTileRows, a.n_pad) : idesc_e4m3(kTileRows, a.n_pad);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (uint32_t i = t_lo; i < t_hi && !*abort; ++i) {
        if (!mbar_wait(&ss.tempty[acc], acc_phase ^ 1, abort, status, a.wait_ns)) break;
        if (!mbar_wait(&ss.full[stage], phase, abort, status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
        const uint32_t sb = sa + a_bytes;
        const uint32_t d = tmem + (uint32_t)(acc * a.n_pad);
        for (int k = 0; k < 4 * halves; ++k) {              // 32-byte K-steps
          const int h = k >> 2, sub = k & 3;
          const uint64_t ad = sdesc_sw128(sa + h * (kTileRows * 128) + sub * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sb + h * b_half + sub * 32, 16, 1024);
          if constexpr (kESize == 2) umma_bf16(d, ad, bd, idesc, k > 0 ? 1u : 0u);
          else umma_e4m3(d, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&ss.empty[stage]);
        umma_commit(&ss.tfull[acc]);
        if (++stage == S) { stage = 0; phase ^= 1; }
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA this thread issued has completed before the CTA frees TMEM and exits
      umma_commit(&ss.drain);
      mbar_drain(&ss.drain, 0);
    }
  } else {
    // ------------------------------ epilogue (warps 2..5) ------------------------------
    // Every epilogue warp walks every tile of the range (even after an abort) so that the
    // named barriers of the histogram flushes always see all four warps.
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;          // entry (or slot) within the tile
    const int etid = tid - 64;                 // 0..127
    int acc = 0;
    uint32_t acc_phase = 0;
    int hq = -1;                               // row whose histogram is being built
    auto flush = [&](int rq) {
      asm volatile("bar.sync 2, 128;" ::: "memory");
      for (int b = etid; b < kHistBins; b += 128) {
        const uint32_t v = shist[b];
        if (v) { atomicAdd(a.hist + (int64_t)rq * kHistBins + b, v); shist[b] = 0; }
        if (a.bhist) {
          const uint32_t u = sbhist[b];
          if (u) { atomicAdd(a.bhist + (int64_t)rq * kHistBins + b, u); sbhist[b] = 0; }
        }
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
    };
    int r = t_lo < t_hi ? find_row(rowp, a.num_q, t_lo) : 0;
    float wr[32];                              // the current query's head weights
    int vis = 0;
    for (uint32_t i = t_lo; i < t_hi; ++i) {
      while (rowp[r + 1] <= i) ++r;
      const int q = a.q0 + r, t = (int)(i - rowp[r]);
      if (q != hq) {
        if (hq >= 0) flush(hq);
        hq = q;
        vis = visible_of(a.seqs, q);
        const float* wq = a.w + (int64_t)q * a.H_I;
#pragma unroll
        for (int h = 0; h < 32; ++h) wr[h] = h < a.H_I ? __ldg(wq + h) : 0.0f;
      }
      const int e = t * kTileRows + row;       // position (Full) or slot (Reindex)
      int jpool = -1;                          // Reindex: this slot's pool block
      if (kGather && e < a.pool_blocks * 8) jpool = __ldg(a.pool + (int64_t)q * a.pool_blocks + (e >> 3));
      // paged cache: entries of a missing page are dropped (and reported)
      bool page_ok = true;
      if (a.seqs.block_table) {
        const int64_t p0 = kGather ? (jpool >= 0 ? 8 * (int64_t)jpool : 0) : (int64_t)t * kTileRows;
        page_ok = row_of_pos(a.seqs, q, p0) >= 0;
        if (!page_ok && (kGather ? jpool >= 0 : e < vis)) report(status, CSA2_ERR_CAPACITY);
      }
      bool ok = mbar_wait(&ss.tfull[acc], acc_phase, abort, status, a.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      float v[32];
      if (ok) {
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * a.n_pad);
        tmem_ld16(taddr, v);
        if (a.n_pad > 16) tmem_ld16(taddr + 16, v + 16);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss.tempty[acc]);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      if (!ok) continue;

      float s = 0.0f;
#pragma unroll
      for (int h = 0; h < 32; ++h)
        if (h < a.H_I) s = fmaf(wr[h], fmaxf(v[h], 0.0f), s);
      uint32_t key = ordered_key(s);
      if (kGather) {
        if (e < a.pool_blocks * 8) {
          if (jpool < 0 || !page_ok || 8 * (int64_t)jpool + (e & 7) >= vis) key = 0u;
          a.keys[(int64_t)q * a.key_stride + e] = key;
          if (key) atomicAdd(&shist[key >> 21], 1u);
        }
      } else {
        if (e >= vis || !page_ok) key = 0u;
        if (e < vis) {
          a.keys[(int64_t)q * a.key_stride + e] = key;
          if (key) atomicAdd(&shist[key >> 21], 1u);
        }
        if (a.bkeys) {
          uint32_t m = key;
          for (int o = 1; o < a.block; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
          if ((e & (a.block - 1)) == 0 && e < vis) {
            a.bkeys[(int64_t)q * a.bkey_stride + e / a.block] = m;
            atomicAdd(&sbhist[m >> 21], 1u);
          }
        }
      }
    }
    if (hq >= 0) flush(hq);
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
  int len_mode;         // 0: visible positions, 1: visible blocks, 2: pool slots
  int block;            // len_mode 1: block size
  const int32_t* pool;  // len_mode 2: output = 8 * pool[slot / 8] + slot % 8
  int pool_blocks;
  const uint32_t* hist; // [rows][kHistBins]
  uint32_t* cand;       // [rows][cand_cap] candidate positions
  uint32_t* cand_key;   // [rows][cand_cap] their keys
  int cand_cap;
  uint32_t* seg;        // [rows][chunks][2]: offset, count of each chunk's candidates
  uint32_t* fill;       // [rows] candidates appended so far
  uint32_t* done;       // [rows] chunks finished
  int chunks;           // grid bound on chunks per row
  int single;           // stride <= kSelSingle: one CTA selects the whole row in shared memory
};
struct SelArgs {
  SelProblem p[2];
  Seqs seqs;
};

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* red);

// Block-wide: entries of row r to select from.  Pool-slot rows cover the active tiles of
// the score kernel (16 pool blocks each), never past the pool's end.
__device__ __forceinline__ int row_len(const SelProblem& p, const Seqs& s, int r, uint32_t* red) {
  if (p.len_mode == 2) {
    const int32_t* pr = p.pool + (int64_t)r * p.pool_blocks;
    uint32_t n = 0;
    for (int i = threadIdx.x; i < p.pool_blocks; i += kSelThreads) n += pr[i] >= 0;
    const uint32_t nv = block_sum(n, red);
    return min(p.pool_blocks * 8, (int)((nv + 15) / 16) * kTileRows);
  }
  const int v = visible_of(s, r);
  return p.len_mode == 0 ? v : (v + p.block - 1) / p.block;
}

struct Top {
  uint32_t b1;       // first-digit bin holding the K-th key
  uint32_t above;    // keys in bins above b1
  uint32_t n_valid;  // candidates of the row
  uint32_t n_cand;   // keys in bins >= b1
  int take_all;      // n_valid <= k: every candidate is selected
};

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  uint32_t t = 0;
  for (int i = 0; i < kSelThreads / 32; ++i) t += red[i];
  return t;
}

// Block-wide: the bin of a `bins`-bin histogram h that holds the k-th largest key, with
// the count of keys above it.  All threads return the same values.
__device__ void find_bin(const uint32_t* h, int bins, uint32_t k, uint32_t* bin, uint32_t* above,
                         uint32_t* red) {
  __shared__ uint32_t s_bin, s_above;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int per = bins / kSelThreads;      // contiguous bins per thread (4 or 2)
  uint32_t c[8];
  uint32_t mine = 0;
  for (int i = 0; i < per; ++i) { c[i] = h[tid * per + i]; mine += c[i]; }
  uint32_t incl = mine;                    // sum over lanes >= mine within the warp
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += y;
  }
  __syncthreads();
  if (lane == 0) red[wid] = incl;
  __syncthreads();
  uint32_t up = 0;
  for (int i = wid + 1; i < kSelThreads / 32; ++i) up += red[i];
  const uint32_t S = incl + up;            // keys in bins >= my first bin
  const uint32_t S_next = S - mine;        // keys in bins above my range
  if (S >= k && S_next < k) {
    uint32_t run = S_next;
    for (int i = per - 1; i >= 0; --i) {
      if (run + c[i] >= k) { s_bin = tid * per + i; s_above = run; break; }
      run += c[i];
    }
  }
  __syncthreads();
  *bin = s_bin;
  *above = s_above;
  __syncthreads();
}

// h: the row's histogram, already in shared memory
__device__ Top resolve_top(const uint32_t* h, uint32_t k, uint32_t* red) {
  Top tp;
  uint32_t n = 0;
#pragma unroll
  for (int b = threadIdx.x; b < kHistBins; b += kSelThreads) n += h[b];
  tp.n_valid = block_sum(n, red);
  tp.take_all = tp.n_valid <= k;
  if (tp.take_all) {
    tp.b1 = 0; tp.above = 0; tp.n_cand = tp.n_valid;
    return tp;
  }
  find_bin(h, kHistBins, k, &tp.b1, &tp.above, red);
  tp.n_cand = tp.above + h[tp.b1];
  return tp;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// exclusive block scan of one value per thread; *total receives the block total
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* total, uint32_t* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) red[wid] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
  for (int i = 0; i < kSelThreads / 32; ++i) {
    if (i < wid) before += red[i];
    tot += red[i];
  }
  *total = tot;
  return before + x - v;
}

// Candidates of a row in ascending position order: either the per-chunk segments of the
// list (kList) or the row's keys filtered by the first digit.
template <bool kList>
struct CandSource {
  const uint32_t* keys;     // the row's keys
  const uint32_t* cand;     // the row's list: positions
  const uint32_t* cand_key; // and their keys
  const uint32_t* seg;      // [chunks][2]
  const uint32_t* pre;      // shared: exclusive prefix of segment counts [nch + 1]
  int nch;
  uint32_t n;               // number of candidates (list) or row length (stream)
  uint32_t b1;
  __device__ __forceinline__ bool pred(uint32_t key) const { return key != 0u && (key >> 21) >= b1; }
  // position of the g-th element of the source (g < n)
  __device__ __forceinline__ uint32_t pos_at(uint32_t g, int& c) const {
    if constexpr (!kList) {
      return g;
    } else {
      while (pre[c + 1] <= g) ++c;
      return cand[seg[2 * c] + (g - pre[c])];
    }
  }
};

// Shared-memory copy of a row's candidates (key, position), in position order.
struct StagedSource {
  const uint32_t* keys;     // shared
  const uint32_t* pos;      // shared
  uint32_t n;
  __device__ __forceinline__ bool pred(uint32_t) const { return true; }
  __device__ __forceinline__ uint32_t key_at(uint32_t g, int&) const { return keys[g]; }
  __device__ __forceinline__ uint32_t pos_at_ordered(uint32_t g, int&) const { return pos[g]; }
};
template <bool kList>
struct GlobalSource {
  CandSource<kList> s;
  uint32_t n;
  __device__ __forceinline__ bool pred(uint32_t key) const { return s.pred(key); }
  // the cursor c only moves forward, so a caller walks g in increasing order
  __device__ __forceinline__ uint32_t pos_at_ordered(uint32_t g, int& c) const { return s.pos_at(g, c); }
  __device__ __forceinline__ uint32_t key_at(uint32_t g, int& c) const {
    if constexpr (kList) {
      const uint32_t i = s.pos_at(g, c), cc = (uint32_t)c;   // advances the cursor
      (void)i;
      return s.cand_key[s.seg[2 * cc] + (g - s.pre[cc])];
    } else {
      return s.keys[g];
    }
  }
};

// Exact selection of the row's Top-K from its candidates (any source in position order).
template <class Src>
__device__ void final_select(const SelProblem& p, int r, const Top& tp, const Src& src,
                             uint32_t* red, uint32_t* hsm, const int32_t* pool_s = nullptr) {
  const int tid = threadIdx.x;
  const uint32_t k = (uint32_t)p.k;
  int32_t* out = p.out + (int64_t)r * p.out_stride;
  const uint32_t n_sel = min(k, tp.n_valid);
  for (uint32_t i = n_sel + tid; i < k; i += kSelThreads) out[i] = -1;
  if (n_sel == 0) return;
  // threshold key T: keys > T are taken, and the first need_eq keys equal to T
  uint32_t T = 0u, need_eq = 0u;
  if (!tp.take_all) {
    uint32_t krem = n_sel - tp.above;      // still to take from bin b1
    uint32_t prefix = tp.b1 << 21;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      const int bins = pass == 0 ? 2048 : 1024;
      const uint32_t pmask = pass == 0 ? 0xFFE00000u : 0xFFFFFC00u;
      for (int b = tid; b < bins; b += kSelThreads) hsm[b] = 0;
      __syncthreads();
      int c = 0;
      for (uint32_t g = tid; g < src.n; g += kSelThreads) {
        const uint32_t key = src.key_at(g, c);
        if (key != 0u && (key & pmask) == prefix) atomicAdd(&hsm[(key >> shift) & (bins - 1)], 1u);
      }
      __syncthreads();
      uint32_t bin, above;
      find_bin(hsm, bins, krem, &bin, &above, red);
      krem -= above;
      prefix |= bin << shift;
    }
    T = prefix;
    need_eq = krem;
  }
  // ordered write: each thread a contiguous run of the source
  const uint32_t per = (src.n + kSelThreads - 1) / kSelThreads;
  const uint32_t g0 = min(src.n, tid * per), g1 = min(src.n, g0 + per);
  uint32_t my_gt = 0, my_eq = 0;
  int c = 0;
  for (uint32_t g = g0; g < g1; ++g) {
    const uint32_t key = src.key_at(g, c);
    if (!src.pred(key)) continue;
    my_gt += key > T;
    my_eq += (key == T);
  }
  uint32_t tot;
  const uint32_t eq_rank = block_excl_scan(my_eq, &tot, red);
  const uint32_t my_take = eq_rank >= need_eq ? 0u : min(my_eq, need_eq - eq_rank);
  uint32_t o = block_excl_scan(my_gt + my_take, &tot, red);
  uint32_t taken = 0;
  c = 0;
  for (uint32_t g = g0; g < g1; ++g) {
    const uint32_t key = src.key_at(g, c);
    if (!src.pred(key)) continue;
    bool sel = key > T;
    if (!sel && key == T) { sel = taken < my_take; ++taken; }
    if (sel && o < k) {   // (keys that disagree with the histogram never write past K)
      const uint32_t pos = src.pos_at_ordered(g, c);
      int32_t v = (int32_t)pos;
      if (p.len_mode == 2)
        v = 8 * (pool_s ? pool_s[pos >> 3] : p.pool[(int64_t)r * p.pool_blocks + (pos >> 3)]) +
            (int32_t)(pos & 7);
      out[o++] = v;
    }
  }
}

// Clears the per-call counters and histograms of the workspace (a kernel rather than a
// memset, so that the launches of one call chain without gaps).
__global__ void __launch_bounds__(256) ws_zero_kernel(uint4* p, uint32_t n16) {
  pdl_trigger();
  pdl_wait();
  for (uint32_t i = blockIdx.x * 256u + threadIdx.x; i < n16; i += gridDim.x * 256u)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// One warp: the bin of the histogram h (32 * kBPL bins) that holds the k-th largest key
// (1 <= k <= total), the count of keys in the bins above it, and the total (k > total:
// bin 0, above 0).  Lane l sums the bins [kBPL l, kBPL l + kBPL) with 16-byte loads in
// rotated order (distinct banks across the warp); a suffix sum over the lanes finds the
// lane range that holds the k-th key; the warp then splits that range, kBPL / 32 bins per
// lane, and a second suffix sum finds the bin.  No step walks bins one by one.
template <int kBPL>
__device__ __forceinline__ void warp_find_bin(const uint32_t* h, uint32_t k, int lane, uint32_t* bin,
                                              uint32_t* above, uint32_t* total) {
  constexpr int kQ = kBPL / 4;               // 16-byte pieces per lane
  constexpr int kB = kBPL / 32;              // bins per lane in the second step
  static_assert(kB >= 1 && kQ >= 1, "32 to 64 bins per lane");
  const uint4* h4 = reinterpret_cast<const uint4*>(h) + lane * kQ;
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < kQ; ++j) {
    const uint4 v = h4[(j + lane) & (kQ - 1)];
    mine += (v.x + v.y) + (v.z + v.w);
  }
  uint32_t S = mine;                         // keys in the bins of lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, S, o);
    if (lane + o < 32) S += y;
  }
  *total = __shfl_sync(0xffffffffu, S, 0);
  const uint32_t who = __ballot_sync(0xffffffffu, S >= k && S - mine < k);
  if (who == 0u) {
    *bin = 0u;
    *above = 0u;
    return;
  }
  const int L = __ffs(who) - 1;
  const uint32_t runL = __shfl_sync(0xffffffffu, S - mine, L);   // keys above lane L's range
  uint32_t cb[kB], mb = 0;
#pragma unroll
  for (int e = 0; e < kB; ++e) { cb[e] = h[L * kBPL + lane * kB + e]; mb += cb[e]; }
  uint32_t Sb = mb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, Sb, o);
    if (lane + o < 32) Sb += y;
  }
  const uint32_t kr = k - runL;              // rank of the k-th key inside lane L's range
  const bool holds = Sb >= kr && Sb - mb < kr;
  uint32_t b = 0u, ab = 0u;
  if (holds) {
    uint32_t run = runL + (Sb - mb);
#pragma unroll
    for (int e = kB - 1; e >= 0; --e) {
      if (run + cb[e] >= k) { b = (uint32_t)(L * kBPL + lane * kB + e); ab = run; break; }
      run += cb[e];
    }
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, holds)) - 1;
  *bin = __shfl_sync(0xffffffffu, b, src);
  *above = __shfl_sync(0xffffffffu, ab, src);
}

// Block-wide exact Top-K of a row of at most 32 * kSelThreads keys held in shared memory
// (0 = not a candidate), given the first digit's threshold bin b1 and the count of keys
// above it.  Thread t owns the contiguous elements [32 t, 32 t + 32); its eight 16-byte
// pieces are stored swizzled (piece j of run t at 16-byte slot 8 t + (j ^ (t & 7))), so
// that a warp's loads of piece j hit distinct banks and land in registers with static
// indices.  One pass marks, as bits, the keys above the threshold bin and in it; the
// second and third digits (counted in h2 [2048] and h3 [1024], zero on entry), the counts
// and the ordered write are predicated on those bits, with the keys in registers.  Each
// digit's bin is found by one warp; one packed scan places the output.  out_of(i) is the
// output value of element i; n_sel = min(k, valid candidates).
__device__ __forceinline__ int swz_slot(int t, int j) { return 8 * t + (j ^ (t & 7)); }

template <class OutOf>
__device__ void resident_select(const uint32_t* keys_s, uint32_t b1, uint32_t above, bool take_all,
                                uint32_t n_sel, uint32_t k, int32_t* out, uint32_t* h2, uint32_t* h3,
                                uint32_t* s_res, uint32_t* wcnt, OutOf out_of) {
  constexpr int kRun = 32;
  static_assert(kSelThreads * kRun >= kSelSingle, "a run of 32 per thread covers a row");
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint32_t kr[kRun];
#pragma unroll
  for (int j = 0; j < kRun / 4; ++j) {
    const uint4 v = reinterpret_cast<const uint4*>(keys_s)[swz_slot(tid, j)];
    kr[4 * j] = v.x; kr[4 * j + 1] = v.y; kr[4 * j + 2] = v.z; kr[4 * j + 3] = v.w;
  }
  // bit i of m_gt / m_eq: element 32 t + i lies above / in the threshold bin (take-all:
  // every candidate is "above")
  uint32_t m_gt = 0u, m_eq = 0u;
#pragma unroll
  for (int i = 0; i < kRun; ++i) {
    const uint32_t d = kr[i] >> 21;
    if (kr[i] != 0u && d > b1) m_gt |= 1u << i;
    if (kr[i] != 0u && d == b1) m_eq |= 1u << i;
  }
  // threshold key T: keys > T are taken, and the first need_eq keys equal to T
  uint32_t T = 0u, need_eq = 0u;
  if (take_all) {
    m_gt |= m_eq;
    m_eq = 0u;
  } else {
    uint32_t krem = n_sel - above;
    if (m_eq) {
#pragma unroll
      for (int i = 0; i < kRun; ++i)
        if ((m_eq >> i) & 1u) atomicAdd(&h2[(kr[i] >> 10) & 2047u], 1u);
    }
    __syncthreads();
    if (wid == 0) {
      uint32_t b2, ab, total;
      warp_find_bin<2048 / 32>(h2, krem, lane, &b2, &ab, &total);
      if (lane == 0) { s_res[0] = b2; s_res[1] = ab; }
    }
    __syncthreads();
    const uint32_t pre2 = (b1 << 11) | s_res[0];           // key bits 31..10
    krem -= s_res[1];
    if (m_eq) {
#pragma unroll
      for (int i = 0; i < kRun; ++i)
        if (((m_eq >> i) & 1u) && (kr[i] >> 10) == pre2) atomicAdd(&h3[kr[i] & 1023u], 1u);
    }
    __syncthreads();
    if (wid == 0) {
      uint32_t b3, ab, total;
      warp_find_bin<1024 / 32>(h3, krem, lane, &b3, &ab, &total);
      if (lane == 0) { s_res[0] = b3; s_res[1] = ab; }
    }
    __syncthreads();
    T = (pre2 << 10) | s_res[0];
    need_eq = krem - s_res[1];
  }
  // one scan of (equal << 16 | greater): the ties taken before this thread are
  // min(equal rank, need_eq), lowest positions first
  uint32_t m_tie = 0u;                                     // keys equal to T
  if (m_eq) {
#pragma unroll
    for (int i = 0; i < kRun; ++i) {
      if (((m_eq >> i) & 1u) && kr[i] > T) m_gt |= 1u << i;
      if (((m_eq >> i) & 1u) && kr[i] == T) m_tie |= 1u << i;
    }
  }
  const uint32_t my_gt = __popc(m_gt), my_eq = __popc(m_tie);
  const uint32_t packed = (my_eq << 16) | my_gt;           // block totals < 2^15 each
  uint32_t incl = packed;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wcnt[wid] = incl;
  __syncthreads();
  uint32_t ex = incl - packed;
  for (int w = 0; w < wid; ++w) ex += wcnt[w];
  const uint32_t gt_rank = ex & 0xFFFFu, eq_rank = ex >> 16;
  // the first my_take ties of this run are taken
  const uint32_t my_take = eq_rank >= need_eq ? 0u : min(my_eq, need_eq - eq_rank);
  uint32_t m_take = m_tie;
  for (uint32_t c = my_eq; c > my_take; --c) m_take &= ~(0x80000000u >> __clz(m_take));   // drop the highest
  uint32_t o = gt_rank + min(eq_rank, need_eq);
  const uint32_t m_sel = m_gt | m_take;
  for (uint32_t m = m_sel; m; m &= m - 1u) {
    if (o >= k) break;                                     // (never past K, even for keys that
    out[o++] = out_of(tid * kRun + __ffs(m) - 1);          // disagree with the histogram)
  }
}

constexpr int kStageCap = 12288;       // candidates staged in shared memory (96 KB)

__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelArgs a) {
  extern __shared__ uint4 stage_raw[];      // chunk keys, later [kStageCap] keys + positions
  uint32_t* stage_buf = reinterpret_cast<uint32_t*>(stage_raw);
  __shared__ uint32_t red[kSelThreads / 32];
  __shared__ uint32_t wcnt[kSelThreads / 32];
  __shared__ uint32_t s_base;
  __shared__ int s_last;
  __shared__ int s_over;
  __shared__ __align__(16) uint32_t hsm[2048];
  __shared__ uint32_t pre[kMaxListChunks + 1];
  __shared__ uint32_t soff[kMaxListChunks];  // list offset of each chunk's candidates
  pdl_trigger();
  pdl_wait();
  const SelProblem& p = a.p[blockIdx.z];
  const int r = blockIdx.y, c = blockIdx.x;
  if (r >= p.num_rows) return;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (p.single) {
    // Short rows: one CTA holds the whole row in shared memory and selects there
    // (resident_select); the first digit's bin comes from the score kernel's histogram,
    // found by one warp.  Seven block barriers in all.  The loads go out before the row
    // length is known; entries at or past it are stale and cleared.
    if (c != 0) return;
    uint32_t* keys_s = stage_buf;                          // [kSelSingle]
    uint32_t* h2 = keys_s + kSelSingle;                    // [2048] second digit (bits 20..10)
    uint32_t* h3 = h2 + 2048;                              // [1024] third digit (bits 9..0)
    int32_t* pool_s = reinterpret_cast<int32_t*>(h3 + 1024);   // [pool_blocks <= 2048]
    __shared__ uint32_t s_res[3];
    constexpr int kPer = kSelSingle / 4 / kSelThreads;    // 16-byte loads per thread
    const uint4 hv = reinterpret_cast<const uint4*>(p.hist + (int64_t)r * kHistBins)[tid];
    const uint4* kg = reinterpret_cast<const uint4*>(p.keys + (int64_t)r * p.stride);
    const int n4 = (int)(p.stride / 4);
    uint4 kv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int u = tid + j * kSelThreads;
      kv[j] = u < n4 ? __ldg(kg + u) : make_uint4(0, 0, 0, 0);
    }
    int len;
    if (p.len_mode == 2) {
      // the row covers the active score tiles: 16 valid pool blocks each
      uint32_t nv = 0;
      for (int i = tid; i < p.pool_blocks; i += kSelThreads) {
        const int32_t b = p.pool[(int64_t)r * p.pool_blocks + i];
        pool_s[i] = b;
        nv += b >= 0;
      }
      nv = block_sum(nv, red);
      len = min(p.pool_blocks * 8, (int)((nv + 15) / 16) * kTileRows);
    } else {
      len = row_len(p, a.seqs, r, red);
    }
    len = min(max(len, 0), (int)p.stride);
    reinterpret_cast<uint4*>(hsm)[tid] = hv;
    for (int b = tid; b < 2048 + 1024; b += kSelThreads) h2[b] = 0u;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int u = tid + j * kSelThreads;
      uint4 v = kv[j];
      if (4 * u + 0 >= len) v.x = 0u;
      if (4 * u + 1 >= len) v.y = 0u;
      if (4 * u + 2 >= len) v.z = 0u;
      if (4 * u + 3 >= len) v.w = 0u;
      reinterpret_cast<uint4*>(keys_s)[swz_slot(u >> 3, u & 7)] = v;
    }
    __syncthreads();                                       // 1
    const uint32_t k = (uint32_t)p.k;
    if (wid == 0) {
      uint32_t b1, ab, total;
      warp_find_bin<kHistBins / 32>(hsm, k, lane, &b1, &ab, &total);
      if (lane == 0) { s_res[0] = b1; s_res[1] = ab; s_res[2] = total; }
    }
    __syncthreads();                                       // 2
    const uint32_t b1 = s_res[0], n_valid = s_res[2];
    const bool take_all = n_valid <= k;
    int32_t* out = p.out + (int64_t)r * p.out_stride;
    const uint32_t n_sel = min(k, n_valid);
    for (uint32_t i = n_sel + tid; i < k; i += kSelThreads) out[i] = -1;
    if (n_sel == 0) return;
    const int32_t* pmap = p.len_mode == 2 ? pool_s : nullptr;
    resident_select(keys_s, b1, s_res[1], take_all, n_sel, k, out, h2, h3, s_res, wcnt,
                    [pmap](int i) -> int32_t { return pmap ? 8 * pmap[i >> 3] + (i & 7) : i; });
    return;
  }
  const int len = row_len(p, a.seqs, r, red);
  const int nch = max(1, (len + kSelChunk - 1) / kSelChunk);
  if (c >= nch || c >= p.chunks) return;
  const uint32_t* keys = p.keys + (int64_t)r * p.stride;
  const int lo = c * kSelChunk, hi = min(len, lo + kSelChunk);
  // the row's histogram and this chunk's keys, each with one round of independent loads
  {
    const uint4* hg = reinterpret_cast<const uint4*>(p.hist + (int64_t)r * kHistBins);
    const uint4 h0 = hg[tid];                // (one 16-byte piece of the histogram per thread)
    uint4 kv[kSelChunk / 4 / kSelThreads];
    const uint4* kg = reinterpret_cast<const uint4*>(keys + lo);
    const int nv = (hi - lo + 3) / 4;
#pragma unroll
    for (int j = 0; j < kSelChunk / 4 / kSelThreads; ++j) {
      const int u = tid + j * kSelThreads;
      kv[j] = u < nv ? kg[u] : make_uint4(0, 0, 0, 0);
    }
    reinterpret_cast<uint4*>(hsm)[tid] = h0;
#pragma unroll
    for (int j = 0; j < kSelChunk / 4 / kSelThreads; ++j) stage_raw[tid + j * kSelThreads] = kv[j];
  }
  __syncthreads();
  const Top tp = resolve_top(hsm, (uint32_t)p.k, red);
  const bool use_list = tp.n_cand <= (uint32_t)p.cand_cap && nch <= kMaxListChunks;
  uint32_t* seg = p.seg + ((int64_t)r * p.chunks + c) * 2;
  if (use_list) {
    // append this chunk's candidates in position order: warp w owns a contiguous sixteenth
    const int sub = kSelChunk / (kSelThreads / 32);
    const int w_lo = wid * sub, w_hi = min(hi - lo, w_lo + sub);   // chunk-relative
    // this warp's keys in registers (key k of lane l: chunk position w_lo + 32 k + l)
    constexpr int kPerLane = kSelChunk / kSelThreads;       // 16
    uint32_t kk[kPerLane];
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const int i = w_lo + 32 * k + lane;
      const uint32_t key = i < w_hi ? stage_buf[i] : 0u;
      kk[k] = (key != 0u && (key >> 21) >= tp.b1) ? key : 0u;   // 0: not a candidate
    }
    uint32_t cnt = 0;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) cnt += __popc(__ballot_sync(0xffffffffu, kk[k] != 0u));
    if (lane == 0) wcnt[wid] = cnt;
    __syncthreads();
    if (tid == 0) {
      uint32_t tot = 0;
      for (int i = 0; i < kSelThreads / 32; ++i) { const uint32_t x = wcnt[i]; wcnt[i] = tot; tot += x; }
      s_base = tot ? atomicAdd(p.fill + r, tot) : 0u;
      // the histogram bounds the list (n_cand <= cand_cap); keys that disagree with it
      // (left by an aborted score kernel) must still not write past the list
      s_over = s_base + tot > (uint32_t)p.cand_cap;
      if (s_over) report(a.seqs.status, CSA2_ERR_CAPACITY);
      seg[0] = s_base;
      seg[1] = s_over ? 0u : tot;
    }
    __syncthreads();
    uint32_t o = s_base + wcnt[wid];
    uint32_t* cand = p.cand + (int64_t)r * p.cand_cap;
    uint32_t* cand_key = p.cand_key + (int64_t)r * p.cand_cap;
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const bool pr = kk[k] != 0u;
      const uint32_t m = __ballot_sync(0xffffffffu, pr);
      if (pr && !s_over) {
        const uint32_t at = o + __popc(m & lt);
        cand[at] = (uint32_t)(lo + w_lo + 32 * k + lane);
        cand_key[at] = kk[k];
      }
      o += __popc(m);
    }
  }
  // the last chunk of the row to finish completes the row (no CTA waits for another)
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.done + r, 1u) == (uint32_t)(nch - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (use_list) {
    // prefix of the chunks' candidate counts (4 chunks per thread)
    const uint32_t* sg = p.seg + (int64_t)r * p.chunks * 2;
    uint32_t cnt4[4], mine = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ci = tid * 4 + j;
      cnt4[j] = ci < nch ? sg[2 * ci + 1] : 0u;
      if (ci < nch) soff[ci] = sg[2 * ci];
      mine += cnt4[j];
    }
    uint32_t tot;
    uint32_t run = block_excl_scan(mine, &tot, red);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ci = tid * 4 + j;
      if (ci < nch) pre[ci] = run;
      run += cnt4[j];
    }
    if (tid == 0) pre[nch] = tot;
    __syncthreads();
    CandSource<true> cs{keys, p.cand + (int64_t)r * p.cand_cap, p.cand_key + (int64_t)r * p.cand_cap,
                        sg, pre, nch, tot, tp.b1};
    if (cs.n <= (uint32_t)kStageCap) {
      // one round of independent loads brings every candidate into shared memory
      uint32_t* sk = stage_buf;
      uint32_t* sp = stage_buf + kStageCap;
      // each thread a contiguous run of the list; its first chunk by binary search
      const uint32_t per = (cs.n + kSelThreads - 1) / kSelThreads;
      const uint32_t g0 = min(cs.n, tid * per), g1 = min(cs.n, g0 + per);
      int cur = 0;
      {
        int lo = 0, hi = nch - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (pre[mid] <= g0) lo = mid; else hi = mid - 1;
        }
        cur = lo;
      }
#pragma unroll 4
      for (uint32_t g = g0; g < g1; ++g) {
        while (pre[cur + 1] <= g) ++cur;
        const uint32_t at = soff[cur] + (g - pre[cur]);
        sp[g] = cs.cand[at];
        sk[g] = cs.cand_key[at];
      }
      __syncthreads();
      StagedSource src{sk, sp, cs.n};
      final_select(p, r, tp, src, red, hsm);
    } else {
      GlobalSource<true> src{cs, cs.n};
      final_select(p, r, tp, src, red, hsm);
    }
  } else {
    CandSource<false> cs{keys, nullptr, nullptr, nullptr, nullptr, nch, (uint32_t)len, tp.b1};
    GlobalSource<false> src{cs, (uint32_t)len};
    final_select(p, r, tp, src, red, hsm);
  }
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------
// the driver's tensor-map encoder, looked up once (a function-local static: thread-safe)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2D map over a row-major [rows][cols] array of bf16 (esize 2) or bytes (esize 1), box =
// one 128-byte column chunk x box_rows rows, 128-byte swizzle, out-of-bounds reads as zero.
bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int cols, int box_rows, int esize) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esize), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(ptr), dims, strides, box,
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

int cand_cap_of(int64_t row_len, int topk) {
  const int64_t cap = std::max<int64_t>(32 * (int64_t)topk, 8192);
  return (int)std::max<int64_t>(1, std::min<int64_t>(cap, row_len));
}

struct ProbLayout {
  int64_t stride;
  int chunks, cand_cap;
  size_t keys, hist, fill, done, cand, seg;
};
struct WsLayout {
  ProbLayout p[2];
  size_t zero_lo, zero_hi, total;
};

// Workspace: status | keys (both problems) | zeroed per call: histograms, fill, done |
// candidate lists | segment tables.
WsLayout layout_of(int num_q, int64_t row_len, int64_t brow_len, int topk, int pool_blocks) {
  WsLayout L{};
  const int64_t lens[2] = {row_len, brow_len};
  const int ks[2] = {topk, std::max(pool_blocks, 1)};
  size_t off = CSA2_STATUS_BYTES;
  for (int i = 0; i < 2; ++i) {
    ProbLayout& P = L.p[i];
    P.stride = (lens[i] + 63) / 64 * 64;
    P.chunks = (int)std::max<int64_t>(1, (lens[i] + kSelChunk - 1) / kSelChunk);
    P.cand_cap = cand_cap_of(lens[i], ks[i]);
    P.keys = off;
    off = align256(off + (size_t)num_q * P.stride * 4);
  }
  L.zero_lo = off;
  for (int i = 0; i < 2; ++i) {
    ProbLayout& P = L.p[i];
    P.hist = off;
    off = align256(off + (size_t)num_q * kHistBins * 4);
    P.fill = off;
    off = align256(off + (size_t)num_q * 4);
    P.done = off;
    off = align256(off + (size_t)num_q * 4);
  }
  L.zero_hi = off;
  for (int i = 0; i < 2; ++i) {
    ProbLayout& P = L.p[i];
    P.cand = off;
    off = align256(off + (size_t)num_q * P.cand_cap * 8);   // positions, then keys
    P.seg = off;
    off = align256(off + (size_t)num_q * P.chunks * 2 * 4);
  }
  L.total = off;
  return L;
}

bool pow2_le32(int b) { return b >= 1 && b <= 32 && (b & (b - 1)) == 0; }

// shared driver for Full (kGather = false) and Reindex (kGather = true), bf16 (kESize = 2)
// or E4M3 (kESize = 1) indexer inputs
template <bool kGather, int kESize = 2>
csa2_status_t run_index(const void* qI, const float* w, int num_q, int H_I, int d_I,
                        const void* idx_k, int64_t cap_rows, csa2_seqs_t seqs,
                        const int32_t* q_visible, int max_visible, int topk, int32_t* indices,
                        int pool_blocks, int block, int32_t* pool_out, const int32_t* pool_in,
                        void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int64_t row_len = kGather ? (int64_t)pool_blocks * 8 : max_visible;
  const int64_t brow_len = (!kGather && pool_blocks > 0) ? (max_visible + block - 1) / block : 0;
  const WsLayout L = layout_of(num_q, row_len, brow_len, topk, kGather ? 0 : pool_blocks);
  if (ws_bytes < L.total) return CSA2_ERR_CAPACITY;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  Seqs sq{seqs.seq_start, seqs.seq_len, q_visible, seqs.q_seq,
          seqs.q_per_seq > 0 ? seqs.q_per_seq : 1, seqs.num_seqs, max_visible, status,
          seqs.block_table, seqs.max_pages};

  {
    const uint32_t n16 = (uint32_t)((L.zero_hi - L.zero_lo) / 16);   // both ends 256-aligned
    const unsigned blocks = std::max(1u, std::min(64u, (n16 + 255u) / 256u));
    if (launch_pdl(ws_zero_kernel, dim3(blocks), dim3(256), 0, stream,
                   reinterpret_cast<uint4*>(wsb + L.zero_lo), n16) != cudaSuccess)
      return CSA2_ERR_CUDA;
  }

  // ---- scores (+ first-digit histograms) ----
  CUtensorMap tm_k, tm_q;
  const int box_rows = kGather ? 8 : kTileRows;
  if (!make_map(&tm_k, idx_k, cap_rows, d_I, box_rows, kESize)) return CSA2_ERR_CUDA;
  if (!make_map(&tm_q, qI, (int64_t)num_q * H_I, d_I, H_I, kESize)) return CSA2_ERR_CUDA;
  ScoreArgs sa{};
  sa.seqs = sq;
  sa.w = w;
  sa.H_I = H_I;
  sa.d_I = d_I;
  sa.n_pad = H_I <= 16 ? 16 : 32;
  sa.pool = pool_in;
  sa.pool_blocks = pool_blocks;
  sa.keys = reinterpret_cast<uint32_t*>(wsb + L.p[0].keys);
  sa.key_stride = L.p[0].stride;
  sa.bkeys = brow_len > 0 ? reinterpret_cast<uint32_t*>(wsb + L.p[1].keys) : nullptr;
  sa.bkey_stride = L.p[1].stride;
  sa.block = block;
  sa.hist = reinterpret_cast<uint32_t*>(wsb + L.p[0].hist);
  sa.bhist = brow_len > 0 ? reinterpret_cast<uint32_t*>(wsb + L.p[1].hist) : nullptr;
  sa.wait_ns = wait_limit_ns();
  const uint32_t stage_bytes = (uint32_t)(d_I * kESize / 128) * (kTileRows * 128 + sa.n_pad * 128);
  const int sms = device_sms();
  if (sms <= 0) return CSA2_ERR_CUDA;
  auto kern = score_kernel<kGather, kESize>;
  for (int q0 = 0; q0 < num_q; q0 += kMaxRowsPerLaunch) {
    sa.q0 = q0;
    sa.num_q = std::min(kMaxRowsPerLaunch, num_q - q0);
    const size_t extra = ((size_t)(sa.num_q + 1 + 31) / 32 * 32 + 2 * kHistBins) * 4;
    sa.stages = std::min<int>(8, (int)((216u * 1024u - extra) / stage_bytes));
    const size_t smem = (size_t)sa.stages * stage_bytes + extra + 1024;
    // at least one tile per CTA on average for the largest plausible work
    const int64_t tiles_bound = (int64_t)sa.num_q * ((row_len + kTileRows - 1) / kTileRows);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sms, tiles_bound));
    if (checked(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return CSA2_ERR_CUDA;
    if (launch_pdl(kern, dim3(grid), dim3(kScoreThreads), smem, stream, tm_k, tm_q, sa) !=
        cudaSuccess)
      return CSA2_ERR_CUDA;
  }

  // ---- selection ----
  SelArgs sel{};
  sel.seqs = sq;
  for (int i = 0; i < 2; ++i) {
    SelProblem& P = sel.p[i];
    const ProbLayout& PL = L.p[i];
    P.keys = reinterpret_cast<const uint32_t*>(wsb + PL.keys);
    P.stride = PL.stride;
    P.num_rows = num_q;
    P.hist = reinterpret_cast<const uint32_t*>(wsb + PL.hist);
    P.cand = reinterpret_cast<uint32_t*>(wsb + PL.cand);
    P.cand_key = P.cand + (size_t)num_q * PL.cand_cap;
    P.cand_cap = PL.cand_cap;
    P.seg = reinterpret_cast<uint32_t*>(wsb + PL.seg);
    P.fill = reinterpret_cast<uint32_t*>(wsb + PL.fill);
    P.done = reinterpret_cast<uint32_t*>(wsb + PL.done);
    P.chunks = PL.chunks;
    P.single = PL.stride <= kSelSingle;
  }
  SelProblem& P = sel.p[0];
  P.k = topk;
  P.out = indices;
  P.out_stride = topk;
  P.len_mode = kGather ? 2 : 0;
  P.pool = pool_in;
  P.pool_blocks = pool_blocks;
  int nprob = 1;
  if (brow_len > 0) {
    SelProblem& B = sel.p[1];
    B.k = pool_blocks;
    B.out = pool_out;
    B.out_stride = pool_blocks;
    B.len_mode = 1;
    B.block = block;
    nprob = 2;
  }
  const dim3 grid(std::max(L.p[0].chunks, nprob == 2 ? L.p[1].chunks : 1), num_q, nprob);
  // chunked rows: [kStageCap] keys + positions (96 KB); one-CTA rows: the row's keys, the
  // second- and third-digit histograms and the pool (at most kSelSingle / 8 blocks): 84 KB
  static_assert((kSelSingle + 2048 + 1024 + kSelSingle / 8) * 4 <= 2 * kStageCap * 4, "select smem");
  const size_t sel_smem = (size_t)2 * kStageCap * 4;
  if (checked(cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)sel_smem)) != cudaSuccess)
    return CSA2_ERR_CUDA;
  return launch_pdl(select_kernel, grid, dim3(kSelThreads), sel_smem, stream, sel) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

csa2_status_t check_common(const void* qI, const float* w, int num_q, int H_I, int d_I,
                           const void* idx_k, int64_t cap_rows, const csa2_seqs_t& seqs,
                           int topk, const int32_t* indices) {
  if (num_q < 0 || num_q > 65535 || H_I < 1 || H_I > 32 || (d_I != 64 && d_I != 128))
    return CSA2_ERR_UNSUPPORTED;
  if (topk < 1 || topk > 4096) return CSA2_ERR_UNSUPPORTED;
  if (cap_rows <= 0 || cap_rows > 0x7FFFFFFF) return CSA2_ERR_INVALID_ARG;
  if (seqs.num_seqs < 1 ||
      (!seqs.q_seq && (seqs.q_per_seq < 1 || (int64_t)seqs.num_seqs * seqs.q_per_seq != num_q)))
    return CSA2_ERR_INVALID_ARG;
  if (seqs.block_table && seqs.max_pages < 1) return CSA2_ERR_INVALID_ARG;
  if (num_q == 0) return CSA2_OK;
  if (!qI || !w || !idx_k || !indices || (!seqs.seq_start && !seqs.block_table) || !seqs.seq_len)
    return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qI) & 15) || (reinterpret_cast<uintptr_t>(idx_k) & 15))
    return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

csa2_status_t check_ws(const void* ws) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

// the Full-mode arguments beyond those of check_common; adjusts `block` when there is no pool
csa2_status_t check_full(int max_visible, int pool_blocks, int& block, const int32_t* pool) {
  if (max_visible < 0) return CSA2_ERR_INVALID_ARG;
  if (pool_blocks < 0 || pool_blocks > 8192) return CSA2_ERR_UNSUPPORTED;
  if (pool_blocks > 0 && (!pool || !pow2_le32(block))) return CSA2_ERR_UNSUPPORTED;
  if (pool_blocks == 0) block = 8;
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_index_full_workspace(int32_t num_q, int32_t max_visible, int32_t topk,
                                            int32_t pool_blocks, int32_t block) {
  if (num_q < 0 || max_visible < 0 || block < 1 || topk < 1) return 0;
  const int64_t brow = pool_blocks > 0 ? ((int64_t)max_visible + block - 1) / block : 0;
  return layout_of(num_q, max_visible, brow, topk, pool_blocks).total;
}

extern "C" size_t csa2_index_pool_workspace(int32_t num_q, int32_t pool_blocks, int32_t block,
                                            int32_t topk) {
  if (num_q < 0 || pool_blocks < 0 || block < 1 || topk < 1) return 0;
  return layout_of(num_q, (int64_t)pool_blocks * block, 0, topk, 0).total;
}

extern "C" csa2_status_t csa2_index_full(const uint16_t* qI, const float* w, int32_t num_q,
                                         int32_t H_I, int32_t d_I, const uint16_t* idx_k,
                                         int64_t cap_rows, csa2_seqs_t seqs,
                                         const int32_t* q_visible, int32_t max_visible,
                                         int32_t topk, int32_t* indices, int32_t pool_blocks,
                                         int32_t block, int32_t* pool, void* workspace,
                                         size_t ws_bytes, void* stream) {
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices);
  if (st != CSA2_OK || num_q == 0) return st;
  if ((st = check_ws(workspace)) != CSA2_OK) return st;
  if ((st = check_full(max_visible, pool_blocks, block, pool)) != CSA2_OK) return st;
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
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices);
  if (st != CSA2_OK || num_q == 0) return st;
  if ((st = check_ws(workspace)) != CSA2_OK) return st;
  if (block != 8 || pool_blocks < 1 || pool_blocks > 8192 || !pool) return CSA2_ERR_UNSUPPORTED;
  // positions inside the pool are bounded by the pool; the visibility bound only clamps
  // q_visible values that exceed the sequence
  return run_index<true>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, 0x7FFFFFFF,
                         topk, indices, pool_blocks, block, nullptr, pool, workspace, ws_bytes,
                         (cudaStream_t)stream);
}

extern "C" csa2_status_t csa2_index_full_e4m3(const uint8_t* qI, const float* w, int32_t num_q,
                                              int32_t H_I, int32_t d_I, const uint8_t* idx_k,
                                              int64_t cap_rows, csa2_seqs_t seqs,
                                              const int32_t* q_visible, int32_t max_visible,
                                              int32_t topk, int32_t* indices, int32_t pool_blocks,
                                              int32_t block, int32_t* pool, void* workspace,
                                              size_t ws_bytes, void* stream) {
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices);
  if (st != CSA2_OK || num_q == 0) return st;
  if (d_I != 128) return CSA2_ERR_UNSUPPORTED;             // one 128-byte row per entry
  if ((st = check_ws(workspace)) != CSA2_OK) return st;
  if ((st = check_full(max_visible, pool_blocks, block, pool)) != CSA2_OK) return st;
  return run_index<false, 1>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible,
                             max_visible, topk, indices, pool_blocks, block, pool, nullptr,
                             workspace, ws_bytes, (cudaStream_t)stream);
}

extern "C" csa2_status_t csa2_index_pool_e4m3(const uint8_t* qI, const float* w, int32_t num_q,
                                              int32_t H_I, int32_t d_I, const uint8_t* idx_k,
                                              int64_t cap_rows, csa2_seqs_t seqs,
                                              const int32_t* q_visible, const int32_t* pool,
                                              int32_t pool_blocks, int32_t block, int32_t topk,
                                              int32_t* indices, void* workspace, size_t ws_bytes,
                                              void* stream) {
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices);
  if (st != CSA2_OK || num_q == 0) return st;
  if (d_I != 128) return CSA2_ERR_UNSUPPORTED;
  if ((st = check_ws(workspace)) != CSA2_OK) return st;
  if (block != 8 || pool_blocks < 1 || pool_blocks > 8192 || !pool) return CSA2_ERR_UNSUPPORTED;
  return run_index<true, 1>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, 0x7FFFFFFF,
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
  // the same argument checks, in the same order, as csa2_index_full; the size check last
  csa2_status_t st = check_common(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, topk, indices);
  if (st != CSA2_OK || num_q == 0) return st;
  if ((st = check_full(max_visible, pool_blocks, block, pool)) != CSA2_OK) return st;
  const size_t need = csa2_index_full_workspace(num_q, max_visible, topk, pool_blocks, block);
  if (need == 0 || need > (size_t)CSA2_INDEX_NOALLOC_SCRATCH_BYTES) return CSA2_ERR_CAPACITY;
  void* ws = index_scratch_address();
  if (!ws) return CSA2_ERR_CUDA;
  // the status word starts clear on every call (the histograms are cleared by run_index)
  if (cudaMemsetAsync(ws, 0, CSA2_STATUS_BYTES, (cudaStream_t)stream) != cudaSuccess)
    return CSA2_ERR_CUDA;
  return run_index<false>(qI, w, num_q, H_I, d_I, idx_k, cap_rows, seqs, q_visible, max_visible,
                          topk, indices, pool_blocks, block, pool, nullptr, ws,
                          (size_t)CSA2_INDEX_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream);
}

extern "C" csa2_status_t csa2_index_full_noalloc_status(void* stream) {
  void* ws = index_scratch_address();
  if (!ws) return CSA2_ERR_CUDA;
  return csa2_status_fetch(ws, stream);
}
