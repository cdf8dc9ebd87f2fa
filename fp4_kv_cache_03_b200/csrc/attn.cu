// a7: sparse attention over the selected FP4 entries joined with the layer's own sliding
// window, one softmax over both sets.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", sections "把 prefill 砍掉一半" (every layer
// keeps a 128-token window), "CSA2：在层的维度上共享缓存" (each layer keeps its own main Q
// and window KV; Reuse layers attend with the latest indices) and "FP4 KV 与部署层的几个改动"
// (E2M1 values with one E4M3 scale per 16 channels).
//
// The key slots of a query form tiles of kT slots (kT = 64 for small batches, 128 once the
// CTAs fill the GPU: tile_keys): ceil(topk / kT) index tiles (the selected cache rows; slots
// past topk are empty) and ceil(window / kT) window tiles (its window positions t-W+1 .. t).
// One CTA takes a contiguous range of one query's tiles for a group of HN heads (the MMAs'
// N): 16 when a small batch leaves SMs idle (more CTAs share a query's work), 32, or all 64
// from a full wave on.  A tcgen05.mma costs about the same for M = 64 as for M = 128 and for
// every N <= 64, and a CTA gathers and dequantises each of its rows once for its heads.
//
// Warp roles (288 threads):
//   warps 0-7  (256 threads) per index tile: thread (row r, quarter p) prefetches its part of
//              row r's FP4 codes and the row's scales into registers one tile ahead (from
//              the cache, or in a Reuse layer from the stash of the group's Full / Reindex
//              call), then dequantises them to bf16 (exact: a 2-bit-mantissa code times a
//              4-bit-mantissa scale) into the KV tile, one 128-dim slab at a time as soon as
//              the previous tile's O MMA has released that slab; then softmax of the tile
//              (one key per TMEM lane, half the heads per warp) writes P; at the end, O.
//   warp 8     one thread: loads Q (TMA, once), the window tiles (TMA, one 16-dim slice per
//              box, straight into the KV tile) and issues every MMA:
//                S^T[key, head]  = KV[key, :] . Q[head, :]       (M = kT keys, K = D)
//                O^T[d, head]   += V^T[d, key] . P^T[key, head]  (M = 128 dims per slab)
//              reading the same 32-byte-swizzled KV tile K-major for S^T and MN-major for O^T.
// The slab barriers let the dequantisation of tile i+1 overlap the O MMAs of tile i, and the
// S MMAs of tile i+1 start slab by slab.  The last tile's O^T is normalised and written
// straight from TMEM; when a query is split over several CTAs they write (m, l, O) partials
// that a small kernel merges by log-sum-exp.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kDqWarps = 8;                  // dequantise / softmax / epilogue warps
constexpr int kDqThreads = kDqWarps * 32;
constexpr int kThreads = kDqThreads + 32;    // + the TMA / MMA warp
constexpr int kTile = 128;                   // key slots per tile, the larger of the two sizes
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;         // rescale O only when a max grows by > 2^8

struct AttnArgs {
  int num_q;
  const uint8_t* codes;
  const uint8_t* scales;
  int64_t cap_rows;
  const int64_t* seq_start;
  const int32_t* seq_len;
  const int32_t* q_seq;                      // or null: q / q_per_seq
  int q_per_seq;
  int num_seqs;
  const int32_t* block_table;                // paged cache, or null
  int max_pages;
  const int32_t* indices;
  int topk;
  const uint16_t* swa;
  int64_t swa_rows;
  const int64_t* swa_start;
  const int64_t* q_pos;
  int window;
  int swa_ring;                              // 0: window rows linear; else a ring of this many
  int mode;                                  // csa2_mode_t
  uint8_t* stash;                            // [num_q][n_idx_tiles][stash tile] or null
  int n_idx_tiles;                           // ceil(topk / kT)
  int n_win_tiles;                           // ceil(window / kT)
  int H;                                     // real heads
  int hsplit;                                // head groups per query (CTAs of HN heads)
  float scale_log2;                          // softmax_scale * log2(e)
  int nsplit, tiles_per_split;
  float* part_o;                             // [num_q][nsplit][H][D]  (nsplit > 1)
  float* part_ml;                            // [num_q][nsplit][H][2]  log2-domain m, l
  float* out;
  float* lse;
  int* status;
  uint64_t wait_ns;                          // bound of every wait
};

constexpr uint32_t align1024(uint32_t x) { return (x + 1023u) & ~1023u; }
constexpr uint32_t tmem_cols_for(uint32_t n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

// Shared-memory geometry of one CTA (offsets from a 1024-byte aligned base); kT = key
// slots per tile (64 or 128: the M of the S^T MMA).
template <int D, int HN, int kT>
struct Geo {
  static constexpr int kSlabs = D / 128;               // 128-dim slabs (O^T MMA M)
  static constexpr int kChunks = D / 64;               // Q: 64-element (128-byte) chunks
  static constexpr uint32_t kQChunk = HN * 128;        // [HN rows][128 B]
  // KV tile: D/16 slices of 16 dims, each [kT keys][32 B] with the 32-byte swizzle, so
  // that one MMA K-step (S^T) or one 16-dim chunk of V^T (O^T) is contiguous
  static constexpr uint32_t kKVSlice = kT * 32;
  static constexpr uint32_t kKVBytes = (D / 16) * kKVSlice;
  static constexpr uint32_t kPChunk = HN * 128;        // P chunk: [HN heads][64 keys]
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = align1024(kChunks * kQChunk);
  static constexpr uint32_t kOffP = kOffKV + kKVBytes;
  static constexpr uint32_t kSmem = 1024 + kOffP + (kT / 64) * kPChunk;
  static constexpr uint32_t kTmemCols = tmem_cols_for(HN * (1 + kSlabs));   // S^T + O^T
  // one stash tile: codes [kT][D/2], scales [kT][D/16], validity [kT]
  static constexpr uint32_t kStashCodes = kT * (D / 2);
  static constexpr uint32_t kStashValid = kStashCodes + kT * (D / 16);
  static constexpr uint32_t kStashBytes = kStashValid + kT;
  static_assert(kStashBytes % 16 == 0, "stash tiles stay 16-byte aligned");
};

template <int HN, int kT>
struct AttnSmem {
  uint64_t bar_q, bar_s, bar_p, bar_o, bar_drain;
  uint64_t full_dq[4], full_tma[4], empty[4];    // per slab
  uint32_t tmem_base;
  int abort;
  int rescale;
  float m_ref[HN];
  float l_acc[HN];
  float alpha[HN];
  float red[4][HN];
  int fail;
  uint8_t valid[2][kT];                      // slot validity of index tiles k (k even / odd)
};

// non-negative e4m3 scale byte -> value (bias 7; exponent field 0 is subnormal m * 2^-9)
__device__ __forceinline__ float e4m3_val(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (b & 0x80u) ? -v : v;
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// bf16x2 product; exact here: an e2m1 value times an e4m3 scale has at most 6 significant
// bits and lies in [2^-10, 2688], so it is representable in bf16
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  const __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                   *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
// Eight E2M1 codes (code i in bits [4i, 4i+4) of w) -> four bf16x2 words, unscaled; word k
// holds code 2k in its low half and code 2k+1 in its high half.  Byte permutes only:
// the 3-bit magnitude selects the bf16 high byte H and low byte L from constant tables
//   magnitude  0     1     2     3     4     5     6     7      (value 0 .5 1 1.5 2 3 4 6)
//   H          0x00  0x3F  0x3F  0x3F  0x40  0x40  0x40  0x40
//   L          0x00  0x00  0x80  0xC0  0x00  0x40  0x80  0xC0
// and the sign bit (bit 3 of a code) becomes bit 15 / 31 of its word.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t* m) {
  const uint32_t sel_lo = w & 0x7777u, sel_hi = (w >> 16) & 0x7777u;
  const uint32_t h0 = __byte_perm(0x3F3F3F00u, 0x40404040u, sel_lo);
  const uint32_t l0 = __byte_perm(0xC0800000u, 0xC0804000u, sel_lo);
  const uint32_t h1 = __byte_perm(0x3F3F3F00u, 0x40404040u, sel_hi);
  const uint32_t l1 = __byte_perm(0xC0800000u, 0xC0804000u, sel_hi);
  const uint32_t se = (w & 0x08080808u) << 4;   // sign of code 2k at bit 7 of byte k
  const uint32_t so = w & 0x80808080u;          // sign of code 2k+1 at bit 7 of byte k
  m[0] = __byte_perm(l0, h0, 0x5140u) ^ (__byte_perm(se, so, 0x4000u) & 0x80008000u);
  m[1] = __byte_perm(l0, h0, 0x7362u) ^ (__byte_perm(se, so, 0x5010u) & 0x80008000u);
  m[2] = __byte_perm(l1, h1, 0x5140u) ^ (__byte_perm(se, so, 0x6020u) & 0x80008000u);
  m[3] = __byte_perm(l1, h1, 0x7362u) ^ (__byte_perm(se, so, 0x7030u) & 0x80008000u);
}

__device__ __forceinline__ float fast_exp2(float x) {   // 2^x (MUFU); 2^-inf = 0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Reduce-scatter of v[0..N) across the 32 lanes of a warp (compile-time recursion over the
// lane bits 16, 8, 4, 2, 1): at each step a lane keeps the half of its values selected by
// its lane bit and combines it with the other half from its partner.  Afterwards lane l
// holds the warp-wide result for heads [kOwn*l, kOwn*l + kOwn) in v[0..kOwn), kOwn = N/32.
template <int N, int BIT, bool kMax>
__device__ __forceinline__ void reduce_scatter_step(float* v, int lane) {
  if constexpr (BIT > 0) {
    static_assert(N >= 2, "needs at least two values per lane");
    constexpr int half = N / 2;
    const bool upper = (lane & BIT) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      const float recv = __shfl_xor_sync(0xffffffffu, send, BIT);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
    reduce_scatter_step<half, BIT / 2, kMax>(v, lane);
  }
}

// Per-head reduction of v[0..N) over the 32 lanes (keys) of a warp: afterwards v[0] of
// lane l is the warp-wide result for head l mod N.
template <int N, bool kMax>
__device__ __forceinline__ void warp_reduce_heads(float* v, int lane) {
  reduce_scatter_step<N, N / 2, kMax>(v, lane);
#pragma unroll
  for (int b = N; b < 32; b <<= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, v[0], b);
    v[0] = kMax ? fmaxf(v[0], y) : v[0] + y;
  }
}

// N (8, 16 or 32) consecutive TMEM columns of the calling thread's lane, one wait.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
  if constexpr (N == 32) tmem_ld32(taddr, taddr + 16, v);
  else tmem_ldn<N>(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float* v) {
  if constexpr (N == 32) { tmem_st16(taddr, v); tmem_st16(taddr + 16, v + 16); }
  else tmem_stn<N>(taddr, v);
}

// the 256 dequantise / softmax threads only (warp 8 never joins)
__device__ __forceinline__ void dq_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int D, int HN, int kT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_swa, const AttnArgs a) {
  static_assert(kT == 64 || kT == 128, "64- or 128-key tiles");
  using G = Geo<D, HN, kT>;
  constexpr int kG = kT / 64;                // 8-row groups per dequantising warp
  constexpr int kSlabs = G::kSlabs;
  constexpr int HW = HN / 2;                 // heads per warp in softmax and epilogue
  constexpr uint32_t kKVSlice = G::kKVSlice;
  // byte offset of 16-byte unit u (dims 8u .. 8u+7) of key row r in the KV tile
  auto kv_off = [](int r, int u) -> uint32_t {
    return (uint32_t)(u >> 1) * kKVSlice + (uint32_t)r * 32 + ((uint32_t)((u & 1) ^ ((r >> 2) & 1)) << 4);
  };
  const int Hr = a.H;

  extern __shared__ uint8_t smem_raw[];
  __shared__ AttnSmem<HN, kT> ss;
  // 1024-byte aligned base, derived from the shared array itself so that the compiler keeps
  // the shared address space (and knows these buffers do not alias `ss`)
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = base + G::kOffQ;
  uint8_t* sKV = base + G::kOffKV;
  uint8_t* sP = base + G::kOffP;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg = blockIdx.x % a.hsplit, split = blockIdx.x / a.hsplit, q = blockIdx.y;
  const int h_lo = hg * HN;                  // first head of this CTA's group
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(a.n_idx_tiles + a.n_win_tiles, t_begin + a.tiles_per_split);
  // processing order: the range's window tiles first (their TMA needs no index), then its
  // index tiles
  const int w_lo = max(t_begin, a.n_idx_tiles);
  const int n_w = max(0, t_end - w_lo);                       // window tiles of the range
  const int i_hi = min(t_end, a.n_idx_tiles);
  const int n_i = max(0, i_hi - t_begin);                     // index tiles of the range
  const int n = n_w + n_i;
  volatile int* abort = &ss.abort;

  // set-up that reads no global memory (it overlaps the previous kernel's tail)
  pdl_trigger();
  if (tid == 0) {
    mbar_init(&ss.bar_q, 1);
    mbar_init(&ss.bar_s, 1);
    mbar_init(&ss.bar_p, 1);
    mbar_init(&ss.bar_o, 1);
    mbar_init(&ss.bar_drain, 1);
    for (int j = 0; j < 4; ++j) {
      mbar_init(&ss.full_dq[j], kDqWarps);
      mbar_init(&ss.full_tma[j], 1);
      mbar_init(&ss.empty[j], 1);
    }
    ss.abort = 0;
    ss.rescale = 0;
    fence_barrier_init();
  }
  if (tid == kDqThreads) {
    tma_prefetch_desc(&tm_q);
    if (a.n_win_tiles > 0 && a.swa_rows > 0) tma_prefetch_desc(&tm_swa);
  }
  if (tid < HN) { ss.m_ref[tid] = -INFINITY; ss.l_acc[tid] = 0.0f; }
  if (warp == 0) { tmem_alloc(&ss.tmem_base, G::kTmemCols); tmem_relinquish(); }
  pdl_wait();

  // the query's sequence and window: read after the dependency wait, below, once the first
  // tile's index (or stash) loads are in flight
  int64_t wrow0 = 0;                         // linear: row of the first window position
  int64_t wbase = 0;                         // ring: row of ring slot 0
  int seqv = 0, slen = 0, n_win = 0;
  int64_t t_q = 0;

  // ---- dequantising threads: the FP4 slots this thread loads and converts ----
  // Warp w covers rows 8kG w .. 8kG w + 8kG - 1 of an index tile (kG = kT / 64 groups of 8
  // rows): lane l takes row 8kG w + 8g + (l & 7) of group g, and of each 128-dim slab j the
  // 16-byte piece pq = 4j + (l >> 3) (32 dims).  A warp load then reads 8 rows x 64
  // contiguous bytes, and a warp store of one 16-byte unit hits 8 rows x 4 slices, which the
  // 32-byte swizzle spreads over all banks.
  const int pl = lane >> 3;                  // piece of the slab (0..3)
  auto row_of = [&](int g) { return 8 * kG * warp + 8 * g + (lane & 7); };
  const bool from_stash = a.stash != nullptr && a.mode == CSA2_MODE_REUSE;
  const bool to_stash = a.stash != nullptr && a.mode != CSA2_MODE_REUSE && hg == 0;
  uint4 cw[kG][kSlabs];                      // codes of (row group, slab)
  uint32_t sc[kG][kSlabs];                   // their two scale bytes (low: first 16 dims)
  bool vld[kG];
  int32_t nidx[kG];                          // indices of the next tile to fetch
#pragma unroll
  for (int g = 0; g < kG; ++g) { vld[g] = false; nidx[g] = -1; }
  // a thread's scale pairs in a stash tile: kSc 16-bit values, (group, slab) in that order
  constexpr int kSc = kG * kSlabs;
  auto fetch_index = [&](int t) {
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int slot = t * kT + row_of(g);
      nidx[g] = (!from_stash && slot < a.topk) ? __ldg(a.indices + (int64_t)q * a.topk + slot) : -1;
    }
  };
  // two scale bytes of row group g, slab j: groups 8j + 2pl, +1 = bytes 2(pl & 1), +1 of
  // word 2j + (pl >> 1) of the row's scales
  auto pick_scales = [&](int g, const uint32_t* wv) {
#pragma unroll
    for (int j = 0; j < kSlabs; ++j) {
      const uint32_t w = (pl >> 1) ? wv[2 * j + 1] : wv[2 * j];
      sc[g][j] = (pl & 1) ? (w >> 16) : (w & 0xFFFFu);
    }
  };
  // Loads index tile t (k-th of the range) into registers and records its slot validity.
  auto fetch_rows = [&](int t, int k) {
    if (from_stash) {
      const uint8_t* st = a.stash + ((int64_t)q * a.n_idx_tiles + t) * G::kStashBytes;
      const uint4* sp = reinterpret_cast<const uint4*>(st) + (size_t)warp * (kG * kSlabs) * 32 + lane;
#pragma unroll
      for (int g = 0; g < kG; ++g)
#pragma unroll
        for (int j = 0; j < kSlabs; ++j) cw[g][j] = __ldg(sp + (g * kSlabs + j) * 32);
      const uint8_t* ssc = st + G::kStashCodes + (size_t)(warp * 32 + lane) * (2 * kSc);
      uint32_t wv[(kSc + 1) / 2];
      if constexpr (kSc == 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(ssc));
        wv[0] = v.x; wv[1] = v.y; wv[2] = v.z; wv[3] = v.w;
      } else if constexpr (kSc == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(ssc));
        wv[0] = v.x; wv[1] = v.y;
      } else if constexpr (kSc == 2) {
        wv[0] = __ldg(reinterpret_cast<const uint32_t*>(ssc));
      } else {
        wv[0] = __ldg(reinterpret_cast<const unsigned short*>(ssc));
      }
#pragma unroll
      for (int g = 0; g < kG; ++g)
#pragma unroll
        for (int j = 0; j < kSlabs; ++j) {
          const int i = g * kSlabs + j;
          sc[g][j] = (wv[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
        }
#pragma unroll
      for (int g = 0; g < kG; ++g) vld[g] = st[G::kStashValid + row_of(g)] != 0;
    } else {
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        const int r = row_of(g);
        const int slot = t * kT + r;
        const int p = nidx[g];
        vld[g] = false;
        int64_t grow = -1;
        if (slot < a.topk) {
          if (p >= 0 && p < slen) grow = entry_row(a.seq_start, a.block_table, a.max_pages, seqv, p);
          if (p >= 0 && p < slen && grow >= 0 && grow < a.cap_rows) {
            vld[g] = true;
          } else if (pl == 0 && (p >= slen || p < -1)) {
            report(a.status, CSA2_ERR_INVALID_ARG);
          } else if (pl == 0 && p >= 0) {
            report(a.status, CSA2_ERR_CAPACITY);
          }
        }
        if (vld[g]) {
          const uint8_t* crow = a.codes + grow * (D / 2) + 16 * pl;
#pragma unroll
          for (int j = 0; j < kSlabs; ++j) cw[g][j] = __ldg(reinterpret_cast<const uint4*>(crow + 64 * j));
          const uint8_t* srow = a.scales + grow * (D / 16);
          uint32_t wv[2 * kSlabs];
          if constexpr (kSlabs >= 2) {
#pragma unroll
            for (int c = 0; c < kSlabs / 2; ++c) {
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(srow) + c);
              wv[4 * c] = v.x; wv[4 * c + 1] = v.y; wv[4 * c + 2] = v.z; wv[4 * c + 3] = v.w;
            }
          } else {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(srow));
            wv[0] = v.x; wv[1] = v.y;
          }
          pick_scales(g, wv);
        } else {
#pragma unroll
          for (int j = 0; j < kSlabs; ++j) { cw[g][j] = make_uint4(0, 0, 0, 0); sc[g][j] = 0u; }
        }
      }
    }
    if (pl == 0) {
#pragma unroll
      for (int g = 0; g < kG; ++g) ss.valid[k & 1][row_of(g)] = vld[g] ? 1 : 0;
    }
  };
  // The first index tile's index (or stash rows) goes out first; then the sequence lookups;
  // then the first tile's rows and the index of the one after (their validity is then in
  // shared memory before the barrier below).
  const bool first_fetch = warp < kDqWarps && n_i > 0;
  if (first_fetch) {
    if (from_stash) fetch_rows(t_begin, 0);
    else fetch_index(t_begin);
  }
  {
    int seq = a.q_seq ? a.q_seq[q] : q / a.q_per_seq;
    const bool seq_ok = seq >= 0 && seq < a.num_seqs;
    if (!seq_ok) {
      if (tid == 0) report(a.status, CSA2_ERR_INVALID_ARG);
      seq = 0;
    }
    seqv = seq;
    slen = seq_ok ? a.seq_len[seq] : 0;
    t_q = a.q_pos[q];
    const int64_t w0 = t_q - a.window + 1 > 0 ? t_q - a.window + 1 : 0;
    n_win = seq_ok ? (int)(t_q + 1 - w0 > 0 ? t_q + 1 - w0 : 0) : 0;
    wbase = (seq_ok && a.window > 0) ? a.swa_start[seq] : 0;
    wrow0 = wbase + w0;
  }
  if (first_fetch && !from_stash) {
    fetch_rows(t_begin, 0);
    if (n_i > 1) fetch_index(t_begin + 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  const uint32_t tS = tmem;                  // S^T: HN columns
  const uint32_t tO = tmem + HN;             // O^T slab j: HN columns from tO + j HN

  if (warp == kDqWarps) {
    // =============================== TMA + MMA issue ===============================
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(kT, HN);                    // KV, Q both K-major
      const uint32_t idesc_o = idesc_bf16(128, HN, true, false);      // V^T (128-dim slab) MN-major, P K-major
      const uint64_t kv_desc = sdesc_sw32(smem_u32(sKV), kKVSlice, 256);
      const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t p_desc = sdesc_sw128(smem_u32(sP), 16, 1024);
      bool ok = true;
      uint32_t n_dq = 0, n_tma = 0;          // completed phases of full_dq / full_tma
      int tma_phase = -1, tma_slabs = 0;     // window slabs issued but not yet awaited
      if (n > 0) {
        // Q of all heads once (heads >= H read as zero: the box runs past the map)
        mbar_arrive_expect_tx(&ss.bar_q, (uint32_t)G::kChunks * G::kQChunk);
        for (int c = 0; c < G::kChunks; ++c)
          tma_load_3d(sQ + c * G::kQChunk, &tm_q, c * 64, h_lo, q, &ss.bar_q);
      }
      for (int i = 0; i < n && ok; ++i) {
        const bool win = i < n_w;
        if (win) {
          // window tile: rows straight into the KV tile, one box per 16-dim slice, each slab
          // once the previous tile's O MMA has released it
          const int wt = w_lo + i - a.n_idx_tiles;
          // (rows are below 2^31; a start that far outside the map loads zeros only)
          const int64_t y = (a.swa_ring ? wbase : wrow0) + (int64_t)wt * kT;
          const int32_t y0 = (y < -(int64_t)(1 << 30) || y > (int64_t)0x7FFFFF00) ? -(1 << 30) : (int32_t)y;
          tma_phase = (int)n_tma;
          tma_slabs = 0;
          for (int j = 0; j < kSlabs && ok; ++j) {
            if (i > 0) ok = mbar_wait(&ss.empty[j], (uint32_t)(i - 1) & 1u, abort, a.status, a.wait_ns);
            if (!ok) break;
            mbar_arrive_expect_tx(&ss.full_tma[j], 8u * kKVSlice);
            for (int sl = 0; sl < 8; ++sl)
              tma_load_2d(sKV + (8 * j + sl) * kKVSlice, &tm_swa, (8 * j + sl) * 16, y0, &ss.full_tma[j]);
            ++tma_slabs;
          }
          if (!ok) break;
        }
        if (i == 0) ok = mbar_wait(&ss.bar_q, 0, abort, a.status, a.wait_ns);
        // S^T = KV . Q^T, slab by slab as the slabs become ready
        for (int j = 0; j < kSlabs && ok; ++j) {
          ok = win ? mbar_wait(&ss.full_tma[j], n_tma & 1u, abort, a.status, a.wait_ns)
                   : mbar_wait(&ss.full_dq[j], n_dq & 1u, abort, a.status, a.wait_ns);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int k = 8 * j + kk;                                    // 16-dim K-step
            const uint32_t qoff = (uint32_t)(k >> 2) * G::kQChunk + (k & 3) * 32;
            umma_bf16(tS, kv_desc + (((uint32_t)k * kKVSlice) >> 4), q_desc + (qoff >> 4), idesc_s,
                      k > 0 ? 1u : 0u);
          }
        }
        if (!ok) break;
        if (win) { ++n_tma; tma_phase = -1; } else { ++n_dq; }
        umma_commit(&ss.bar_s);
        ok = mbar_wait(&ss.bar_p, (uint32_t)i & 1u, abort, a.status, a.wait_ns);
        if (!ok) break;
        tc_fence_after();
        // O^T += V^T . P^T, slab by slab; each slab is released when its MMAs complete
        for (int j = 0; j < kSlabs; ++j) {
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk) {
            const uint32_t poff = (uint32_t)(kk >> 2) * G::kPChunk + (kk & 3) * 32;
            const uint32_t off = (uint32_t)(8 * j) * kKVSlice + kk * 512;   // 16 keys = 2 atoms
            umma_bf16(tO + j * HN, kv_desc + (off >> 4), p_desc + (poff >> 4), idesc_o,
                      (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&ss.empty[j]);
        }
      }
      if (ok) {
        if (n > 0) umma_commit(&ss.bar_o);
      } else {
        // abort: the other roles stop waiting; then nothing this thread issued may still be
        // running at exit (every MMA, the window slabs in flight, Q)
        *abort = 1;
        umma_commit(&ss.bar_drain);
        mbar_drain(&ss.bar_drain, 0);
        if (tma_phase >= 0)
          for (int j = 0; j < tma_slabs; ++j) mbar_drain(&ss.full_tma[j], (uint32_t)tma_phase & 1u);
        if (n > 0) mbar_drain(&ss.bar_q, 0);
      }
    }
  } else {
    // ====================== dequantise, softmax, epilogue (warps 0-7) ======================
    const int qd = warp & 3;                   // TMEM lane quadrant of this warp
    const int h0 = (warp >> 2) * HW;           // this warp's heads [h0, h0 + HW)
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;

    // A failed wait (an abort) never leaves the loop early: every thread passes the same
    // sequence of named barriers, skipping the waits and the MMA hand-offs once failed.
    bool ok = true;
    uint32_t ph_s = 0;
    for (int i = 0; i < n; ++i) {
      const bool win = i < n_w;
      const int t = win ? (w_lo + i) : (t_begin + (i - n_w));
      const int k = i - n_w;                   // index tile number within the range
      if (!win) {
        if (to_stash && ok) {
          // the stash holds the tile in this thread order, so a Reuse layer's loads coalesce
          uint8_t* st = a.stash + ((int64_t)q * a.n_idx_tiles + t) * G::kStashBytes;
          uint4* sp = reinterpret_cast<uint4*>(st) + (size_t)warp * (kG * kSlabs) * 32 + lane;
#pragma unroll
          for (int g = 0; g < kG; ++g)
#pragma unroll
            for (int j = 0; j < kSlabs; ++j) sp[(g * kSlabs + j) * 32] = cw[g][j];
          uint8_t* ssc = st + G::kStashCodes + (size_t)(warp * 32 + lane) * (2 * kSc);
          uint32_t wv[(kSc + 1) / 2];
#pragma unroll
          for (int w = 0; w < (kSc + 1) / 2; ++w) wv[w] = 0u;
#pragma unroll
          for (int g = 0; g < kG; ++g)
#pragma unroll
            for (int j = 0; j < kSlabs; ++j) {
              const int i = g * kSlabs + j;
              wv[i >> 1] |= sc[g][j] << (16 * (i & 1));
            }
          if constexpr (kSc == 8) {
            *reinterpret_cast<uint4*>(ssc) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          } else if constexpr (kSc == 4) {
            *reinterpret_cast<uint2*>(ssc) = make_uint2(wv[0], wv[1]);
          } else if constexpr (kSc == 2) {
            *reinterpret_cast<uint32_t*>(ssc) = wv[0];
          } else {
            *reinterpret_cast<unsigned short*>(ssc) = (unsigned short)wv[0];
          }
          if (pl == 0) {
#pragma unroll
            for (int g = 0; g < kG; ++g) st[G::kStashValid + row_of(g)] = vld[g] ? 1 : 0;
          }
        }
        // dequantise slab by slab into the swizzled tile as the previous tile's O MMA
        // releases each slab.  The loop is not unrolled (a short body keeps the kernel's
        // code small: each SM runs it cold); slab j's registers rotate into position 0.
#pragma unroll 1
        for (int j = 0; j < kSlabs; ++j) {
          if (i > 0 && ok) {
            int wok = 1;
            if (lane == 0) wok = mbar_wait(&ss.empty[j], (uint32_t)(i - 1) & 1u, abort, a.status, a.wait_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, wok, 0) != 0;
          }
          if (ok) {
#pragma unroll
            for (int g = 0; g < kG; ++g) {
              const uint4 c4 = cw[g][0];
              const float s0 = e4m3_val(sc[g][0] & 0xFFu), s1 = e4m3_val(sc[g][0] >> 8);
              const uint32_t s02 = pack_bf16(s0, s0), s12 = pack_bf16(s1, s1);   // exact in bf16
              const uint32_t w4[4] = {c4.x, c4.y, c4.z, c4.w};
              const int r = row_of(g);
#pragma unroll
              for (int u4 = 0; u4 < 4; ++u4) {
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
                e2m1x8_to_bf16(w4[u4], ow);
                const uint32_t s2 = u4 < 2 ? s02 : s12;
#pragma unroll
                for (int e = 0; e < 4; ++e) ow[e] = mul_bf16x2(ow[e], s2);
                *reinterpret_cast<uint4*>(sKV + kv_off(r, 4 * (4 * j + pl) + u4)) = o;
              }
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&ss.full_dq[j]);
#pragma unroll
          for (int g = 0; g < kG; ++g) {
#pragma unroll
            for (int jj = 0; jj + 1 < kSlabs; ++jj) { cw[g][jj] = cw[g][jj + 1]; sc[g][jj] = sc[g][jj + 1]; }
          }
        }
        // next index tile: its rows (index already fetched), then the index after it
        if (ok && k + 1 < n_i) {
          fetch_rows(t + 1, k + 1);
          if (k + 2 < n_i && !from_stash) fetch_index(t + 2);
        }
      }
      // ------------------------------ softmax of tile t ------------------------------
      if (ok) {
        int wok = 1;
        if (lane == 0) wok = mbar_wait(&ss.bar_s, ph_s, abort, a.status, a.wait_ns) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, wok, 0) != 0;
      }
      ph_s ^= 1u;
      tc_fence_after();
      // this thread's key row.  M = 128: TMEM lane = key.  M = 64: key m sits in lane
      // 32 (m / 16) + m % 16, so lanes 16-31 of each quadrant hold no key ("dead": they take
      // part in the warp's loads and reductions with p = 0 and store nothing)
      const bool live = kT == 128 || lane < 16;
      const int key = kT == 128 ? qd * 32 + lane : qd * 16 + (lane & 15);
      bool valid = false;
      if (!live) {
      } else if (win) {
        const int u = (t - a.n_idx_tiles) * kT + key;               // window slot / ring slot
        if (a.swa_ring) {
          // ring slot u holds the window position t_q - d, d = (t_q - u) mod ring
          const int64_t d = ((t_q - u) % a.swa_ring + a.swa_ring) % a.swa_ring;
          const int64_t grow = wbase + u;
          const bool in_win = d < n_win;
          valid = in_win && grow >= 0 && grow < a.swa_rows;
          if (in_win && !valid && h0 == 0) report(a.status, CSA2_ERR_CAPACITY);
        } else {
          const int64_t grow = wrow0 + u;
          valid = u < n_win && grow >= 0 && grow < a.swa_rows;
          if (u < n_win && !valid && h0 == 0) report(a.status, CSA2_ERR_CAPACITY);
        }
      } else {
        valid = ss.valid[k & 1][key] != 0;       // written a tile ahead, before a barrier
      }
      float v[HW];
      tmem_ld_cols<HW>(tS + lane_base + h0, v);
      bool over = false;                         // a score above the lazy reference + 2^8
#pragma unroll
      for (int e = 0; e < HW; ++e) {
        v[e] = valid ? v[e] * a.scale_log2 : -INFINITY;
        over = over || (v[e] > ss.m_ref[h0 + e] + kRescaleLog2);
      }
      if (over) ss.rescale = 1;
      dq_sync();
      if (ss.rescale) {
        // the tile's exact per-head max, then every head's reference moves up to its
        // running max; O and l scale by alpha
        {
          float red[HW];
#pragma unroll
          for (int e = 0; e < HW; ++e) red[e] = v[e];
          warp_reduce_heads<HW, true>(red, lane);   // lane holds head h0 + lane % HW
          if (lane < HW) ss.red[qd][h0 + lane] = red[0];
        }
        dq_sync();
        if (tid < HN) {
          const float mt = fmaxf(fmaxf(ss.red[0][tid], ss.red[1][tid]), fmaxf(ss.red[2][tid], ss.red[3][tid]));
          const float mo = ss.m_ref[tid];
          const float mn = fmaxf(mo, mt);
          const float al = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
          ss.alpha[tid] = al;
          ss.l_acc[tid] *= al;
          ss.m_ref[tid] = mn;
        }
        if (tid == 0) ss.rescale = 0;
        dq_sync();
        if (i > 0) {   // O holds earlier tiles (their MMAs completed before S of this tile)
          float al[HW];
#pragma unroll
          for (int e = 0; e < HW; ++e) al[e] = ss.alpha[h0 + e];
#pragma unroll 1
          for (int j = 0; j < kSlabs; ++j) {
            float o[HW];
            const uint32_t ta = tO + lane_base + j * HN + h0;
            tmem_ld_cols<HW>(ta, o);
#pragma unroll
            for (int e = 0; e < HW; ++e) o[e] *= al[e];
            tmem_st_cols<HW>(ta, o);
          }
          tmem_wait_st();
        }
      }
      {
        // p = 2^(s - m_ref), rounded to bf16, written as P[head][key] (a K-major operand:
        // kT / 64 chunks of [HN rows x 64 keys x 2 B], 128-byte swizzle); v becomes the
        // rounded p.  An empty slot (s = -inf) gives p = 0 even while m_ref is still -inf.
        uint8_t* prow = sP + (key >> 6) * G::kPChunk;
        const uint32_t unit = (uint32_t)(key & 63) >> 3, byte = (uint32_t)(key & 7) * 2;
#pragma unroll
        for (int e = 0; e < HW; ++e) {
          const int hh = h0 + e;
          const float pe = v[e] == -INFINITY ? 0.0f : fast_exp2(v[e] - ss.m_ref[hh]);
          const __nv_bfloat16 pb = __float2bfloat16_rn(pe);
          v[e] = __bfloat162float(pb);
          if (live) *reinterpret_cast<__nv_bfloat16*>(prow + hh * 128 + ((unit ^ (hh & 7)) << 4) + byte) = pb;
        }
        warp_reduce_heads<HW, false>(v, lane);
        if (lane < HW) ss.red[qd][h0 + lane] = v[0];
        fence_proxy_async_smem();
        tc_fence_before();
      }
      dq_sync();
      if (tid == 0 && ok) mbar_arrive(&ss.bar_p);
      if (tid < HN) ss.l_acc[tid] += (ss.red[0][tid] + ss.red[1][tid]) + (ss.red[2][tid] + ss.red[3][tid]);
    }

    // ------------------------------ epilogue ------------------------------
    bool done_ok = ok && !*abort;
    if (n > 0 && done_ok) {
      int wok = 1;
      if (lane == 0) wok = mbar_wait(&ss.bar_o, 0, abort, a.status, a.wait_ns) ? 1 : 0;
      done_ok = __shfl_sync(0xffffffffu, wok, 0) != 0;
    }
    // (a vote among the 256 threads: all of them write, or none)
    if (tid == 0) ss.fail = 0;
    dq_sync();
    if (!done_ok) ss.fail = 1;
    dq_sync();
    done_ok = ss.fail == 0;
    tc_fence_after();
    const bool partial = a.nsplit > 1;
    const int n_h = min(HN, Hr - h_lo);          // real heads of this group
    if (done_ok && partial) {
      // Split: the unnormalised O (relative to m_ref) as this split's [H][D] partial, written
      // straight from TMEM (a thread holds one dim of its HW heads, so each warp store is 32
      // consecutive dims of one head: a full 128-byte line), plus (m, l) per head.
      float* dst = a.part_o + (((int64_t)q * a.nsplit + split) * Hr + h_lo) * D;
#pragma unroll 1
      for (int j = 0; j < kSlabs; ++j) {
        const int d = j * 128 + qd * 32 + lane;
        float o[HW];
        if (n > 0) {
          tmem_ld_cols<HW>(tO + lane_base + j * HN + h0, o);
        } else {
#pragma unroll
          for (int e = 0; e < HW; ++e) o[e] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < HW; ++e)
          if (h0 + e < n_h) dst[(size_t)(h0 + e) * D + d] = o[e];
      }
      if (tid < n_h) {
        const float m = ss.m_ref[tid], l = ss.l_acc[tid];
        float* ml = a.part_ml + (((int64_t)q * a.nsplit + split) * Hr + h_lo + tid) * 2;
        ml[0] = (n > 0 && l > 0.0f) ? m : -INFINITY;
        ml[1] = n > 0 ? l : 0.0f;
      }
    } else if (done_ok) {
      // Unsplit: out = O / l, from TMEM into shared memory as [head][D] fp32 rows (the KV
      // tile is free: every MMA has completed), then bulk copies of the H rows.
      float* sO = reinterpret_cast<float*>(sKV);
      float osc[HW];
#pragma unroll
      for (int e = 0; e < HW; ++e) {
        const float l = ss.l_acc[h0 + e];
        osc[e] = n == 0 ? 0.0f : (l > 0.0f ? 1.0f / l : 0.0f);
      }
#pragma unroll 1
      for (int j = 0; j < kSlabs; ++j) {
        const int d = j * 128 + qd * 32 + lane;
        float o[HW];
        if (n > 0) {
          tmem_ld_cols<HW>(tO + lane_base + j * HN + h0, o);
        } else {
#pragma unroll
          for (int e = 0; e < HW; ++e) o[e] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < HW; ++e) sO[(h0 + e) * D + d] = o[e] * osc[e];
      }
      fence_proxy_async_smem();
      dq_sync();
      float* dst = a.out + (int64_t)q * Hr * D;
      if (tid < 32) {
        for (int hh = tid; hh < n_h; hh += 32)
          bulk_s2g(dst + (size_t)(h_lo + hh) * D, sO + (size_t)hh * D, D * 4);
        bulk_commit();
        bulk_wait_all();
      }
      if (tid >= 32 && tid < 32 + n_h && a.lse) {
        const int hh = tid - 32;
        const float m = ss.m_ref[hh], l = ss.l_acc[hh];
        a.lse[(int64_t)q * Hr + h_lo + hh] = (l > 0.0f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

// Merge of the split partials of one query: per head the weights 2^(m_s - M) / L with
// M = max_s m_s and L = sum_s 2^(m_s - M) l_s.  Partials are [head][D] rows, so a thread
// combines one 4-dim group of one head with 16-byte loads, every load in flight at once.
constexpr int kMaxSplit = 16;
// (small CTAs: at batch 1 the merge's partials spread over many SMs)
constexpr int kMergeThreads = 64;
__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(const AttnArgs a, int H, int D) {
  pdl_trigger();
  pdl_wait();
  const int q = blockIdx.y, ns = a.nsplit;
  const int n4 = H * D / 4;                  // 4-dim groups of one partial
  const int g = blockIdx.x * kMergeThreads + threadIdx.x;
  if (g >= n4) return;
  const int h = (g * 4) / D;
  const float4* po = reinterpret_cast<const float4*>(a.part_o + (int64_t)q * ns * H * D) + g;
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml + (int64_t)q * ns * H * 2) + h;
  float4 v[kMaxSplit];
  float2 m[kMaxSplit];
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    if (s < ns) {
      v[s] = __ldg(po + (int64_t)s * n4);
      m[s] = __ldg(ml + s * H);
    } else {
      v[s] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      m[s] = make_float2(-INFINITY, 0.0f);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) M = fmaxf(M, m[s].x);
  float L = 0.0f;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    const float w = (m[s].x == -INFINITY) ? 0.0f : exp2f(m[s].x - M);
    L = fmaf(w, m[s].y, L);
    acc.x = fmaf(w, v[s].x, acc.x);
    acc.y = fmaf(w, v[s].y, acc.y);
    acc.z = fmaf(w, v[s].z, acc.z);
    acc.w = fmaf(w, v[s].w, acc.w);
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  reinterpret_cast<float4*>(a.out + (int64_t)q * H * D)[g] =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (a.lse && g * 4 == h * D)
    a.lse[(int64_t)q * H + h] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// ---------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------
inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

int idx_tiles_of(int topk, int kt) { return (topk + kt - 1) / kt; }
int win_tiles_of(int window, int kt) { return (window + kt - 1) / kt; }

int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Key splits per query: enough CTAs to cover the SMs when the batch is small (each split
// adds a partial of H x D fp32 that the merge reads back), one split from a full wave on.
int nsplit_of(int num_q, int n_tiles) {
  if (n_tiles <= 1 || num_q <= 0) return 1;
  const int per_q = std::max(1, sm_count() / num_q);
  return std::max(1, std::min(std::min(n_tiles, kMaxSplit), per_q));
}

// Keys per tile.  64 when twice the CTAs of 128-key tiles (one per tile and group of 16
// heads) still fit in one wave: each CTA then dequantises half the rows and issues half the
// O MMAs (a tcgen05.mma of M = 64 costs what one of M = 128 does), which shortens a small
// batch's chain.  128 otherwise: fewer, fuller MMAs for batches that fill the GPU.  A pure
// function of the call's shape, so every layer of a group (and the stash) agrees.
int tile_keys(int num_q, int H, int topk, int window) {
  const int64_t n128 = std::max(1, idx_tiles_of(topk, 128) + win_tiles_of(window, 128));
  const int64_t ctas = (int64_t)num_q * std::min<int64_t>(n128, kMaxSplit) * ((H + 15) / 16);
  return 2 * ctas <= sm_count() ? 64 : 128;
}

bool attn_shape_ok(int H, int D) {
  return H >= 1 && H <= 64 && (D == 128 || D == 256 || D == 512);
}

size_t stash_tile_bytes(int D, int kt) { return (size_t)kt * ((size_t)D / 2 + (size_t)D / 16 + 1); }

// the driver's tensor-map encoder, looked up once (a function-local static: thread-safe)
PFN_cuTensorMapEncodeTiled_v12000 attn_encode_fn() {
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

// Q as a [num_q][H][D] bf16 map with boxes of 64 dims x HN heads: heads >= H fall outside
// the map and read as zero.
bool make_q_map(CUtensorMap* tm, const uint16_t* q, int num_q, int H, int D, int HN) {
  auto fn = attn_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)num_q};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)HN, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The window rows as a [swa_rows][D] bf16 map with boxes of 16 dims x kt rows and the
// 32-byte swizzle: one box is one slice of the KV tile.  Rows outside the map read as zero.
bool make_swa_map(CUtensorMap* tm, const uint16_t* swa, int64_t rows, int D, int kt) {
  auto fn = attn_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {16u, (cuuint32_t)kt};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(swa), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int HN, int kT>
cudaError_t launch(AttnArgs a, const uint16_t* q, cudaStream_t st) {
  using G = Geo<D, HN, kT>;
  CUtensorMap tm;
  if (!make_q_map(&tm, q, a.num_q, a.H, D, HN)) return checked(cudaErrorInvalidValue);
  CUtensorMap tm_swa;
  std::memset(&tm_swa, 0, sizeof(tm_swa));  // not read without window tiles
  if (a.n_win_tiles > 0 && a.swa_rows > 0 && !make_swa_map(&tm_swa, a.swa, a.swa_rows, D, kT))
    return checked(cudaErrorInvalidValue);
  cudaError_t e = checked(cudaFuncSetAttribute(attn_tc_kernel<D, HN, kT>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(attn_tc_kernel<D, HN, kT>, dim3(a.nsplit * a.hsplit, a.num_q), dim3(kThreads),
                 (size_t)G::kSmem, st, tm, tm_swa, a);
  if (e != cudaSuccess || a.nsplit <= 1) return e;
  return launch_pdl(attn_merge_kernel, dim3((a.H * D / 4 + kMergeThreads - 1) / kMergeThreads, a.num_q),
                    dim3(kMergeThreads), 0, st, a, a.H, D);
}

// Heads per CTA.  Every CTA gathers and dequantises its query's tiles once for all of its
// heads, and an MMA costs about the same for N = 16 as for N = 64; but a CTA's softmax,
// output and split partial scale with its heads.  Small batches that leave SMs idle split
// the heads into groups of 16 (or 32); from a full wave on, one CTA takes all heads.
int heads_per_cta(int num_q, int nsplit, int H) {
  const int64_t ctas = (int64_t)num_q * nsplit;
  if (ctas * ((H + 15) / 16) <= sm_count()) return 16;
  if (ctas * ((H + 31) / 32) <= sm_count()) return 32;
  return 64;
}

template <int D>
cudaError_t launch_d(AttnArgs a, const uint16_t* q, int kt, cudaStream_t st) {
  if (kt == 64) {                                           // small batches: groups of 16 heads
    a.hsplit = (a.H + 15) / 16;
    return launch<D, 16, 64>(a, q, st);
  }
  const int all = a.H <= 16 ? 16 : a.H <= 32 ? 32 : 64;     // one group of all heads
  const int g = std::min(heads_per_cta(a.num_q, a.nsplit, a.H), all);
  a.hsplit = (a.H + g - 1) / g;
  if (g == 16) return launch<D, 16, 128>(a, q, st);
  if (g == 32) return launch<D, 32, 128>(a, q, st);
  return launch<D, 64, 128>(a, q, st);
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_sparse_attn_stash_bytes(int32_t num_q, int32_t D, int32_t topk) {
  if (num_q < 0 || D < 1 || topk < 0) return 0;
  // (sized for 128-key tiles: at least what 64-key tiles of the same slots take)
  return (size_t)num_q * idx_tiles_of(topk, kTile) * stash_tile_bytes(D, kTile);
}

extern "C" size_t csa2_sparse_attn_workspace(int32_t num_q, int32_t H, int32_t D, int32_t topk,
                                             int32_t window) {
  if (num_q < 0 || H < 1 || D < 1 || topk < 0 || window < 0) return 0;
  const int kt = tile_keys(num_q, H, topk, window);
  const int ns = nsplit_of(num_q, idx_tiles_of(topk, kt) + win_tiles_of(window, kt));
  size_t off = CSA2_STATUS_BYTES;
  if (ns > 1) {
    off = a256(off + (size_t)num_q * ns * H * D * 4);
    off = a256(off + (size_t)num_q * ns * H * 2 * 4);
  }
  return off;
}

extern "C" csa2_status_t csa2_sparse_attn(const uint16_t* q, int32_t num_q, int32_t H, int32_t D,
                                          const uint8_t* kv_codes, const uint8_t* kv_scales,
                                          int64_t cap_rows, csa2_seqs_t seqs,
                                          const int32_t* indices, int32_t topk,
                                          const uint16_t* swa_kv, int64_t swa_rows,
                                          const int64_t* swa_start, const int64_t* q_pos,
                                          int32_t window, int32_t swa_ring,
                                          float softmax_scale, float* out,
                                          float* lse, csa2_mode_t mode, void* kv_stash,
                                          size_t stash_bytes, void* workspace, size_t ws_bytes,
                                          void* stream) {
  if (num_q < 0 || topk < 0 || topk > 2048 || window < 0 || window > 1024) return CSA2_ERR_INVALID_ARG;
  if (swa_ring < 0 || (swa_ring > 0 && (swa_ring % kTile != 0 || swa_ring < window || swa_ring > 1024)))
    return CSA2_ERR_INVALID_ARG;
  if (seqs.block_table && seqs.max_pages < 1) return CSA2_ERR_INVALID_ARG;
  if (!attn_shape_ok(H, D)) return CSA2_ERR_UNSUPPORTED;
  if (seqs.num_seqs < 1 ||
      (!seqs.q_seq && (seqs.q_per_seq < 1 || (int64_t)seqs.num_seqs * seqs.q_per_seq != num_q)))
    return CSA2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < csa2_sparse_attn_workspace(num_q, H, D, topk, window))
    return CSA2_ERR_CAPACITY;
  if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
    return CSA2_ERR_INVALID_ARG;
  if (kv_stash && (reinterpret_cast<uintptr_t>(kv_stash) & 15)) return CSA2_ERR_INVALID_ARG;
  if (kv_stash && stash_bytes < csa2_sparse_attn_stash_bytes(num_q, D, topk)) return CSA2_ERR_CAPACITY;
  if (num_q == 0) return CSA2_OK;
  if (num_q > 65535) return CSA2_ERR_UNSUPPORTED;       // queries are a grid dimension
  if (!q || !out || !q_pos || !seqs.seq_len) return CSA2_ERR_INVALID_ARG;
  if (topk > 0 && !seqs.seq_start && !seqs.block_table) return CSA2_ERR_INVALID_ARG;
  if (topk > 0 && (!indices || !kv_codes || !kv_scales || cap_rows <= 0)) return CSA2_ERR_INVALID_ARG;
  if (window > 0 && (!swa_kv || !swa_start || swa_rows < 0)) return CSA2_ERR_INVALID_ARG;
  if (swa_rows > 0x7FFFFFFF) return CSA2_ERR_UNSUPPORTED;    // window rows are TMA coordinates
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kv_codes) & 15) ||
      (reinterpret_cast<uintptr_t>(kv_scales) & 15) || (reinterpret_cast<uintptr_t>(swa_kv) & 15) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(out) & 15))
    return CSA2_ERR_INVALID_ARG;
  AttnArgs a{};
  a.num_q = num_q;
  a.codes = kv_codes; a.scales = kv_scales; a.cap_rows = cap_rows;
  a.seq_start = seqs.seq_start; a.seq_len = seqs.seq_len;
  a.block_table = seqs.block_table; a.max_pages = seqs.max_pages;
  a.q_seq = seqs.q_seq; a.q_per_seq = seqs.q_per_seq > 0 ? seqs.q_per_seq : 1;
  a.num_seqs = seqs.num_seqs;
  a.indices = indices; a.topk = topk;
  a.swa = swa_kv; a.swa_rows = swa_rows; a.swa_start = swa_start; a.q_pos = q_pos;
  a.window = window;
  a.swa_ring = window > 0 ? swa_ring : 0;
  a.mode = (int)mode;
  a.stash = static_cast<uint8_t*>(kv_stash);
  const int kt = tile_keys(num_q, H, topk, window);
  a.n_idx_tiles = idx_tiles_of(topk, kt);
  a.n_win_tiles = (swa_rows > 0 && window > 0) ? (a.swa_ring ? a.swa_ring / kt : win_tiles_of(window, kt)) : 0;
  a.H = H;
  a.scale_log2 = softmax_scale * kLog2e;
  const int n_tiles = a.n_idx_tiles + a.n_win_tiles;
  // (the split count depends on the call's shape only, as the workspace size does)
  a.nsplit = nsplit_of(num_q, idx_tiles_of(topk, kt) + win_tiles_of(window, kt));
  a.tiles_per_split = std::max(1, (n_tiles + a.nsplit - 1) / a.nsplit);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  size_t off = CSA2_STATUS_BYTES;
  a.part_o = reinterpret_cast<float*>(ws + off);
  off = a256(off + (size_t)num_q * a.nsplit * H * D * 4);
  a.part_ml = reinterpret_cast<float*>(ws + off);
  a.out = out; a.lse = lse;
  a.wait_ns = wait_limit_ns();

  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (D == 128) e = launch_d<128>(a, q, kt, st);
  else if (D == 256) e = launch_d<256>(a, q, kt, st);
  else e = launch_d<512>(a, q, kt, st);
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
