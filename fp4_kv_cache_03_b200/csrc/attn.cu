// a7: sparse attention over the selected FP4 entries joined with the layer's own sliding
// window, one softmax over both sets.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", sections "把 prefill 砍掉一半" (every layer
// keeps a 128-token window), "CSA2：在层的维度上共享缓存" (each layer keeps its own main Q
// and window KV; Reuse layers attend with the latest indices) and "FP4 KV 与部署层的几个改动"
// (E2M1 values with one E4M3 scale per 16 channels).
//
// One CTA handles a range of 128-key tiles of one query for one group of 16 or 32 heads
// (the key slots of a query are [indices[q][0..topk) ; window positions t-W+1 .. t]).
// Per tile:
//   stage    the selected rows' FP4 codes and scales are copied with cp.async (row-
//            contiguous, 16-byte pieces) into a staging area -- or, in a Reuse layer with
//            a stash, come back as one bulk copy of the stage image (with the slots'
//            validity) that the group's Full / Reindex call stored, so that the layer
//            reads no indices; window rows go straight into the tile, by TMA (one box
//            per slice) for a tile of window slots only, else by cp.async;
//   dequant  all 8 warps decode the staged rows to bf16 (exact: a 2-bit-mantissa code times
//            a 4-bit-mantissa scale) into the KV tile: D/16 slices of [128 keys x 32 B]
//            with the 32-byte swizzle, which both MMAs read as contiguous 4 KB blocks;
//   S^T      one thread issues tcgen05.mma: S^T[key, head] = KV[key, :] . Q[head, :]
//            (M = 128 keys, N = the CTA's heads, K = D; Q arrives once by TMA);
//   softmax  all 8 warps read S^T from TMEM (one key per thread, half the heads per warp),
//            form per-head maxima and sums with warp reduce-scatters, keep a lazily
//            rescaled running max per head, and write P (bf16) as [head][key] rows;
//   O^T      tcgen05.mma: O^T[d, head] += V^T[d, key] . P^T[key, head], reading the same
//            swizzled KV tile as an MN-major operand (M = 128 dims per slab).
// The last tile's O^T is normalised and written straight from TMEM; when a query is split
// over several CTAs they write (m, l, O) partials that a small kernel merges by
// log-sum-exp.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kThreads = 256;                // 8 warps
constexpr int kTile = 128;                   // keys per tile (MMA M)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;         // rescale O only when a max grows by > 2^8
constexpr int kScaleStride = 48;             // bytes per staged scale row (16-aligned)

struct AttnArgs {
  int num_q;
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
  int mode;                                  // csa2_mode_t
  uint8_t* stash;                            // [num_q][n_idx_tiles][stage bytes] or null
  int n_idx_tiles;                           // tiles holding index slots: ceil(topk / 128)
  int H;                                     // real heads
  int hsplit;                                // head groups (CTAs) per query and split
  float scale_log2;                          // softmax_scale * log2(e)
  int n_tiles;                               // tiles of the slot list
  int nsplit, tiles_per_split;
  float* part_o;                             // [num_q][nsplit][H][D]  (nsplit > 1)
  float* part_ml;                            // [num_q][nsplit][H][2]  log2-domain m, l
  float* out;
  float* lse;
  int* status;
};

// Shared-memory geometry of one CTA (offsets from a 1024-byte aligned base).
template <int D, int HN>
struct Geo {
  static constexpr int kChunks = D / 64;               // 64-element (128-byte) column chunks
  static constexpr int kSlabs = D / 128;               // O^T slabs of 128 dims (MMA M)
  static constexpr uint32_t kQChunk = HN * 128;        // Q chunk: [HN rows][128 B]
  // KV tile: D/16 slices of 16 dims, each [128 keys][32 B] with the 32-byte swizzle, so
  // that one MMA K-step (S^T) or one 16-dim chunk of V^T (O^T) is a contiguous 4 KB
  static constexpr uint32_t kKVSlice = kTile * 32;
  static constexpr uint32_t kKVBytes = (D / 16) * kKVSlice;
  static constexpr uint32_t kPChunk = HN * 128;        // P chunk: [HN heads][64 keys]
  static constexpr uint32_t kCodeStride = D / 2 + 16;  // staged code row (padded: no bank conflicts)
  static constexpr uint32_t kStageCodes = kTile * kCodeStride;
  static constexpr uint32_t kStageValid = kStageCodes + kTile * kScaleStride;  // 1 byte per slot
  static constexpr uint32_t kStageBytes = kStageValid + kTile;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = (kChunks * kQChunk + 1023) / 1024 * 1024;
  static constexpr uint32_t kOffP = kOffKV + kKVBytes;
  static constexpr uint32_t kOffStage = kOffP + (2 * kPChunk + 1023) / 1024 * 1024;
  static constexpr uint32_t kSmem = 1024 + kOffStage + kStageBytes;
  // S^T as kSAcc partial accumulators (independent MMA chains), then the O^T slabs
  static constexpr int kSAcc = 4;
  static constexpr uint32_t kTmemCols = (kSAcc * HN + kSlabs * HN) <= 128 ? 128 : 256;
  static_assert(kStageBytes % 16 == 0 && D / 16 <= kScaleStride, "stage layout");
};

template <int HN>
struct AttnSmem {
  uint64_t bar_q, bar_s, bar_o, bar_kv;
  uint32_t tmem_base;
  int abort;
  int rescale;
  float m_ref[HN];
  float l_acc[HN];
  float alpha[HN];
  float red[4][HN];
  int kind[kTile];                           // 0 invalid, 1 FP4 row, 2 window row
  int64_t src[kTile];                        // cache row (kind 1) or window row (kind 2)
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

template <int D, int HN>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_swa, const AttnArgs a) {
  using G = Geo<D, HN>;
  constexpr int kChunks = G::kChunks, kSlabs = G::kSlabs;
  constexpr int HW = HN / 2;                 // heads per warp in softmax and epilogue
  constexpr int kParts = D / 32;             // 16-byte code pieces (32 values) of a row
  constexpr int kRowsPerIter = kThreads / kParts;
  constexpr int kIters = kTile / kRowsPerIter;
  constexpr uint32_t kKVSlice = G::kKVSlice;
  // byte offset of 16-byte unit u (dims 8u .. 8u+7) of key row r in the KV tile
  auto kv_off = [](int r, int u) -> uint32_t {
    return (uint32_t)(u >> 1) * kKVSlice + (uint32_t)r * 32 + ((uint32_t)((u & 1) ^ ((r >> 2) & 1)) << 4);
  };
  const int Hr = a.H;

  extern __shared__ uint8_t smem_raw[];
  __shared__ AttnSmem<HN> ss;
  // 1024-byte aligned base, derived from the shared array itself so that the compiler keeps
  // the shared address space (and knows these buffers do not alias `ss`)
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = base + G::kOffQ;
  uint8_t* sKV = base + G::kOffKV;
  uint8_t* sP = base + G::kOffP;
  uint8_t* sStage = base + G::kOffStage;
  uint8_t* sScale = sStage + G::kStageCodes;
  uint8_t* sValid = sStage + G::kStageValid;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3;                 // TMEM lane quadrant of this warp
  const int h0 = (warp >> 2) * HW;           // this warp's heads [h0, h0 + HW) of the group
  const int hg = blockIdx.x % a.hsplit, split = blockIdx.x / a.hsplit, q = blockIdx.y;
  const int h_lo = hg * HN;                  // first head of the CTA's group
  const int seq = q / a.q_per_seq;
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(a.n_tiles, t_begin + a.tiles_per_split);
  volatile int* abort = &ss.abort;

  // set-up that reads no global memory (it overlaps the previous kernel's tail)
  pdl_trigger();
  if (tid == 0) {
    mbar_init(&ss.bar_q, 1);
    mbar_init(&ss.bar_s, 1);
    mbar_init(&ss.bar_o, 1);
    mbar_init(&ss.bar_kv, 1);
    ss.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    if (a.window > 0 && a.swa_rows > 0) tma_prefetch_desc(&tm_swa);
  }
  if (tid < HN) { ss.m_ref[tid] = -INFINITY; ss.l_acc[tid] = 0.0f; }
  if (warp == 0) { tmem_alloc(&ss.tmem_base, G::kTmemCols); tmem_relinquish(); }
  pdl_wait();
  // Q of the group first, by one thread (heads >= H read as zero: the box runs past the map),
  // and a first stash tile, whose address needs nothing from memory
  const bool stash_first = a.stash != nullptr && a.mode == CSA2_MODE_REUSE && t_begin < t_end &&
                           t_begin < a.n_idx_tiles;
  if (tid == 0) {
    mbar_arrive_expect_tx(&ss.bar_q, (uint32_t)kChunks * G::kQChunk);
    for (int c = 0; c < kChunks; ++c)
      tma_load_3d(sQ + c * G::kQChunk, &tm_q, c * 64, h_lo, q, &ss.bar_q);
    if (stash_first) {
      mbar_arrive_expect_tx(&ss.bar_kv, G::kStageBytes);
      bulk_g2s(sStage, a.stash + ((int64_t)q * a.n_idx_tiles + t_begin) * G::kStageBytes,
               G::kStageBytes, &ss.bar_kv);
    }
  }
  // index of row `tid` of a tile (threads < 128), fetched one tile ahead
  int32_t my_idx = 0;
  auto fetch_idx = [&](int t) {
    const int slot = t * kTile + tid;
    const bool stashed = a.stash != nullptr && a.mode == CSA2_MODE_REUSE && t < a.n_idx_tiles;
    if (tid < kTile && slot < a.topk && !stashed) my_idx = __ldg(a.indices + (int64_t)q * a.topk + slot);
  };
  if (t_begin < t_end) fetch_idx(t_begin);

  const int64_t row0 = a.seq_start[seq];
  const int slen = a.seq_len[seq];
  const int64_t t_q = a.q_pos[q];
  const int64_t w0 = t_q - a.window + 1 > 0 ? t_q - a.window + 1 : 0;
  const int n_win = (int)(t_q + 1 - w0 > 0 ? t_q + 1 - w0 : 0);
  const int64_t wrow0 = a.swa_start[seq] + w0;

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  const uint32_t tS = tmem;                  // S^T partial a: columns [a HN, (a+1) HN)
  const uint32_t tO = tmem + G::kSAcc * HN;  // O^T slab j: HN columns from tO + j HN
  const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

  const uint32_t idesc_s = idesc_bf16(kTile, HN);                  // KV, Q both K-major
  const uint32_t idesc_o = idesc_bf16(kTile, HN, true, false);     // V^T MN-major, P K-major
  uint32_t ph_s = 0, ph_o = 0, ph_kv = 0;
  bool q_ready = false, o_init = false, o_pending = false, store_pending = false;

  for (int t = t_begin; t < t_end; ++t) {
    // Reuse with a stash: the tile's selected rows come back as the stage image that the
    // Full / Reindex call (head group 0) stored after its gather.
    const bool stash_tile = a.stash != nullptr && t < a.n_idx_tiles;
    const bool from_stash = stash_tile && a.mode == CSA2_MODE_REUSE;
    const bool to_stash = stash_tile && a.mode != CSA2_MODE_REUSE && hg == 0;
    uint8_t* stile = stash_tile ? a.stash + ((int64_t)q * a.n_idx_tiles + t) * G::kStageBytes : nullptr;
    // a tile of window slots only comes in by TMA: D/16 boxes of [128 rows x 16 dims], each
    // one slice of the tile (rows outside the window are masked, and zeroed below)
    const bool win_tile = t * kTile >= a.topk;
    // the previous tile's O^T MMA and stash store must be done before its buffers are rewritten
    if (store_pending && tid == 0) bulk_wait_read();
    if (o_pending) {
      const bool ok = mbar_wait(&ss.bar_o, ph_o, abort, a.status);
      if (__syncthreads_or(!ok)) break;
      ph_o ^= 1;
      o_pending = false;
      tc_fence_after();
    } else if (store_pending) {
      __syncthreads();
    }
    store_pending = false;
    if (tid == 0 && from_stash && !(t == t_begin && stash_first)) {   // needs no index
      mbar_arrive_expect_tx(&ss.bar_kv, G::kStageBytes);
      bulk_g2s(sStage, stile, G::kStageBytes, &ss.bar_kv);
    } else if (tid == 0 && win_tile) {
      if (a.swa_rows > 0) {
        // (rows are below 2^31; a start that far outside the map loads zeros only)
        const int64_t y = wrow0 + ((int64_t)t * kTile - a.topk);
        const int32_t y0 = (y < -(int64_t)(1 << 30) || y > (int64_t)0x7FFFFF00) ? -(1 << 30) : (int32_t)y;
        mbar_arrive_expect_tx(&ss.bar_kv, (uint32_t)(D / 16) * kKVSlice);
        for (int sl = 0; sl < D / 16; ++sl)
          tma_load_2d(sKV + sl * kKVSlice, &tm_swa, sl * 16, y0, &ss.bar_kv);
      } else {
        mbar_arrive(&ss.bar_kv);             // no rows: every slot is masked and zeroed
      }
    }
    // ------------------------- slots -> sources (one thread per row) -------------------------
    bool ok = true;
    if (from_stash && tid < kTile) ok = mbar_wait(&ss.bar_kv, ph_kv, abort, a.status);
    if (from_stash) ph_kv ^= 1;
    if (tid < kTile) {
      const int slot = t * kTile + tid;
      int kind = 0;
      int64_t src = 0;
      if (slot < a.topk && from_stash) {
        kind = sValid[tid] ? 1 : 0;              // rows are in the stage already
      } else if (slot < a.topk) {
        const int p = my_idx;
        if (p >= 0 && p < slen && row0 + p < a.cap_rows) {
          kind = 1;
          src = row0 + p;
        } else if (p >= slen || p < -1) {
          report(a.status, CSA2_ERR_INVALID_ARG);
        } else if (p >= 0) {
          report(a.status, CSA2_ERR_CAPACITY);
        }
      } else if (slot - a.topk < n_win) {
        const int64_t grow = wrow0 + (slot - a.topk);
        if (grow >= 0 && grow < a.swa_rows) {
          kind = 2;
          src = grow;
        } else {
          report(a.status, CSA2_ERR_CAPACITY);
        }
      }
      ss.kind[tid] = kind;
      ss.src[tid] = src;
      if (to_stash && slot < a.topk) sValid[tid] = kind != 0;
    }
    if (__syncthreads_or(!ok)) break;
    if (t + 1 < t_end) fetch_idx(t + 1);
    // ------------------------- loads (a row's threads are contiguous) -------------------------
    {
      const int lp = tid % kParts;
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        const int r = it * kRowsPerIter + tid / kParts;
        const int kind = ss.kind[r];
        if (kind == 1 && !from_stash) {
          const int64_t grow = ss.src[r];
          cp_async16(sStage + r * G::kCodeStride + lp * 16, a.codes + grow * (D / 2) + lp * 16);
          if constexpr (D / 16 >= 16) {
            if (lp * 16 < D / 16) cp_async16(sScale + r * kScaleStride + lp * 16, a.scales + grow * (D / 16) + lp * 16);
          } else {
            if (lp == 0) cp_async8(sScale + r * kScaleStride, a.scales + grow * (D / 16));
          }
        } else if (kind == 2 && !win_tile) {
          const uint16_t* src = a.swa + ss.src[r] * D;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = 4 * lp + i;
            cp_async16(sKV + kv_off(r, u), src + u * 8);
          }
        } else if (kind == 0 && to_stash && t * kTile + r < a.topk) {
          // an index slot without a row is stored as zero codes and scales
          *reinterpret_cast<uint4*>(sStage + r * G::kCodeStride + lp * 16) = make_uint4(0, 0, 0, 0);
          if (lp * 16 < D / 16) {
            if constexpr (D / 16 >= 16)
              *reinterpret_cast<uint4*>(sScale + r * kScaleStride + lp * 16) = make_uint4(0, 0, 0, 0);
            else
              *reinterpret_cast<uint2*>(sScale + r * kScaleStride) = make_uint2(0, 0);
          }
        }
      }
    }
    cp_async_wait_all();
    if (win_tile) {
      ok = mbar_wait(&ss.bar_kv, ph_kv, abort, a.status);
      ph_kv ^= 1;
    }
    if (to_stash) fence_proxy_async_smem();  // staged rows -> the bulk store below
    if (__syncthreads_or(!ok)) break;
    if (to_stash) {
      if (tid == 0) {
        bulk_s2g(stile, sStage, G::kStageBytes);
        bulk_commit();
      }
      store_pending = true;                  // uniform: every thread takes the same branches
    }
    // ------------------------- dequantise into the swizzled tile -------------------------
    // consecutive threads take consecutive rows: the 8 threads of a quarter warp then store
    // one 16-byte unit of each of 8 consecutive rows of a slice, which the 32-byte swizzle
    // spreads over all 32 banks
    {
      const int rsub = tid % kRowsPerIter;
      const int part = tid / kRowsPerIter;
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        const int r = it * kRowsPerIter + rsub;
        const int kind = ss.kind[r];
        // a stash holds zero codes for index slots without a row
        const bool dec = from_stash ? (t * kTile + r < a.topk) : (kind == 1);
        if (dec) {
          const uint4 cw = *reinterpret_cast<const uint4*>(sStage + r * G::kCodeStride + part * 16);
          const uint32_t sc = *reinterpret_cast<const uint16_t*>(sScale + r * kScaleStride + part * 2);
          const float s0 = e4m3_val(sc & 0xFFu), s1 = e4m3_val((sc >> 8) & 0xFFu);
          const uint32_t s02 = pack_bf16(s0, s0), s12 = pack_bf16(s1, s1);   // exact in bf16
          const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {              // unit i: 8 values of word w4[i]
            const uint32_t s2 = i < 2 ? s02 : s12;
            uint4 o;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
            e2m1x8_to_bf16(w4[i], ow);
#pragma unroll
            for (int k = 0; k < 4; ++k) ow[k] = mul_bf16x2(ow[k], s2);
            const int u = 4 * part + i;
            *reinterpret_cast<uint4*>(sKV + kv_off(r, u)) = o;
          }
        } else if (kind == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = 4 * part + i;
            *reinterpret_cast<uint4*>(sKV + kv_off(r, u)) = make_uint4(0, 0, 0, 0);
          }
        }
      }
    }
    fence_proxy_async_smem();
    const int any = __syncthreads_or(tid < kTile && ss.kind[tid] != 0);
    if (!any) continue;

    // ------------------------------ S^T = KV . Q^T ------------------------------
    if (tid == 0) {
      bool okq = true;
      if (!q_ready) { okq = mbar_wait(&ss.bar_q, 0, abort, a.status); q_ready = okq; }
      if (okq) {
        tc_fence_after();
        const uint64_t kv_desc_k = sdesc_sw32(smem_u32(sKV), kKVSlice, 256);  // KV as K-major A
        const uint64_t q_desc_k = sdesc_sw128(smem_u32(sQ), 16, 1024);     // Q as K-major B
        // K-step k accumulates into partial k mod kSAcc: kSAcc independent chains
#pragma unroll 4
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (uint32_t)k * kKVSlice;
          const uint32_t qoff = (uint32_t)(k >> 2) * G::kQChunk + (k & 3) * 32;
          umma_bf16(tS + (uint32_t)(k % G::kSAcc) * HN, kv_desc_k + (off >> 4),
                    q_desc_k + (qoff >> 4), idesc_s, k >= G::kSAcc ? 1u : 0u);
        }
        umma_commit(&ss.bar_s);
      }
    }

    // ------------------------------ softmax (all 8 warps) ------------------------------
    // warp w: keys of TMEM lane quadrant (w & 3), heads [h0, h0 + HW)
    const int r = quad * 32 + lane;               // key row = TMEM lane
    float v[HW];
    ok = mbar_wait(&ss.bar_s, ph_s, abort, a.status);
    ok = __syncthreads_and(ok);
    ph_s ^= 1;
    if (!ok) break;
    tc_fence_after();
    tmem_ld_sum4<HW>(tS + lane_base + h0, HN, v);   // S^T = the sum of the partials
    {
      const bool valid = ss.kind[r] != 0;
#pragma unroll
      for (int h = 0; h < HW; ++h) v[h] = valid ? v[h] * a.scale_log2 : -INFINITY;
      float red[HW];
#pragma unroll
      for (int h = 0; h < HW; ++h) red[h] = v[h];
      warp_reduce_heads<HW, true>(red, lane);     // lane holds head h0 + lane % HW
      if (lane < HW) ss.red[quad][h0 + lane] = red[0];
    }
    if (tid == 0) ss.rescale = 0;
    __syncthreads();
    if (tid < HN) {
      const float mt = fmaxf(fmaxf(ss.red[0][tid], ss.red[1][tid]), fmaxf(ss.red[2][tid], ss.red[3][tid]));
      ss.alpha[tid] = mt;                          // stash the tile max
      if (mt > ss.m_ref[tid] + kRescaleLog2) ss.rescale = 1;
    }
    __syncthreads();
    if (ss.rescale) {
      // move every head's reference max up to its running max; O and l scale by alpha
      if (tid < HN) {
        const float mo = ss.m_ref[tid];
        const float mn = fmaxf(mo, ss.alpha[tid]);
        const float al = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
        ss.alpha[tid] = al;
        ss.l_acc[tid] *= al;
        ss.m_ref[tid] = mn;
      }
      __syncthreads();
      if (o_init) {
        float al[HW];
#pragma unroll
        for (int i = 0; i < HW; ++i) al[i] = ss.alpha[h0 + i];
#pragma unroll 1
        for (int j = 0; j < kSlabs; ++j) {
          float o[HW];
          const uint32_t ta = tO + lane_base + j * HN + h0;
          tmem_ldn<HW>(ta, o);
#pragma unroll
          for (int i = 0; i < HW; ++i) o[i] *= al[i];
          tmem_stn<HW>(ta, o);
        }
        tmem_wait_st();
      }
    }
    {
      // p = 2^(s - m_ref), rounded to bf16, written as P[head][key] (a K-major operand:
      // two 64-key chunks of [HN rows x 128 B], 128-byte swizzle); v becomes the rounded p
      uint8_t* prow = sP + (r >> 6) * G::kPChunk;
      const uint32_t unit = (uint32_t)(r & 63) >> 3, byte = (uint32_t)(r & 7) * 2;
#pragma unroll
      for (int i = 0; i < HW; ++i) {
        const int h = h0 + i;
        const __nv_bfloat16 pb = __float2bfloat16_rn(fast_exp2(v[i] - ss.m_ref[h]));
        v[i] = __bfloat162float(pb);
        *reinterpret_cast<__nv_bfloat16*>(prow + h * 128 + ((unit ^ (h & 7)) << 4) + byte) = pb;
      }
      warp_reduce_heads<HW, false>(v, lane);
      if (lane < HW) ss.red[quad][h0 + lane] = v[0];
      fence_proxy_async_smem();
      tc_fence_before();
    }
    __syncthreads();
    if (tid < HN) ss.l_acc[tid] += (ss.red[0][tid] + ss.red[1][tid]) + (ss.red[2][tid] + ss.red[3][tid]);
    // ------------------------------ O^T += V^T . P^T ------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint64_t kv_desc_mn = sdesc_sw32(smem_u32(sKV), kKVSlice, 256);    // V^T, MN-major A
      const uint64_t p_desc_k = sdesc_sw128(smem_u32(sP), 16, 1024);           // P, K-major B
      // key steps outermost: consecutive MMAs go to the kSlabs independent slabs
#pragma unroll 2
      for (int k = 0; k < kTile / 16; ++k) {
        const uint32_t poff = (uint32_t)(k >> 2) * G::kPChunk + (k & 3) * 32;
#pragma unroll
        for (int j = 0; j < kSlabs; ++j) {
          const uint32_t off = (uint32_t)(8 * j) * kKVSlice + k * 512;   // 16 keys = 2 atoms
          umma_bf16(tO + j * HN, kv_desc_mn + (off >> 4), p_desc_k + (poff >> 4), idesc_o,
                    (o_init || k > 0) ? 1u : 0u);
        }
      }
      umma_commit(&ss.bar_o);
    }
    o_init = true;
    o_pending = true;
  }

  // ------------------------------ epilogue ------------------------------
  if (store_pending && tid == 0) bulk_wait_read();
  bool done_ok = !*abort;
  if (o_pending) done_ok = mbar_wait(&ss.bar_o, ph_o, abort, a.status) && done_ok;
  done_ok = __syncthreads_and(done_ok);
  tc_fence_after();
  const bool partial = a.nsplit > 1;
  if (done_ok) {
    // Straight from TMEM: a thread holds one dim of HW heads, so a warp stores one full
    // 128-byte line per head.  Unsplit: out = O / l.  Split: the unnormalised O (relative
    // to m_ref) as [H][D] rows of this split, plus (m, l) per head.
    float* dst = partial ? a.part_o + ((int64_t)q * a.nsplit + split) * Hr * D
                         : a.out + (int64_t)q * Hr * D;
    float osc[HW];
#pragma unroll
    for (int i = 0; i < HW; ++i) {
      const float l = ss.l_acc[h0 + i];
      osc[i] = !o_init ? 0.0f : (partial ? 1.0f : (l > 0.0f ? 1.0f / l : 0.0f));
    }
#pragma unroll 1
    for (int j = 0; j < kSlabs; ++j) {
      const int d = j * 128 + quad * 32 + lane;
      float o[HW];
      if (o_init) {
        tmem_ldn<HW>(tO + lane_base + j * HN + h0, o);
      } else {
#pragma unroll
        for (int i = 0; i < HW; ++i) o[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < HW; ++i) {
        const int h = h_lo + h0 + i;
        if (h < Hr) dst[h * D + d] = o[i] * osc[i];
      }
    }
    if (tid < HN && h_lo + tid < Hr) {
      const int h = h_lo + tid;
      const float m = ss.m_ref[tid], l = ss.l_acc[tid];
      if (partial) {
        float* ml = a.part_ml + (((int64_t)q * a.nsplit + split) * Hr + h) * 2;
        ml[0] = (o_init && l > 0.0f) ? m : -INFINITY;
        ml[1] = o_init ? l : 0.0f;
      } else if (a.lse) {
        a.lse[(int64_t)q * Hr + h] = (l > 0.0f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
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
// (small CTAs: at batch 1 the merge's 640 KB of partials spread over 128 SMs)
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

int n_tiles_of(int topk, int window) { return (topk + window + kTile - 1) / kTile; }

int nsplit_of(int num_q, int n_tiles) {
  if (n_tiles <= 1) return 1;
  return std::max(1, std::min(std::min(n_tiles, kMaxSplit), 512 / std::max(1, num_q)));
}

bool attn_shape_ok(int H, int D) {
  return H >= 1 && H <= 64 && (D == 128 || D == 256 || D == 512);
}

// bytes of one staged tile (and of one stash tile): padded code rows, scale rows, then one
// validity byte per slot
size_t stage_bytes_of(int D) { return (size_t)kTile * ((size_t)D / 2 + 16 + kScaleStride + 1); }

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

// Heads per CTA: groups of 16 while every CTA of the call fits on the GPU at once (the
// latency-bound small batches), else 32 (fewer repeated gathers per query).
int head_group_of(int num_q, int nsplit, int H) {
  return (int64_t)num_q * nsplit * ((H + 15) / 16) <= sm_count() ? 16 : 32;
}

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

// Q as a [num_q][H][D] bf16 map with boxes of 64 dims x HN heads: heads >= H of the last
// group fall outside the map and read as zero.
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

// The window rows as a [swa_rows][D] bf16 map with boxes of 16 dims x 128 rows and the
// 32-byte swizzle: one box is one slice of the KV tile.  Rows outside the map read as zero.
bool make_swa_map(CUtensorMap* tm, const uint16_t* swa, int64_t rows, int D) {
  auto fn = attn_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {16u, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(swa), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int HN>
cudaError_t launch(AttnArgs a, const uint16_t* q, cudaStream_t st) {
  using G = Geo<D, HN>;
  CUtensorMap tm;
  if (!make_q_map(&tm, q, a.num_q, a.H, D, HN)) return cudaErrorInvalidValue;
  CUtensorMap tm_swa;
  std::memset(&tm_swa, 0, sizeof(tm_swa));  // not read without window slots
  if (a.window > 0 && a.swa_rows > 0 && !make_swa_map(&tm_swa, a.swa, a.swa_rows, D))
    return cudaErrorInvalidValue;
  a.hsplit = (a.H + HN - 1) / HN;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, HN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(attn_tc_kernel<D, HN>, dim3(a.nsplit * a.hsplit, a.num_q), dim3(kThreads),
                 (size_t)G::kSmem, st, tm, tm_swa, a);
  if (e != cudaSuccess || a.nsplit <= 1) return e;
  return launch_pdl(attn_merge_kernel, dim3((a.H * D / 4 + kMergeThreads - 1) / kMergeThreads, a.num_q),
                    dim3(kMergeThreads), 0, st, a, a.H, D);
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_sparse_attn_stash_bytes(int32_t num_q, int32_t D, int32_t topk) {
  if (num_q < 0 || D < 1 || topk < 0) return 0;
  return (size_t)num_q * ((topk + kTile - 1) / kTile) * stage_bytes_of(D);
}

extern "C" size_t csa2_sparse_attn_workspace(int32_t num_q, int32_t H, int32_t D, int32_t topk,
                                             int32_t window) {
  if (num_q < 0 || H < 1 || D < 1 || topk < 0 || window < 0) return 0;
  const int ns = nsplit_of(num_q, n_tiles_of(topk, window));
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
                                          int32_t window, float softmax_scale, float* out,
                                          float* lse, csa2_mode_t mode, void* kv_stash,
                                          size_t stash_bytes, void* workspace, size_t ws_bytes,
                                          void* stream) {
  if (num_q < 0 || topk < 0 || topk > 2048 || window < 0 || window > 1024) return CSA2_ERR_INVALID_ARG;
  if (!attn_shape_ok(H, D)) return CSA2_ERR_UNSUPPORTED;
  if (seqs.num_seqs < 1 || seqs.q_per_seq < 1 || (int64_t)seqs.num_seqs * seqs.q_per_seq != num_q)
    return CSA2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < csa2_sparse_attn_workspace(num_q, H, D, topk, window))
    return CSA2_ERR_CAPACITY;
  if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
    return CSA2_ERR_INVALID_ARG;
  if (kv_stash && (stash_bytes < csa2_sparse_attn_stash_bytes(num_q, D, topk) ||
                   (reinterpret_cast<uintptr_t>(kv_stash) & 15)))
    return kv_stash && (reinterpret_cast<uintptr_t>(kv_stash) & 15) ? CSA2_ERR_INVALID_ARG
                                                                    : CSA2_ERR_CAPACITY;
  if (num_q == 0) return CSA2_OK;
  if (num_q > 65535) return CSA2_ERR_UNSUPPORTED;       // queries are a grid dimension
  if (!q || !out || !q_pos || !seqs.seq_start || !seqs.seq_len) return CSA2_ERR_INVALID_ARG;
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
  a.seq_start = seqs.seq_start; a.seq_len = seqs.seq_len; a.q_per_seq = seqs.q_per_seq;
  a.indices = indices; a.topk = topk;
  a.swa = swa_kv; a.swa_rows = swa_rows; a.swa_start = swa_start; a.q_pos = q_pos;
  a.window = window;
  a.mode = (int)mode;
  a.stash = static_cast<uint8_t*>(kv_stash);
  a.n_idx_tiles = (topk + kTile - 1) / kTile;
  a.H = H;
  a.scale_log2 = softmax_scale * kLog2e;
  a.n_tiles = n_tiles_of(topk, window);
  a.nsplit = nsplit_of(num_q, a.n_tiles);
  a.tiles_per_split = (a.n_tiles + a.nsplit - 1) / a.nsplit;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  size_t off = CSA2_STATUS_BYTES;
  a.part_o = reinterpret_cast<float*>(ws + off);
  off = a256(off + (size_t)num_q * a.nsplit * H * D * 4);
  a.part_ml = reinterpret_cast<float*>(ws + off);
  a.out = out; a.lse = lse;

  cudaStream_t st = (cudaStream_t)stream;
  const bool g16 = head_group_of(num_q, a.nsplit, H) == 16;
  cudaError_t e = cudaSuccess;
  if (D == 128) e = g16 ? launch<128, 16>(a, q, st) : launch<128, 32>(a, q, st);
  else if (D == 256) e = g16 ? launch<256, 16>(a, q, st) : launch<256, 32>(a, q, st);
  else e = g16 ? launch<512, 16>(a, q, st) : launch<512, 32>(a, q, st);
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
