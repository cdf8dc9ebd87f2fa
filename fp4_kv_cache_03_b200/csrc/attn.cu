// a7: sparse attention over the selected FP4 entries joined with the layer's own sliding
// window, one softmax over both sets.
// Pages: aprilzz.com "DeepSeek V4.1 Flash 发布…", sections "把 prefill 砍掉一半" (every layer
// keeps a 128-token window), "CSA2：在层的维度上共享缓存" (each layer keeps its own main Q
// and window KV; Reuse layers attend with the latest indices) and "FP4 KV 与部署层的几个改动"
// (E2M1 values with one E4M3 scale per 16 channels).
//
// One CTA handles a range of 128-key tiles of one query.  The key slots of a query are
// [indices[q][0..topk) ; window positions t-W+1 .. t].  Per tile:
//   gather   all 8 warps load the tile's rows -- FP4 rows are dequantised in registers to
//            bf16 (exact: a 2-bit-mantissa code times a 4-bit-mantissa scale), window rows
//            are copied with cp.async -- into a 128-byte-swizzled [128 keys x D] tile;
//   S^T      one thread issues tcgen05.mma: S^T[key, head] = KV[key, :] . Q[head, :]
//            (M = 128 keys, N = heads, K = D; Q arrives once by TMA);
//   softmax  warps 0-3 read S^T from TMEM (one key per thread), form per-head maxima and
//            sums with warp reduce-scatters, keep a lazily rescaled running max per head,
//            and write P (bf16) as [key][head] rows -- an MN-major operand;
//   O^T      tcgen05.mma: O^T[d, head] += V^T[d, key] . P^T[key, head], reading the same
//            swizzled KV tile as an MN-major operand (M = 128 dims per slab, N = heads).
// The last tile's O^T is normalised and written; when a query is split over several CTAs
// they write (m, l, O) partials that a small kernel merges by log-sum-exp.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"

namespace csa2 {
namespace {

constexpr int kThreads = 256;                // 8 warps
constexpr int kTile = 128;                   // keys per tile (MMA M)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;         // rescale O only when a max grows by > 2^8

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
  uint8_t* stash;                            // [num_q][n_idx_tiles][tile bytes] or null
  int n_idx_tiles;                           // tiles holding index slots: ceil(topk / 128)
  int H;                                     // real heads (<= kN); the rest are padding
  float scale_log2;                          // softmax_scale * log2(e)
  int n_tiles;                               // tiles of the slot list
  int nsplit, tiles_per_split;
  float* part_o;                             // [num_q][nsplit][H][D]  (nsplit > 1)
  float* part_ml;                            // [num_q][nsplit][H][2]  log2-domain m, l
  float* out;
  float* lse;
  int* status;
};

constexpr int kN = 64;                       // MMA N: heads, padded to 64

template <int H>
struct AttnSmem {
  uint64_t bar_q, bar_s, bar_o, bar_kv;
  uint32_t tmem_base;
  int abort;
  int rescale;
  float m_ref[H];
  float l_acc[H];
  float alpha[H];
  float red[4][H];
  int valid[kTile];
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const AttnArgs a) {
  constexpr int H = kN;
  constexpr int kChunks = D / 64;            // 64-element (128-byte) column chunks
  constexpr int kSlabs = D / 128;            // O^T slabs of 128 dims (MMA M)
  constexpr uint32_t kQChunk = H * 128;      // bytes of one Q chunk ([H rows][128 B])
  constexpr uint32_t kQBytes = kChunks * kQChunk;
  constexpr uint32_t kKVChunk = kTile * 128;  // 16 KB
  constexpr uint32_t kTmemCols = (H + kSlabs * H) <= 128 ? 128 : ((H + kSlabs * H) <= 256 ? 256 : 512);
  static_assert(D % 128 == 0 && D <= 512, "shape");
  const int Hr = a.H;

  extern __shared__ uint8_t smem_raw[];
  __shared__ AttnSmem<H> ss;
  // 1024-byte aligned base, derived from the shared array itself so that the compiler keeps
  // the shared address space (and knows these buffers do not alias `ss`)
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = base;
  uint8_t* sKV = sQ + ((kQBytes + 1023) / 1024) * 1024;
  uint8_t* sP = sKV + kChunks * kKVChunk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3;                 // TMEM lane quadrant of this warp
  const int hh = warp >> 2;                  // head half (softmax / epilogue columns)
  const int split = blockIdx.x, q = blockIdx.y;
  const int seq = q / a.q_per_seq;
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(a.n_tiles, t_begin + a.tiles_per_split);
  volatile int* abort = &ss.abort;

  // Q goes out first: barrier init, then its TMA, by one thread
  if (tid == 0) {
    mbar_init(&ss.bar_q, 1);
    mbar_init(&ss.bar_s, 1);
    mbar_init(&ss.bar_o, 1);
    mbar_init(&ss.bar_kv, 1);
    ss.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    mbar_arrive_expect_tx(&ss.bar_q, (uint32_t)kChunks * Hr * 128);
    for (int c = 0; c < kChunks; ++c) tma_load_2d(sQ + c * kQChunk, &tm_q, c * 64, q * Hr, &ss.bar_q);
  }

  const int64_t row0 = a.seq_start[seq];
  const int slen = a.seq_len[seq];
  const int64_t t_q = a.q_pos[q];
  const int64_t w0 = t_q - a.window + 1 > 0 ? t_q - a.window + 1 : 0;
  const int n_win = (int)(t_q + 1 - w0 > 0 ? t_q + 1 - w0 : 0);
  const int64_t wrow0 = a.swa_start[seq] + w0;

  // gather geometry: kParts threads per row, each covering 32 columns (4 units of 8 bf16)
  constexpr int kParts = D / 32;
  constexpr int kRowsPerIter = kThreads / kParts;
  constexpr int kIters = kTile / kRowsPerIter;
  // consecutive threads take consecutive rows: the 8 threads of a quarter warp then store
  // to 8 different rows, whose 128-byte swizzle puts their 16-byte units in 8 bank groups
  const int rsub = tid % kRowsPerIter;
  const int part = tid / kRowsPerIter;
  int kind[kIters];                          // 0 invalid, 1 FP4 row, 2 window row
  int32_t gidx[kIters];                      // FP4: sequence position; window: offset in window
  // Phase 1 of a tile's gather: slot -> source (the index load is only issued here).
  auto issue_slots = [&](int t) {
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int slot = t * kTile + it * kRowsPerIter + rsub;
      kind[it] = 0;
      gidx[it] = 0;
      if (slot < a.topk) {
        gidx[it] = __ldg(a.indices + (int64_t)q * a.topk + slot);
        kind[it] = 1;
      } else if (slot - a.topk < n_win) {
        gidx[it] = slot - a.topk;
        kind[it] = 2;
      }
    }
  };
  if (t_begin < t_end) issue_slots(t_begin);

  if (tid < H) { ss.m_ref[tid] = -INFINITY; ss.l_acc[tid] = 0.0f; }
  if (Hr < H) {  // rows of padding heads must read as zero; TMA writes rows < Hr only
    const uint32_t pad = (uint32_t)(H - Hr) * 128;
    for (uint32_t i = tid * 16; i < kChunks * pad; i += kThreads * 16) {
      const uint32_t c = i / pad, o = i % pad;
      *reinterpret_cast<uint4*>(sQ + c * kQChunk + (uint32_t)Hr * 128 + o) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 0) { tmem_alloc(&ss.tmem_base, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  const uint32_t tS = tmem;                  // S^T: columns [0, H)
  const uint32_t tO = tmem + H;              // O^T slab j: columns [H + jH, H + (j+1)H)
  const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

  const uint32_t idesc_s = idesc_bf16(kTile, H);
  const uint32_t idesc_o = idesc_bf16(kTile, H, true, true);
  uint32_t ph_s = 0, ph_o = 0, ph_kv = 0;
  bool q_ready = false, o_init = false, o_pending = false, store_pending = false;
  constexpr uint32_t kTileBytes = kChunks * kKVChunk;

  for (int t = t_begin; t < t_end; ++t) {
    // Reuse with a stash: this tile's selected rows come back as the bf16 tile a Full /
    // Reindex call stored; Full / Reindex with a stash store their tile after the gather.
    const bool stash_tile = a.stash != nullptr && t < a.n_idx_tiles;
    const bool from_stash = stash_tile && a.mode == CSA2_MODE_REUSE;
    const bool to_stash = stash_tile && a.mode != CSA2_MODE_REUSE;
    uint8_t* stile = stash_tile ? a.stash + ((int64_t)q * a.n_idx_tiles + t) * kTileBytes : nullptr;
    if (t != t_begin) issue_slots(t);        // in flight while the previous O^T finishes
    // the previous tile's O^T MMA must be done before its KV / P buffers are rewritten
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
    if (from_stash) {
      if (tid == 0) {
        mbar_arrive_expect_tx(&ss.bar_kv, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          bulk_g2s(sKV + c * kKVChunk, stile + c * kKVChunk, kKVChunk, &ss.bar_kv);
      }
      const bool ok = mbar_wait(&ss.bar_kv, ph_kv, abort, a.status);
      ph_kv ^= 1;
      if (__syncthreads_or(!ok)) break;
    }
    // ------------------------------ gather ------------------------------
    // Phase 2: the rows -- FP4 codes + scales into registers, window rows by cp.async
    // straight to shared memory; phase 3: dequantise (LUT + exact bf16 multiply) and store
    // into the 128-byte-swizzled [128 keys x D] tile.
    uint4 cw[kIters];
    uint32_t sc[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int r = it * kRowsPerIter + rsub;
      uint8_t* row_smem = sKV + r * 128;
      if (kind[it] == 1) {
        const int p = gidx[it];
        if (p >= 0 && p < slen && row0 + p < a.cap_rows) {
          if (from_stash) {
            kind[it] = 3;                          // row already in the tile (from the stash)
          } else {
            const int64_t grow = row0 + p;
            cw[it] = __ldg(reinterpret_cast<const uint4*>(a.codes + grow * (D / 2) + part * 16));
            sc[it] = __ldg(reinterpret_cast<const uint16_t*>(a.scales + grow * (D / 16) + part * 2));
          }
        } else {
          if (p >= slen || p < -1) report(a.status, CSA2_ERR_INVALID_ARG);
          else if (p >= 0) report(a.status, CSA2_ERR_CAPACITY);
          kind[it] = 0;
        }
      } else if (kind[it] == 2) {
        const int64_t grow = wrow0 + gidx[it];
        if (grow >= 0 && grow < a.swa_rows) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = 4 * part + i;
            cp_async16(row_smem + (u >> 3) * kKVChunk + (((u & 7) ^ (r & 7)) << 4),
                       a.swa + grow * D + u * 8);
          }
        } else {
          report(a.status, CSA2_ERR_CAPACITY);
          kind[it] = 0;
        }
      }
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int r = it * kRowsPerIter + rsub;
      uint8_t* row_smem = sKV + r * 128;
      if (part == 0) ss.valid[r] = kind[it] != 0;
      if (kind[it] == 1) {
        const float s0 = e4m3_val(sc[it] & 0xFFu), s1 = e4m3_val((sc[it] >> 8) & 0xFFu);
        const uint32_t s02 = pack_bf16(s0, s0), s12 = pack_bf16(s1, s1);   // exact in bf16
        const uint32_t w4[4] = {cw[it].x, cw[it].y, cw[it].z, cw[it].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {              // unit i: 8 values of word w4[i]
          const uint32_t s2 = i < 2 ? s02 : s12;
          uint4 o;
          uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
          e2m1x8_to_bf16(w4[i], ow);
#pragma unroll
          for (int k = 0; k < 4; ++k) ow[k] = mul_bf16x2(ow[k], s2);
          const int u = 4 * part + i;
          *reinterpret_cast<uint4*>(row_smem + (u >> 3) * kKVChunk + (((u & 7) ^ (r & 7)) << 4)) = o;
        }
      } else if (kind[it] == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int u = 4 * part + i;
          *reinterpret_cast<uint4*>(row_smem + (u >> 3) * kKVChunk + (((u & 7) ^ (r & 7)) << 4)) =
              make_uint4(0, 0, 0, 0);
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    const int any = __syncthreads_or(ss.valid[tid & (kTile - 1)]);
    if (to_stash) {                            // keep the dequantised tile for Reuse layers
      if (tid == 0) {
        for (int c = 0; c < kChunks; ++c) bulk_s2g(stile + c * kKVChunk, sKV + c * kKVChunk, kKVChunk);
        bulk_commit();
      }
      store_pending = true;                    // uniform: every thread takes the same branches
    }
    if (!any) continue;

    // ------------------------------ S^T = KV . Q^T ------------------------------
    if (tid == 0) {
      bool ok = true;
      if (!q_ready) { ok = mbar_wait(&ss.bar_q, 0, abort, a.status); q_ready = ok; }
      if (ok) {
        tc_fence_after();
        const uint64_t kv_desc_k = sdesc_sw128(smem_u32(sKV), 16, 1024);   // KV as K-major A
        const uint64_t q_desc_k = sdesc_sw128(smem_u32(sQ), 16, 1024);     // Q as K-major B
#pragma unroll 4
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * kKVChunk + (k & 3) * 32;
          const uint32_t qoff = (uint32_t)(k >> 2) * kQChunk + (k & 3) * 32;
          umma_bf16(tS, kv_desc_k + (off >> 4), q_desc_k + (qoff >> 4), idesc_s, k > 0 ? 1u : 0u);
        }
        umma_commit(&ss.bar_s);
      }
    }

    // ------------------------------ softmax (all 8 warps) ------------------------------
    // warp w: keys of TMEM lane quadrant (w & 3), heads [32 * (w >> 2), +32)
    const int r = quad * 32 + lane;               // key row = TMEM lane
    const int h0 = hh * 32;
    float v[32];
    bool ok = mbar_wait(&ss.bar_s, ph_s, abort, a.status);
    ok = __syncthreads_and(ok);
    ph_s ^= 1;
    if (!ok) break;
    tc_fence_after();
    tmem_ld32(tS + lane_base + h0, tS + lane_base + h0 + 16, v);
    {
      const bool valid = ss.valid[r] != 0;
#pragma unroll
      for (int h = 0; h < 32; ++h) v[h] = valid ? v[h] * a.scale_log2 : -INFINITY;
      float red[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) red[h] = v[h];
      reduce_scatter_step<32, 16, true>(red, lane);     // lane holds head h0 + lane
      ss.red[quad][h0 + lane] = red[0];
    }
    if (tid == 0) ss.rescale = 0;
    __syncthreads();
    if (tid < H) {
      const float mt = fmaxf(fmaxf(ss.red[0][tid], ss.red[1][tid]), fmaxf(ss.red[2][tid], ss.red[3][tid]));
      ss.alpha[tid] = mt;                          // stash the tile max
      if (mt > ss.m_ref[tid] + kRescaleLog2) ss.rescale = 1;
    }
    __syncthreads();
    if (ss.rescale) {
      // move every head's reference max up to its running max; O and l scale by alpha
      if (tid < H) {
        const float mo = ss.m_ref[tid];
        const float mn = fmaxf(mo, ss.alpha[tid]);
        const float al = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
        ss.alpha[tid] = al;
        ss.l_acc[tid] *= al;
        ss.m_ref[tid] = mn;
      }
      __syncthreads();
      if (o_init) {
        float al[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) al[i] = ss.alpha[h0 + i];
#pragma unroll 1
        for (int j = 0; j < kSlabs; ++j) {
          float o[32];
          const uint32_t ta = tO + lane_base + j * H + h0;
          tmem_ld32(ta, ta + 16, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= al[i];
          tmem_st16(ta, o);
          tmem_st16(ta + 16, o + 16);
        }
        tmem_wait_st();
      }
    }
    {
      // p = 2^(s - m_ref), rounded to bf16; P row r = [heads] (the MN-major B operand)
      // (v is overwritten with the bf16-rounded p for the per-head sums)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4 pk;
        uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int h = 8 * u + 2 * k;
          const float p0 = fast_exp2(v[h] - ss.m_ref[h0 + h]);
          const float p1 = fast_exp2(v[h + 1] - ss.m_ref[h0 + h + 1]);
          pw[k] = pack_bf16(p0, p1);
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[k]));
          v[h] = f.x;
          v[h + 1] = f.y;
        }
        const int unit = 4 * hh + u;
        *reinterpret_cast<uint4*>(sP + r * 128 + ((unit ^ (r & 7)) << 4)) = pk;
      }
      reduce_scatter_step<32, 16, false>(v, lane);
      ss.red[quad][h0 + lane] = v[0];
      fence_proxy_async_smem();
      tc_fence_before();
    }
    __syncthreads();
    if (tid < H) ss.l_acc[tid] += (ss.red[0][tid] + ss.red[1][tid]) + (ss.red[2][tid] + ss.red[3][tid]);
    // ------------------------------ O^T += V^T . P^T ------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint64_t kv_desc_mn = sdesc_sw128(smem_u32(sKV), kKVChunk, 1024);  // V^T, MN-major A
      const uint64_t p_desc_mn = sdesc_sw128(smem_u32(sP), 8192, 1024);        // P^T, MN-major B
#pragma unroll 1
      for (int j = 0; j < kSlabs; ++j) {
#pragma unroll 4
        for (int k = 0; k < kTile / 16; ++k) {
          const uint32_t off = (uint32_t)(2 * j) * kKVChunk + k * 2048;
          umma_bf16(tO + j * H, kv_desc_mn + (off >> 4), p_desc_mn + ((uint32_t)(k * 2048) >> 4),
                    idesc_o, (o_init || k > 0) ? 1u : 0u);
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
  if (partial) {
    // Split query: write this CTA's unnormalised O (relative to m_ref) as [D][Hr] rows,
    // straight from TMEM (16-byte stores of 32 heads per thread), plus (m, l) per head.
    if (done_ok) {
      float* po = a.part_o + ((int64_t)q * a.nsplit + split) * D * Hr;
      const int hbase = hh * 32;
#pragma unroll 1
      for (int j = 0; j < kSlabs; ++j) {
        const int d = j * 128 + quad * 32 + lane;
        float o[32];
        if (o_init) {
          const uint32_t ta = tO + lane_base + j * H + hbase;
          tmem_ld32(ta, ta + 16, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.0f;
        }
        float* row = po + (int64_t)d * Hr + hbase;
        if (hbase + 32 <= Hr && (Hr & 3) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(row + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (hbase + i < Hr) row[i] = o[i];
        }
      }
      if (tid < Hr) {
        const float m = ss.m_ref[tid], l = ss.l_acc[tid];
        float* ml = a.part_ml + (((int64_t)q * a.nsplit + split) * Hr + tid) * 2;
        ml[0] = (o_init && l > 0.0f) ? m : -INFINITY;
        ml[1] = o_init ? l : 0.0f;
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  if (tid < H) {  // reciprocal of l for the normalised (unsplit) output
    const float l = ss.l_acc[tid];
    ss.alpha[tid] = (!partial && l > 0.0f) ? 1.0f / l : 1.0f;
  }
  __syncthreads();
  // The KV tile is free once the last O^T MMA has completed: stage O there as [head][D]
  // fp32, then copy it out with 16-byte stores.
  float* so = reinterpret_cast<float*>(sKV);        // [Hr][D] (Hr * D * 4 <= 128 KB)
  if (done_ok) {
    const int hbase = hh * 32;
    float oscale[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      oscale[i] = (o_init && ss.l_acc[hbase + i] > 0.0f) ? ss.alpha[hbase + i] : 0.0f;
#pragma unroll 1
    for (int j = 0; j < kSlabs; ++j) {
      const int d = j * 128 + quad * 32 + lane;
      float o[32];
      if (o_init) {
        const uint32_t ta = tO + lane_base + j * H + hbase;
        tmem_ld32(ta, ta + 16, o);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int h = hbase + i;
        if (h < Hr) so[h * D + d] = o_init ? o[i] * oscale[i] : 0.0f;
      }
    }
    if (tid < Hr) {
      const float m = ss.m_ref[tid], l = ss.l_acc[tid];
      if (partial) {
        float* ml = a.part_ml + (((int64_t)q * a.nsplit + split) * Hr + tid) * 2;
        ml[0] = (l > 0.0f) ? m : -INFINITY;
        ml[1] = l;
      } else if (a.lse) {
        a.lse[(int64_t)q * Hr + tid] = (l > 0.0f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }
  __syncthreads();
  if (done_ok) {
    float4* dst4 = reinterpret_cast<float4*>(partial ? a.part_o + (((int64_t)q * a.nsplit + split) * Hr) * D
                                                     : a.out + (int64_t)q * Hr * D);
    const float4* src4 = reinterpret_cast<const float4*>(so);
    const int n4 = Hr * D / 4;
#pragma unroll 4
    for (int i = tid; i < n4; i += kThreads) dst4[i] = src4[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge of the split partials of one query over a 32-dim block: per head the weights
// 2^(m_s - M) / L, M = max_s m_s, L = sum_s 2^(m_s - M) l_s; partials are [D][H] rows, so the
// block is read with consecutive threads on consecutive heads and transposed through
// shared memory for the [H][D] output.
constexpr int kMergeD = 8;               // output dims per merge CTA
constexpr int kMaxSplit = 16;
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnArgs a, int H, int D) {
  __shared__ float wgt[kMaxSplit][kN];
  __shared__ float tile[kN][kMergeD + 1];
  const int q = blockIdx.x, d0 = blockIdx.y * kMergeD, tid = threadIdx.x;
  const int ns = a.nsplit;
  // partial values first: every load of this thread in flight at once
  const float* base = a.part_o + (int64_t)q * ns * D * H + (int64_t)d0 * H;
  const int n_el = kMergeD * H;          // <= 512: two per thread
  float v[2][kMaxSplit];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = tid + 256 * k;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s)
      v[k][s] = (e < n_el && s < ns) ? __ldg(base + (int64_t)s * D * H + e) : 0.0f;
  }
  if (tid < H) {
    const float* ml = a.part_ml + (int64_t)q * ns * H * 2;
    float m[kMaxSplit], l[kMaxSplit];
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) {
      m[s] = s < ns ? ml[(s * H + tid) * 2] : -INFINITY;
      l[s] = s < ns ? ml[(s * H + tid) * 2 + 1] : 0.0f;
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) M = fmaxf(M, m[s]);
    float L = 0.0f;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) {
      const float w = (m[s] == -INFINITY) ? 0.0f : exp2f(m[s] - M);
      wgt[s][tid] = w;
      L += w * l[s];
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) wgt[s][tid] *= inv;
    if (a.lse && blockIdx.y == 0)
      a.lse[(int64_t)q * H + tid] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = tid + 256 * k;
    if (e < n_el) {
      const int dd = e / H, h = e - dd * H;
      float acc = 0.0f;
#pragma unroll
      for (int s = 0; s < kMaxSplit; ++s) acc = fmaf(wgt[s][h], v[k][s], acc);
      tile[h][dd] = acc;
    }
  }
  __syncthreads();
  float* out = a.out + (int64_t)q * H * D + d0;
  for (int e = tid; e < n_el; e += 256) {
    const int h = e / kMergeD, dd = e - h * kMergeD;
    out[(int64_t)h * D + dd] = tile[h][dd];
  }
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

size_t attn_smem_bytes(int D) {
  const size_t q = ((size_t)(D / 64) * kN * 128 + 1023) / 1024 * 1024;
  return 1024 + q + (size_t)(D / 64) * kTile * 128 + kTile * 128;
}

bool attn_shape_ok(int H, int D) {
  return H >= 1 && H <= kN && (D == 128 || D == 256 || D == 512);
}

PFN_cuTensorMapEncodeTiled_v12000 attn_encode_fn() {
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

template <int D>
cudaError_t launch(const AttnArgs& a, const CUtensorMap& tm, cudaStream_t st) {
  const size_t smem = attn_smem_bytes(D);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D><<<dim3(a.nsplit, a.num_q), kThreads, smem, st>>>(tm, a);
  if (a.nsplit > 1) attn_merge_kernel<<<dim3(a.num_q, D / kMergeD), 256, 0, st>>>(a, a.H, D);
  return cudaGetLastError();
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_sparse_attn_stash_bytes(int32_t num_q, int32_t D, int32_t topk) {
  if (num_q < 0 || D < 1 || topk < 0) return 0;
  return (size_t)num_q * ((topk + kTile - 1) / kTile) * (size_t)D * 256;
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
  if ((int64_t)num_q * H > 0x7FFFFFFF) return CSA2_ERR_UNSUPPORTED;
  if (!q || !out || !q_pos || !seqs.seq_start || !seqs.seq_len) return CSA2_ERR_INVALID_ARG;
  if (topk > 0 && (!indices || !kv_codes || !kv_scales || cap_rows <= 0)) return CSA2_ERR_INVALID_ARG;
  if (window > 0 && (!swa_kv || !swa_start || swa_rows < 0)) return CSA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kv_codes) & 15) ||
      (reinterpret_cast<uintptr_t>(kv_scales) & 1) || (reinterpret_cast<uintptr_t>(swa_kv) & 15) ||
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

  auto fn = attn_encode_fn();
  if (!fn) return CSA2_ERR_CUDA;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_q * H};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)H};
  cuuint32_t estr[2] = {1u, 1u};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(q), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return CSA2_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (D == 128) e = launch<128>(a, tm, st);
  else if (D == 256) e = launch<256>(a, tm, st);
  else e = launch<512>(a, tm, st);
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
