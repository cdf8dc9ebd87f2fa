/*
 * csa2.h -- C ABI of the CSA2 attention step over an FP4 global KV cache (B200, sm_100a).
 *
 * What is computed follows the DeepSeek-V4.1-Flash pages:
 *   [MTP]  aprilzz.com "DeepSeek V4.1 Flash 发布：KV cache 降到 890 字节/token…",
 *          sections "CSA2：在层的维度上共享缓存" (Full / Reindex / Reuse, Top-512, the
 *          2048 x 8 candidate pool), "FP4 KV 与部署层的几个改动" (E2M1 values, one E4M3
 *          scale per 16 channels, no global scale), "把 prefill 砍掉一半" (128-token window)
 *   [SURV] gkm0120.cn "DeepSeek-V4.1-Flash 技术调研报告", §2.2.2 (modes table) and
 *          §2.2.3 (hierarchical sparse indexer)
 *   [OVR]  "DeepSeek-V4.1-Flash：推动 KV 缓存压缩极限", 摘要 (FP4 KV + cross-layer reuse)
 * Details the pages leave open are fixed as stated at each entry point.
 *
 * Conventions shared by every entry point
 *   - Pointers marked "device" are CUDA device pointers; "host" values are plain
 *     integers.  The caller owns every buffer; the library allocates nothing and keeps
 *     no state between calls.
 *   - bf16 data is passed as its raw 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *     enqueues work on it and returns; results are ready when the stream is.  Kernels
 *     are launched as programmatic dependents of the work before them in the stream: a
 *     kernel may start its set-up while the previous kernel still runs, but reads no
 *     memory until that kernel has completed, so stream order is kept.
 *   - Shape, pointer and workspace-size errors are detected on the host and returned
 *     before anything is enqueued.  Values that live in device memory (lengths, row
 *     ids, indices) are checked by the kernels: a bad value is skipped and the first
 *     such error is recorded in the status word at the start of `workspace`, which
 *     csa2_status_fetch() returns.  Kernels never trap; every wait inside a kernel is
 *     bounded and reports CSA2_ERR_TIMEOUT when its bound runs out.
 *   - `workspace` is caller-allocated device memory of at least the size the matching
 *     *_workspace() function returns, 256-byte aligned.  Its first CSA2_STATUS_BYTES
 *     hold the sticky status word: clear it once with csa2_status_reset(); calls never
 *     clear it.  Two calls that overlap on the GPU must not share a workspace.
 *   - Launch failures map to CSA2_ERR_CUDA.
 *
 * Cache layout in HBM (row-major, one row per compressed entry)
 *   kv_codes  uint8 [cap_rows][D/2]   E2M1 codes, byte k = code[2k] | code[2k+1] << 4
 *   kv_scales uint8 [cap_rows][D/16]  E4M3 scale of channels 16g .. 16g+15
 *   idx_k     bf16  [cap_rows][d_I]   indexer keys
 *   That is 9D/16 bytes of main KV per entry: 288 B at D = 512.
 *   Sequence s owns rows [seq_start[s], seq_start[s] + seq_len[s]); a position p of
 *   the sequence is row seq_start[s] + p.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Static per-layer mode ([SURV] §2.2.2, [MTP] "CSA2：…"):
 *   FULL    - own indexer over every visible entry, new Top-K (the decoder's first Full
 *             layer also builds the candidate pool);
 *   REINDEX - reuses main KV and indexer K, scores only the pool with its own indexer Q;
 *   REUSE   - no indexer; attends with the latest Full/Reindex indices. */
typedef enum { CSA2_MODE_FULL = 0, CSA2_MODE_REINDEX = 1, CSA2_MODE_REUSE = 2 } csa2_mode_t;

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,  /* bad shape / pointer, or a device-side value out of range */
  CSA2_ERR_UNSUPPORTED = 2,  /* a shape this build has no kernel for */
  CSA2_ERR_CAPACITY = 3,     /* workspace too small, or a row outside the cache */
  CSA2_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  CSA2_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel ran out */
} csa2_status_t;

#define CSA2_STATUS_BYTES 256

/* Ragged batch description, shared by every call.
 * Query q belongs to sequence q_seq[q] when q_seq is not NULL (any mix of decode queries
 * and chunks of several queries per sequence; a value outside [0, num_seqs) makes that
 * query see nothing and records CSA2_ERR_INVALID_ARG), else to sequence q / q_per_seq, in
 * which case num_seqs * q_per_seq must equal num_q.
 * Cache rows: linear (block_table NULL): position p of sequence s is row seq_start[s] + p.
 * Paged ([MTP] "FP4 KV 与部署层的几个改动": the global cache outlives the session and is
 * managed by the serving layer): the cache is a pool of CSA2_PAGE_ROWS-row pages and
 * position p of sequence s is row block_table[s][p / 128] * 128 + p % 128; seq_start may be
 * NULL.  Entries of a page < 0 (or beyond the cache) are skipped and CSA2_ERR_CAPACITY is
 * recorded.  Every index and attention call takes either layout. */
#define CSA2_PAGE_ROWS 128
typedef struct {
  int32_t num_seqs;           /* host: number of sequences (>= 1) */
  int32_t q_per_seq;          /* host: queries per sequence when q_seq is NULL (decode: 1) */
  const int64_t* seq_start;   /* device [num_seqs]: cache row of position 0 (linear layout) */
  const int32_t* seq_len;     /* device [num_seqs]: entries stored for the sequence */
  const int32_t* q_seq;       /* device [num_q] or NULL: the sequence of every query */
  const int32_t* block_table; /* device [num_seqs][max_pages] or NULL: page of positions
                                 128i .. 128i+127 */
  int32_t max_pages;          /* host: columns of block_table */
} csa2_seqs_t;

/* ---------------------------------------------------------------------------------
 * a1. Quantise + append main-KV rows ([MTP] "FP4 KV 与部署层的几个改动": E2M1 values with
 * one E4M3 scale per 16 channels, no global scale).  For each row r and channel group g:
 *   amax  = max |x[r][16g .. 16g+15]|
 *   scale = E4M3(amax / 6)                  fp32 divide, round-to-nearest-even, saturate
 *   code  = E2M1(x / dec(scale))            fp32 divide, RNE, saturate to +-6, sign kept;
 *                                           a zero scale gives signed-zero codes
 * and writes codes/scale into cache row dst_row[r].  If idx_k_in is not NULL, its row r
 * (d_I bf16) is copied to idx_k row dst_row[r] as well.
 *   x         device fp32 [rows][D]          D a multiple of 32, 32 <= D <= 4096
 *   dst_row   device int64 [rows]            must be in [0, cap_rows): else skipped and
 *                                            CSA2_ERR_CAPACITY is recorded
 *   kv_codes, kv_scales  device, layout above, cap_rows rows
 *   idx_k_in  device bf16 [rows][d_I] or NULL;  idx_k device bf16 [cap_rows][d_I]
 *   workspace >= csa2_quant_append_workspace() bytes (status word only)
 * rows = 0 is a no-op. */
CSA2_API size_t csa2_quant_append_workspace(void);
CSA2_API csa2_status_t csa2_quant_append(const float* x, int32_t rows, int32_t D, const int64_t* dst_row,
                                uint8_t* kv_codes, uint8_t* kv_scales, int64_t cap_rows,
                                const uint16_t* idx_k_in, uint16_t* idx_k, int32_t d_I,
                                void* workspace, size_t ws_bytes, void* stream);
/* The same append into a compact indexer-K cache: idx_k is E4M3 bytes [cap_rows][d_I]; row r
 * of the bf16 idx_k_in is converted element by element (round to nearest even, saturating
 * to +-448; integers in [-16, 16] are exact).  idx_k 8-byte aligned. */
CSA2_API csa2_status_t csa2_quant_append_e4m3k(const float* x, int32_t rows, int32_t D,
                                      const int64_t* dst_row, uint8_t* kv_codes, uint8_t* kv_scales,
                                      int64_t cap_rows, const uint16_t* idx_k_in, uint8_t* idx_k,
                                      int32_t d_I, void* workspace, size_t ws_bytes, void* stream);
/* n bf16 values -> n E4M3 bytes (round to nearest even, saturating to +-448): for indexer
 * queries and bulk indexer-K rows of the compact path. */
CSA2_API csa2_status_t csa2_e4m3_from_bf16(const uint16_t* in, uint8_t* out, int64_t n, void* stream);

/* ---------------------------------------------------------------------------------
 * Sequence-axis compressor fused with a1 ([SURV] §2.2.1: every m tokens become one
 * compressed entry; [MTP] "CSA2：…": the encoder groups run at ratio 2).  The pages do not
 * give the compressor's form; here it is a linear map of the entry's m token rows:
 *   entry_j[n] = sum_k xcat_j[k] * w_t[n][k],  xcat_j = [x_{jm}; ...; x_{jm+m-1}], K = m*D_in
 * (bf16 inputs, fp32 tensor-core accumulation), quantised exactly as csa2_quant_append does
 * (E4M3 scale of amax/6 per 16 channels, E2M1 codes) into cache row dst_row[j].
 *   x         device bf16 [n_entries * m][D_in] (token rows, consecutive per entry)
 *   w_t       device bf16 [D][m * D_in]          m * D_in a multiple of 64
 *   D         128, 256 or 512
 *   dst_row   device int64 [n_entries]; rows outside [0, cap_rows) are skipped and
 *             CSA2_ERR_CAPACITY is recorded
 *   x, w_t 16-byte aligned; workspace >= CSA2_STATUS_BYTES (status word only) */
CSA2_API csa2_status_t csa2_compress_append(const uint16_t* x, int32_t n_entries, int32_t m,
                                   int32_t D_in, const uint16_t* w_t, int32_t D,
                                   const int64_t* dst_row, uint8_t* kv_codes, uint8_t* kv_scales,
                                   int64_t cap_rows, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ---------------------------------------------------------------------------------
 * a2 + a3 (+ a4).  Full-mode indexer ([MTP] "CSA2：…": Full selects a new Top-512;
 * [SURV] §2.2.3: the decoder's first Full layer bounds the search of deeper layers).
 * For query q of sequence s with visible entries V = q_visible[q] (seq_len[s] if
 * q_visible is NULL), and every position e < V:
 *   score[q][e] = sum_h w[q][h] * max(0, sum_d qI[q][h][d] * idx_k[seq_start[s]+e][d])
 * (bf16 inputs, fp32 tensor-core accumulation: exact for the integer-valued inputs the
 * tests use).  indices[q][*] = the topk positions ranked first by (score desc, position
 * asc), written in ascending position order, padded with -1 when V < topk.
 * If pool_blocks > 0 it also builds the candidate pool: block j covers positions
 * [block*j, block*j + block) below V, its score is the max of their scores, and
 * pool[q][*] = the pool_blocks block ids ranked first by (block score desc, id asc),
 * ascending, -1 padded.
 *   qI        device bf16 [num_q][H_I][d_I]      1 <= H_I <= 32, d_I in {64, 128}
 *   w         device fp32 [num_q][H_I]
 *   idx_k     device bf16 [cap_rows][d_I], base 16-byte aligned, cap_rows < 2^31
 *   q_visible device int32 [num_q] or NULL; values above seq_len are clamped and
 *             CSA2_ERR_INVALID_ARG is recorded
 *   max_visible host bound on every V (sizes the workspace); larger V are clamped and
 *             CSA2_ERR_CAPACITY is recorded
 *   topk      1 <= topk <= 4096;  indices device int32 [num_q][topk]
 *   pool_blocks 0 or 1..8192; block a power of two in 1..32 (the pages use 8);
 *             pool device int32 [num_q][pool_blocks] (may be NULL when pool_blocks = 0)
 *   workspace >= csa2_index_full_workspace(...) bytes */
CSA2_API size_t csa2_index_full_workspace(int32_t num_q, int32_t max_visible, int32_t topk,
                                 int32_t pool_blocks, int32_t block);
CSA2_API csa2_status_t csa2_index_full(const uint16_t* qI, const float* w, int32_t num_q, int32_t H_I,
                              int32_t d_I, const uint16_t* idx_k, int64_t cap_rows,
                              csa2_seqs_t seqs, const int32_t* q_visible, int32_t max_visible,
                              int32_t topk, int32_t* indices,
                              int32_t pool_blocks, int32_t block, int32_t* pool,
                              void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * csa2_index_full without a workspace: for callers that cannot allocate device memory.
 * (The pages have no counterpart; this is a deployment convenience.)  Some callers run
 * where cudaMalloc is unavailable or forbidden -- inside a host framework that owns the
 * allocator, a real-time loop that must not allocate, or code that is not allowed to grow
 * device memory after start-up -- and so cannot provide csa2_index_full's workspace.
 * This entry point computes exactly what csa2_index_full computes (same arguments minus
 * the workspace) using scratch memory that the library holds in a fixed-size device array
 * of CSA2_INDEX_NOALLOC_SCRATCH_BYTES, present on every GPU that loads the library until
 * the process exits.  It calls no cudaMalloc / cudaFree and no allocating routine.
 *   - Size limit: if csa2_index_full_workspace(num_q, max_visible, topk, pool_blocks, block)
 *     exceeds CSA2_INDEX_NOALLOC_SCRATCH_BYTES the call returns CSA2_ERR_CAPACITY and
 *     enqueues nothing (8 MiB covers one query over 1,048,576 entries with a pool).
 *   - Set-up: the first call on a device looks up the array's device address (with that
 *     device current) and caches it; make that first call before any stream capture.  A
 *     cudaDeviceReset() invalidates the cached address: do not call this entry point on a
 *     device after resetting it in the same process.
 *   - Sharing: every call on a device uses the same array and leaves its contents there;
 *     each call clears what must start at zero.  Calls that overlap on the GPU (different
 *     streams, or different host threads) race on the array: serialise them.
 *   - Arguments are checked in the same order and with the same status codes as
 *     csa2_index_full; the size limit is checked after them.
 *   - Device-side value errors are handled as in csa2_index_full (skipped / clamped) and
 *     recorded in the array's own status word, which each call clears when it starts:
 *     csa2_index_full_noalloc_status() returns it for the latest call on the current
 *     device. */
#define CSA2_INDEX_NOALLOC_SCRATCH_BYTES (8u << 20)
CSA2_API csa2_status_t csa2_index_full_noalloc(const uint16_t* qI, const float* w, int32_t num_q,
                                               int32_t H_I, int32_t d_I, const uint16_t* idx_k,
                                               int64_t cap_rows, csa2_seqs_t seqs,
                                               const int32_t* q_visible, int32_t max_visible,
                                               int32_t topk, int32_t* indices,
                                               int32_t pool_blocks, int32_t block, int32_t* pool,
                                               void* stream);
/* Wait for `stream`, then return the status word of the latest csa2_index_full_noalloc call
 * on the current device (CSA2_OK if its kernels recorded no error). */
CSA2_API csa2_status_t csa2_index_full_noalloc_status(void* stream);

/* ---------------------------------------------------------------------------------
 * Compact indexer K (E4M3): csa2_index_full and csa2_index_pool with qI and idx_k as E4M3
 * bytes ([num_q][H_I][d_I] and [cap_rows][d_I], d_I = 128, base 16-byte aligned) instead of
 * bf16.  The score is the same formula over the E4M3 values (fp32 accumulation of the exact
 * products): for integer-valued indexer inputs in [-16, 16] it, and so every index and pool,
 * is identical to the bf16 path's, while the Full scan reads 128 instead of 256 bytes per
 * entry.  The pages put the whole global cache at 890 bytes per token ([OVR] 摘要), which
 * leaves little room for a 2-byte indexer key.  Workspace sizes are those of the bf16 calls. */
CSA2_API csa2_status_t csa2_index_full_e4m3(const uint8_t* qI, const float* w, int32_t num_q,
                                   int32_t H_I, int32_t d_I, const uint8_t* idx_k,
                                   int64_t cap_rows, csa2_seqs_t seqs, const int32_t* q_visible,
                                   int32_t max_visible, int32_t topk, int32_t* indices,
                                   int32_t pool_blocks, int32_t block, int32_t* pool,
                                   void* workspace, size_t ws_bytes, void* stream);
CSA2_API csa2_status_t csa2_index_pool_e4m3(const uint8_t* qI, const float* w, int32_t num_q,
                                   int32_t H_I, int32_t d_I, const uint8_t* idx_k,
                                   int64_t cap_rows, csa2_seqs_t seqs, const int32_t* q_visible,
                                   const int32_t* pool, int32_t pool_blocks, int32_t block,
                                   int32_t topk, int32_t* indices, void* workspace,
                                   size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * a5. Reindex over the pool ([SURV] §2.2.2: Reindex reuses main KV and indexer K but has
 * its own indexer Q and re-selects; [MTP] "CSA2：…": Reindex layers only score inside the
 * bounded pool).  Candidates of query q: positions block*pool[q][i] + r, r < block, for
 * every pool entry >= 0, that are below V.  Each is scored with this layer's qI/w as in
 * csa2_index_full; indices[q][*] = the topk candidates ranked first by (score desc,
 * position asc), ascending, -1 padded.  pool must list block ids in ascending order
 * followed by -1 padding, as csa2_index_full writes it.
 *   block must be 8 (the pages' block size); pool_blocks 1..8192; other arguments as
 *   csa2_index_full. */
CSA2_API size_t csa2_index_pool_workspace(int32_t num_q, int32_t pool_blocks, int32_t block,
                                 int32_t topk);
CSA2_API csa2_status_t csa2_index_pool(const uint16_t* qI, const float* w, int32_t num_q, int32_t H_I,
                              int32_t d_I, const uint16_t* idx_k, int64_t cap_rows,
                              csa2_seqs_t seqs, const int32_t* q_visible,
                              const int32_t* pool, int32_t pool_blocks, int32_t block,
                              int32_t topk, int32_t* indices,
                              void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * a7. Sparse attention with the joint sliding window ([MTP] "把 prefill 砍掉一半": every
 * layer keeps a 128-token window; "CSA2：…": each layer keeps its own main Q and window
 * KV).  For query q of sequence s at token position t = q_pos[q], the key/value rows are
 *   - for every i with p = indices[q][i] >= 0: the dequantised cache row seq_start[s] + p
 *     (e2m1(code) * e4m3(scale), exact in bf16); p >= seq_len[s] is skipped and
 *     CSA2_ERR_INVALID_ARG recorded;
 *   - the window: token positions u = max(0, t - window + 1) .. t, at swa_kv row
 *     swa_start[s] + u (swa_ring = 0), or, with a ring of swa_ring rows per sequence
 *     (swa_ring a multiple of 128, window <= swa_ring <= 1024), at row
 *     swa_start[s] + (u mod swa_ring), the ring holding the latest swa_ring tokens (rows
 *     outside [0, swa_rows) are skipped and CSA2_ERR_CAPACITY recorded).
 * Keys equal values (one vector per row).  Per head h:
 *   l_j = softmax_scale * q[q][h] . row_j;  out[q][h] = sum_j softmax(l)_j row_j;
 *   lse[q][h] = log(sum_j exp(l_j)) (natural log); no rows at all gives out = 0,
 *   lse = -inf.  The two sets share one softmax; a row in both counts twice.
 * Cross-layer reuse ([SURV] §2.2.2, [MTP] "CSA2：…": a Reuse layer takes the main KV and the
 * latest Top-K of an earlier layer): with a non-NULL `kv_stash`,
 *   - mode FULL or REINDEX also stores the selected rows' FP4 codes and scales (per tile
 *     of 64 or 128 slots, a choice made from num_q, H, topk and window, in the kernel's
 *     staging layout) into kv_stash;
 *   - mode REUSE takes the selected rows from kv_stash instead of the FP4 cache.  The
 *     stash must hold the rows of exactly these indices for these queries, as written by
 *     the latest FULL/REINDEX call with the same num_q, H, D, topk and window; the window
 *     rows are always read from swa_kv.  Results equal those of a stateless call.
 *   With kv_stash == NULL every mode reads the FP4 cache (the call is stateless).
 *   q         device bf16 [num_q][H][D]        1 <= H <= 64, D in {128, 256, 512},
 *             num_q <= 65535 (other shapes return CSA2_ERR_UNSUPPORTED); base 16-byte
 *             aligned
 *   kv_codes, kv_scales  the cache (layout above), both 16-byte aligned
 *   indices   device int32 [num_q][topk]       0 <= topk <= 2048
 *   swa_kv    device bf16 [swa_rows][D], swa_rows < 2^31;  swa_start device int64
 *             [num_seqs] (may be negative).  Only rows of window positions take part;
 *             other rows inside [0, swa_rows) may be read by the tile loads but are
 *             masked and do not change the result.
 *   q_pos     device int64 [num_q]
 *   window    0 .. 1024
 *   out       device fp32 [num_q][H][D];  lse device fp32 [num_q][H] or NULL
 *   mode      csa2_mode_t (only used with a stash)
 *   kv_stash  device, >= csa2_sparse_attn_stash_bytes(num_q, D, topk) bytes, 16-byte
 *             aligned, or NULL
 *   workspace >= csa2_sparse_attn_workspace(...) bytes */
CSA2_API size_t csa2_sparse_attn_workspace(int32_t num_q, int32_t H, int32_t D, int32_t topk,
                                  int32_t window);
CSA2_API size_t csa2_sparse_attn_stash_bytes(int32_t num_q, int32_t D, int32_t topk);
CSA2_API csa2_status_t csa2_sparse_attn(const uint16_t* q, int32_t num_q, int32_t H, int32_t D,
                               const uint8_t* kv_codes, const uint8_t* kv_scales,
                               int64_t cap_rows, csa2_seqs_t seqs,
                               const int32_t* indices, int32_t topk,
                               const uint16_t* swa_kv, int64_t swa_rows,
                               const int64_t* swa_start, const int64_t* q_pos,
                               int32_t window, int32_t swa_ring, float softmax_scale,
                               float* out, float* lse,
                               csa2_mode_t mode, void* kv_stash, size_t stash_bytes,
                               void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * A layer of the schedule. */
/* One layer of the CSA2 schedule, driven by its mode ([SURV] §2.2.2 modes table; [MTP]
 * "CSA2：在层的维度上共享缓存": Full and Reindex layers run their own indexer, Reuse layers
 * attend with the latest indices):
 *   FULL     csa2_index_full (building the pool when indexer->pool_blocks > 0) into
 *            `indices`, then csa2_sparse_attn with mode FULL;
 *   REINDEX  csa2_index_pool over indexer->pool into `indices`, then csa2_sparse_attn with
 *            mode REINDEX;
 *   REUSE    csa2_sparse_attn with mode REUSE and `indices` as given (the latest
 *            FULL/REINDEX layer's); `indexer` may be NULL.
 * Every argument keeps the meaning, layout and limits of the call it is passed to; the
 * two structs only group them.  The first error is returned and nothing after it is
 * enqueued.  Only host logic: the work is that of the two calls. */
typedef struct {
  const void* qI;            /* device [num_q][H_I][d_I]: bf16, or E4M3 bytes when e4m3 */
  const float* w;            /* device fp32 [num_q][H_I] */
  int32_t H_I, d_I;
  const void* idx_k;         /* device [cap_rows][d_I]: bf16, or E4M3 bytes when e4m3 */
  const int32_t* q_visible;  /* device int32 [num_q] or NULL */
  int32_t max_visible;       /* FULL: bound on any query's visible entries */
  int32_t pool_blocks;       /* FULL: 0 = no pool; REINDEX: the pool's blocks per query */
  int32_t block;             /* pool block size (8) */
  int32_t* pool;             /* FULL: written when pool_blocks > 0; REINDEX: read */
  void* workspace;           /* csa2_index_full_workspace / csa2_index_pool_workspace bytes */
  size_t ws_bytes;
  int32_t e4m3;              /* 0: bf16 qI / idx_k; 1: the compact E4M3 path */
} csa2_indexer_t;
typedef struct {
  const uint16_t* q;         /* device bf16 [num_q][H][D] */
  int32_t H, D;
  const uint16_t* swa_kv;    /* device bf16 [swa_rows][D] */
  int64_t swa_rows;
  const int64_t* swa_start;  /* device int64 [num_seqs] */
  const int64_t* q_pos;      /* device int64 [num_q] */
  int32_t window;
  int32_t swa_ring;          /* 0: linear window rows; else ring rows per sequence */
  float softmax_scale;
  float* out;                /* device fp32 [num_q][H][D] */
  float* lse;                /* device fp32 [num_q][H] or NULL */
  void* kv_stash;            /* or NULL (stateless) */
  size_t stash_bytes;
  void* workspace;           /* csa2_sparse_attn_workspace bytes */
  size_t ws_bytes;
} csa2_attention_t;
CSA2_API csa2_status_t csa2_layer_step(csa2_mode_t mode, int32_t num_q, const uint8_t* kv_codes,
                              const uint8_t* kv_scales, int64_t cap_rows, csa2_seqs_t seqs,
                              int32_t topk, int32_t* indices, const csa2_indexer_t* indexer,
                              const csa2_attention_t* attn, void* stream);

/* ---------------------------------------------------------------------------------
 * Paged cache helpers (persistent-cache export and import: [MTP] "FP4 KV 与部署层的几个改动"
 * -- the global cache is kept for hours, the window is rebuilt, so a sequence's cached
 * entries move between this cache and slower storage). */
/* rows[i] = the cache row of position pos[i] of sequence seq[i] under `seqs` (linear or
 * paged); -1 for a sequence or page that does not exist.  seq, pos device int32 [n]; rows
 * device int64 [n]. */
CSA2_API csa2_status_t csa2_cache_rows(csa2_seqs_t seqs, const int32_t* seq, const int32_t* pos,
                              int32_t n, int64_t* rows, void* stream);
/* dst[i] = table[rows[i]] for rows of row_bytes bytes (rows[i] outside [0, cap_rows) give a
 * zero row): e.g. a sequence's FP4 codes, scales or indexer keys into a contiguous buffer
 * for export.  table, dst 16-byte aligned, row_bytes a multiple of 4. */
CSA2_API csa2_status_t csa2_gather_rows(const uint8_t* table, int64_t cap_rows, int32_t row_bytes,
                               const int64_t* rows, int32_t n, uint8_t* dst, void* stream);
/* table[rows[i]] = src[i] (rows outside [0, cap_rows) are skipped): the import. */
CSA2_API csa2_status_t csa2_scatter_rows(const uint8_t* src, int32_t row_bytes, const int64_t* rows,
                                int32_t n, uint8_t* table, int64_t cap_rows, void* stream);

/* ---------------------------------------------------------------------------------
 * Status word helpers. */
/* Enqueue a clear of the status word at the start of `workspace`. */
CSA2_API csa2_status_t csa2_status_reset(void* workspace, void* stream);
/* Wait for `stream`, then return the first error any kernel recorded in the status
 * word of `workspace` since the last reset (CSA2_OK if none). */
CSA2_API csa2_status_t csa2_status_fetch(const void* workspace, void* stream);
/* Static text for a status code. */
CSA2_API const char* csa2_status_string(csa2_status_t status);
/* The CUDA runtime's message for the latest CUDA failure (a call that returned
 * CSA2_ERR_CUDA) made by the calling host thread, or "no error".  Static storage. */
CSA2_API const char* csa2_last_cuda_error(void);
/* Bound, in nanoseconds of the GPU's global timer, of every wait inside the library's
 * kernels, for launches made after this call (process-wide; 0 restores the default of
 * 2 s).  A wait that runs out makes its kernel stop every role, wait for the copies and
 * MMAs it has itself issued, free its tensor memory and record CSA2_ERR_TIMEOUT.  Returns
 * the previous bound.  Meant for tests of that path and for callers that want a tighter
 * bound than the default. */
CSA2_API uint64_t csa2_set_wait_limit_ns(uint64_t ns);
/* Number of streaming multiprocessors of the current device (0 on error). */
CSA2_API int32_t csa2_device_sms(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
