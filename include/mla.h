/*
 * mla.h - C ABI of the MLA latent-KV decode library (libmla.so).
 *
 * Multi-head Latent Attention caches, per token and layer, one compressed
 * latent c_KV (d_c values) plus one small decoupled rotary key k_R (d_r
 * values, shared by all heads) instead of per-head K and V.  At decode time
 * the key/value up-projections are folded into the query and output sides
 * (matrix absorption), so per-head K and V are never materialised.
 *
 * Sources (by page title and section):
 *  [P2] "Multi-head Latent Attention (MLA) Nedir?" (yapayzekasozluk.tr),
 *       section "MLA nasıl çalışır?" (Compression, Decompression, Decoupled
 *       RoPE, query compression) and "MLA ve diğer optimizasyonlarla
 *       ilişkisi" (page-based caches hold the smaller latent vectors).
 *  [P4] "GQA, MQA ve MLA: attention KV cache'i nasıl belirler" (LLMScale),
 *       section "Multi-head latent attention (MLA)" (what one cache row holds).
 *  [P5] "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
 *       section 1 "Định nghĩa" (absorption into the query and output
 *       matrices; RoPE kept on a separate branch), section 2 "Luồng" (project
 *       hidden to latent -> write the cache -> read and project the output).
 *
 * Conventions shared by every entry point
 *  - Row-vector convention y = x W.  Every weight is stored [in, out],
 *    row-major, in the config's storage dtype (bf16 or f32).
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    except where an argument says otherwise.  `stream` is a cudaStream_t
 *    (NULL = legacy default stream).  Every call is asynchronous on `stream`
 *    and never synchronises, except mla_get_device_error.
 *  - Kernels are launched with programmatic stream serialization: one may
 *    begin its set-up (barriers, tensor-memory allocation, warming L2 with
 *    weights) while the previous kernel in the stream is finishing, but it
 *    reads or writes no argument or workspace before that kernel completes,
 *    so stream order is kept exactly.
 *  - Ownership: the caller owns every buffer, including the workspaces whose
 *    sizes the *_workspace_size queries return.  The library allocates no
 *    device memory.  Its only device state, per device, is one error word
 *    and the fixed scratch of mla_cache_append_noalloc (file-scope
 *    __device__ variables).
 *  - Synchronous errors (null pointers, unsupported dimensions, workspace too
 *    small, a failed launch) return a negative mla_status before or at launch
 *    and leave outputs untouched.  Data-dependent errors found on the device
 *    (a block id outside the pool, a position past a sequence's block table,
 *    a sequence shorter than its query count) skip the offending work,
 *    record the first such error in the device error word, and surface
 *    through mla_get_device_error.  No C++ exception crosses this ABI.
 *  - Alignment: on the bf16 path, every tensor argument of mla_absorb_q,
 *    mla_decode, mla_combine and mla_out_proj, and the workspaces, must start
 *    on a 16-byte boundary (cudaMalloc and PyTorch allocations do); the
 *    kernels read and write them with TMA and 16-byte vector accesses.  A
 *    pointer that does not returns MLA_ERR_INVALID_ARG.  mla_cache_append
 *    takes any alignment (unaligned operands take a slower kernel).
 *  - Storage dtype: MLA_BF16 (bf16 storage, fp32 accumulation) or MLA_F32
 *    (fp32 storage and arithmetic on CUDA cores, for small shapes); with
 *    MLA_BF16 the cache alone may be FP8 (MLA_FLAG_FP8_CACHE).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 2

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,  /* null pointer, negative size, inconsistent config */
  MLA_ERR_UNSUPPORTED = -2,  /* dimensions this build has no kernel for */
  MLA_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed */
  MLA_ERR_BOUNDS = -4,       /* (device) block id / position / length out of range */
  MLA_ERR_TIMEOUT = -5,      /* (device) a bounded wait gave up */
  MLA_ERR_WORKSPACE = -6     /* workspace too small, or not written by mla_decode */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Per-layer MLA dimensions. */
typedef struct {
  int32_t hidden;        /* model width */
  int32_t n_heads;       /* H */
  int32_t d_c;           /* latent width (kv_lora_rank) */
  int32_t d_r;           /* decoupled RoPE key width (even), one key shared by all heads */
  int32_t qk_nope;       /* per-head no-position query/key width */
  int32_t v_head;        /* per-head value width */
  int32_t q_lora;        /* query latent width; 0 = no query compression (W_Q used directly) */
  double rope_theta;     /* RoPE base; pair (2i, 2i+1) turns by pos * theta^(-2i/d_r) */
  float softmax_scale;   /* 0 -> 1/sqrt(qk_nope + d_r) */
  int32_t block_size;    /* tokens per cache page */
  int32_t dtype;         /* mla_dtype */
  int32_t flags;         /* OR of MLA_FLAG_* */
} mla_config;

/* Decode with the query held as a bf16 hi + lo pair on the tensor cores
 * (about 16 significant bits instead of 8), for strongly peaked softmaxes
 * where a bf16 query alone perturbs the dominant probabilities by ~1%.
 * Costs extra score work in the bf16 decode kernel; no effect on fp32 storage. */
#define MLA_FLAG_SPLIT_QUERY 1

/* Latent cache in FP8 (OCP E4M3: 4 exponent bits, bias 7, 3 mantissa bits,
 * largest finite 448) with one fp32 scale per cached row ([P2] "MLA ve diğer
 * optimizasyonlarla ilişkisi": quantization is orthogonal to MLA and used
 * together with it; the pages fix no format, this is the plainest per-row
 * one).  A stored row [c_KV | k_R] stands for codes * scale with
 *   scale = the smallest power of two with max_i |row_i| / scale <= 448
 *           (1 for a zero row), stored as fp32,
 *   code_i = E4M3(row_i / scale)        nearest, ties to even, from the exact
 *                                       fp64 row.
 * A power-of-two scale makes code * scale exact in bf16.
 * Requires dtype MLA_BF16 (weights and activations stay bf16) and
 * mla_cache.row_scale.  A 576-value row takes 580 bytes instead of 1152.
 * The decode of an FP8 cache runs on the CUDA-core path of mla_decode; the
 * packed-query entry points return MLA_ERR_UNSUPPORTED for it. */
#define MLA_FLAG_FP8_CACHE 2

/* Paged latent cache of one layer ([P2] "MLA ve diğer optimizasyonlarla ilişkisi").
 * pool:        [num_blocks, block_size, d_c + d_r] storage dtype (E4M3 codes,
 *              one byte each, with MLA_FLAG_FP8_CACHE); row = [c_KV | k_R].
 * block_table: int32 [batch, max_blocks_per_seq]; entry (b, k) is the pool block
 *              holding positions [k*block_size, (k+1)*block_size) of sequence b.
 * row_scale:   float32 [num_blocks, block_size], the scale of each row, with
 *              MLA_FLAG_FP8_CACHE (4-byte aligned); NULL otherwise (ignored).
 * The library reads and writes the pool in place; the caller owns all of it. */
typedef struct {
  void* pool;
  int32_t num_blocks;
  const int32_t* block_table;
  int32_t batch;
  int32_t max_blocks_per_seq;
  float* row_scale;
} mla_cache;

/* ---------------------------------------------------------------------------
 * Step 1 - latent append ([P5] section 2 "Luồng", steps 1-2; [P2] Compression
 * and Decoupled RoPE; [P4] one row = d_c latent values + d_r rotary values).
 * For each new token t:  c = x_t W_DKV,  k_R = RoPE(x_t W_KR, pos[t]),
 * and the row [c | k_R], rounded once to the storage dtype, is stored at
 * pool[block_table[seq_idx[t]][pos[t] / block_size]][pos[t] % block_size].
 * The bf16 path reproduces the exactly rounded value of the real-number dot
 * product (fp64 accumulation), so the cache is bit-identical to x W rounded
 * once to bf16.
 *   x        [n_tok, hidden]        storage dtype
 *   W_DKV    [hidden, d_c], W_KR [hidden, d_r]
 *   seq_idx  int32 [n_tok]   sequence of each token (row of block_table)
 *   pos      int32 [n_tok]   0-based absolute position of each token
 *   workspace >= mla_cache_append_workspace_size(cfg, n_tok) bytes
 * Device errors: a block id outside [0, num_blocks) or a page index outside
 * [0, max_blocks_per_seq) -> MLA_ERR_BOUNDS, row not written.
 * ------------------------------------------------------------------------- */
size_t mla_cache_append_workspace_size(const mla_config* cfg, int32_t n_tok);
mla_status mla_cache_append(const mla_config* cfg, const void* x, int32_t n_tok,
                            const void* W_DKV, const void* W_KR,
                            const int32_t* seq_idx, const int32_t* pos,
                            const mla_cache* cache, void* workspace, size_t ws_bytes,
                            void* stream);

/* ---------------------------------------------------------------------------
 * Latent append for callers that cannot allocate device memory.  The pages
 * have no counterpart for this entry point; it exists for callers such as a
 * serving engine that has already reserved all device memory for its own
 * pool and forbids any further cudaMalloc, or plain C callers without a
 * device allocator, which cannot provide the workspace mla_cache_append
 * asks for.
 * Same arguments and result as mla_cache_append, minus the workspace: its
 * scratch is a fixed array of MLA_APPEND_NOALLOC_SCRATCH_BYTES in device
 * memory, built into the library, which every GPU that loads the library
 * holds until the process exits.  The call allocates nothing and frees
 * nothing.  The caller still passes all inputs and outputs.
 *  - Size limit: n_tok must satisfy
 *      mla_cache_append_workspace_size(cfg, n_tok) <= MLA_APPEND_NOALLOC_SCRATCH_BYTES
 *    (n_tok <= 910 for d_c + d_r = 576); larger requests return
 *    MLA_ERR_WORKSPACE before any launch.
 *  - First call on a device: it looks up the device address of the array
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture on that device.
 *  - All calls on a device share the one array.  Calls that may overlap on
 *    the GPU (different streams, no ordering between them) race on it and
 *    corrupt each other's result; serialise them, e.g. on one stream.
 * ------------------------------------------------------------------------- */
#define MLA_APPEND_NOALLOC_SCRATCH_BYTES (4u << 20)
mla_status mla_cache_append_noalloc(const mla_config* cfg, const void* x, int32_t n_tok,
                                    const void* W_DKV, const void* W_KR,
                                    const int32_t* seq_idx, const int32_t* pos,
                                    const mla_cache* cache, void* stream);

/* ---------------------------------------------------------------------------
 * Step 2 - queries with W_UK absorbed ([P2] query compression; [P5] section 1
 * "Định nghĩa": the decompression matrix is folded into the query matrix, the
 * RoPE part stays separate).
 *   c_Q = x W_DQ (q_lora > 0) ;  q = c_Q W_UQ   (q_lora == 0: q = x W_Q, pass W_Q as W_UQ, W_DQ = NULL)
 *   head h owns q columns [h(qk_nope+d_r), (h+1)(qk_nope+d_r)): qk_nope no-position
 *   values then d_r rotary values;  q_rope_h = RoPE(q_R_h, pos[t]);
 *   q_lat_h = q_nope_h W_UK_h^T  with  W_UK_h = W_UK[:, h qk_nope : (h+1) qk_nope].
 *   x      [n_tok, hidden];  W_DQ [hidden, q_lora];  W_UQ [q_lora or hidden, H (qk_nope + d_r)]
 *   W_UK   [d_c, H qk_nope];  pos int32 [n_tok]
 *   q_lat  float32 [n_tok, H, d_c] (out);  q_rope float32 [n_tok, H, d_r] (out)
 *   The query side keeps fp32 intermediates (c_Q, q, q_nope) and fp32
 *   outputs: a bf16 query perturbs strongly peaked softmaxes by ~1%.
 *   workspace >= mla_absorb_q_workspace_size(cfg, n_tok) bytes
 * ------------------------------------------------------------------------- */
size_t mla_absorb_q_workspace_size(const mla_config* cfg, int32_t n_tok);
mla_status mla_absorb_q(const mla_config* cfg, const void* x, int32_t n_tok,
                        const void* W_DQ, const void* W_UQ, const void* W_UK,
                        const int32_t* pos, float* q_lat, float* q_rope,
                        void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Step 3 - split-KV decode in latent space ([P5] section 2 "Luồng" step 3:
 * scores and output from the merged matrices or an equivalent kernel; [P2]
 * "MLA'nın avantajları ve hesap maliyeti": recompute from the small latent
 * instead of storing K/V).  For sequence b, query j (token t = b n_q + j,
 * position p = seq_lens[b] - n_q + j) and head h:
 *   s_u = (q_lat[t,h] . c_u + q_rope[t,h] . kR_u) * scale   for rows u <= p
 *   o_lat[t,h] = sum_u softmax(s)_u c_u
 * The pages of all query rows are split into contiguous ranges of about
 * equal cost, one per scheduled worker (the plan is computed on the device
 * from seq_lens); each piece writes its output normalised over its own rows
 * and its log2-sum-exp into `workspace`, and mla_combine merges them.  On the
 * bf16 path the workspace also holds a packed bf16 copy of the query.
 *   q_lat float32 [batch n_q, H, d_c], q_rope float32 [batch n_q, H, d_r]:
 *            from mla_absorb_q (row v = b n_q + j)
 *   seq_lens int32 [batch]: rows of each sequence INCLUDING the n_q new rows
 *            (already appended); must satisfy n_q <= seq_lens[b] <=
 *            max_blocks_per_seq * block_size, or seq_lens[b] = 0: an empty
 *            sequence (a shard without rows of it, see mla_merge_shards),
 *            whose query rows get o_lat = 0 and lse = -inf.
 *   max_workers: upper bound on parallel workers (0 = sized to the device).
 *   workspace >= mla_decode_workspace_size(cfg, batch, n_q, max_workers)
 * Device errors: bad lengths or block ids -> MLA_ERR_BOUNDS (that sequence's
 * output is zero).
 * ------------------------------------------------------------------------- */
size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t n_q,
                                 int32_t max_workers);
mla_status mla_decode(const mla_config* cfg, const float* q_lat, const float* q_rope,
                      int32_t batch, int32_t n_q, const mla_cache* cache,
                      const int32_t* seq_lens, int32_t max_workers,
                      void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 cache on the tensor-core decode (MLA_FLAG_FP8_CACHE; not on the pages):
 * the visible pages of the step are expanded into a caller-owned bf16 scratch
 * cache, which the bf16 entry points then decode (packed query, fused
 * combine), with the configuration without MLA_FLAG_FP8_CACHE.
 *   mla_fp8_scratch_bytes: bytes of that scratch for `batch` sequences of
 *     up to `max_blocks_per_seq` pages (0 for a configuration without the
 *     flag).  Layout: int32 block table [batch, max_blocks_per_seq], then,
 *     256-byte aligned, bf16 pages [batch * max_blocks_per_seq, block_size,
 *     d_c + d_r]; page (b, k) is scratch block b * max_blocks_per_seq + k.
 *   mla_cache_dequant_fp8: for every sequence b < batch and page k holding
 *     rows below seq_lens[b], scratch page (b, k) = bf16(code * row scale)
 *     of cache page block_table[b][k]; writes the whole scratch block table.
 *     Form the scratch cache as { pages, batch * max_blocks_per_seq, table,
 *     batch, max_blocks_per_seq, NULL }.  The cache pool and the scratch must
 *     be 16-byte aligned; d_c + d_r a multiple of 16.
 * Errors: MLA_ERR_INVALID_ARG (flag missing, NULL or misaligned pointers, no
 * row scales), MLA_ERR_WORKSPACE (scratch too small); bad lengths or block
 * ids -> MLA_ERR_BOUNDS on the device error word (that page is not written).
 * ------------------------------------------------------------------------- */
size_t mla_fp8_scratch_bytes(const mla_config* cfg, int32_t batch, int32_t max_blocks_per_seq);
mla_status mla_cache_dequant_fp8(const mla_config* cfg, const mla_cache* cache, int32_t batch,
                                 const int32_t* seq_lens, void* scratch, size_t scratch_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Steps 2 and 3 with the query handed over in the decode's own layout
 * (tensor-core path, bf16 storage).  mla_absorb_q_packed computes the same
 * absorbed query as mla_absorb_q but writes it straight from the projection's
 * accumulators as bf16 rows, one per (token, head), of d_c + d_r values:
 * q_lat then the rotated q_rope; in split-query mode (MLA_FLAG_SPLIT_QUERY)
 * a second array of the same shape follows with the bf16 remainders
 * (value - bf16(value)).  mla_decode_packed reads that buffer directly
 * (mla_decode would first convert fp32 q_lat / q_rope into it).  The
 * rounding is the one mla_decode applies, so results are identical.
 *   q_packed  bf16 [n_tok, H, d_c + d_r] (x2 in split-query mode):
 *             mla_query_packed_bytes(cfg, n_tok) bytes, 16-byte aligned
 *   Other arguments as in mla_absorb_q / mla_decode; the decode workspace
 *   is sized by mla_decode_workspace_size (its query region stays unused).
 * MLA_ERR_UNSUPPORTED for fp32 storage or shapes without the tensor-core path.
 * ------------------------------------------------------------------------- */
size_t mla_query_packed_bytes(const mla_config* cfg, int32_t n_tok);
mla_status mla_absorb_q_packed(const mla_config* cfg, const void* x, int32_t n_tok,
                               const void* W_DQ, const void* W_UQ, const void* W_UK,
                               const int32_t* pos, void* q_packed,
                               void* workspace, size_t ws_bytes, void* stream);
mla_status mla_decode_packed(const mla_config* cfg, const void* q_packed, int32_t batch, int32_t n_q,
                             const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers,
                             void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The decode's split plan on its own (not on the pages: how the cached pages
 * are cut among the SMs).  The plan depends only on seq_lens, the cache's
 * block geometry, batch, n_q and max_workers, so a caller can compute it
 * early (e.g. on a second stream beside the query projections) and then run
 * mla_decode_packed_planned, which skips it.
 *   mla_decode_plan: writes the plan into `workspace` (the region
 *     mla_decode_packed would write); arguments as in mla_decode_packed.
 *   mla_decode_packed_planned: mla_decode_packed without the planning launch;
 *     `workspace` must hold the plan of an mla_decode_plan call with the same
 *     cfg, batch, n_q, cache geometry, seq_lens contents and max_workers,
 *     ordered before this call (same stream, or an event).  Results are
 *     identical to mla_decode_packed.  A plan that does not match these
 *     arguments is caught only partly (its header is checked by the decode and
 *     the merge; a stale plan for other sequence lengths gives wrong output).
 * Errors as mla_decode_packed.
 * ------------------------------------------------------------------------- */
mla_status mla_decode_plan(const mla_config* cfg, int32_t batch, int32_t n_q, const mla_cache* cache,
                           const int32_t* seq_lens, int32_t max_workers, void* workspace, size_t ws_bytes,
                           void* stream);
mla_status mla_decode_packed_planned(const mla_config* cfg, const void* q_packed, int32_t batch, int32_t n_q,
                                     const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers,
                                     void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Step 4a - split combine (not on the pages; the standard log-sum-exp merge):
 *   o_lat[t,h] = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),  M = max_s lse_s
 * over the partials that mla_decode left in `workspace` (same batch, n_q).
 *   o_lat  float32 [batch n_q, H, d_c] (out)
 * Returns MLA_ERR_WORKSPACE on the device error word if the workspace was not
 * written by a matching mla_decode call.
 * ------------------------------------------------------------------------- */
mla_status mla_combine(const mla_config* cfg, const void* workspace, size_t ws_bytes,
                       int32_t batch, int32_t n_q, float* o_lat, void* stream);

/* ---------------------------------------------------------------------------
 * Sequence split across GPUs (not on the pages: the step-4a merge one level
 * up, for contexts too long for one GPU's cache or time budget).  The cached
 * pages of a sequence are cut into contiguous page ranges ("shards") held by
 * different GPUs.  Each GPU decodes its shard (its own cache and block-table
 * rows, the shard's number of visible rows as seq_lens, n_q = 1 per query
 * row), takes per-row (o_lat, lse) with mla_combine_lse, the pairs of all
 * shards are exchanged (e.g. an all-gather over NVLink), and
 * mla_merge_shards merges them:
 *   o[t,h] = sum_r 2^(lse_r - M) o_r / sum_r 2^(lse_r - M),  M = max_r lse_r
 *   lse[t,h] = M + log2 sum_r 2^(lse_r - M)
 * which equals the decode over the whole key set up to fp32 rounding.
 *   mla_combine_lse: mla_combine, plus
 *     lse      float32 [batch n_q, H] (out): the base-2 log-sum-exp of the
 *              scaled scores (scale log2 e) over the keys decoded; -inf for a
 *              row with no key (its o_lat is then 0).
 *   mla_merge_shards:
 *     o_parts  float32 [n_shards, rows, H, d_c] (in), 16-byte aligned
 *     lse_parts float32 [n_shards, rows, H] (in)
 *     o_lat    float32 [rows, H, d_c] (out), 16-byte aligned
 *     lse      float32 [rows, H] (out, may be NULL)
 *   A row whose shards all have lse = -inf gets o = 0, lse = -inf.
 * Errors: MLA_ERR_INVALID_ARG for NULL / misaligned pointers or counts < 0
 * (n_shards < 1); MLA_ERR_UNSUPPORTED for d_c not a multiple of 8 or > 2048.
 * ------------------------------------------------------------------------- */
mla_status mla_combine_lse(const mla_config* cfg, const void* workspace, size_t ws_bytes,
                           int32_t batch, int32_t n_q, float* o_lat, float* lse, void* stream);
mla_status mla_merge_shards(const mla_config* cfg, int32_t n_shards, int32_t rows, const float* o_parts,
                            const float* lse_parts, float* o_lat, float* lse, void* stream);

/* ---------------------------------------------------------------------------
 * Step 4b - output side with W_UV absorbed ([P5] section 1 "Định nghĩa":
 * the decompression matrix folded into the output matrix).
 *   o_h = o_lat_h W_UV_h  (W_UV_h = W_UV[:, h v_head : (h+1) v_head]),
 *   y   = concat_h(o_h) W_O
 *   o_lat float32 [n_tok, H, d_c];  W_UV [d_c, H v_head];  W_O [H v_head, hidden]
 *   y     [n_tok, hidden] storage dtype (out)
 *   workspace >= mla_out_proj_workspace_size(cfg, n_tok) bytes
 * ------------------------------------------------------------------------- */
size_t mla_out_proj_workspace_size(const mla_config* cfg, int32_t n_tok);
mla_status mla_out_proj(const mla_config* cfg, const float* o_lat, int32_t n_tok,
                        const void* W_UV, const void* W_O, void* y,
                        void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Steps 4a + 4b fused - split combine inside the W_UV projection, then W_O
 * ([P5] section 1 "Định nghĩa": W_UV folded into the output side; the merge
 * of the splits is the standard log-sum-exp merge, not on the pages).  Since
 * o_h = o_lat_h W_UV_h is linear in o_lat, W_UV_h is applied to every
 * segment's partial output and the segments of a row are merged on the
 * projection's fp32 accumulators:
 *   o_h[t] = sum_s w_s,h (O_s,h W_UV_h),  w_s,h = 2^(lse_s,h - M) / sum_s' 2^(lse_s',h - M)
 *   y[t]   = concat_h(o_h[t]) W_O
 * The latent output o_lat is never written (use mla_combine for it).
 *   decode_ws: the workspace of the mla_decode call of this step (same
 *              batch, n_q and max_workers); read only.
 *   W_UV [d_c, H v_head];  W_O [H v_head, hidden];  y [batch n_q, hidden] (out)
 *   workspace >= mla_combine_out_proj_workspace_size(cfg, batch, n_q) bytes
 * bf16 storage only (MLA_ERR_UNSUPPORTED otherwise, or when v_head != 128 or
 * the decode has more than 512 segments: batch n_q + workers - 1 > 512).
 * mla_combine_out_proj_workspace_size returns 0 for shapes the fused path
 * does not take at the default worker count (then use mla_combine +
 * mla_out_proj).
 * A decode workspace that mla_decode did not write for this batch makes y
 * zero and records MLA_ERR_WORKSPACE on the device error word.
 * ------------------------------------------------------------------------- */
size_t mla_combine_out_proj_workspace_size(const mla_config* cfg, int32_t batch, int32_t n_q);
mla_status mla_combine_out_proj(const mla_config* cfg, const void* decode_ws, size_t decode_ws_bytes,
                                int32_t batch, int32_t n_q, int32_t max_workers,
                                const void* W_UV, const void* W_O, void* y,
                                void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Errors and introspection
 * ------------------------------------------------------------------------- */
/* Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (MLA_OK if none) and clears it.
 * detail (may be NULL) receives 3 ints describing the failing item. */
mla_status mla_get_device_error(void* stream, int32_t* detail);
/* Check of the bounded-wait path (not on the pages; a test of this library's
 * hang protection).  Every wait of the tensor-core kernels on a barrier gives
 * up after a time limit (2 s in the decode), records MLA_ERR_TIMEOUT in the
 * device error word and lets the kernel return, so a lost arrival surfaces
 * as an error instead of a hung GPU.  This call launches a one-warp kernel
 * that waits on a barrier whose second arrival never comes, with the given
 * limit (1 ns .. 10 s); after it, mla_get_device_error returns
 * MLA_ERR_TIMEOUT (detail[0] = 1) and the stream stays usable.
 * Returns MLA_ERR_INVALID_ARG for a limit out of range. */
mla_status mla_check_wait_timeout(int64_t limit_ns, void* stream);
/* Static description of a status code. */
const char* mla_status_string(mla_status status);
/* MLA_ABI_VERSION of the loaded library. */
int32_t mla_abi_version(void);
/* Number of CUDA kernels this library has launched in this process, on all
 * devices (a host-side counter; it never synchronises). */
int64_t mla_kernel_launches(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MLA_H_ */
