/*
 * ckv.h: C ABI of libckv, the compressed-KV sparse decode-attention library for NVIDIA B200
 * (sm_100a).
 *
 * The library implements the decode-time attention path of compressed-KV serving described on
 * these pages (cited by title and section):
 *
 *   [HR] 24-ai.news, "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom: milijun tokena konteksta na
 *        standardnom GPU hardveru", sections "Kako funkcionira optimizacija KV cachea?" (shared
 *        K=V vectors with inverse RoPE, compression by a weighted sum of tokens, top-k sparse
 *        attention, local sliding window) and "Sto je vLLM morao rijesiti u integraciji?" (CSA
 *        ratio 4 / HCA ratio 128, fixed 256-position logical blocks with a per-layer
 *        logical-to-physical mapping, the compressor remainder kept as sliding-window state).
 *   [DE] the German translation of [HR] on 24-ai.news, same sections.
 *   [CZ] aidevelopers.cz, "DeepSeek-V4.1-Flash ve vLLM: kde se vzala 5,3x vyssi propustnost",
 *        sections "Proc je obnova sliding-window cache draha" (FP8 window of the last 128
 *        positions, FP4 compressed cache) and "Vykon neprinesl jeden kernel" (Sparse MQA logits
 *        over candidate positions; attention over an NVFP4 compressed cache).
 *
 * Conventions used by every call:
 *   - Pointers named d_* are DEVICE pointers (CUDA global memory of the current device); other
 *     pointers are host pointers. The caller owns every buffer. Device buffers must be 16-byte
 *     aligned. The library allocates no device memory, never synchronizes the device, and
 *     enqueues all work on the CUDA stream passed as `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Calls are stream-ordered.
 *   - Host-side argument errors return a negative ckv_status before anything is enqueued.
 *   - Problems only visible on the device (a table entry outside the pool, a length above the
 *     stated maximum, an index out of range) are OR-ed as CKV_DEV_* bits into the caller's
 *     device word *d_status; the offending item is skipped (treated as absent) and the kernel
 *     returns normally. The caller zeroes *d_status and reads it after synchronizing. No kernel
 *     traps or waits on another block.
 *   - Layout of the rotary dims: the last rope_dim of head_dim, as interleaved pairs
 *     (D-d_r+2i, D-d_r+2i+1) rotated by angle p * rope_base^(-2i/d_r) (angles in fp64).
 */
#ifndef CKV_H_
#define CKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CKV_OK = 0,
  CKV_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, bad size or inconsistent config   */
  CKV_ERR_UNSUPPORTED = -2,   /* a dtype or shape this build has no kernel for               */
  CKV_ERR_OUT_OF_BLOCKS = -3, /* block pool exhausted (nothing was allocated)               */
  CKV_ERR_WORKSPACE = -4,     /* workspace smaller than the matching *_workspace_bytes()    */
  CKV_ERR_CUDA = -5           /* a CUDA runtime call or kernel launch failed                */
} ckv_status;

/* Bits OR-ed into *d_status by the kernels. */
#define CKV_DEV_BAD_BLOCK 0x1u   /* a needed table entry was < 0 or >= the pool's block count  */
#define CKV_DEV_BAD_LENGTH 0x2u  /* a length < 0 (append) / < 1 (decode) or > max_seq_len     */
#define CKV_DEV_BAD_INDEX 0x4u   /* a selected entry index outside [0, floor(L/r))            */
#define CKV_DEV_TIMEOUT 0x8u     /* a bounded wait for the tensor cores gave up (the split's
                                    partial is marked empty)                                  */

typedef enum {
  CKV_F32 = 0,       /* fp32                                                         */
  CKV_BF16 = 1,      /* bf16 (compressed cache)                                      */
  CKV_FP8_E4M3 = 2,  /* e4m3 codes + one fp32 scale per token (window cache)         */
  CKV_NVFP4 = 3      /* e2m1 codes (2 per byte, even element in the low nibble) + one
                        e4m3 scale per 16 consecutive elements (compressed cache)    */
} ckv_dtype;

/* One attention layer. */
typedef struct {
  int32_t num_heads;  /* H query heads; all share one K=V vector per key (MQA)            */
  int32_t head_dim;   /* D: multiple of 32 (NVFP4: of 64), 32..1024                       */
  int32_t rope_dim;   /* d_r: even, 0..D; the last d_r dims are rotary                   */
  int32_t ratio;      /* r: tokens folded into one compressed entry; a power of two 1..256
                         (4 for CSA and 128 for HCA layers in [HR] section B)             */
  int32_t window;     /* W: most recent tokens attended uncompressed, 0..256 ([CZ]: 128) */
  int32_t comp_dtype; /* CKV_F32 | CKV_BF16 | CKV_NVFP4                                   */
  int32_t win_dtype;  /* CKV_F32 | CKV_FP8_E4M3                                           */
  float sm_scale;     /* softmax scale; 0 selects 1/sqrt(D)                               */
  float rope_base;    /* rotary base; 0 selects 10000                                     */
} ckv_layer_cfg;

/*
 * The paged caches of one layer ([HR] section B). Logical block l of a request covers token
 * positions [256 l, 256 l + 256). A compressed pool block holds the 256/r entries whose tokens
 * lie in one logical block (entry i covers tokens [i r, i r + r)); a window pool block holds 256
 * tokens. Physical row of compressed entry i of request b:
 *     comp_table[b * table_stride + (i r) / 256] * (256 / r) + i % (256 / r)
 * and of window token t:   win_table[b * table_stride + t / 256] * 256 + t % 256.
 * Entry / token code bytes per row: F32 4D, BF16 2D, NVFP4 D/2 (+ D/16 scale bytes in
 * comp_scales), FP8_E4M3 D (+ one fp32 in win_scales). Use ckv_cache_row_bytes().
 */
typedef struct {
  void* comp_codes;            /* d: [comp_blocks][256/r][entry code bytes]                 */
  void* comp_scales;           /* d: NVFP4 only: [comp_blocks][256/r][D/16] e4m3; else NULL */
  void* win_codes;             /* d: [win_blocks][256][token code bytes]                    */
  float* win_scales;           /* d: FP8 only: [win_blocks][256] fp32; else NULL            */
  float* residue_kv;           /* d: [batch][r][D] fp32, rotated tokens of the unfinished
                                  group, slot = position % r ([HR] section B)               */
  float* residue_logit;        /* d: [batch][r] fp32 compressor logits of those tokens      */
  const int32_t* comp_table;   /* d: [batch][table_stride] physical block ids, -1 unmapped  */
  const int32_t* win_table;    /* d: [batch][table_stride]                                  */
  int32_t table_stride;        /* ints per table row, >= ceil(max_seq_len / 256)            */
  int32_t comp_blocks;         /* blocks in the compressed pool (device bounds checks)      */
  int32_t win_blocks;          /* blocks in the window pool                                 */
} ckv_layer_cache;

/* ---------------------------------------------------------------------------------------- */
/* Block pools ([HR] section B: fixed 256-position logical blocks mapped to physical blocks).
 * A pool is a HOST object handing out physical block ids 0..num_blocks-1 for one cache of one
 * layer; the caller writes the ids into the device tables. Ids come from a LIFO free list
 * whose initial order yields 0, 1, 2, ...; pools are not thread-safe. */

typedef struct ckv_pool ckv_pool;

/* Creates a pool of num_blocks (> 0) ids in *out. */
int kv_block_pool_create(int32_t num_blocks, ckv_pool** out);
/* Destroys the pool (NULL is a no-op). */
int kv_block_pool_destroy(ckv_pool* pool);
/* Writes n ids to out_ids (host array of n), all or nothing: CKV_ERR_OUT_OF_BLOCKS when fewer
 * than n are free, with nothing allocated. n == 0 is allowed. */
int kv_block_alloc(ckv_pool* pool, int32_t n, int32_t* out_ids);
/* Returns n ids (host array) to the pool, pushed in array order. An id out of range, already
 * free, or repeated in the array gives CKV_ERR_INVALID_ARG and frees nothing. */
int kv_block_free(ckv_pool* pool, const int32_t* ids, int32_t n);
/* Number of free ids, or a negative status. */
int32_t kv_block_pool_num_free(const ckv_pool* pool);

/* ---------------------------------------------------------------------------------------- */
/* Sizes. */

/* Bytes per pool row (one compressed entry / one window token) of each plane; unused planes
 * get 0. Returns CKV_OK or CKV_ERR_INVALID_ARG / CKV_ERR_UNSUPPORTED for a bad config. */
int ckv_cache_row_bytes(const ckv_layer_cfg* cfg, size_t* comp_code_bytes,
                        size_t* comp_scale_bytes, size_t* win_code_bytes,
                        size_t* win_scale_bytes);

/* Floats per request row of the optional score output of sparse_indexer_topk:
 * floor(max_seq_len / r) rounded up to a multiple of 64. */
int64_t ckv_score_stride(const ckv_layer_cfg* cfg, int32_t max_seq_len);

/* Workspace bytes needed by sparse_indexer_topk / compressed_window_attention for these sizes
 * (0 on a bad config). max_selected: idx_stride for a sparse call, or 0 for a dense call. */
size_t ckv_indexer_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch, int32_t max_seq_len,
                                   int32_t top_k);
size_t ckv_attention_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch,
                                     int32_t max_seq_len, int32_t max_selected);

/* ---------------------------------------------------------------------------------------- */
/* Step 1: the KV compressor ([HR] section A: compression by a weighted sum of tokens; section B:
 * the remainder kept as sliding-window state).
 *
 * Appends n_b raw (un-rotated) tokens to request b at positions prev_len[b] .. prev_len[b]+n_b-1.
 * Each token x is rotated at its own position (fp64 angle) and stored as fp32:
 *   - into the window cache if its position is >= prev_len[b] + n_b - W (FP8: per-token scale
 *     s = amax|x| / 448, codes = e4m3 round-to-nearest-even satfinite of x/s; s = 1 if x == 0);
 *   - into the residue ring slot (position % r) if its group stays unfinished after the call;
 *   - a token whose position + 1 is a multiple of r completes its group g = (position+1)/r - 1:
 *     the weights are the softmax of the group's r logits and entry g = sum_t w_t * x_t (fp32),
 *     stored as fp32, bf16 (round to nearest even) or NVFP4 (per 16 elements: scale = e4m3
 *     RNE-satfinite of amax/6; codes = e2m1 RNE-satfinite of x/scale, all 0 if scale is 0).
 * Tokens of the group before prev_len[b] are read from the residue ring (written by earlier
 * calls). The call only writes; nothing it writes is read by a later block of the same call.
 *
 *   d_prev_len  [batch] int32: tokens already appended (>= 0).
 *   d_cu_new    [batch+1] int32 prefix offsets into the rows of d_kv_new, or NULL for exactly one
 *               token per request (row b).
 *   max_new     host upper bound of n_b (1 when d_cu_new is NULL); sizes the grid. With
 *               max_new == 1 (decode) a request with n_b > 1 is rejected on the device
 *               (CKV_DEV_BAD_LENGTH, nothing written for it).
 *   max_seq_len host upper bound of prev_len[b] + n_b (table bounds).
 *   d_kv_new    [sum n_b][D] fp32;  d_logit_new [sum n_b] fp32.
 * The tables must map every logical block written: the blocks holding the completed entries
 * and the window positions above.
 */
int kv_compress_append(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                       const int32_t* d_prev_len, const int32_t* d_cu_new, int32_t max_new,
                       int32_t max_seq_len, const float* d_kv_new, const float* d_logit_new,
                       uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* SWA bounded replay ([CZ] section "Proc je obnova sliding-window cache draha": after a
 * prefix-cache hit only the last window is run through the model again, and the dependence on
 * positions before it is cut; [CZ] section "Polovina vrstev nemusi cist cely prompt" names the
 * switch). The model recomputes the window's K=V vectors; this call puts them in the cache.
 *
 * For request b with L = seq_len[b] and n_w = min(W, L): the raw (un-rotated) tokens of positions
 * L - n_w .. L - 1 are rotated at their own positions and written to the window cache with the
 * rules of kv_compress_append; those in the unfinished group [floor(L/r) r, L) also go to the
 * residue ring (slot = position % r) with their compressor logits, so that the next append folds
 * them. Compressed entries are not touched (they come from the prefix cache). Ring slots of the
 * unfinished group's positions before L - n_w (only possible when r - 1 > W) are left as they are.
 *
 *   d_seq_len   [batch] int32, 1 <= L <= max_seq_len (else CKV_DEV_BAD_LENGTH, request skipped).
 *   d_kv        [batch][W][D] fp32: row i of request b is position L - n_w + i (rows >= n_w unused).
 *   d_logit     [batch][W] fp32 compressor logits, same rows.
 * The window table must map the blocks of positions [L - n_w, L). W == 0 enqueues nothing. */
int kv_window_replay(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                     const int32_t* d_seq_len, int32_t max_seq_len, const float* d_kv, const float* d_logit,
                     uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* Step 2: the sparse MQA indexer and top-k ([HR] section A: sparse attention over the top-k
 * compressed tokens; [CZ] section C: "Sparse MQA logits" scores the candidate positions).
 *
 * For request b with context L = seq_len[b] (including the decode token at position L-1), the
 * candidates are the N_c = floor(L / r) completed entries. The query q[b] ([H][D] fp32, raw) is
 * rotated at position L-1 and each candidate j gets the head-averaged MQA logit
 *     s_j = sm_scale * (1/H) * sum_h q~_h . k_j          (fp32 on the device)
 * The min(top_k, N_c) largest scores are selected (ties to the lower index) and written to
 * d_idx[b][0..] in ascending index order, padded with -1 up to top_k; d_cnt[b] = min(top_k, N_c).
 *
 *   d_seq_len   [batch] int32, 1 <= L <= max_seq_len.   d_q [batch][H][D] fp32.
 *   top_k       >= 1.   d_idx [batch][top_k] int32.   d_cnt [batch] int32.
 *   d_scores    optional [batch][ckv_score_stride()] fp32 output of every s_j (NULL = none).
 *   d_ws        workspace of ws_bytes >= ckv_indexer_workspace_bytes(cfg, batch, max_seq_len,
 *               top_k); its contents need not be initialised and are clobbered.
 */
int sparse_indexer_topk(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                        const int32_t* d_seq_len, int32_t max_seq_len, const float* d_q,
                        int32_t top_k, int32_t* d_idx, int32_t* d_cnt, float* d_scores,
                        void* d_ws, size_t ws_bytes, uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* Step 3: attention over the selected compressed entries plus the window ([HR] section A: top-k
 * compressed tokens and a local window with full vectors; one shared K=V vector with inverse
 * RoPE).
 *
 * For request b: keys = the entries d_idx[b][0 .. d_cnt[b]) (or, when d_idx is NULL, every
 * completed entry 0 .. floor(L/r)-1: a dense HCA layer) followed by the window tokens
 * [max(0, L-W), L). Each key vector is also its value. With q~_h the query rotated at L-1:
 *     o_h = sum_j softmax_j(sm_scale * q~_h . x_j) x_j      (one softmax over all keys)
 * and the rotary dims of o_h are rotated back by -(L-1). No keys gives o_h = 0.
 *
 *   d_idx       [batch][idx_stride] int32 entry indices in [0, floor(L/r)) or NULL (dense).
 *   d_cnt       [batch] int32 counts (ignored when d_idx is NULL), 0 <= cnt <= idx_stride.
 *   d_out       [batch][H][D] fp32.
 *   d_ws        workspace of ws_bytes >= ckv_attention_workspace_bytes(cfg, batch, max_seq_len,
 *               d_idx ? idx_stride : 0).
 */
int compressed_window_attention(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache,
                                int32_t batch, const int32_t* d_seq_len, int32_t max_seq_len,
                                const float* d_q, const int32_t* d_idx, const int32_t* d_cnt,
                                int32_t idx_stride, float* d_out, void* d_ws, size_t ws_bytes,
                                uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* sparse_indexer_topk without a caller-allocated workspace. The pages have no counterpart to
 * this entry point; it exists for callers that cannot allocate device memory (an extension
 * inside a host program that owns all device memory and gives extensions no allocator, or a
 * latency-critical path where an allocation would synchronize the device).
 *
 * Same arguments, results and errors as sparse_indexer_topk minus d_ws / ws_bytes: the scratch
 * comes from a 16 MiB array owned by the library, which every GPU that loads the library holds
 * until the process exits. Sizes whose ckv_indexer_workspace_bytes() exceeds 16 MiB return
 * CKV_ERR_WORKSPACE before anything is enqueued. No allocation of any kind is made.
 *
 * The first call on a device looks up the array's device address on that device (a host-side
 * runtime query, no allocation); make that first call before any stream capture. Later calls only
 * check, with host-side driver queries, that the device's context is still the one the address
 * was found in; the first call after the context was replaced (cudaDeviceReset) looks it up again
 * and should also come before any stream capture. All calls share
 * the array and it keeps the last call's contents: the kernels reset the parts that must start at
 * zero on every call, and calls whose kernels overlap on the GPU (other streams, or unordered
 * threads) race on it. */
int sparse_indexer_topk_noalloc(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache,
                                int32_t batch, const int32_t* d_seq_len, int32_t max_seq_len,
                                const float* d_q, int32_t top_k, int32_t* d_idx, int32_t* d_cnt,
                                float* d_scores, uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* Fused decode step of one layer: steps 1-3 in one call (the three descriptions above apply).
 * [HR] section A lists the path's parts (compression, top-k over compressed tokens, window,
 * shared K=V attention); [CZ] section C credits the speed-up to fused kernels. One token per
 * request is appended at position seq_len[b] - 1, the layer's top_k entries are selected
 * (top_k > 0, CSA) or all entries are attended (top_k == 0, HCA), and the output is written.
 * Compared with the three calls, the append of the new token runs beside the indexer's query pass
 * (in one kernel when the batch fills the GPU), and that pass also writes the cos/sin table the
 * attention's merge needs; every result is bit-identical to the three calls'.
 *
 *   d_seq_len    [batch] int32: L_b including the new token (1 .. max_seq_len).
 *   d_q          [batch][H][D] fp32 raw query; d_kv_new [batch][D] fp32 raw token; d_logit_new
 *                [batch] fp32 compressor logit.
 *   top_k        0 for a dense layer; else the selection size, and d_idx [batch][top_k] / d_cnt
 *                [batch] receive the selection (as sparse_indexer_topk writes it).
 *   d_out        [batch][H][D] fp32.
 *   d_ws         workspace of ckv_decode_step_workspace_bytes(cfg, batch, max_seq_len, top_k)
 *                bytes, 16-byte aligned; its contents need no initialisation.
 * Errors as for the three calls (host codes before any launch, device status bits after).
 */
size_t ckv_decode_step_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch, int32_t max_seq_len,
                                       int32_t top_k);
int ckv_decode_step(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                    const int32_t* d_seq_len, int32_t max_seq_len, const float* d_q,
                    const float* d_kv_new, const float* d_logit_new, int32_t top_k, int32_t* d_idx,
                    int32_t* d_cnt, float* d_out, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                    void* stream);

/* ---------------------------------------------------------------------------------------- */
/* Multi-head indexer ([CZ] section C: "Sparse MQA logits" scores only the candidate positions).
 * The pages name the indexer and give no formula; this is its multi-head reading, next to the
 * head-averaged one of sparse_indexer_topk. The indexer has H_I heads of width d_I and its own
 * compressed index key per entry:
 *   - per token the caller supplies an index key (d_I fp32, position encoding already applied;
 *     the projections that make index keys and queries are outside this library);
 *   - the keys of a group of r tokens are folded with the softmax weights of the same compressor
 *     logits as the K=V tokens ([HR] section A: compression by a weighted sum), entry = sum_t w_t
 *     key_t in fp32, and stored as FP8 e4m3 with one fp32 scale per entry (s = amax / 448, 1 for a
 *     zero entry; codes = e4m3 RNE-satfinite of x / s: the window's FP8 rule);
 *   - at decode time each head's index query q_h (d_I fp32) is stored by the same FP8 rule
 *     (codes q~_h, scale t_h = amax_h / 448) and, with one fp32 weight w_h per head, candidate j
 *     (an entry < floor(L/r), codes c_j, scale s_j) scores
 *         score_j = s_j * sum_h (w_h t_h) * max(0, q~_h . c_j)      (e4m3 products, fp32 sums)
 *     i.e. sum_h w_h max(0, q^_h . k_j) for the decoded query and entry; the top-k rule and
 *     outputs are those of sparse_indexer_topk.
 * The index plane lives in the rows of the layer's compressed pool: entry i of request b is row
 * comp_table[b * table_stride + (i r) / 256] * (256 / r) + i % (256 / r) of `codes` / `scales`. */
typedef struct {
  int32_t index_heads; /* H_I: a multiple of 16, 16..128                                   */
  int32_t index_dim;   /* d_I: 128 or 256                                                  */
} ckv_index_cfg;

typedef struct {
  void* codes;          /* d: [comp_blocks][256/r][d_I] e4m3 index entries                 */
  float* scales;        /* d: [comp_blocks][256/r] fp32 entry scales                       */
  float* residue_k;     /* d: [batch][r][d_I] fp32 index keys of the unfinished group,
                           slot = position % r (kv_index_append only)                      */
  float* residue_logit; /* d: [batch][r] fp32 their logits; a ring of its own, not the
                           layer's residue_logit (kv_index_append only)                    */
} ckv_index_cache;

/* Appends n_b index keys to request b at positions prev_len[b] .. prev_len[b]+n_b-1 (the same
 * tokens, in the same calls, as kv_compress_append): a key whose position + 1 is a multiple of r
 * completes its group, which is folded and stored as above; the keys of an unfinished group go
 * to the residue ring. Arguments as for kv_compress_append, with cfg / cache the layer's (ratio,
 * compressed table and pool size) and d_k_new [sum n_b][d_I] fp32. Nothing outside the index
 * plane and its ring is written. */
int kv_index_append(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, const ckv_index_cfg* icfg,
                    const ckv_index_cache* icache, int32_t batch, const int32_t* d_prev_len,
                    const int32_t* d_cu_new, int32_t max_new, int32_t max_seq_len, const float* d_k_new,
                    const float* d_logit_new, uint32_t* d_status, void* stream);

/* Workspace bytes of sparse_mh_indexer_topk (0 on a bad config). */
size_t ckv_mh_indexer_workspace_bytes(const ckv_layer_cfg* cfg, const ckv_index_cfg* icfg, int32_t batch,
                                      int32_t max_seq_len, int32_t top_k);

/* Scores every candidate of each request with the multi-head rule and selects the top_k, with the
 * outputs, padding, tie rule, optional d_scores and device errors of sparse_indexer_topk.
 *   d_q_index  [batch][H_I][d_I] fp32.   d_weights [batch][H_I] fp32.
 *   batch      1 .. 2048, ratio r 1, 2 or 4 (256/r >= 64 entries per pool block); otherwise
 *              CKV_ERR_UNSUPPORTED.
 *   d_ws       workspace of ws_bytes >= ckv_mh_indexer_workspace_bytes(...).
 * A wait for the tensor cores that gives up sets CKV_DEV_TIMEOUT (the scores of the tiles not
 * reached are not written). */
int sparse_mh_indexer_topk(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, const ckv_index_cfg* icfg,
                           const ckv_index_cache* icache, int32_t batch, const int32_t* d_seq_len,
                           int32_t max_seq_len, const float* d_q_index, const float* d_weights, int32_t top_k,
                           int32_t* d_idx, int32_t* d_cnt, float* d_scores, void* d_ws, size_t ws_bytes,
                           uint32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* Diagnostics. */

/* Static text of a ckv_status. */
const char* ckv_status_str(int status);
/* Number of kernel launches enqueued by this process since load (all entry points). */
uint64_t ckv_launch_count(void);

/* Failure-path hook for tests. While request >= 0, the lane that issues the tensor-core MMAs of
 * every attention CTA of that request (tensor-core layers: H = 64, D = 512, bf16 or NVFP4
 * compressed cache, FP8 window) first waits on a barrier that nothing completes; the bounded wait
 * runs out, the CTA takes its failure path (nothing is issued, CKV_DEV_TIMEOUT is set, its
 * partial is marked empty) and that request's output is zero, while the other requests and the
 * CUDA context are unaffected. request = -1 turns it off (the default). The setting is a device
 * variable of the current device, written with a blocking copy; not thread-safe. */
int ckv_debug_force_timeout(int32_t request);

/* Diagnostic timing. While set, every later call records the CUDA events ev_begin (just before)
 * and ev_end (just after) the launch of one kernel, on the call's stream:
 *   CKV_PROF_SCORE      the scoring kernel of sparse_indexer_topk
 *   CKV_PROF_ATTENTION  the attention kernels of compressed_window_attention (the attention
 *                       kernel and the merge of its splits, which writes the output)
 * ev_begin / ev_end are cudaEvent_t handles created by the caller; NULL, NULL stops recording.
 * Process-wide setting, not thread-safe. Returns CKV_ERR_INVALID_ARG for an unknown `which` or
 * only one NULL handle. */
#define CKV_PROF_SCORE 0
#define CKV_PROF_ATTENTION 1
int ckv_profile_events(int which, void* ev_begin, void* ev_end);

#ifdef __cplusplus
}
#endif

#endif /* CKV_H_ */
