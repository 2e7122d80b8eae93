/*
 * csa2.h -- C ABI of libcsa2.so: the CSA2 decode step (Compressed Sparse
 * Attention 2) with its Hierarchical Sparse Indexer over an FP4 main-KV cache,
 * as hand-written sm_100a (B200) CUDA kernels.
 *
 * Where each operation is defined (page title and section):
 *   - Layer modes Full / Reindex / Reuse: readance summary of the
 *     DeepSeek-V4.1-Flash report, section 4.2; 4sapi "DeepSeek V4.1 Flash
 *     CED/CSA2" blog, section 二 (mode table).
 *   - Indexer (32 heads x 128, Top-512) and the hierarchical pool (2048 blocks
 *     x 8 positions kept by the first Full layer; Reindex layers choose inside
 *     it): 4sapi blog, section 四; alphalab "DeepSeek-V4.1-Flash 深度分析",
 *     section 2 CSA2; animattoys article, section 層與層之間拼車.
 *   - Main KV in FP4 E2M1 with one E4M3 scale per 16 channels, no global
 *     scale, quantised after RoPE: 4sapi blog, section 五 FP4 KV; animattoys
 *     article, section 把精度降到4比特; alphalab analysis, section 3 FP4.
 *   The pages leave open the indexer dtype, the score and block functions and
 *   every tie rule; the readings implemented here are:
 *     indexer K and Q: FP8 E4M3 codes with one power-of-two scale per row
 *       (sigma = 2^e, e the smallest integer with 448 * 2^e >= max|row|,
 *       e >= -126; stored byte e + 127);
 *     score s_t = sigma_t * sum_h w_h * ReLU(sigma^q_h * <q^_h, k^_t>);
 *     block score = max over the block's visible positions;
 *     ties in every selection go to the lower index; selections are returned
 *     sorted ascending and padded with -1.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers owned by the caller unless marked
 *     "host".  The library never allocates, frees or synchronises (except
 *     csa2_get_error) and keeps no state between calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued asynchronously on it.
 *   - Shapes and pointers are validated on the host before any launch; a
 *     violation returns CSA2_ERR_ARG / CSA2_ERR_SHAPE / CSA2_ERR_UNSUPPORTED
 *     and launches nothing.  csa2_last_error_message() then describes it.
 *   - Data-dependent violations found on the device (a page id outside
 *     [0, num_pages), a position outside the request's capacity, a Top-k
 *     index outside the visible context) never trap: the kernel records the
 *     first one in cache->err_word and skips or neutralises the offending
 *     element; csa2_get_error() reads it back.
 *   - A ctx_len[b] outside [0, capacity] is such a violation too: every
 *     kernel that reads it records CSA2_ERR_DEVICE_BOUNDS with index = the
 *     length and treats request b as empty (no scan, an all -1 pool and
 *     Top-k, zero attention output): a corrupt length never silently
 *     truncates a request.
 *   - Launch failures return CSA2_ERR_CUDA.
 *   - Each kernel's launch attributes (dynamic shared memory size, cluster
 *     size) are set once per CUDA context, on its first launch there: one
 *     process may drive several devices, and a context that is destroyed and
 *     created again is set up anew.
 *   - Kernels are launched with programmatic dependent launch: each one waits
 *     for the kernel before it on the stream before reading anything that
 *     kernel may write, and lets its own successor start early.  The
 *     attention entry points load their query rows `q` before that wait, so
 *     q must not be written by an immediately preceding kernel that itself
 *     signals early completion (griddepcontrol.launch_dependents); ordinary
 *     kernels, copies and events before the call are safe.
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

typedef enum {
  CSA2_FULL = 0,     /* Top-k from this layer's own Full scan            */
  CSA2_REINDEX = 1,  /* re-score the pool with this layer's own query    */
  CSA2_REUSE = 2     /* take the previous layer's Top-k unchanged        */
} csa2_mode;

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_ARG = 1,            /* null / misaligned pointer, bad enum    */
  CSA2_ERR_SHAPE = 2,          /* size outside the supported range        */
  CSA2_ERR_CUDA = 3,           /* a CUDA runtime call failed              */
  CSA2_ERR_DEVICE_BOUNDS = 4,  /* (err_word) out-of-range page/position   */
  CSA2_ERR_TIMEOUT = 5,        /* (err_word) a pipeline wait gave up      */
  CSA2_ERR_UNSUPPORTED = 6     /* device is not sm_100 / feature missing  */
} csa2_status;

/* Positions per pool block and cache row sizes (bytes). */
#define CSA2_BLOCK 8
#define CSA2_INDEX_HEADS 32
#define CSA2_INDEX_DIM 128
#define CSA2_KV_DIM 512
#define CSA2_KV_CODE_BYTES 256   /* 512 E2M1 codes, 2 per byte            */
#define CSA2_KV_SCALE_BYTES 32   /* one E4M3 scale per 16 channels         */

/*
 * The paged cache of one layer group.  A "row" is one cached position; rows
 * live in pages of `page_size` consecutive rows.  Position t of request b is
 * row  page_table[b * max_pages_per_req + t / page_size] * page_size
 *      + t % page_size.
 * Arrays (row-major, device memory, 16-byte aligned base pointers):
 *   kv_codes   uint8 [num_pages * page_size][256]  E2M1 pairs: byte i holds
 *              channel 2i in its low nibble, channel 2i+1 in its high nibble
 *   kv_scales  uint8 [num_pages * page_size][32]   E4M3 scale of channels
 *              16g..16g+15
 *   ik_codes   uint8 [num_pages * page_size][128]  E4M3 indexer key
 *   ik_exp     uint8 [num_pages * page_size]       sigma_t = 2^(byte - 127)
 *   page_table int32 [batch][max_pages_per_req]
 *   ctx_len    int32 [batch]  visible positions of each request
 *   err_word   int32 [4]      {code, kernel, request, index} of the first
 *              device-side error; the caller zeroes it once.
 * page_size must be a positive multiple of 128.
 */
typedef struct csa2_cache {
  uint8_t* kv_codes;
  uint8_t* kv_scales;
  uint8_t* ik_codes;
  uint8_t* ik_exp;
  const int32_t* page_table;
  const int32_t* ctx_len;
  int32_t num_pages;
  int32_t page_size;
  int32_t max_pages_per_req;
  int32_t batch;
  int32_t* err_word;
} csa2_cache;

/* Capacity of one request in positions: max_pages_per_req * page_size.  The
 * per-request strides of the score and block-max buffers below derive from it:
 *   scores   float [batch][capacity]
 *   blockmax float [batch][capacity / 8]                                    */

/*
 * csa2_append_kv -- quantise-on-append (main KV to FP4, indexer K to FP8) and
 * write n_rows rows into their page slots.
 *   kv_new  float [n_rows][512]  main KV rows (already rotated: the pages
 *                                state quantisation happens after RoPE)
 *   ik_new  float [n_rows][128]  indexer keys
 *   req     int32 [n_rows]       request of each row; NULL = row i -> request i
 *   pos     int32 [n_rows]       position of each row inside its request
 * Per 16 channels: s = E4M3 nearest (ties to even, saturating) of amax/6;
 * codes = E2M1 nearest of x/s (ties to even code, saturating at 6, -0 -> +0).
 * Indexer: sigma as above, codes = E4M3 nearest of k/sigma.
 * ctx_len is not modified: the caller advances it.
 * Device errors: req outside [0,batch), pos outside [0,capacity), page id
 * outside [0,num_pages) -> CSA2_ERR_DEVICE_BOUNDS, row skipped.
 */
CSA2_API csa2_status csa2_append_kv(const csa2_cache* cache, int32_t n_rows, const float* kv_new,
                           const float* ik_new, const int32_t* req, const int32_t* pos,
                           void* stream);

/*
 * csa2_compress_append -- the sequence compressor of the encoder groups,
 * then quantise-on-append: entry i is the mean of the m token rows
 * m*i .. m*i + m - 1 and is stored, quantised exactly as by csa2_append_kv,
 * at position pos[i] of request req[i] [4sapi blog, section 三: the
 * encoder's 1 Full + 5 Reuse groups compress the sequence with m = 2].
 * Reading (the pages name m only): a plain mean, summed in float64 in token
 * order, scaled by 1/m and rounded once to fp32; m in {1, 2, 4, 8}.  Rotary
 * position encoding, which the pages place before quantisation, is the
 * caller's: the token rows arrive rotated.
 *   n_entries  entries to write (>= 0; 0 does nothing)
 *   m          tokens per entry
 *   kv_tok     float [n_entries * m][512]  main-KV token rows
 *   ik_tok     float [n_entries * m][128]  indexer-K token rows
 *   req        int32 [n_entries] request of each entry, or NULL (request 0)
 *   pos        int32 [n_entries] entry position inside its request
 * Device errors as csa2_append_kv.
 */
CSA2_API csa2_status csa2_compress_append(const csa2_cache* cache, int32_t n_entries, int32_t m,
                                          const float* kv_tok, const float* ik_tok, const int32_t* req,
                                          const int32_t* pos, void* stream);

/*
 * Histogram of the block maxima passed from csa2_index_full to
 * csa2_pool_select: uint32 [batch][CSA2_POOL_HIST_BINS], one count per
 * visible block in the bin of its score's leading 12 order-key bits (the fp32
 * bit pattern with the sign bit flipped, or all bits flipped when negative:
 * sign, exponent and 3 mantissa bits, so that one bin spans an eighth of an
 * octave; the block maxima of a request crowd into few octaves).
 * The scan adds to it, so it must hold zeros when the scan starts;
 * csa2_pool_select reads it and zeroes it again.  Zero it once (for instance
 * cudaMemsetAsync) before its first use.  It only saves time: a histogram
 * that does not hold exactly one count per block, or whose threshold bin and
 * the bins above it disagree with the block maxima (not zeroed, shared by two
 * scans, a scan that gave up) is detected and ignored by csa2_pool_select,
 * which then selects without it, exactly, and still zeroes it.
 */
#define CSA2_POOL_HIST_BINS 4096

/*
 * csa2_index_full -- Full-mode indexer scan of every visible position of every
 * request (Hierarchical Sparse Indexer, first stage).
 *   q        float [batch][32][128]  indexer query (quantised inside, FP8 rule)
 *   w        float [batch][32]       head weights
 *   blockmax float [batch][capacity/8]  out: m_j = max score of block j over
 *            positions < ctx_len; entries past ceil(ctx_len/8) are untouched
 *   scores   float [batch][capacity] or NULL  out: per-position scores s_t
 *   hist     uint32 [batch][CSA2_POOL_HIST_BINS] or NULL (16-byte aligned):
 *            the block maxima's histogram for csa2_pool_select (see above)
 * Runs on tcgen05 FP8 tensor cores (scores are fp32; the float64 reference
 * differs by fp32 accumulation rounding only).
 */
CSA2_API csa2_status csa2_index_full(const csa2_cache* cache, const float* q, const float* w,
                            float* blockmax, float* scores, uint32_t* hist, void* stream);

/*
 * csa2_pool_select -- the hierarchical pool: the pool_blocks blocks with the
 * largest block max (ties -> lower block id), sorted ascending, -1 padded.
 * With ceil(ctx_len/8) <= pool_blocks the pool is every block.
 *   blockmax float [batch][capacity/8]   (from csa2_index_full)
 *   hist     uint32 [batch][CSA2_POOL_HIST_BINS] from the same scan, or NULL:
 *            with it the selection starts from the bin that holds the
 *            threshold instead of radix passes over every block; it is left
 *            zeroed.  The result is the same with or without it.
 *   pool     int32 [batch][pool_blocks]  out
 * pool_blocks in [1, 4096] (the pages use 2048); ceil(capacity/8) must not
 * exceed 16 * 16384 blocks (2,097,152 positions per request).
 */
CSA2_API csa2_status csa2_pool_select(const csa2_cache* cache, const float* blockmax, uint32_t* hist,
                             int32_t pool_blocks, int32_t* pool, void* stream);

/*
 * Context-sharded pool.  One request's context split into consecutive slices,
 * one per device (slice g holds positions [start_g, start_g + len_g), start_g
 * a multiple of 8), each device holding its slice in a cache of its own whose
 * positions count from the slice start [alphalab analysis, limits section: a
 * 1M context may have to be sharded across machines, with the exchange as
 * its cost].  Per device: csa2_index_full and csa2_pool_select on the slice,
 * then csa2_pool_candidates; the devices exchange the candidates (an
 * all-gather of pool_blocks * 8 bytes per request and device); every device
 * (or the one that continues) calls csa2_pool_merge.  The merged pool is
 * exactly the pool csa2_pool_select returns for the unsharded request: a
 * block of that pool has fewer than pool_blocks blocks ahead of it in its own
 * slice, so its slice kept it.
 *
 * csa2_pool_candidates -- a slice's local pool as (block max, global block id)
 * pairs.
 *   shard        the slice's cache (ctx_len = the slice's visible length)
 *   blockmax     float [batch][capacity/8] of the slice's scan
 *   pool         int32 [batch][pool_blocks] of the slice's csa2_pool_select
 *   block_offset global block id of the slice's block 0 (start_g / 8)
 *   values       float [batch][pool_blocks] out (0 where the pool is -1)
 *   ids          int32 [batch][pool_blocks] out: pool + block_offset, or -1
 * Device errors: a pool entry outside [-1, ceil(ctx_len/8)) ->
 * CSA2_ERR_DEVICE_BOUNDS, entry emptied.
 *
 * csa2_pool_merge -- the request's pool from the G slices' candidates.
 *   values float [n_shards][batch][pool_blocks], ids int32 [same], the slices
 *          in ascending order of their start (as gathered by rank), each list
 *          ascending with -1 last (as csa2_pool_candidates writes it): the
 *          candidate order is then the global block order that decides ties
 *   pool   int32 [batch][pool_blocks] out: the pool_blocks best (block max
 *          desc, global id asc), ascending, -1 padded
 * n_shards in [1, CSA2_MAX_SHARDS], n_shards * pool_blocks <= 32768.  One
 * CTA per request; no workspace.
 */
#define CSA2_MAX_SHARDS 16
CSA2_API csa2_status csa2_pool_candidates(const csa2_cache* shard, const float* blockmax, const int32_t* pool,
                                          int32_t pool_blocks, int32_t block_offset, float* values,
                                          int32_t* ids, void* stream);
CSA2_API csa2_status csa2_pool_merge(int32_t n_shards, int32_t batch, int32_t pool_blocks, const float* values,
                                     const int32_t* ids, int32_t* pool, void* stream);

/*
 * FP4 indexer variant [animattoys article, section 把精度降到4比特: V4 kept
 * the indexer's Q and K in FP4].  Reading (the pages give no format): the
 * main-KV format on the indexer's 128-element row, E2M1 codes with one E4M3
 * scale per 16 elements, s = E4M3(amax / 6) (nearest, ties to even,
 * saturating), no row scale, for the cached keys and for each query head; the
 * score is s_t = sum_h w_h * ReLU(<q~_h, k~_t>) over the dequantised values.
 * 72 bytes per position instead of the FP8 indexer's 129.  The keys live next
 * to the cache (same rows, same page table):
 *   codes   uint8 [num_pages * page_size][64]: element 2i in the low nibble
 *           of byte i, element 2i + 1 in the high nibble
 *   scales  uint8 [num_pages * page_size / 128][1024]: the scales of each
 *           128-row tile (rows r .. r + 127 with r a multiple of 128), the
 *           scale of tile row m and element group g (elements 16g .. 16g+15)
 *           at byte  (g / 4) * 512 + (m % 32) * 16 + (m / 32) * 4 + g % 4,
 *           the order in which the tensor cores read block scales
 * Both 16-byte aligned, caller-owned.
 */
#define CSA2_IK4_CODE_BYTES 64
#define CSA2_IK4_TILE_SCALE_BYTES 1024
typedef struct csa2_ik4 {
  uint8_t* codes;
  uint8_t* scales;
} csa2_ik4;

/*
 * csa2_append_ik4 -- quantise n_rows indexer keys (float [n_rows][128]) to
 * the FP4 indexer format and store them at (req[i], pos[i]) (req NULL: row i
 * -> request i).  Device errors as csa2_append_kv.
 *
 * csa2_index_full_fp4 -- csa2_index_full over the FP4 indexer keys: q float
 * [batch][32][128] is quantised per head to the same format inside; w, blockmax,
 * scores and hist as csa2_index_full.  The contraction runs on the tensor
 * cores as block-scaled FP4 (tcgen05 kind::mxf4nvf4, E4M3 scales per 16
 * elements), fp32 accumulation.
 *
 * csa2_reindex_layers_fp4 -- csa2_reindex_layers over the FP4 indexer keys
 * (every layer's query quantised per head to FP4); n_layers in [1, 4], other
 * arguments and the workspace as csa2_reindex_layers.
 */
CSA2_API csa2_status csa2_append_ik4(const csa2_cache* cache, const csa2_ik4* ik4, int32_t n_rows,
                                     const float* ik_new, const int32_t* req, const int32_t* pos, void* stream);
CSA2_API csa2_status csa2_index_full_fp4(const csa2_cache* cache, const csa2_ik4* ik4, const float* q,
                                         const float* w, float* blockmax, float* scores, uint32_t* hist,
                                         void* stream);
CSA2_API csa2_status csa2_reindex_layers_fp4(const csa2_cache* cache, const csa2_ik4* ik4, int32_t n_layers,
                                             const int32_t* pool, int32_t pool_blocks, const float* const* q,
                                             const float* const* w, int32_t k, int32_t* const* topk,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * csa2_reindex -- Top-k of one layer of the group, by mode:
 *   CSA2_FULL    the k best positions of this layer's own Full scan among the
 *                candidates.  Scores come from full_scores when it is not NULL,
 *                else they are recomputed from (q, w) with the exact arithmetic
 *                of csa2_index_full (bit-identical).
 *   CSA2_REINDEX re-score only the candidates with this layer's own (q, w).
 *   CSA2_REUSE   copy prev_topk into topk (nothing is done when they alias).
 * Candidates: the positions of the pool's blocks (pool int32 [batch]
 * [pool_blocks], ascending, -1 padded), or every visible position when pool is
 * NULL (then the request capacity must not exceed 65,536 positions).
 *   q float [batch][32][128], w float [batch][32]  (FULL without full_scores,
 *                                                   and REINDEX)
 *   full_scores float [batch][capacity] or NULL
 *   prev_topk int32 [batch][k]  (REUSE)
 *   topk      int32 [batch][k]  out: positions ascending, -1 padded
 * k in [1, 4096], pool_blocks in [1, 4096].
 */
CSA2_API csa2_status csa2_reindex(const csa2_cache* cache, csa2_mode mode, const int32_t* pool,
                         int32_t pool_blocks, const float* q, const float* w,
                         const float* full_scores, const int32_t* prev_topk, int32_t k,
                         int32_t* topk, void* stream);

/*
 * csa2_reindex_layers -- csa2_reindex over a pool for n_layers layers at once:
 * layer l's Top-k is the k best positions of the pool by the score of
 * (q[l], w[l]), exactly as csa2_reindex in mode CSA2_REINDEX would return it;
 * a Full layer passes its own (q, w) and gets the Top-k of its scan's scores
 * (the arithmetic is bit-identical).  Reuse layers take no part: they alias
 * the Top-k of the layer they follow.  Every pool block is gathered from the
 * cache once for all layers, and all layers are scored in one tensor-core
 * pass; one select launch then serves every (request, layer).
 *   n_layers     in [1, CSA2_MAX_SCORE_LAYERS]
 *   pool         int32 [batch][pool_blocks] (from csa2_pool_select)
 *   q, w         host arrays [n_layers] of device pointers: float
 *                [batch][32][128] (16-byte aligned) and float [batch][32]
 *   k            in [1, 4096]
 *   topk         host array [n_layers] of device pointers, int32 [batch][k]
 *                out: positions ascending, -1 padded (ties -> lower position)
 *   workspace    caller-owned device memory of at least
 *                csa2_reindex_layers_workspace_bytes(batch, n_layers,
 *                pool_blocks) bytes, 16-byte aligned: the layers' pool scores
 *                and one histogram of their leading 12 bits per (request,
 *                layer).  Zero it once before its first use; each call leaves
 *                the histograms zeroed again.  As with the pool's histogram,
 *                a histogram that is not zero at the start only costs time
 *                (it is detected, ignored and zeroed).  Two calls in flight at
 *                once must not share a workspace.
 * Launches two kernels.  Device errors as csa2_reindex; on CSA2_ERR_TIMEOUT
 * the outputs are undefined.
 */
#define CSA2_MAX_SCORE_LAYERS 8
#define CSA2_RESCORE_HIST_BINS 4096
CSA2_API size_t csa2_reindex_layers_workspace_bytes(int32_t batch, int32_t n_layers, int32_t pool_blocks);
CSA2_API csa2_status csa2_reindex_layers(const csa2_cache* cache, int32_t n_layers, const int32_t* pool,
                                         int32_t pool_blocks, const float* const* q, const float* const* w,
                                         int32_t k, int32_t* const* topk, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * csa2_sparse_attn -- sparse MQA attention over the gathered Top-k rows:
 *   o_h = sum_i softmax_i(scale * q_h . v_i) v_i,  K = V = dequantised row,
 * skipping -1 entries; a query with no valid entry gets o = 0.
 *   n_queries  queries in this call
 *   q_req      int32 [n_queries] request of each query, or NULL (query i ->
 *              request i; then n_queries <= batch)
 *   topk       int32 [n_queries][k]   positions in the query's request
 *   q          bf16  [n_queries][H][512] (uint16 bit patterns)
 *   out        bf16  [n_queries][H][512] out
 * H in {16, 32, 64}; k in [1, 4096].  Dequantised rows are exact in fp16,
 * logits and softmax are fp32, P.V uses fp16 probabilities with fp32 sums.
 * A query's rows are split over 4, 2 or 1 CTAs (H = 16: always 4) by the
 * number of queries in the call (up to 6, up to 12, more), and the partial
 * results are merged in fp32: a query's output is bit-identical across calls
 * with the same number of queries, whatever the number of layers, and may
 * differ in the last bits between calls with different numbers.
 * Device errors: a Top-k entry >= ctx_len or < -1 -> CSA2_ERR_DEVICE_BOUNDS,
 * entry skipped; a q_req entry outside [0, batch) -> CSA2_ERR_DEVICE_BOUNDS
 * (request = that value, index = -1), the query's output is 0.
 */
CSA2_API csa2_status csa2_sparse_attn(const csa2_cache* cache, int32_t n_queries, const int32_t* q_req,
                             const int32_t* topk, int32_t k, const uint16_t* q, int32_t H,
                             float scale, uint16_t* out, void* stream);

/*
 * csa2_prefill_index -- causal prefill indexer: for each of n_queries queries
 * of request `req`, the Top-k visible entries by the score of
 * csa2_index_full, with no pool.  This is the indexer of the pages' encoder
 * group (1 Full + 5 Reuse layers over a sequence compressed m = 2, two tokens
 * per cached entry) [4sapi blog, section 三; Top-512 and indexer shape, section
 * 四].  Causal rule (a reading; the pages state none): entry e covers tokens
 * ratio*e .. ratio*e + ratio - 1 and is visible to the query at token p iff
 * ratio*e + ratio - 1 <= p, i.e. e < floor((p + 1) / ratio); entries at or past
 * ctx_len[req] are never visible.
 *   req        request holding the entries, 0 <= req < batch
 *   n_queries  queries in this call (>= 0; 0 does nothing)
 *   q_pos      int32 [n_queries] token position of each query (negative: sees
 *              nothing)
 *   ratio      tokens per entry, >= 1
 *   q          float [n_queries][32][128] indexer queries (FP8 rule inside)
 *   w          float [n_queries][32]      head weights
 *   k          Top-k per query, in [1, CSA2_PREFILL_MAX_K]
 *   topk       int32 [n_queries][k] out: entries ascending, -1 padded
 *   workspace  device scratch of at least csa2_prefill_workspace_bytes(
 *              n_queries) bytes, 16-byte aligned, owned by the caller; its
 *              contents on entry do not matter and are undefined after.  Two
 *              calls in flight at once must not share it.
 *   workspace_bytes  its size
 * The scores are an FP8 tensor-core GEMM (n_queries*32 x 128 by 128 x
 * entries) reduced over the heads in fp32; each query keeps a list of at most
 * CSA2_PREFILL_CANDIDATES candidates in the workspace, so the score matrix is
 * never stored.  Ties go to the lower entry, as everywhere.  Launches two
 * kernels.  Device errors: a page id outside [0, num_pages) ->
 * CSA2_ERR_DEVICE_BOUNDS (outputs undefined); a pipeline wait that runs out
 * -> CSA2_ERR_TIMEOUT (see csa2_set_wait_limit_ns).
 */
#define CSA2_PREFILL_MAX_K 1024
#define CSA2_PREFILL_CANDIDATES 4096
CSA2_API size_t csa2_prefill_workspace_bytes(int32_t n_queries);
CSA2_API csa2_status csa2_prefill_index(const csa2_cache* cache, int32_t req, int32_t n_queries,
                                        const int32_t* q_pos, int32_t ratio, const float* q, const float* w,
                                        int32_t k, int32_t* topk, void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * csa2_prefill_index_static -- csa2_prefill_index without a workspace
 * argument.  The pages have no counterpart: this entry point exists for
 * callers that cannot hand the library scratch memory.  The candidate lists
 * live in a file-scope static device array of the library sized for
 * CSA2_PREFILL_STATIC_MAX_QUERIES queries (about 8.4 MB per device); a call
 * with more queries returns CSA2_ERR_SHAPE and launches nothing.  Nothing in
 * the array needs to start at zero (every list length is written before it is
 * read).  The array's device address is looked up with cudaGetSymbolAddress
 * on the first call in each CUDA context (each device, and again in a context
 * created anew), so make that first call outside any stream capture.  Every call on a device uses the same array: two calls in
 * flight at once on one device (other streams, other host threads) race and
 * corrupt each other's results; serialise them.  Arguments, outputs and
 * device errors are those of csa2_prefill_index.
 */
#define CSA2_PREFILL_STATIC_MAX_QUERIES 256
CSA2_API csa2_status csa2_prefill_index_static(const csa2_cache* cache, int32_t req, int32_t n_queries,
                                               const int32_t* q_pos, int32_t ratio, const float* q,
                                               const float* w, int32_t k, int32_t* topk, void* stream);

/*
 * csa2_sparse_attn_layers -- csa2_sparse_attn for n_layers layers in one
 * launch, each layer over its own Top-k (a Reuse layer passes the Top-k of the
 * layer it follows, and keeps its own main query [readance summary, section
 * 4.2]).
 *   topk host array [n_layers] of device pointers, each int32 [n_queries][k]
 *        (layers may share one)
 *   q    host array [n_layers] of device pointers, each bf16 [n_queries][H][512]
 *   out  host array [n_layers] of device pointers, each bf16 [n_queries][H][512]
 *   workspace  NULL, or caller-owned device memory of at least
 *              csa2_attn_workspace_bytes(n_layers, n_queries, H) bytes,
 *              16-byte aligned, used as scratch by this call only (contents
 *              need no initialisation; no two calls in flight may share it).
 *              Each (layer, query) is split over four CTAs by Top-k entries;
 *              with a workspace they merge their partial outputs through it
 *              (L2), without one through each other's shared memory.  Both
 *              give bit-identical results; the workspace is faster when few
 *              queries are in flight (decode).
 * n_layers in [1, CSA2_ATTN_MAX_LAYERS]; everything else as csa2_sparse_attn.
 * A workspace that is misaligned or smaller than required -> CSA2_ERR_ARG /
 * CSA2_ERR_SHAPE, nothing launched.
 */
#define CSA2_ATTN_MAX_LAYERS 8
CSA2_API csa2_status csa2_sparse_attn_layers(const csa2_cache* cache, int32_t n_layers, int32_t n_queries,
                                             const int32_t* q_req, const int32_t* const* topk, int32_t k,
                                             const uint16_t* const* q, int32_t H, float scale,
                                             uint16_t* const* out, void* workspace, size_t workspace_bytes,
                                             void* stream);
/* Workspace bytes of csa2_sparse_attn_layers: n_layers * n_queries * 4 splits
 * * (H * 512 + 2 * H) floats (0 for negative arguments). */
CSA2_API size_t csa2_attn_workspace_bytes(int32_t n_layers, int32_t n_queries, int32_t H);

/*
 * Sliding-window (SWA) branch.  Every layer, Reuse layers included, keeps its
 * own local KV of the most recent tokens, in FP8 where the global KV is FP4
 * [4sapi blog, section 二 (Reuse layers keep their own SWA state) and section
 * 五 (the local SWA KV stays FP8)].  The window size and the way the window
 * is merged with the sparse attention are not on the pages; the readings:
 * the window is the last `window` tokens up to and including the query's
 * own; its rows are FP8 E4M3 with one power-of-two scale per row (the
 * indexer's rule); attention takes one softmax over the union of the Top-k
 * rows and the window rows (K = V for both).
 * Layout (one layer): swa_codes uint8 [batch][window][512], swa_exp uint8
 * [batch][window]; token t of request b lives in slot t % window.
 *
 * csa2_swa_append -- quantise n_rows SWA rows and store them in their slots.
 *   x    float [n_rows][512];  req int32 [n_rows] or NULL (row i -> request i);
 *   pos  int32 [n_rows] token positions.
 * Device errors: req outside [0, batch) or pos < 0 -> CSA2_ERR_DEVICE_BOUNDS.
 *
 * csa2_sparse_attn_swa -- csa2_sparse_attn of one layer with its window merged
 * in: query i attends over its Top-k rows and the window tokens
 * max(0, q_pos[i] - window + 1) .. q_pos[i] of its request (q_pos int32
 * [n_queries], device).  window in [1, CSA2_SWA_MAX_WINDOW].  Window rows are
 * decoded to fp16 like the Top-k rows: exact while the row's largest
 * magnitude stays below 2^15 (a larger row overflows fp16 and the query's
 * output is undefined); rows below about 2^-14 lose low bits to fp16
 * subnormals.
 */
#define CSA2_SWA_MAX_WINDOW 4096
CSA2_API csa2_status csa2_swa_append(const csa2_cache* cache, int32_t window, uint8_t* swa_codes,
                                     uint8_t* swa_exp, int32_t n_rows, const float* x, const int32_t* req,
                                     const int32_t* pos, void* stream);
CSA2_API csa2_status csa2_sparse_attn_swa(const csa2_cache* cache, int32_t n_queries, const int32_t* q_req,
                                          const int32_t* topk, int32_t k, const uint8_t* swa_codes,
                                          const uint8_t* swa_exp, int32_t window, const int32_t* q_pos,
                                          const uint16_t* q, int32_t H, float scale, uint16_t* out,
                                          void* stream);

/*
 * csa2_get_error -- synchronise `stream`, copy cache->err_word to the host
 * array out[4] (host pointer) and return out[0] as a status (CSA2_OK when no
 * device error was recorded).  Does not clear the word.
 */
CSA2_API csa2_status csa2_get_error(const csa2_cache* cache, int32_t* out, void* stream);

/*
 * csa2_set_wait_limit_ns -- process-wide bound, in nanoseconds, on every
 * pipeline wait inside the tensor-core kernels (csa2_index_full, the
 * re-scoring csa2_reindex and csa2_prefill_index); default 2e9.  A wait that runs out makes the
 * kernel record CSA2_ERR_TIMEOUT in err_word, wait (with a fixed bound) for its
 * own copies in flight, free its tensor memory and return; the call's outputs
 * are then undefined.  0 gives up on the first wait that is not already
 * satisfied (used by the tests of that path).  Not thread-safe with
 * concurrent launches.
 */
CSA2_API void csa2_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code. */
CSA2_API const char* csa2_status_string(csa2_status status);

/* Thread-local description of the last host-side failure of this thread. */
CSA2_API const char* csa2_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
