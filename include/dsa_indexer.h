/*
 * dsa_indexer.h - C ABI of the B200 (sm_100a) DeepSeek Sparse Attention lightning indexer,
 * its top-k selection, IndexCache cross-layer index reuse and the cross-layer top-k overlap.
 *
 * What is computed (pages by title and section):
 *   "IndexShare deep-dive report" (深度解读报告) §1.1: the lightning indexer is a multi-head,
 *   ReLU-gated dot product over FP8 inputs that scores the whole prefix and keeps the top-k
 *   keys (k = 2048 in the abstract). It is read here as
 *       I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]),
 *       q[t,j] = q_scale[t] * e4m3(q8[t][j][:]),   k[s] = k_scale[s] * e4m3(k8[s][:]),
 *   over the causal prefix s <= t ("ADIndex以分组蒸馏重构长上下文稀疏注意力索引", section
 *   索引器为何成为长上下文瓶颈). Each query keeps the top-k keys, ties going to the lower key
 *   index; rows are written by (score descending, index ascending), and a row with fewer
 *   than topk visible keys is padded with index -1 (score -inf).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers (or managed memory) of the current CUDA
 *     device, row-major and densely packed as stated. The caller owns every buffer,
 *     including the workspace; the library allocates no device memory and keeps no state
 *     between calls. Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; outputs are valid once the stream reaches them.
 *   - FP8 inputs are OCP E4M3 byte codes; the NaN codes 0x7F / 0xFF are not valid input.
 *     Scales must be finite and > 0.
 *   - Arguments are validated on the host before anything is enqueued; a rejected call
 *     returns DSA_ERR_INVALID (malformed) or DSA_ERR_UNSUPPORTED (valid but not built)
 *     and enqueues nothing. A failed CUDA runtime call returns DSA_ERR_CUDA.
 *   - Device-side checks (block-table entries, sequence lengths, index ranges) and
 *     bounded pipeline waits record the FIRST failure in the workspace header; read it
 *     with dsa_read_device_status. Kernels never trap and never wait without a bound
 *     (env DSA_WAIT_BUDGET_NS, default 2e9 ns per wait).
 *   - A workspace's first DSA_WS_HEADER_BYTES must be zeroed once before first use
 *     (dsa_workspace_init). Calls that share a workspace must not overlap on the GPU.
 *   - Supported shapes, per entry point: prefill takes (H, d) in {(8, 64), (64, 128)}; decode
 *     (and its allocation-free variant) takes only (H, d) = (64, 128) with block_size = 64.
 *     Every entry point takes 1 <= topk <= 2048. Other shapes return DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_INDEXER_H
#define DSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_API __attribute__((visibility("default")))

#define DSA_ABI_VERSION 1
#define DSA_WS_HEADER_BYTES 256
#define DSA_MAX_TOPK 2048
#define DSA_MAX_LAYERS 64

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID = 1,     /* malformed argument (null, size, alignment, pattern) */
  DSA_ERR_UNSUPPORTED = 2, /* well-formed but not supported by this build (H, d, topk) */
  DSA_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed */
  DSA_ERR_TIMEOUT = 4,     /* device-side: a pipeline wait exceeded its bound */
  DSA_ERR_DEVICE = 5       /* device-side: an input check failed (see detail) */
} dsa_status;

enum { DSA_MODE_PREFILL = 0, DSA_MODE_DECODE = 1 };

/* Library ABI version (DSA_ABI_VERSION). */
DSA_API int32_t dsa_abi_version(void);

/* Static description of a status code; never NULL. */
DSA_API const char* dsa_status_string(int32_t status);

/* Zeroes the workspace header (the first DSA_WS_HEADER_BYTES) on `stream`.
 * workspace_bytes must be >= DSA_WS_HEADER_BYTES. */
DSA_API dsa_status dsa_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then returns in *status_out / *detail_out the first device-side
 * failure recorded in the workspace header since it was last cleared (DSA_OK / 0 if
 * none) and clears it. Either output pointer may be NULL. */
DSA_API dsa_status dsa_read_device_status(void* workspace, void* stream, int32_t* status_out,
                                          int32_t* detail_out);

/* ---------------------------------------------------------------------------------------
 * Prefill indexer ("IndexShare deep-dive report" §1.1; "Index Share逻辑详解" §2: every
 * layer scores the whole length and takes the top-k).
 *
 * Queries i = 0..Lq-1 sit at positions t = q_pos0 + i and see keys s = 0..t (a chunk of a
 * longer prefill is one call with q_pos0 > 0 against all keys before its end; the result
 * equals the unchunked one).
 *   q        [Lq][H][d]   u8 E4M3, 16-byte aligned      q_scale [Lq]  f32
 *   w        [Lq][H]      f32 head weights
 *   k        [Lk][d]      u8 E4M3, 16-byte aligned      k_scale [Lk]  f32
 *   out_idx  [Lq][topk]   i32, written                   out_score [Lq][topk] f32 or NULL
 * Requires q_pos0 >= 0, Lq >= 1, q_pos0 + Lq <= Lk.
 * workspace: >= dsa_prefill_workspace_bytes(Lq, H, d, topk) bytes, 256-byte aligned.
 * -------------------------------------------------------------------------------------*/
DSA_API size_t dsa_prefill_workspace_bytes(int32_t Lq, int32_t H, int32_t d, int32_t topk);

DSA_API dsa_status dsa_indexer_prefill(const uint8_t* q, const float* q_scale, const float* w,
                                       const uint8_t* k, const float* k_scale, int32_t Lk,
                                       int32_t q_pos0, int32_t Lq, int32_t H, int32_t d,
                                       int32_t topk, int32_t* out_idx, float* out_score,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Decode indexer ("Index Share逻辑详解" §2: the decode step runs the indexer in every layer
 * at every step; "多层索引器" abstract: the indexer scans the whole cache and keeps
 * k = 2048 tokens).
 *
 * Request b has one new query at position seq_lens[b]-1 whose own key is already cached;
 * it scores all seq_lens[b] cached keys. Logical key s of request b lives in physical
 * block block_table[b][s / block_size], slot s % block_size.
 *   q             [B][H][d]                      u8 E4M3      q_scale [B] f32, w [B][H] f32
 *   k_cache       [n_blocks][block_size][d]      u8 E4M3, 16-byte aligned
 *   k_scale_cache [n_blocks][block_size]         f32
 *   block_table   [B][max_blocks]                i32 (entries past a request's last block
 *                                                 are not read)
 *   seq_lens      [B]                            i32, 1 <= seq_lens[b] <= max_blocks*block_size
 *   out_idx       [B][topk] i32 logical positions;  out_score [B][topk] f32 or NULL
 * Decode is built for H = 64, d = 128 and block_size = 64 only, and for B at most
 * DSA_DECODE_MAX_REQUESTS; any other shape returns DSA_ERR_UNSUPPORTED with nothing
 * enqueued. A block-table entry outside [0, n_blocks) or a bad length is recorded as
 * DSA_ERR_DEVICE (the request's keys are then read from block 0 / clamped).
 * workspace: >= dsa_decode_workspace_bytes(B, max_blocks*block_size, H, d, topk) bytes.
 * -------------------------------------------------------------------------------------*/
#define DSA_DECODE_MAX_REQUESTS 65535

DSA_API size_t dsa_decode_workspace_bytes(int32_t B, int32_t max_len, int32_t H, int32_t d,
                                          int32_t topk);

DSA_API dsa_status dsa_indexer_decode(const uint8_t* q, const float* q_scale, const float* w,
                                      const uint8_t* k_cache, const float* k_scale_cache,
                                      int32_t n_blocks, int32_t block_size,
                                      const int32_t* block_table, int32_t max_blocks,
                                      const int32_t* seq_lens, int32_t B, int32_t H, int32_t d,
                                      int32_t topk, int32_t* out_idx, float* out_score,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Decode indexer that allocates nothing (the pages have no counterpart to this entry point).
 *
 * For callers that cannot allocate device memory when they run the indexer: e.g. a plugin
 * inside a host application whose allocator owns all device memory, or a decode loop that must
 * not call cudaMalloc / cudaFree at step time (cudaFree synchronises the whole device). It
 * computes exactly what dsa_indexer_decode computes, with the same arguments except that,
 * instead of a workspace, its scratch is a fixed array inside the library:
 * DSA_WS_HEADER_BYTES + DSA_NOALLOC_MAX_SCORES * 4 + DSA_NOALLOC_MAX_REQUESTS * (8192 + 16 +
 * 65536) bytes (34 MiB + 4352 B), held on every GPU that loads the library until the process
 * exits.
 *   - B must not exceed DSA_NOALLOC_MAX_REQUESTS and B * max_blocks * block_size must not exceed
 *     DSA_NOALLOC_MAX_SCORES; a larger call returns DSA_ERR_UNSUPPORTED and enqueues nothing.
 *     Other errors are those of dsa_indexer_decode.
 *   - Shapes: as dsa_indexer_decode, i.e. H = 64, d = 128, block_size = 64.
 *   - device_status_out: optional DEVICE int32[2] that receives the call's device-side status
 *     and detail (as dsa_read_device_status reports them). The fixed scratch's status header
 *     is cleared on the stream at the start of every call, so each call reports only its own
 *     device-side errors; pass NULL only if those errors are not wanted.
 *   - The first call on each device looks up the scratch's device address (cudaGetSymbolAddress)
 *     with that device current and caches it; make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array and may leave data in it: calls whose
 *     work overlaps on the GPU (other streams, other host threads) race and must be serialised
 *     by the caller.
 * -------------------------------------------------------------------------------------*/
#define DSA_NOALLOC_MAX_SCORES 4194304
#define DSA_NOALLOC_MAX_REQUESTS 256

DSA_API dsa_status dsa_indexer_decode_noalloc(const uint8_t* q, const float* q_scale, const float* w,
                                              const uint8_t* k_cache, const float* k_scale_cache,
                                              int32_t n_blocks, int32_t block_size,
                                              const int32_t* block_table, int32_t max_blocks,
                                              const int32_t* seq_lens, int32_t B, int32_t H,
                                              int32_t d, int32_t topk, int32_t* out_idx,
                                              float* out_score, int32_t* device_status_out,
                                              void* stream);

/* ---------------------------------------------------------------------------------------
 * IndexCache layer driver ("IndexShare deep-dive report" §2.1: Full layers run the indexer
 * and overwrite the cached indices, Shared layers take T <- T_f(l) with
 * f(l) = max{j < l : c_j = F}, the first layer is always F, and the cache costs no extra
 * memory; "Index Share逻辑详解" §4.2: one branch per layer).
 *
 * pattern: n_layers characters over {F, S}, first 'F' (no whitespace).
 * shape:   the per-layer call shape. mode = DSA_MODE_PREFILL uses H, d, topk, Lk, q_pos0,
 *          Lq; mode = DSA_MODE_DECODE uses H, d, topk, n_blocks, block_size, block_table,
 *          max_blocks, seq_lens, B.
 * layers:  [n_layers] per-layer inputs; entries of S layers are not read. For decode,
 *          k / k_scale are that layer's paged k_cache / k_scale_cache.
 * f_bufs:  output index buffers, each [rows][topk] i32 (rows = Lq or B). n_fbufs = 1: every
 *          F layer overwrites f_bufs[0] (the pages' single cache). n_fbufs = number of F
 *          layers: the m-th F layer writes f_bufs[m] and all layer outputs stay readable.
 * out_layer_idx: [n_layers] host array, filled with the buffer holding each layer's indices
 *          (an S layer gets its source F layer's buffer: no copy, no launch).
 * after_layer: optional host callback invoked after layer l's work has been ENQUEUED (not
 *          completed) with the buffer holding layer l's indices; work the callback enqueues
 *          on the same stream runs before the next F layer overwrites a shared buffer.
 * workspace: >= dsa_indexcache_workspace_bytes(shape) bytes (one layer's worth, reused).
 * -------------------------------------------------------------------------------------*/
typedef struct dsa_layer_inputs {
  const uint8_t* q;
  const float* q_scale;
  const float* w;
  const uint8_t* k;       /* prefill keys [Lk][d] or decode k_cache [n_blocks][block_size][d] */
  const float* k_scale;   /* prefill [Lk] or decode k_scale_cache [n_blocks][block_size]     */
  float* out_score;       /* optional [rows][topk] scores of this layer, or NULL             */
} dsa_layer_inputs;

typedef struct dsa_indexer_shape {
  int32_t mode;
  int32_t H, d, topk;
  int32_t Lk, q_pos0, Lq;                 /* prefill */
  int32_t n_blocks, block_size;           /* decode  */
  const int32_t* block_table;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t B;
} dsa_indexer_shape;

typedef void (*dsa_after_layer_fn)(int32_t layer, const int32_t* layer_idx, void* user);

DSA_API size_t dsa_indexcache_workspace_bytes(const dsa_indexer_shape* shape);

DSA_API dsa_status indexcache_run(const char* pattern, int32_t n_layers,
                                  const dsa_indexer_shape* shape, const dsa_layer_inputs* layers,
                                  int32_t* const* f_bufs, int32_t n_fbufs,
                                  const int32_t** out_layer_idx, dsa_after_layer_fn after_layer,
                                  void* user, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* ---------------------------------------------------------------------------------------
 * Multi-layer-indexer (lagged) variant of indexcache_run ("多层索引器：DeepSeek 稀疏注意力中的重叠
 * 选择与注意力", abstract: adjacent layers select nearly the same tokens, so a layer can attend the
 * selection of the previous indexer layer instead of its own; that removes the dependency and
 * lets every indexer run concurrently with the attention of its layer, and it composes with
 * IndexCache).
 *
 * Arguments as indexcache_run, plus indexer_stream (a second cudaStream_t). Every Full layer's
 * indexer runs on indexer_stream; `consume` is called for every layer in order and enqueues that
 * layer's consumer (attention) on `stream`. The buffer layer l's consumer gets is that of the
 * last Full layer BEFORE l: for a Full layer the previous indexer layer's selection (its own
 * indexer runs meanwhile), for a Shared layer its source Full layer's (the IndexCache rule).
 * Layer 0 has no earlier indexer layer and gets its own selection. Before each call of `consume`,
 * `stream` is made to wait (cudaStreamWaitEvent) for the indexer work that wrote the buffer it
 * passes; before each Full layer's indexer, indexer_stream waits for all work enqueued on
 * `stream` so far (the layer's inputs, and every consumer that may still read the buffer about
 * to be rewritten). When the call returns, `stream` also waits for the last indexer.
 * 2 <= n_fbufs <= max(2, number of Full layers) (1 is allowed when there is one Full layer):
 * Full layer m writes f_bufs[m % n_fbufs]; n_fbufs = number of Full layers keeps every layer's
 * indices. stream and indexer_stream must differ. `consume` may be NULL (then only out_layer_idx is filled).
 * The workspace is used on indexer_stream only. Errors as indexcache_run.
 * -------------------------------------------------------------------------------------*/
DSA_API dsa_status indexcache_run_lagged(const char* pattern, int32_t n_layers,
                                         const dsa_indexer_shape* shape,
                                         const dsa_layer_inputs* layers, int32_t* const* f_bufs,
                                         int32_t n_fbufs, const int32_t** out_layer_idx,
                                         dsa_after_layer_fn consume, void* user, void* workspace,
                                         size_t workspace_bytes, void* stream, void* indexer_stream);

/* ---------------------------------------------------------------------------------------
 * Sparse attention over the selected latents ("Index Share逻辑详解" §2: after the indexer's
 * top-k selection, the core MLA attention runs on only those k latents). A consumer of the
 * decode index buffer: one query per request with Hq = 128 heads over a dqk = 576-wide bf16
 * latent cache whose first dv = 512 entries are the values. For request b and head h,
 *     out[b][h] = sum_s softmax_s(scale * q[b][h] . K[s]) V[s],  K[s] = latent[row(b, s)],
 *     V[s] = K[s][0:512],  row(b, s) = block_table[b][s / block_size] * block_size + s % block_size,
 * over the logical positions s = idx[b][0..topk) (entries -1 select nothing; a request that
 * selects nothing gets zeros).
 *   q           [B][128][576]                    bf16 (as uint16), 16-byte aligned
 *   latent      [n_blocks * block_size][576]     bf16, 16-byte aligned (the paged cache's rows)
 *   block_table [B][max_blocks] i32, seq_lens [B] i32 (positions >= seq_lens[b] are invalid)
 *   idx         [B][topk] i32 logical positions, as dsa_indexer_decode writes them
 *   out         [B][128][512] f32, 16-byte aligned
 * topk must be a multiple of 256, at most 2048; scale > 0. Products run on the tensor cores in
 * bf16 with fp32 accumulation; the softmax weights are rounded to bf16 before the value product
 * (their sum is taken over the rounded weights). A position outside [0, seq_lens[b]) other than
 * -1, a bad length or a block-table entry outside [0, n_blocks) is recorded as DSA_ERR_DEVICE
 * and the key is left out.
 * workspace: >= dsa_sparse_attention_workspace_bytes(B, topk) bytes, 256-byte aligned.
 * -------------------------------------------------------------------------------------*/
DSA_API size_t dsa_sparse_attention_workspace_bytes(int32_t B, int32_t topk);

DSA_API dsa_status dsa_sparse_attention_decode(const uint16_t* q, const uint16_t* latent,
                                               int32_t n_blocks, int32_t block_size,
                                               const int32_t* block_table, int32_t max_blocks,
                                               const int32_t* seq_lens, const int32_t* idx,
                                               int32_t B, int32_t Hq, int32_t dqk, int32_t dv,
                                               int32_t topk, float scale, float* out,
                                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Cross-layer top-k overlap ("IndexShare deep-dive report" §1.2: the overlap of layers i
 * and j is |T(i) ∩ T(j)| / k; adjacent layers overlap 70-100% in blocks).
 *
 * layer_idx: HOST array of n_layers (<= DSA_MAX_LAYERS) device pointers, each [rows][topk]
 *          i32 index rows as the indexer writes them (distinct entries in [0, n_keys), -1
 *          padding). Pointers may repeat (aliased S layers).
 * out_counts [n_layers][n_layers] u64: C[i][j] = sum over rows of |T_i(row) ∩ T_j(row)|.
 * out_valid  [1] u64: V = number of non-negative entries of layer 0 (= C[0][0], since a row lists a
 *          key at most once).
 * out_overlap [n_layers][n_layers] f64 = C / V, or NULL.
 * An entry outside [-1, n_keys) is skipped and recorded as DSA_ERR_DEVICE.
 * rows >= 0; with rows = 0 the counts, V and the overlap are 0 and the layer pointers are not
 * read (they may be NULL, as an empty tensor's are).
 * workspace: >= DSA_WS_HEADER_BYTES bytes. n_keys <= 1,500,000 (larger: DSA_ERR_UNSUPPORTED).
 * -------------------------------------------------------------------------------------*/
DSA_API dsa_status topk_overlap(const int32_t* const* layer_idx, int32_t n_layers, int32_t rows,
                                int32_t topk, int32_t n_keys, uint64_t* out_counts,
                                uint64_t* out_valid, double* out_overlap, void* workspace,
                                size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Exact merge of top-k lists selected over disjoint key ranges of the same rows. The pages
 * serve one model replica per GPU ("IndexShare deep-dive report" §4.2, Table 1: SGLang with
 * dp = 8 on one node); they have no counterpart to splitting one request's keys over GPUs.
 * That split is exact because the top-k of a row ("IndexShare deep-dive report" §1.1) is
 * contained in the union of the top-k lists of any partition of its keys: each GPU selects
 * the top-k of its own range (dsa_indexer_decode on its share of the block table), the lists
 * are gathered, and this call takes the top-k of their union.
 *   scores     [n_lists][rows][topk] f32   each list row as the indexer writes it: score
 *   idx        [n_lists][rows][topk] i32   descending, ties by ascending index, -1 / -inf padding
 *   idx_offset [n_lists][rows] i32 or NULL: added to every valid index of that list row (the
 *              first key position of the range the list was selected from)
 *   out_idx    [rows][topk] i32, written; out_score [rows][topk] f32 or NULL
 * The result is ordered and padded like the indexer's rows, ties going to the lower index. The
 * lists of one row must hold distinct key positions (disjoint ranges); duplicates are not
 * removed. 1 <= n_lists <= DSA_MAX_LAYERS, 1 <= topk <= 2048, rows >= 1; outputs must not
 * alias inputs.
 * -------------------------------------------------------------------------------------*/
DSA_API dsa_status dsa_topk_merge(const float* scores, const int32_t* idx, const int32_t* idx_offset,
                                  int32_t n_lists, int32_t rows, int32_t topk, int32_t* out_idx,
                                  float* out_score, void* stream);

/* ---------------------------------------------------------------------------------------
 * Layer-pattern diagnostics from an overlap matrix (host functions; no device work).
 * "IndexShare deep-dive report" §1.2 / §3.1: the cross-layer overlap of a DSA model forms blocks
 * of layers whose selections agree, separated by a few transition layers, which uniform F/S
 * interleaving ignores. §5.2 of the same report: a similarity proxy does not predict model
 * quality, so these describe an overlap matrix; they do not choose a serving pattern.
 *
 * overlap: HOST [n_layers][n_layers] f64 (as topk_overlap writes out_overlap, copied to the host),
 * 1 <= n_layers <= DSA_MAX_LAYERS.
 *
 * dsa_overlap_blocks: block_of_layer[l] (HOST [n_layers] i32) = index of the block of layer l,
 *   where a new block starts at every layer l > 0 with overlap[l][l-1] < threshold. Returns the
 *   number of blocks, or -1 for invalid arguments.
 * dsa_pattern_from_overlap: writes to pattern_out (HOST, n_layers + 1 chars, NUL-terminated) the
 *   F/S pattern with exactly n_full Full layers, layer 0 Full, that maximises the overlap kept,
 *   sum_l overlap[l][f(l)] with f(l) the last Full layer at or before l (overlap[l][l] taken as
 *   1); *retained_out (nullable) = that maximum / n_layers. Exact (dynamic programming); ties go
 *   to the pattern the recursion meets first. DSA_ERR_INVALID for bad arguments.
 * -------------------------------------------------------------------------------------*/
DSA_API int32_t dsa_overlap_blocks(const double* overlap, int32_t n_layers, double threshold,
                                   int32_t* block_of_layer);

DSA_API dsa_status dsa_pattern_from_overlap(const double* overlap, int32_t n_layers, int32_t n_full,
                                            char* pattern_out, double* retained_out);

/* ---------------------------------------------------------------------------------------
 * Failure-detection self-test (no counterpart on the pages): launches one CTA that waits,
 * with the given bound, on an mbarrier that nothing completes, so that the bounded-wait
 * path records DSA_ERR_TIMEOUT in the workspace header and the kernel returns normally.
 * -------------------------------------------------------------------------------------*/
DSA_API dsa_status dsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                             uint64_t budget_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEXER_H */
