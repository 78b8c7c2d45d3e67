/*
 * libspx -- the sparse-attention layer of a hybrid long-context decoder on
 * NVIDIA B200 (sm_100a).
 *
 * One sparse-attention layer takes four steps per query token:
 *   1. IndexPool cache write: every 4 consecutive raw indexer keys are folded
 *      into one pooled key k_pool = sum_i w_i k_i with learned weights that
 *      sum to 1.  Source: [W1] section "IndexPool: 인덱서 KV 캐시를 4배 압축".
 *   2. Lightning indexer: every complete pooled block b is scored against the
 *      query, s[b] = sum_h w_h ReLU(q_h . k_pool[b]), 32 heads x 128 dims.
 *      Source: [W4] section "수렴점 2 — 4배 압축 후 2,048 토큰만 유지" (32-head
 *      indexer, top-2048) and [W3] section "GLM-5.3 Sparse Attention이 실제로
 *      바꾸는 것" (the DeepSeek sparse-attention indexer; its ReLU-weighted form
 *      is the one fixed by the workload specification, the pages give none).
 *   3. Top-k: the 512 highest-scoring blocks (= 2048 tokens) are kept; equal
 *      scores go to the lower block index.  Source: [W4] "수렴점 2".
 *   4. Sparse MLA attention: softmax attention of every head over the latent
 *      rows of the tokens of the selected blocks plus the query's partial
 *      tail block (tokens that have no pooled key yet).  With 2051 visible
 *      tokens or fewer every token is kept, i.e. the layer is exactly dense
 *      attention.  Sources: [W3] "실제로 바꾸는 것" (MLA on the selected
 *      positions only; dense below the 2048-position budget) and [W4] section
 *      "의견이 갈리는 지점 — 위치 인코딩" (NoPE: no rotary component).
 *
 * Pages cited:
 *   [W1] "GLM-5.3-Flash: 하이브리드 희소·선형 어텐션과 IndexPool·EPD로 1M 컨텍스트를
 *        오픈 소스로 서빙하는 방법"
 *   [W3] "GLM-5.3 Sparse Attention은 연산량을 줄이지만 HBM 수요는 지속된다"
 *   [W4] "GLM-5.3-Flash vs Qwen3.8-Flash-Next: 두 중국 AI 연구소가 독립적으로 같은
 *        모델 설계로 수렴한 이유"
 *
 * Conventions shared by every call
 *   - All tensor arguments are DEVICE pointers to caller-owned memory, dense
 *     row-major, with the shapes given per call.  bf16 tensors are passed as
 *     void* (IEEE bfloat16 bit patterns).  The library never allocates, frees
 *     or synchronises; scratch memory is a caller buffer sized by the
 *     matching *_workspace_size call (256-byte aligned).
 *   - Calls are asynchronous on the given stream (a cudaStream_t; NULL is the
 *     legacy default stream).  A call that returns SPX_OK has enqueued its
 *     kernels; device-side faults surface at the caller's next
 *     synchronisation.  The library holds no per-call state and is safe to
 *     call from several host threads.
 *   - Arguments are validated on the host before anything is launched: a call
 *     that returns an error has enqueued nothing.
 *   - Per-sequence lengths live on the device (int64).  `max_len` is a host
 *     upper bound on every visible length of the call; kernels clamp the
 *     device lengths to it, so a length above the bound is read as the bound
 *     and never causes an out-of-range access.
 *   - v1 supports idx_heads = 32, idx_dim = 128, pool = 4, topk_blocks = 512,
 *     latent = 512 and heads a multiple of 16 in [16, 128]; other values
 *     return SPX_ERR_UNSUPPORTED.
 */
#ifndef SPX_H_
#define SPX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPX_API __attribute__((visibility("default")))
#else
#define SPX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same handle type, declared here without CUDA headers). */
typedef struct CUstream_st* spx_stream;

typedef enum spx_status {
  SPX_OK = 0,
  SPX_ERR_INVALID_ARG = 1, /* null pointer, non-finite or negative scalar   */
  SPX_ERR_SHAPE = 2,       /* sizes, strides or capacities inconsistent     */
  SPX_ERR_UNSUPPORTED = 3, /* dims outside what v1 implements                */
  SPX_ERR_WORKSPACE = 4,   /* workspace null, misaligned or too small        */
  SPX_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed    */
  SPX_ERR_DEVICE = 6       /* a kernel reported a device-side error          */
} spx_status;

/* Layer dimensions. */
typedef struct spx_dims {
  int32_t idx_heads;   /* indexer heads (32)                         */
  int32_t idx_dim;     /* indexer key/query width (128)              */
  int32_t pool;        /* tokens per pooled block (4)                */
  int32_t topk_blocks; /* blocks kept per query (512)                */
  int32_t heads;       /* MLA query heads (multiple of 16, <= 128)   */
  int32_t latent;      /* MLA latent width (512)                     */
  float sm_scale;      /* softmax scale applied to q . c (finite, > 0) */
} spx_dims;

/* Optional CUDA events (cudaEvent_t handles, or NULL) that the fused calls
 * record on their stream immediately before and after the indexer-scoring
 * launch, so a caller can time that kernel inside a larger step. */
typedef struct spx_timing {
  void* score_begin;
  void* score_end;
} spx_timing;

/* Name of a status code ("SPX_OK", ...).  Never NULL. */
SPX_API const char* spx_status_string(spx_status s);

/* Library version string. */
SPX_API const char* spx_version(void);

/* Fills *d with the dimensions of the layer described by the pages
 * (32 x 128 indexer, pool 4, top-512 blocks, latent 512) and the given MLA
 * head count and softmax scale. */
SPX_API spx_status spx_dims_init(spx_dims* d, int32_t heads, float sm_scale);

/* Number of kernels this process has launched through the library so far
 * (all devices, all threads).  Lets a caller count launches in a region. */
SPX_API uint64_t spx_launch_count(void);

/* Reads and clears the device-side error word that kernels set when one of
 * their bounded waits gives up (a pipeline that did not make progress within
 * about two seconds).  Synchronises the given stream.  *code is 0 when no
 * kernel reported an error since the last call. */
SPX_API spx_status spx_device_error(int32_t* code, spx_stream stream);

/* Self-test of the failure path of the kernels' bounded waits.  The pages
 * describe no such call: it is library plumbing, so that a test can make a
 * device-side wait run out on purpose and check that the host learns of it
 * while the context stays usable.  It launches one CTA in which one thread
 * starts a 1 KiB bulk copy into shared memory and then waits, with a limit of
 * limit_ns nanoseconds, on an mbarrier that nothing will ever complete; a
 * second thread waits on another such barrier with a limit 1000 times longer.
 * The first wait gives up, sets the device error word (read it with
 * spx_device_error: code 1) and the CTA's abort flag, which makes the second
 * thread give up at once; the first thread then waits for its copy to land,
 * as every kernel of the library does before it exits after a timeout.
 *
 *   limit_ns  1,000 .. 1,000,000,000
 *   result    DEVICE int64 [6]: [0] first wait succeeded (0: it gave up),
 *             [1] second wait succeeded (0: it gave up), [2] the copy landed
 *             (1), [3] and [4] nanoseconds each thread waited, [5] the copied
 *             bytes are right (1)
 * Errors: SPX_ERR_INVALID_ARG for a null or misaligned result or a limit
 * outside the range.  Asynchronous on the stream, like every other call. */
SPX_API spx_status spx_selftest_wait_timeout(int64_t limit_ns, int64_t* result,
                                             spx_stream stream);

/* ---------------------------------------------------------------------------
 * Step 1 -- IndexPool cache write.  [W1] "IndexPool": k_pool = sum_i w_i k_i,
 * i = 1..4, sum_i w_i = 1, learned w.
 *
 * Appends n_new raw indexer keys per sequence.  Token p of sequence b (0-based
 * position in the sequence) belongs to block p / 4 at slot p % 4.  For every
 * block that the append completes, the pooled key
 *     pooled_k[b][blk][d] = bf16_rne( sum_{i=0..3} pool_w[i] * key(4 blk + i)[d] )
 * is written (the sum is formed in fp64, where each product of a bf16 key
 * and an fp32 weight is exact, adding the four in time order from +0, and
 * rounded once to bf16), taking the older keys of the block from `tail`.  Keys of the still-incomplete last
 * block are stored in tail[b][p % 4].  The caller advances its lengths by
 * n_new afterwards.
 *
 *   raw_k     bf16 [B, n_new, idx_dim]        keys of the appended tokens
 *   pool_w    HOST float [pool]               sum must be 1 within 1e-6
 *   tail      bf16 [B, pool-1, idx_dim]       raw keys of incomplete blocks (in/out)
 *   pooled_k  bf16 [B, cap_blk, idx_dim]      pooled-key cache (out)
 *   len_dev   DEVICE int64 [B]                tokens already appended per sequence
 *   max_len   host bound: len_dev[b] + n_new <= max_len <= pool * cap_blk
 * Errors: SPX_ERR_INVALID_ARG for null pointers or weights that do not sum
 * to 1; SPX_ERR_SHAPE for B < 1, n_new < 0 or max_len out of range.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_pool_append(const spx_dims* d, int32_t B, const void* raw_k,
                           int32_t n_new, const float* pool_w, void* tail,
                           void* pooled_k, int64_t cap_blk,
                           const int64_t* len_dev, int64_t max_len,
                           spx_stream stream);

/* ---------------------------------------------------------------------------
 * spx_pool_append_tok -- step 1 with a weight per token.  [W1] "IndexPool"
 * says the pooling weights are learned; this is the data-dependent reading of
 * that sentence: token p arrives with its own weight (for example a learned
 * gate's output normalised over its block), and the pooled key of block blk is
 *     pooled_k[b][blk][d] = bf16_rne( sum_{i=0..3} wt(4 blk + i) * key(4 blk + i)[d] )
 * formed in fp64 and rounded once, as in spx_pool_append.  The four weights
 * of a block are expected to sum to 1; they live on the device, so the call
 * does not check that.  Weights of the still-incomplete block wait in tail_w
 * beside the keys in tail.
 *
 *   raw_w     DEVICE float [B, n_new]    weights of the appended tokens
 *   tail_w    DEVICE float [B, pool-1]   weights of the tail tokens (in/out)
 * Other arguments, limits and errors as for spx_pool_append; compose with
 * spx_decode_fused (raw_k = NULL) or the separate calls for the other steps.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_pool_append_tok(const spx_dims* d, int32_t B, const void* raw_k,
                                       const float* raw_w, int32_t n_new, void* tail,
                                       float* tail_w, void* pooled_k, int64_t cap_blk,
                                       const int64_t* len_dev, int64_t max_len,
                                       spx_stream stream);

/* ---------------------------------------------------------------------------
 * Step 2 -- lightning-indexer scores of every complete block (decode: one
 * query per sequence).  [W4] "수렴점 2" (32-head lightning indexer);
 * formula as fixed by the workload specification:
 *     scores[b][blk] = sum_h w_head[b][h] * max(0, sum_d q_idx[b][h][d] * pooled_k[b][blk][d])
 * for blk < n_vis[b] / pool.  Products are exact, sums are fp32.
 *
 *   q_idx     bf16 [B, idx_heads, idx_dim]
 *   w_head    float [B, idx_heads]
 *   pooled_k  bf16 [B, cap_blk, idx_dim]
 *   n_vis     DEVICE int64 [B]   visible tokens per sequence (clamped to max_len)
 *   scores    float [B, score_stride]; entries blk >= n_vis[b]/pool untouched
 *   Requires max_len <= pool * cap_blk and score_stride >= max_len / pool.
 * Runs on the tensor cores (tcgen05) with TMA-staged key tiles.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_index_score(const spx_dims* d, int32_t B, const void* q_idx,
                           const float* w_head, const void* pooled_k,
                           int64_t cap_blk, const int64_t* n_vis,
                           int64_t max_len, float* scores, int64_t score_stride,
                           spx_stream stream);

/* ---------------------------------------------------------------------------
 * Step 3 -- top-k blocks per row.  [W4] "수렴점 2": keep the 512
 * highest-scoring blocks (2048 tokens).  Ties go to the lower block index;
 * -0 and +0 are equal; scores must be finite.  Rows with nblk <= topk_blocks
 * keep every block ([W3]: no larger pool to reduce -> dense).
 *
 *   scores    float [rows, score_stride]   only blk < n_vis[r]/pool are read
 *   n_vis     DEVICE int64 [rows]
 *   idx       int32 [rows, topk_blocks]    selected block ids, ascending,
 *                                          padded with -1 after count[r]
 *   count     int32 [rows]                 min(topk_blocks, n_vis[r]/pool)
 *   ws        workspace of spx_topk_workspace_size(d, rows, max_len) bytes
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_topk_workspace_size(const spx_dims* d, int32_t rows,
                                   int64_t max_len, size_t* bytes);
SPX_API spx_status spx_topk_blocks(const spx_dims* d, int32_t rows,
                           const float* scores, int64_t score_stride,
                           const int64_t* n_vis, int64_t max_len, int32_t* idx,
                           int32_t* count, void* ws, size_t ws_bytes,
                           spx_stream stream);

/* ---------------------------------------------------------------------------
 * spx_topk_blocks_noalloc -- the same selection as spx_topk_blocks, for
 * callers that cannot allocate or pass scratch memory (for example code that
 * runs inside a framework whose allocator owns all device memory, or a
 * serving path where cudaMalloc's device-wide synchronisation is not
 * allowed).  The pages describe no such entry point; it is an addition of
 * this library.
 *
 * The candidate lists live in one array built into the library, of
 * SPX_TOPK_NOALLOC_SCRATCH_BYTES bytes, held on every GPU that loads the
 * library until the process exits.  The call allocates nothing.  Calls whose
 * scratch need (spx_topk_workspace_size) exceeds that size return
 * SPX_ERR_WORKSPACE before launching anything.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress), so make that
 * first call before any stream capture; the address is kept for the life of
 * the process, which assumes the device is not reset (cudaDeviceReset) in
 * between.  All calls share the array: calls
 * whose kernels overlap on the GPU race and must be serialised by the caller.
 * Arguments and results are those of spx_topk_blocks.
 * ------------------------------------------------------------------------- */
#define SPX_TOPK_NOALLOC_SCRATCH_BYTES (4u << 20)
SPX_API spx_status spx_topk_blocks_noalloc(const spx_dims* d, int32_t rows,
                                           const float* scores, int64_t score_stride,
                                           const int64_t* n_vis, int64_t max_len,
                                           int32_t* idx, int32_t* count,
                                           spx_stream stream);

/* ---------------------------------------------------------------------------
 * Step 4 -- sparse MLA attention over the selected latent rows.
 * [W3] "실제로 바꾸는 것": attention runs on the selected positions only;
 * absorbed MLA with NoPE ([W4] "위치 인코딩"): the latent row c_t is both key
 * and value, shared by all heads.  For row r the attended set is
 *     S_r = { 4 idx[r][j] + i : j < count[r], i < 4 }  U  { 4 floor(n/4) .. n-1 }
 * with n = n_vis[r], and for every head h
 *     out[r][h] = sum_{t in S_r} softmax_t(sm_scale * q[r][h] . c_t) c_t,
 *     lse[r][h] = log sum_t exp(sm_scale * q[r][h] . c_t)   (natural log).
 * Block ids outside [0, n/4) are skipped.  An empty set gives out = 0 and
 * lse = -inf.
 *
 *   q         bf16 [rows, heads, latent]
 *   latent    bf16; row r reads tokens latent + r*seq_stride + t*latent,
 *             t < cap_tok (seq_stride 0: all rows share one cache).  Device
 *             memory or pinned host memory mapped into the device's address
 *             space (only the selected rows are read)
 *   idx,count as produced by spx_topk_blocks (or by an earlier layer's
 *             spx_decode_fused: one selection may serve several layers)
 *   n_vis     DEVICE int64 [rows]   (clamped to min(max_len, cap_tok))
 *   out       bf16 [rows, heads, latent]
 *   lse       float [rows, heads] or NULL
 *   ws        workspace of spx_attn_workspace_size(d, rows, max_len) bytes
 *             (zero when each row runs in one CTA; otherwise the splits of a
 *             row combine through it: their rows normalised by their own
 *             softmax sum, in bf16, and their (max, sum) in fp32)
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_attn_workspace_size(const spx_dims* d, int32_t rows,
                                   int64_t max_len, size_t* bytes);
SPX_API spx_status spx_sparse_mla_attn(const spx_dims* d, int32_t rows, const void* q,
                               const void* latent, int64_t seq_stride,
                               int64_t cap_tok, const int32_t* idx,
                               const int32_t* count, const int64_t* n_vis,
                               int64_t max_len, void* out, float* lse, void* ws,
                               size_t ws_bytes, spx_stream stream);

/* ---------------------------------------------------------------------------
 * FP8 (E4M3) latent cache.  [W1] section "양자화: W8A8와 혼합 캐시": recent,
 * important cache entries are kept in FP8.  The page gives no format or
 * scale; libspx stores a 512-wide latent row x as E4M3 codes (4 exponent
 * bits with bias 7, 3 mantissa bits, largest 448, subnormal step 2^-9) of
 * x / 2^e, rounded to nearest (ties to even), with one power-of-two scale
 * per row: e the smallest integer with max |x| <= 448 * 2^e (not below -149;
 * 0 for an all-zero row).  Half the bytes of the bf16 cache; a dequantised
 * row (code value * 2^e) is exact in bf16.
 *
 * spx_latent_quant_fp8 writes n rows: codes uint8 [n, 512] (16-byte aligned)
 * and exps int32 [n] from latent bf16 [n, 512] (all DEVICE memory); the
 * caller points it at the rows of its cache that are new.
 *
 * spx_sparse_mla_attn_fp8 is step 4 over such a cache: the same attended set
 * and result definition as spx_sparse_mla_attn, with the latent rows read as
 * their dequantised values.  codes uint8: row r reads tokens
 * codes + r*seq_stride + t*512 (seq_stride 0: a shared cache; a multiple of
 * 512), exps int32 at r*(seq_stride/512) + t.  It first gathers the attended
 * rows, dequantised, into the workspace (about 2.1 MB per row), then runs the
 * attention kernel on them; ws is spx_attn_fp8_workspace_size bytes.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_latent_quant_fp8(const void* latent, int64_t n, void* codes,
                                        int32_t* exps, spx_stream stream);
SPX_API spx_status spx_attn_fp8_workspace_size(const spx_dims* d, int32_t rows,
                                               int64_t max_len, size_t* bytes);
SPX_API spx_status spx_sparse_mla_attn_fp8(const spx_dims* d, int32_t rows, const void* q,
                                           const void* codes, const int32_t* exps,
                                           int64_t seq_stride, int64_t cap_tok,
                                           const int32_t* idx, const int32_t* count,
                                           const int64_t* n_vis, int64_t max_len, void* out,
                                           float* lse, void* ws, size_t ws_bytes,
                                           spx_stream stream);

/* ---------------------------------------------------------------------------
 * Step 4 with the latent cache in host memory and a device working set.
 * [W3] "HiSparse는 전체 이력을 GPU 밖으로 옮긴다": the full history stays in
 * host memory, recently used entries stay on the GPU, and a step fetches only
 * the selected entries that are not resident.  The result is the same, bit
 * for bit, as spx_sparse_mla_attn over the same rows in device memory.
 *
 * The working set of a row is a pool of nslots slots of one 4-token block
 * (4 KiB) each, plus one slot for the partial tail block of the step.  A
 * block selected by the step stays resident; each missing block takes the
 * next slot, in ring order from the row's hand, that the step does not use,
 * and is fetched from host memory (the tail tokens are fetched every call).
 *
 *   host_latent  bf16, pinned host memory mapped into the device's address
 *                space (row r reads tokens host_latent + r*seq_stride + t*512)
 *   pool         DEVICE bf16 [rows, nslots + 1, 4, 512]
 *   nslots       >= 512 slots per row
 *   slot_blk     DEVICE int32 [rows, nslots]       block in each slot; -1 at first
 *   blk_slot     DEVICE int32 [rows, cap_tok / 4]  slot of each block; -1 at first
 *   slot_stamp   DEVICE int32 [rows, nslots]       last step a slot was used; -1 at first
 *   hand         DEVICE int32 [rows]               next slot in ring order; 0 at first
 *   step         a value that differs from the previous call's
 *   stats        DEVICE int64 [rows, 2]            hits and fetched blocks, accumulated
 *   ws           spx_ws_workspace_size(d, rows, nslots) bytes
 * Other arguments as for spx_sparse_mla_attn.  The state buffers belong to
 * one cache: calls on it must not overlap on the GPU.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_ws_workspace_size(const spx_dims* d, int32_t rows, int32_t nslots,
                                         size_t* bytes);
SPX_API spx_status spx_sparse_mla_attn_ws(const spx_dims* d, int32_t rows, const void* q,
                                          const void* host_latent, int64_t seq_stride,
                                          int64_t cap_tok, const int32_t* idx,
                                          const int32_t* count, const int64_t* n_vis,
                                          int64_t max_len, void* pool, int32_t nslots,
                                          int32_t* slot_blk, int32_t* blk_slot,
                                          int32_t* slot_stamp, int32_t* hand, int32_t step,
                                          int64_t* stats, void* out, float* lse, void* ws,
                                          size_t ws_bytes, spx_stream stream);

/* ---------------------------------------------------------------------------
 * Fused decode step: steps 1-4 for one new token per sequence, in one call.
 * If raw_k is non-NULL the step first appends raw_k[b] (bf16 [B, 1, idx_dim])
 * at position len_dev[b], and the query sees n = len_dev[b] + 1 tokens;
 * with raw_k NULL nothing is appended and n = len_dev[b].  The result is
 * identical, bit for bit, to calling spx_pool_append, spx_index_score,
 * spx_topk_blocks and spx_sparse_mla_attn in turn.
 *
 *   latent    bf16 [B, cap_tok, latent]  (the new token's latent row must
 *             already be stored at position len_dev[b])
 *   idx_out, count_out   optional (NULL) copies of the selection, e.g. to
 *             reuse it in the next layers
 *   max_len   host bound on n for every sequence; <= pool*cap_blk, <= cap_tok;
 *             above 16,777,216 tokens the call returns SPX_ERR_UNSUPPORTED
 *   ws        workspace of spx_decode_workspace_size(d, B, max_len) bytes
 *             (holds the scores, their key histogram, the selection lists
 *             and, for spx_decode_fused_i8, the quantised indexer queries)
 *   timing    optional events around the scoring launch (may be NULL); the
 *             kernels of the call may otherwise start before their
 *             predecessor in the call has finished (they wait for its data)
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_decode_workspace_size(const spx_dims* d, int32_t B,
                                     int64_t max_len, size_t* bytes);
SPX_API spx_status spx_decode_fused(const spx_dims* d, int32_t B, const void* raw_k,
                            const float* pool_w, void* tail, void* pooled_k,
                            int64_t cap_blk, const int64_t* len_dev,
                            const void* q_idx, const float* w_head,
                            const void* q, const void* latent, int64_t cap_tok,
                            int64_t max_len, void* out, float* lse,
                            int32_t* idx_out, int32_t* count_out, void* ws,
                            size_t ws_bytes, const spx_timing* timing,
                            spx_stream stream);

/* ---------------------------------------------------------------------------
 * INT8 pooled-key cache.  [W1] section "양자화: W8A8와 혼합 캐시": the
 * indexer's far, compressed cache entries are kept in INT8.  The page gives
 * no scale convention; libspx stores each pooled block as 128 int8 codes
 * plus one power-of-two scale:
 *     e = the smallest integer with max_d |x_d| <= 127 * 2^e  (not below
 *         -149; 0 for an all-zero block),
 *     code_d = round-half-even(x_d / 2^e)  in [-127, 127],
 *     k_scale = 2^e  (fp32),
 * where x is the block's pooled value summed in fp64 (as spx_pool_append,
 * before any rounding).  The scoring calls quantise every query head
 * the same way (codes and 2^e_h) and compute
 *     scores[b][blk] = k_scale[b][blk] * sum_h (w_head[b][h] * 2^e_h) *
 *                      max(0, sum_d qcode[b][h][d] * code[b][blk][d])
 * with the integer dot products exact (tcgen05 kind::i8, s32) and the head
 * sum in fp32.  The key scan reads half the bytes of the bf16 cache.
 *
 *   pooled_k8  int8 [B, cap_blk, idx_dim]   codes (16-byte aligned base)
 *   k_scale    float [B, cap_blk]           block scales (4-byte aligned)
 * Other arguments, limits and errors as for the bf16 calls above; the
 * raw-key tail stays bf16.
 *
 * spx_index_score_i8 needs a workspace of spx_index_score_i8_workspace_size
 * bytes (the quantised queries); SPX_ERR_WORKSPACE if it is smaller, NULL
 * or not 16-byte aligned.  spx_decode_fused_i8 takes the workspace of
 * spx_decode_workspace_size and runs the same four launches as
 * spx_decode_fused (the queries are quantised by its first kernel); its
 * result equals spx_pool_append_i8, spx_index_score_i8, spx_topk_blocks and
 * spx_sparse_mla_attn called in turn.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_pool_append_i8(const spx_dims* d, int32_t B, const void* raw_k,
                              int32_t n_new, const float* pool_w, void* tail,
                              void* pooled_k8, float* k_scale, int64_t cap_blk,
                              const int64_t* len_dev, int64_t max_len,
                              spx_stream stream);
SPX_API spx_status spx_index_score_i8_workspace_size(const spx_dims* d, int32_t B,
                                             size_t* bytes);
SPX_API spx_status spx_index_score_i8(const spx_dims* d, int32_t B, const void* q_idx,
                              const float* w_head, const void* pooled_k8,
                              const float* k_scale, int64_t cap_blk,
                              const int64_t* n_vis, int64_t max_len, float* scores,
                              int64_t score_stride, void* ws, size_t ws_bytes,
                              spx_stream stream);
SPX_API spx_status spx_decode_fused_i8(const spx_dims* d, int32_t B, const void* raw_k,
                               const float* pool_w, void* tail, void* pooled_k8,
                               float* k_scale, int64_t cap_blk,
                               const int64_t* len_dev, const void* q_idx,
                               const float* w_head, const void* q,
                               const void* latent, int64_t cap_tok,
                               int64_t max_len, void* out, float* lse,
                               int32_t* idx_out, int32_t* count_out, void* ws,
                               size_t ws_bytes, const spx_timing* timing,
                               spx_stream stream);

/* ---------------------------------------------------------------------------
 * Chunked causal prefill of one sequence: T new tokens appended after pos0
 * cached tokens.  Query t (0-based in the chunk, absolute position pos0 + t)
 * sees n_t = pos0 + t + 1 tokens: it scores the floor(n_t/4) complete blocks
 * (including blocks completed inside this chunk), keeps the top 512, and
 * always keeps its own partial block.  Steps: IndexPool append of the T raw
 * keys, causal indexer scoring as one tensor-core GEMM (keys x (queries x
 * heads)), per-query top-k, sparse attention.
 *
 *   raw_k     bf16 [T, idx_dim];  q_idx bf16 [T, idx_heads, idx_dim]
 *   w_head    float [T, idx_heads];  q bf16 [T, heads, latent]
 *   tail, pooled_k   the sequence's caches, as for spx_pool_append (B = 1)
 *   pos0      HOST int64: tokens already cached; pos0 + T <= pool*cap_blk
 *   latent    bf16 [cap_tok, latent], rows 0 .. pos0+T-1 filled
 *   out       bf16 [T, heads, latent];  lse float [T, heads] or NULL
 *   ws        workspace of spx_prefill_workspace_size(d, T, pos0) bytes
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_prefill_workspace_size(const spx_dims* d, int32_t T,
                                      int64_t pos0, size_t* bytes);
SPX_API spx_status spx_prefill_chunk(const spx_dims* d, int32_t T, const void* raw_k,
                             const float* pool_w, void* tail, void* pooled_k,
                             int64_t cap_blk, int64_t pos0, const void* q_idx,
                             const float* w_head, const void* q,
                             const void* latent, int64_t cap_tok, void* out,
                             float* lse, int32_t* idx_out, int32_t* count_out,
                             void* ws, size_t ws_bytes,
                             const spx_timing* timing, spx_stream stream);

/* ---------------------------------------------------------------------------
 * Chunked prefill on the INT8 pooled-key cache ([W1] section "양자화: W8A8와
 * 혼합 캐시"; codes, scales and scores as for the INT8 calls above).  The
 * chunk's complete blocks are appended as codes and scales (as
 * spx_pool_append_i8 does), the T indexer queries are quantised per head,
 * and each query scores the codes of its floor(n_t/4) blocks on the int8
 * tensor cores; top-k and attention as in spx_prefill_chunk.
 *
 *   pooled_k8  int8 [1, cap_blk, idx_dim]  codes (16-byte aligned base)
 *   k_scale    float [1, cap_blk]          block scales (4-byte aligned)
 *   ws         workspace of spx_prefill_workspace_size(d, T, pos0) bytes
 * Other arguments, limits and errors as for spx_prefill_chunk.
 * ------------------------------------------------------------------------- */
SPX_API spx_status spx_prefill_chunk_i8(const spx_dims* d, int32_t T, const void* raw_k,
                                const float* pool_w, void* tail, void* pooled_k8,
                                float* k_scale, int64_t cap_blk, int64_t pos0,
                                const void* q_idx, const float* w_head,
                                const void* q, const void* latent,
                                int64_t cap_tok, void* out, float* lse,
                                int32_t* idx_out, int32_t* count_out, void* ws,
                                size_t ws_bytes, const spx_timing* timing,
                                spx_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SPX_H_ */
