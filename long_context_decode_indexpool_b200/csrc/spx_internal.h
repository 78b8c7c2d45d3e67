// Internal interface between the C-ABI layer (spx_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "spx.h"

namespace spx {

// Host check of the layer dimensions shared by every entry point:
// SPX_ERR_INVALID_ARG for a null pointer or a non-finite / non-positive
// softmax scale, SPX_ERR_UNSUPPORTED for dimensions v1 does not implement.
spx_status check_dims(const spx_dims* d);

// Dimensions v1 implements (the layer the pages describe).
constexpr int kIdxHeads = 32;
constexpr int kIdxDim = 128;
constexpr int kPool = 4;
constexpr int kTopK = 512;
constexpr int kLatent = 512;
constexpr int kHeadGroup = 16;  // MLA heads per attention CTA
constexpr int kMaxHeads = 128;

struct PoolAppendArgs {
  int B;
  const void* raw_k;
  int n_new;
  float w[4];
  const float* raw_w;  // optional per-token weights [B, n_new]; tail_w [B, 3] then
  float* tail_w;
  void* tail;
  void* pooled_k;
  int64_t cap_blk;
  const int64_t* len_dev;  // or nullptr -> len_host
  int64_t len_host;
  int64_t max_len;
  int64_t* nvis_out;  // optional: receives len + n_new per sequence
  // optional per-sequence initialisation of the decode selection state:
  // hist[b][..] = 0, done[b] = 0 for b < B, and done[B] = 0
  uint32_t* init_hist;
  int32_t* init_done;
  // INT8 cache: pooled_k holds int8 codes [B, cap_blk, 128] and k_scale the
  // per-block scales [B, cap_blk]; with q_idx set, CTA 0 of each row also
  // quantises that row's indexer query (q8 [B, 32, 128], wq [B, 32] =
  // w_head times the head's scale) for the scoring kernel.
  bool i8;
  float* k_scale;
  const void* q_idx;
  const float* w_head;
  int8_t* q8;
  float* wq;
  bool pdl;  // may start while the previous kernel of the stream finishes
};
cudaError_t launch_pool_append(const PoolAppendArgs& a, cudaStream_t stream);
// Query quantisation alone (one CTA per row), as in launch_pool_append.
cudaError_t launch_quant_q(int B, const void* q_idx, const float* w_head, int8_t* q8, float* wq,
                           cudaStream_t stream);
cudaError_t launch_prefill_nvis(int64_t* n_vis, int T, int64_t pos0, cudaStream_t stream);

// Indexer scoring as a tcgen05 GEMM: tiles of 128 pooled keys (M) against
// query groups of nq queries x 32 heads (N = 32 nq), K = 128.
struct ScoreArgs {
  int nq;             // queries per group: 1 (decode) or 8 (prefill)
  // INT8 cache (nq == 1): q_idx holds int8 query codes, w_head the weights
  // with the head scales folded in, pooled_k int8 key codes and k_scale
  // [key_batches, cap_blk] the block scales
  bool i8;
  const float* k_scale;
  int rows;           // query rows
  int key_batches;    // batches of the pooled-key cache (decode: rows; prefill: 1)
  const void* q_idx;  // [rows, 32, 128] bf16
  const float* w_head;  // [rows, 32]
  const void* pooled_k;  // [key_batches, cap_blk, 128] bf16
  int64_t cap_blk;
  const int64_t* n_vis;  // [rows]
  // optional (decode): the lengths before the append that writes n_vis,
  // n_vis = clamp(len_spec, 0, max_len - n_add) + n_add; read before the
  // wait on the previous kernel to plan the work, then checked against n_vis
  const int64_t* len_spec;
  int n_add;
  int64_t max_len;
  float* scores;        // [rows, score_stride]
  int64_t score_stride;
  int num_sms;
  // decode (nq == 1): when set, the keys of the scores are also counted in
  // a per-row histogram of their top 11 bits (zero on entry), the input of
  // launch_select_blocks.
  uint32_t* sel_ghist;  // [rows, kSelHistBins]
  int* work_counter;    // optional, zero on entry: tiles are then shared out dynamically
  bool pdl;             // may start while the previous kernel finishes
};
constexpr int kSelHistBins = 2048;
// Grid size of the scoring kernel for the given call shape.
int score_grid(int nq, int rows, int64_t max_len, int num_sms);
cudaError_t launch_index_score(const ScoreArgs& a, cudaStream_t stream);

// Decode top-k from scores and their complete key histogram: per row, the
// histogram locates the bin of the 512th-largest key; chunks of the row keep
// their blocks at or above it (at most 512 each, index order) and the last
// chunk to finish selects the row's 512 block ids (ascending, -1 padded) and
// count.  done[] must be zero on entry and is zero again on exit.
constexpr int kSelChunk = 8192;     // scores per selection CTA
constexpr int kMaxSelChunks = 512;  // chunks per row (rows up to 16M tokens)
struct SelectBlocksArgs {
  int rows;
  const float* scores;
  int64_t score_stride;
  const int64_t* n_vis;
  int64_t max_len;
  const uint32_t* ghist;  // [rows, kSelHistBins]
  int nchunk;             // ceil(max_len / kPool / kSelChunk) <= 512
  uint32_t* list_key;     // [rows * nchunk, 512]
  int32_t* list_idx;      // [rows * nchunk, 512]
  int32_t* list_cnt;      // [rows * nchunk]
  int32_t* done;          // [rows]
  int32_t* out_idx;
  int32_t* out_cnt;
  bool pdl;
};
cudaError_t launch_select_blocks(const SelectBlocksArgs& a, cudaStream_t stream);
// Fills the rows' key histograms (ghist, zero on entry) from scores written
// without one (prefill); uses rows, scores, score_stride, n_vis, max_len,
// ghist, nchunk and pdl of the same arguments.
cudaError_t launch_key_hist(const SelectBlocksArgs& a, cudaStream_t stream);
// Prefill top-k, one CTA per row (rows of at most select_rows_fits(max_len)
// blocks): a sampled threshold and one pass over the row's scores, then the
// exact choice on the survivors; rows the sample misjudges are redone by a
// second kernel with the row staged in shared memory.  Uses rows, scores,
// score_stride, n_vis, max_len, out_idx, out_cnt, pdl, and done ([rows]
// flags between the two kernels; no initial value needed).  Same result as
// the two kernels above.
bool select_rows_fits(int64_t max_len);
cudaError_t launch_select_rows(const SelectBlocksArgs& a, int num_sms, cudaStream_t stream);

// Top-k blocks.
struct TopkPlan {
  int rows;
  int64_t max_blk;
  int chunk;      // scores per first-level CTA
  int nchunks;    // first-level lists per row
  int levels;     // merge levels after the first (0: first level is final)
  int lists[8];   // lists per row entering each merge level
  size_t ws_bytes;
};
TopkPlan plan_topk(int rows, int64_t max_len);
cudaError_t launch_topk(const TopkPlan& p, const float* scores, int64_t score_stride,
                        const int64_t* n_vis, int64_t max_len, int32_t* idx, int32_t* count,
                        void* ws, cudaStream_t stream);

// Sparse MLA attention.
struct AttnPlan {
  int rows, heads, groups;
  int nsplit;        // token-list splits per (row, head group)
  int split_tokens;  // tokens per split (multiple of 64)
  size_t ws_bytes;
};
AttnPlan plan_attn(int rows, int heads, int64_t max_len, int num_sms);
struct AttnArgs {
  const void* q;
  const void* latent;
  int64_t seq_stride;
  int64_t cap_tok;
  const int32_t* idx;    // the selected blocks [rows, 512]
  const int32_t* count;  // [rows]
  const int64_t* n_vis;
  int64_t max_len;
  float sm_scale;
  void* out;
  float* lse;
  void* ws;
  bool pdl;
};
cudaError_t launch_attn(const AttnPlan& p, const AttnArgs& a, cudaStream_t stream);

// FP8 (E4M3) latent cache (latent_fp8.cu): quantisation of n bf16 rows into
// codes [n, 512] and row exponents [n]; gather of a rows' attended tokens,
// dequantised, into a compact bf16 buffer [rows, kFp8Dense, 512] with the
// ids, counts and lengths that describe it to launch_attn.
constexpr int kFp8Dense = kTopK * kPool + kPool;  // 2052 rows per query
cudaError_t launch_latent_quant_fp8(const void* lat, int64_t n, uint8_t* codes, int32_t* exps,
                                    cudaStream_t stream);
cudaError_t launch_gather_fp8(int rows, const uint8_t* codes, const int32_t* exps,
                              int64_t seq_stride, int64_t len_cap, const int32_t* idx,
                              const int32_t* count, const int64_t* n_vis, void* dense,
                              int64_t dense_stride, int32_t* c_idx, int32_t* c_cnt,
                              int64_t* c_nvis, cudaStream_t stream);

// Device working set of a host-resident latent cache (working_set.cu): the
// per-step hit/miss pass and the fetch of the missed blocks and tail tokens
// into the slot pool [rows, nslots + 1, 4, 512].
struct WsArgs {
  int rows;
  const int32_t* idx;
  const int32_t* count;
  const int64_t* n_vis;
  int64_t len_cap;  // min(max_len, cap_tok)
  int64_t cap_blk;  // blk_slot entries per sequence
  int nslots;
  int32_t* slot_blk;
  int32_t* blk_slot;
  int32_t* slot_stamp;
  int32_t* hand;
  int32_t step;
  int64_t* stats;
  const void* host_latent;
  int64_t seq_stride;
  void* pool;
  int32_t* r_idx;   // [rows, 512] ids remapped to slots
  int32_t* r_cnt;   // [rows]
  int64_t* r_nvis;  // [rows] nslots*4 + tail
  int32_t* fill_blk;   // [rows, 512]
  int32_t* fill_slot;  // [rows, 512]
  int32_t* fill_n;     // [rows]
};
cudaError_t launch_ws_update(const WsArgs& a, cudaStream_t stream);

// Self-test of the bounded waits (one CTA; see selftest.cu).  res: device
// int64 [6].
cudaError_t launch_wait_selftest(uint64_t limit_ns, int64_t* res, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                       const void* base, const uint64_t* dims, const uint64_t* strides_bytes,
                       const uint32_t* box, CUtensorMapSwizzle swizzle);

int device_sm_count();

// Adds n to the process-wide launch counter (spx_launch_count).
void count_launches(int n);

}  // namespace spx
