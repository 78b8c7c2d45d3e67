// Internal interface between the C-ABI layer (spx_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace spx {

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
  void* tail;
  void* pooled_k;
  int64_t cap_blk;
  const int64_t* len_dev;  // or nullptr -> len_host
  int64_t len_host;
  int64_t max_len;
  int64_t* nvis_out;  // optional: receives len + n_new per sequence
  // optional per-sequence initialisation of the fused selection state:
  // hist[b][..] = 0, first[b] = last[b] = -1, idx[b][0..512) = -1, cnt[b] = 0
  uint32_t* init_hist;
  int32_t* init_first;
  int32_t* init_last;
  int32_t* init_idx;
  int32_t* init_cnt;
};
cudaError_t launch_pool_append(const PoolAppendArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_nvis(int64_t* n_vis, int T, int64_t pos0, cudaStream_t stream);

// Indexer scoring as a tcgen05 GEMM: tiles of 128 pooled keys (M) against
// query groups of nq queries x 32 heads (N = 32 nq), K = 128.
struct ScoreArgs {
  int nq;             // queries per group: 1 (decode) or 8 (prefill)
  int rows;           // query rows
  int key_batches;    // batches of the pooled-key cache (decode: rows; prefill: 1)
  const void* q_idx;  // [rows, 32, 128] bf16
  const float* w_head;  // [rows, 32]
  const void* pooled_k;  // [key_batches, cap_blk, 128] bf16
  int64_t cap_blk;
  const int64_t* n_vis;  // [rows]
  int64_t max_len;
  float* scores;        // written unless the selection is fused
  int64_t score_stride;
  int num_sms;
  // fused top-k, first stage (decode, nq == 1): set sel_ghist to enable;
  // see index_score.cu.  ghist must be zero and row_first/row_last -1 on
  // entry.  The second stage is launch_select_merge.
  uint32_t* sel_ghist;     // [rows, kSelHistBins]
  uint32_t* sel_list_key;  // [score_grid + rows, 512]
  int32_t* sel_list_idx;   // [score_grid + rows, 512]
  int32_t* sel_list_cnt;   // [score_grid + rows]
  int32_t* sel_row_first;  // [rows]
  int32_t* sel_row_last;   // [rows]
  int64_t* sel_total;      // [1]
};
constexpr int kSelHistBins = 2048;
// Grid size of the scoring kernel for the given call shape.
int score_grid(int nq, int rows, int64_t max_len, int num_sms);
cudaError_t launch_index_score(const ScoreArgs& a, cudaStream_t stream);

// Second stage of the fused decode selection: per row, the complete
// histogram gives an exact lower bound; the CTA lists are filtered and merged
// into the row's 512 block ids (ascending, -1 padded) and count.
struct SelectMergeArgs {
  int rows;
  int grid;  // grid of the scoring launch
  const uint32_t* ghist;
  const uint32_t* list_key;
  const int32_t* list_idx;
  const int32_t* list_cnt;
  const int32_t* row_first;
  const int32_t* row_last;
  const int64_t* total;
  int32_t* out_idx;
  int32_t* out_cnt;
};
cudaError_t launch_select_merge(const SelectMergeArgs& a, cudaStream_t stream);

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
  const int32_t* idx;
  const int32_t* count;
  const int64_t* n_vis;
  int64_t max_len;
  float sm_scale;
  void* out;
  float* lse;
  void* ws;
};
cudaError_t launch_attn(const AttnPlan& p, const AttnArgs& a, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                       const void* base, const uint64_t* dims, const uint64_t* strides_bytes,
                       const uint32_t* box, CUtensorMapSwizzle swizzle);

int device_sm_count();

// Adds n to the process-wide launch counter (spx_launch_count).
void count_launches(int n);

}  // namespace spx
