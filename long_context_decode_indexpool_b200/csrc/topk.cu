// Top-k block selection.
//
// [W4] "GLM-5.3-Flash vs Qwen3.8-Flash-Next: 두 중국 AI 연구소가 독립적으로 같은
// 모델 설계로 수렴한 이유", section "수렴점 2 — 4배 압축 후 2,048 토큰만 유지":
// the 512 highest-scoring 4-token blocks are kept (2,048 tokens).  Equal
// scores go to the lower block index (the tie rule of the workload
// specification); a row with 512 blocks or fewer keeps all of them.
//
// Order: scores become 32-bit keys whose unsigned order is the float order
// (-0 folded onto +0).  The selection is the first K elements of the strict
// total order (key descending, block ascending), so it is unique.
//
// Level 1: a CTA takes a contiguous chunk of one row's scores (8192 by
// default), finds the K-th largest key by four 8-bit radix passes over
// shared-memory histograms (warp-aggregated atomics), then keeps every key
// above it and the lowest-index keys equal to it.  A block-wide exclusive
// scan places the survivors in index order, so every list is ascending.
// Level 2+: a CTA merges up to 32 lists of one row (concatenated in chunk
// order, hence still ascending) with the same routine.  The last level
// writes the row's block ids, ascending, padded with -1.
// The K best of a union are among the K best of each part, under the same
// strict order, so the result equals a full sort of the row.
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kThreads = 512;
constexpr int kMergeFanIn = 32;  // lists merged per CTA

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelectSmem {
  int hist[256];
  int scan[33];
  int digit;
  int above;
};

// Selects the best min(K, n_valid) of the candidates held by the block:
// thread i holds E candidates at positions i*E .. i*E+E-1 (valid if bit set).
// Calls emit(slot, out_pos) for each survivor, in position order per thread
// with out_pos increasing with position across the block.  Returns the
// number of survivors (same in every thread).
template <int E, typename Emit>
__device__ __forceinline__ int block_select(const uint32_t (&key)[E], uint32_t valid, int K,
                                            SelectSmem& sm, Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31;
  int total;
  {
    int n_all;
    int pos = block_excl_scan(__popc(valid), sm.scan, &n_all);
    if (n_all <= K) {  // uniform: keep every candidate
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((valid >> i) & 1u) emit(i, pos++);
      return n_all;
    }
  }

  uint32_t prefix = 0, pmask = 0;
  int remaining = K;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += blockDim.x) sm.hist[b] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const bool ok = ((valid >> i) & 1u) && ((key[i] & pmask) == prefix);
      const uint32_t dig = ok ? ((key[i] >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (ok && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[dig], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      // lane L owns bins 255-8L .. 248-8L (descending)
      int local[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        local[j] = sm.hist[255 - (lane * 8 + j)];
        lsum += local[j];
      }
      int incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      int cum = incl - lsum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (cum < remaining && remaining <= cum + local[j]) {
          sm.digit = 255 - (lane * 8 + j);
          sm.above = cum;
        }
        cum += local[j];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sm.digit) << shift;
    pmask |= 255u << shift;
    remaining -= sm.above;
    __syncthreads();
  }
  // prefix is the K-th largest key; `remaining` ties at it are kept.
  int ngt = 0, neq = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      ngt += key[i] > prefix;
      neq += key[i] == prefix;
    }
  }
  int eq_tot;
  const int eq_before = block_excl_scan(neq, sm.scan, &eq_tot);
  int take = remaining - eq_before;
  take = take < 0 ? 0 : (take > neq ? neq : take);
  int pos = block_excl_scan(ngt + take, sm.scan, &total);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      if (key[i] > prefix) {
        emit(i, pos++);
      } else if (key[i] == prefix && take > 0) {
        --take;
        emit(i, pos++);
      }
    }
  }
  return total;
}

__device__ __forceinline__ int64_t clamp_blocks(const int64_t* n_vis, int r, int64_t max_len) {
  int64_t n = n_vis[r];
  n = n < 0 ? 0 : (n > max_len ? max_len : n);
  return n / kPool;
}

// Level 1: chunk of raw scores -> list (or final output when final_out).
template <int E>
__global__ void __launch_bounds__(kThreads)
    k_topk_chunk(const float* __restrict__ scores, int64_t score_stride,
                 const int64_t* __restrict__ n_vis, int64_t max_len, int nchunks,
                 uint32_t* __restrict__ out_key, int32_t* __restrict__ out_idx,
                 int32_t* __restrict__ out_cnt, int32_t* __restrict__ final_idx,
                 int32_t* __restrict__ final_cnt) {
  __shared__ SelectSmem sm;
  const int r = blockIdx.y, c = blockIdx.x;
  const int64_t nblk = clamp_blocks(n_vis, r, max_len);
  const int64_t start = static_cast<int64_t>(c) * (kThreads * E);
  const int64_t my0 = start + static_cast<int64_t>(threadIdx.x) * E;
  const float* row = scores + static_cast<int64_t>(r) * score_stride;
  uint32_t key[E];
  uint32_t valid = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int64_t b = my0 + i;
    key[i] = 0;
    if (b < nblk) {
      key[i] = order_key(row[b]);
      valid |= 1u << i;
    }
  }
  const int list = r * nchunks + c;
  if (final_idx) {
    int32_t* dst = final_idx + static_cast<int64_t>(r) * kTopK;
    const int n = block_select<E>(key, valid, kTopK, sm, [&](int i, int pos) {
      dst[pos] = static_cast<int32_t>(my0 + i);
    });
    for (int j = n + threadIdx.x; j < kTopK; j += kThreads) dst[j] = -1;
    if (threadIdx.x == 0) final_cnt[r] = n;
  } else {
    uint32_t* kd = out_key + static_cast<int64_t>(list) * kTopK;
    int32_t* id = out_idx + static_cast<int64_t>(list) * kTopK;
    const int n = block_select<E>(key, valid, kTopK, sm, [&](int i, int pos) {
      kd[pos] = key[i];
      id[pos] = static_cast<int32_t>(my0 + i);
    });
    if (threadIdx.x == 0) out_cnt[list] = n;
  }
}

// Level 2+: merge up to kMergeFanIn lists of one row.
template <int E>
__global__ void __launch_bounds__(kThreads)
    k_topk_merge(const uint32_t* __restrict__ in_key, const int32_t* __restrict__ in_idx,
                 const int32_t* __restrict__ in_cnt, int in_lists, int out_lists,
                 uint32_t* __restrict__ out_key, int32_t* __restrict__ out_idx,
                 int32_t* __restrict__ out_cnt, int32_t* __restrict__ final_idx,
                 int32_t* __restrict__ final_cnt) {
  __shared__ SelectSmem sm;
  const int r = blockIdx.y, c = blockIdx.x;
  const int first_list = c * kMergeFanIn;
  const int nl = min(kMergeFanIn, in_lists - first_list);
  // positions p = l*K + j, l < nl; thread holds E consecutive positions
  uint32_t key[E];
  int32_t idx[E];
  uint32_t valid = 0;
  const int p0 = threadIdx.x * E;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int p = p0 + i;
    const int l = p / kTopK, j = p % kTopK;
    key[i] = 0;
    idx[i] = -1;
    if (l < nl) {
      const int64_t list = static_cast<int64_t>(r) * in_lists + first_list + l;
      if (j < in_cnt[list]) {
        key[i] = in_key[list * kTopK + j];
        idx[i] = in_idx[list * kTopK + j];
        valid |= 1u << i;
      }
    }
  }
  if (final_idx) {
    int32_t* dst = final_idx + static_cast<int64_t>(r) * kTopK;
    const int n = block_select<E>(key, valid, kTopK, sm, [&](int i, int pos) { dst[pos] = idx[i]; });
    for (int j = n + threadIdx.x; j < kTopK; j += kThreads) dst[j] = -1;
    if (threadIdx.x == 0) final_cnt[r] = n;
  } else {
    const int64_t list = static_cast<int64_t>(r) * out_lists + c;
    uint32_t* kd = out_key + list * kTopK;
    int32_t* id = out_idx + list * kTopK;
    const int n = block_select<E>(key, valid, kTopK, sm, [&](int i, int pos) {
      kd[pos] = key[i];
      id[pos] = idx[i];
    });
    if (threadIdx.x == 0) out_cnt[list] = n;
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <int E>
cudaError_t launch_merge_e(dim3 grid, cudaStream_t s, const uint32_t* ik, const int32_t* ii,
                           const int32_t* ic, int in_lists, int out_lists, uint32_t* ok,
                           int32_t* oi, int32_t* oc, int32_t* fi, int32_t* fc) {
  k_topk_merge<E><<<grid, kThreads, 0, s>>>(ik, ii, ic, in_lists, out_lists, ok, oi, oc, fi, fc);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

TopkPlan plan_topk(int rows, int64_t max_len) {
  TopkPlan p{};
  p.rows = rows;
  p.max_blk = max_len / kPool;
  // Level-1 chunk: 8192 scores per CTA; shorter rows use 2048 so that small
  // batches still spread over the GPU.
  p.chunk = (p.max_blk > 8 * 8192 || rows >= 64) ? 8192 : 2048;
  int64_t nch = (p.max_blk + p.chunk - 1) / p.chunk;
  if (nch < 1) nch = 1;
  p.nchunks = static_cast<int>(nch);
  p.levels = 0;
  int lists = p.nchunks;
  size_t ws = 0;
  if (lists > 1) {
    // buffer A: level-1 lists; buffer B: lists after the first merge
    ws += align256(static_cast<size_t>(rows) * lists * kTopK * 8) +
          align256(static_cast<size_t>(rows) * lists * 4);
    int next = (lists + kMergeFanIn - 1) / kMergeFanIn;
    if (next > 1)
      ws += align256(static_cast<size_t>(rows) * next * kTopK * 8) +
            align256(static_cast<size_t>(rows) * next * 4);
    while (lists > 1) {
      p.lists[p.levels++] = lists;
      lists = (lists + kMergeFanIn - 1) / kMergeFanIn;
    }
  }
  p.ws_bytes = ws;
  return p;
}

cudaError_t launch_topk(const TopkPlan& p, const float* scores, int64_t score_stride,
                        const int64_t* n_vis, int64_t max_len, int32_t* idx, int32_t* count,
                        void* ws, cudaStream_t stream) {
  if (p.rows == 0) return cudaSuccess;
  const bool single = p.nchunks == 1;
  // Buffers: A holds level-1 lists, B the first merge output; later levels
  // ping-pong between them (each level needs at most as much as the last).
  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t a_keys = single ? 0 : align256(static_cast<size_t>(p.rows) * p.nchunks * kTopK * 8);
  const size_t a_cnt = single ? 0 : align256(static_cast<size_t>(p.rows) * p.nchunks * 4);
  uint32_t* A_key = reinterpret_cast<uint32_t*>(w);
  int32_t* A_idx = reinterpret_cast<int32_t*>(w + static_cast<size_t>(p.rows) * p.nchunks * kTopK * 4);
  int32_t* A_cnt = reinterpret_cast<int32_t*>(w + a_keys);
  uint8_t* wb = w + a_keys + a_cnt;
  const int l2 = (p.nchunks + kMergeFanIn - 1) / kMergeFanIn;
  uint32_t* B_key = reinterpret_cast<uint32_t*>(wb);
  int32_t* B_idx = reinterpret_cast<int32_t*>(wb + static_cast<size_t>(p.rows) * l2 * kTopK * 4);
  int32_t* B_cnt = reinterpret_cast<int32_t*>(wb + align256(static_cast<size_t>(p.rows) * l2 * kTopK * 8));

  dim3 g1(p.nchunks, p.rows);
  if (p.chunk == 8192)
    k_topk_chunk<16><<<g1, kThreads, 0, stream>>>(scores, score_stride, n_vis, max_len, p.nchunks,
                                                  A_key, A_idx, A_cnt, single ? idx : nullptr,
                                                  single ? count : nullptr);
  else
    k_topk_chunk<4><<<g1, kThreads, 0, stream>>>(scores, score_stride, n_vis, max_len, p.nchunks,
                                                 A_key, A_idx, A_cnt, single ? idx : nullptr,
                                                 single ? count : nullptr);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || single) return e;

  const uint32_t* in_k = A_key;
  const int32_t* in_i = A_idx;
  const int32_t* in_c = A_cnt;
  bool in_is_a = true;
  for (int lv = 0; lv < p.levels; ++lv) {
    const int in_lists = p.lists[lv];
    const int out_lists = (in_lists + kMergeFanIn - 1) / kMergeFanIn;
    const bool last = out_lists == 1;
    uint32_t* ok = in_is_a ? B_key : A_key;
    int32_t* oi = in_is_a ? B_idx : A_idx;
    int32_t* oc = in_is_a ? B_cnt : A_cnt;
    // positions per CTA: min(fan-in, lists) * K -> E per thread
    const int per_cta = (in_lists < kMergeFanIn ? in_lists : kMergeFanIn) * kTopK;
    const int E = (per_cta + kThreads - 1) / kThreads;
    dim3 g(out_lists, p.rows);
    int32_t* fi = last ? idx : nullptr;
    int32_t* fc = last ? count : nullptr;
    if (E <= 2)
      e = launch_merge_e<2>(g, stream, in_k, in_i, in_c, in_lists, out_lists, ok, oi, oc, fi, fc);
    else if (E <= 4)
      e = launch_merge_e<4>(g, stream, in_k, in_i, in_c, in_lists, out_lists, ok, oi, oc, fi, fc);
    else if (E <= 8)
      e = launch_merge_e<8>(g, stream, in_k, in_i, in_c, in_lists, out_lists, ok, oi, oc, fi, fc);
    else if (E <= 16)
      e = launch_merge_e<16>(g, stream, in_k, in_i, in_c, in_lists, out_lists, ok, oi, oc, fi, fc);
    else
      e = launch_merge_e<32>(g, stream, in_k, in_i, in_c, in_lists, out_lists, ok, oi, oc, fi, fc);
    if (e != cudaSuccess) return e;
    in_k = ok;
    in_i = oi;
    in_c = oc;
    in_is_a = !in_is_a;
  }
  return cudaSuccess;
}

}  // namespace spx
