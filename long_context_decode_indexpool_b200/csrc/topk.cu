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
// shared-memory histograms, then keeps every key
// above it and the lowest-index keys equal to it.  A block-wide exclusive
// scan places the survivors in index order, so every list is ascending.
// Level 2+: a CTA merges up to 32 lists of one row (concatenated in chunk
// order, hence still ascending) with the same routine.  The last level
// writes the row's block ids, ascending, padded with -1.
// The K best of a union are among the K best of each part, under the same
// strict order, so the result equals a full sort of the row.
#include <atomic>

#include "select.cuh"
#include "spx_internal.h"
#include "spx_launch.cuh"

namespace spx {

namespace {

constexpr int kThreads = 512;
constexpr int kMergeFanIn = 32;  // lists merged per CTA

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
  uint32_t thr;
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
    const int n = group_select<E, kThreads, 0>(key, valid, kTopK, threadIdx.x, sm, &thr, [&](int i, int pos) {
      dst[pos] = static_cast<int32_t>(my0 + i);
    });
    for (int j = n + threadIdx.x; j < kTopK; j += kThreads) dst[j] = -1;
    if (threadIdx.x == 0) final_cnt[r] = n;
  } else {
    uint32_t* kd = out_key + static_cast<int64_t>(list) * kTopK;
    int32_t* id = out_idx + static_cast<int64_t>(list) * kTopK;
    const int n = group_select<E, kThreads, 0>(key, valid, kTopK, threadIdx.x, sm, &thr, [&](int i, int pos) {
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
  uint32_t thr;
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
    const int n = group_select<E, kThreads, 0>(key, valid, kTopK, threadIdx.x, sm, &thr, [&](int i, int pos) { dst[pos] = idx[i]; });
    for (int j = n + threadIdx.x; j < kTopK; j += kThreads) dst[j] = -1;
    if (threadIdx.x == 0) final_cnt[r] = n;
  } else {
    const int64_t list = static_cast<int64_t>(r) * out_lists + c;
    uint32_t* kd = out_key + list * kTopK;
    int32_t* id = out_idx + list * kTopK;
    const int n = group_select<E, kThreads, 0>(key, valid, kTopK, threadIdx.x, sm, &thr, [&](int i, int pos) {
      kd[pos] = key[i];
      id[pos] = idx[i];
    });
    if (threadIdx.x == 0) out_cnt[list] = n;
  }
}

// Decode selection (k_select_blocks below): keys are counted by their top 11
// bits (sign, exponent, 2 mantissa bits) in 2048 bins.
constexpr int kSelBins = kSelHistBins;
constexpr int kSelShift = 32 - 11;
constexpr int kMergeCap = kThreads * 16;  // candidates held at once (16 per thread)
constexpr int kMergePer = 4;              // list entries per thread per round (long rows)
constexpr int kSpecChunks = kThreads / 16;  // rows of at most this many chunks: one-round list load
constexpr int kSpecPer = 4;                  // entries per thread loaded before the counts are known
constexpr int kRowCap = 49152;               // k_select_rows: scores of a row staged at once (192 KiB)

// Key histogram of scores written by another kernel (prefill): grid
// (chunks of kSelChunk, rows); each CTA counts its chunk's keys in shared
// memory and adds the non-zero bins into the row's histogram (zero on entry).
__global__ void __launch_bounds__(kThreads)
    k_key_hist(const float* __restrict__ scores, int64_t score_stride,
               const int64_t* __restrict__ n_vis, int64_t max_len, uint32_t* __restrict__ ghist) {
  __shared__ uint32_t hist[kSelBins];
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x;
  pdl_trigger();
  for (int b = tid; b < kSelBins; b += kThreads) hist[b] = 0;
  pdl_wait();  // the scores come from the scoring kernel
  const int64_t nblk = clamp_blocks(n_vis, r, max_len);
  const int64_t b0 = static_cast<int64_t>(c) * kSelChunk + tid * 16;
  const float* row = scores + static_cast<int64_t>(r) * score_stride;
  float4 sv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)  // rows are padded to a multiple of 4 scores
    sv[q] = b0 + 4 * q < nblk ? __ldcg(reinterpret_cast<const float4*>(row + b0 + 4 * q))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 v = sv[i >> 2];
    const float f = (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
    if (b0 + i < nblk) atomicAdd(&hist[order_key(f) >> kSelShift], 1u);
  }
  __syncthreads();
  uint32_t* gh = ghist + static_cast<int64_t>(r) * kSelBins;
  for (int b = tid; b < kSelBins; b += kThreads) {
    const uint32_t n = hist[b];
    if (n) atomicAdd(gh + b, n);
  }
}

// Decode selection from the row's scores and its complete key histogram.
// Grid (nchunk, rows), one CTA per chunk of kSelChunk scores (16 per thread):
//   1. the histogram gives the bin of the row's 512th-largest key (every CTA
//      of the row finds the same bin);
//   2. the chunk's keys at or above that bin's lower edge are candidates; an
//      exact top-512 of them (ties: lower block, the chunk's index order)
//      becomes the chunk's list;
//   3. the last CTA of the row to finish (a counter) gathers the lists (CTA
//      order = index order) and makes the final choice.
// The union of per-chunk exact top-512 lists holds the row's top-512, so the
// result is exact.
__global__ void __launch_bounds__(kThreads)
    k_select_blocks(const float* __restrict__ scores, int64_t score_stride,
                    const int64_t* __restrict__ n_vis, int64_t max_len,
                    const uint32_t* __restrict__ ghist, int nchunk, uint32_t* __restrict__ list_key,
                    int32_t* __restrict__ list_idx, int32_t* __restrict__ list_cnt,
                    int32_t* __restrict__ done, int32_t* __restrict__ out_idx,
                    int32_t* __restrict__ out_cnt) {
  extern __shared__ uint8_t dyn[];
  uint32_t* buf_key = reinterpret_cast<uint32_t*>(dyn);
  int32_t* buf_idx = reinterpret_cast<int32_t*>(buf_key + pad32(kMergeCap));
  __shared__ SelectSmem sm;
  __shared__ MergeSmem ms;
  __shared__ int seg_off[kThreads + 1];
  __shared__ int s_bin, s_above, s_last;
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();  // scores and histogram come from the scoring kernel
  // Loads first: the histogram (thread t owns bins kSelBins-1-4t ..
  // kSelBins-4-4t) and this thread's 16 scores.
  const uint32_t* h = ghist + static_cast<int64_t>(r) * kSelBins;
  int hc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) hc[j] = static_cast<int>(__ldcg(h + kSelBins - 1 - (tid * 4 + j)));
  const int64_t nblk = clamp_blocks(n_vis, r, max_len);
  const int64_t b0 = static_cast<int64_t>(c) * kSelChunk + tid * 16;
  const float* row = scores + static_cast<int64_t>(r) * score_stride;
  float4 sv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)  // rows are padded to a multiple of 4 scores
    sv[q] = b0 + 4 * q < nblk ? __ldcg(reinterpret_cast<const float4*>(row + b0 + 4 * q))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b = tid; b < 3 * 128; b += kThreads) (&ms.rh[0][0])[b] = 0;
  if (tid < 3) {
    ms.dig[tid] = 0;
    ms.abv[tid] = 0;
  }
  if (tid == 0) {
    s_bin = -1;
    s_above = 0;
    ms.kmin = 0xFFFFFFFFu;
    ms.kmax = 0;
  }

  // 1. the cut bin from the complete histogram
  {
    int sum = hc[0] + hc[1] + hc[2] + hc[3];
    int tot;
    int cum = group_excl_scan<kThreads, 0>(sum, tid, sm.scan, &tot);
    if (tot > kTopK) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (cum < kTopK && kTopK <= cum + hc[j]) {
          s_bin = kSelBins - 1 - (tid * 4 + j);
          s_above = cum;  // keys in higher bins: all of them are selected
        }
        cum += hc[j];
      }
    }
    __syncthreads();
  }
  const int cut_bin = s_bin, above = s_above;
  const uint32_t theta = cut_bin < 0 ? 0u : static_cast<uint32_t>(cut_bin) << kSelShift;

  // 2. this chunk's list
  {
    uint32_t key[16];
    uint32_t valid = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 v = sv[i >> 2];
      const float f = (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
      key[i] = order_key(f);
      if (b0 + i < nblk && key[i] >= theta) valid |= 1u << i;
    }
    const int64_t slot = static_cast<int64_t>(r) * nchunk + c;
    uint32_t* kd = list_key + slot * kTopK;
    int32_t* id = list_idx + slot * kTopK;
    uint32_t thr;
    const int n = group_select<16, kThreads, 0>(key, valid, kTopK, tid, sm, &thr, [&](int i, int pos) {
      kd[pos] = key[i];
      id[pos] = static_cast<int32_t>(b0 + i);
    });
    if (tid == 0) list_cnt[slot] = n;
  }

  // 3. the last CTA of the row continues.  After the CTA barrier one
  // acquire-release count per CTA orders every thread's list writes before
  // it and the last CTA's reads after it (a fence in every thread instead
  // cost 0.6 us per 1M decode step).
  __syncthreads();
  if (tid == 0) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(done + r)
                 : "memory");
    s_last = old == nchunk - 1;
  }
  __syncthreads();
  if (!s_last) return;
  int32_t* dst = out_idx + static_cast<int64_t>(r) * kTopK;
  const int64_t slot0 = static_cast<int64_t>(r) * nchunk;
  if (tid == 0) done[r] = 0;  // ready for the next launch
  if (nchunk <= kSpecChunks) {  // uniform
    // One round trip for the common case: thread t reads the count of chunk
    // t / 16 and, speculatively, entries t % 16 + 16 u (u < 4) of its list
    // (a list slot always holds 512 entries, so the reads stay in bounds;
    // entries past the count are ignored).
    const int cc = tid >> 4, jj = tid & 15;
    int cnt_c = 0;
    uint32_t k4[kSpecPer];
    int32_t i4[kSpecPer];
    if (cc < nchunk) {
      cnt_c = __ldcg(list_cnt + slot0 + cc);
#pragma unroll
      for (int u = 0; u < kSpecPer; ++u) {
        const int64_t e = (slot0 + cc) * kTopK + jj + 16 * u;
        k4[u] = __ldcg(list_key + e);
        i4[u] = __ldcg(list_idx + e);
      }
    }
    if (jj == 0 && cc < nchunk) seg_off[cc] = cnt_c;
    __syncthreads();
    if (tid < 32) {
      const int x = tid < nchunk ? seg_off[tid] : 0;
      const int xi = warp_incl_scan(x);
      __syncwarp();
      if (tid < nchunk) seg_off[tid] = xi - x;
      if (tid == 31) seg_off[kThreads] = xi;  // the total
    }
    __syncthreads();
    const int mtot = seg_off[kThreads];
    if (tid == 0) seg_off[nchunk] = mtot;
    if (mtot <= kMergeCap) {  // uniform
      if (cc < nchunk) {
        const int base = seg_off[cc];
#pragma unroll
        for (int u = 0; u < kSpecPer; ++u) {
          const int j = jj + 16 * u;
          if (j < cnt_c) {
            buf_key[pad32(base + j)] = k4[u];
            buf_idx[pad32(base + j)] = i4[u];
          }
        }
        // longer lists (crowded cut bins): the rest in a second round
#pragma unroll 1
        for (int j = jj + 16 * kSpecPer; j < cnt_c; j += 16) {
          const int64_t e = (slot0 + cc) * kTopK + j;
          buf_key[pad32(base + j)] = __ldcg(list_key + e);
          buf_idx[pad32(base + j)] = __ldcg(list_idx + e);
        }
      }
      __syncthreads();
      merge_final<kThreads, 0>(buf_key, buf_idx, mtot, theta, cut_bin, above, sm, ms, dst,
                               out_cnt + r, tid);
      return;
    }
    __syncthreads();  // (seg_off[nchunk] is read below)
  } else {
    const int m = tid < nchunk ? __ldcg(list_cnt + slot0 + tid) : 0;
    int tot;
    const int off = group_excl_scan<kThreads, 0>(m, tid, sm.scan, &tot);
    if (tid < nchunk) seg_off[tid] = off;
    if (tid == 0) seg_off[nchunk] = tot;
    __syncthreads();
  }
  const int mtot = seg_off[nchunk];
  if (mtot <= kMergeCap) {  // uniform: every list entry into the buffer
#pragma unroll 1
    for (int f = tid; f < mtot; f += kThreads) {
      int lo_s = 0, hi_s = nchunk - 1;  // last segment with seg_off <= f
      while (lo_s < hi_s) {
        const int mid = (lo_s + hi_s + 1) >> 1;
        if (seg_off[mid] <= f) lo_s = mid; else hi_s = mid - 1;
      }
      const int64_t e = (slot0 + lo_s) * kTopK + (f - seg_off[lo_s]);
      buf_key[pad32(f)] = __ldcg(list_key + e);
      buf_idx[pad32(f)] = __ldcg(list_idx + e);
    }
    __syncthreads();
    merge_final<kThreads, 0>(buf_key, buf_idx, mtot, theta, cut_bin, above, sm, ms, dst,
                             out_cnt + r, tid);
    return;
  }

  // More candidates than fit at once (rows with a crowded cut bin): gather
  // in rounds, compacting to the best 512 when the buffer fills up.
  uint32_t thr_keep = theta, thr_admit = theta;
  int nbuf = 0;
  for (int base = 0; base < mtot; base += kThreads * kMergePer) {
    uint32_t k[kMergePer];
    int32_t ix[kMergePer];
    int npass = 0;
    uint32_t pass = 0;
#pragma unroll
    for (int u = 0; u < kMergePer; ++u) {
      const int f = base + tid * kMergePer + u;
      k[u] = 0;
      ix[u] = 0;
      if (f < mtot) {
        int lo_s = 0, hi_s = nchunk - 1;  // last segment with seg_off <= f
        while (lo_s < hi_s) {
          const int mid = (lo_s + hi_s + 1) >> 1;
          if (seg_off[mid] <= f) lo_s = mid; else hi_s = mid - 1;
        }
        const int64_t e = (slot0 + lo_s) * kTopK + (f - seg_off[lo_s]);
        k[u] = __ldcg(list_key + e);
        ix[u] = __ldcg(list_idx + e);
        if (k[u] >= thr_admit) {
          pass |= 1u << u;
          ++npass;
        }
      }
    }
    int ptot;
    int pos = nbuf + group_excl_scan<kThreads, 0>(npass, tid, sm.scan, &ptot);
#pragma unroll
    for (int u = 0; u < kMergePer; ++u) {
      if ((pass >> u) & 1u) {
        buf_key[pad32(pos)] = k[u];
        buf_idx[pad32(pos)] = ix[u];
        ++pos;
      }
    }
    nbuf += ptot;
    if (nbuf > kMergeCap - kThreads * kMergePer) {  // compact in place
      __syncthreads();
      uint32_t kk[16];
      int32_t ii[16];
      uint32_t valid = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = tid * 16 + i;
        kk[i] = 0;
        ii[i] = 0;
        if (q < nbuf) {
          kk[i] = buf_key[pad32(q)];
          ii[i] = buf_idx[pad32(q)];
          if (kk[i] >= thr_keep) valid |= 1u << i;
        }
      }
      __syncthreads();
      uint32_t thr;
      nbuf = group_select<16, kThreads, 0>(kk, valid, kTopK, tid, sm, &thr, [&](int i, int p) {
        buf_key[pad32(p)] = kk[i];
        buf_idx[pad32(p)] = ii[i];
      });
      if (thr != 0) {
        // a later entry equal to thr has a higher block id: it loses
        const uint32_t t1 = thr == 0xFFFFFFFFu ? thr : thr + 1;
        thr_admit = t1 > thr_admit ? t1 : thr_admit;
        thr_keep = thr > thr_keep ? thr : thr_keep;
      }
    }
    __syncthreads();
  }
  merge_final<kThreads, 0>(buf_key, buf_idx, nbuf, thr_keep, cut_bin, above, sm, ms, dst,
                           out_cnt + r, tid);
}

// Prefill top-k, fast path, one CTA per row.  The row comes into shared
// memory with bulk copies (per-thread loads of a 135 KiB row were bound by
// the misses an SM keeps in flight: 11 us a row).  2048 evenly spaced scores
// give a threshold theta, a 22-bit key prefix above which about
// 2 x 512 x 2048 / nblk of the samples lie, found by two 11-bit radix
// passes over the samples.  Each warp then keeps the keys at or above theta
// of a contiguous range and appends them, in block order, to a list of its
// own (ballots place them).  If
// at least 512 keys survive, the row's top 512 are all among them (theta is
// at most the 512th key), and the exact choice of the selection kernels
// (merge_final, ties to the lower block) finishes on the survivors in block
// order.  A row whose sample misjudges it (fewer than 512 survivors, or more
// than a warp list holds, as with thousands of tied scores) is flagged in
// need_full[r] for k_select_rows_full; every row's flag is written.
constexpr int kWarpCap = 256;                 // survivors per warp list
constexpr int kCandCap = (kThreads / 32) * kWarpCap;  // 4096
constexpr int kTargetSurvivors = 1024;        // 2 x 512 expected
constexpr int kSampPer = 4;                   // samples per thread (2048 per row)
constexpr int kFastRowCap = 36864;            // scores of a row staged by the fast path (144 KiB)

__global__ void __launch_bounds__(kThreads, 1)
    k_select_rows_fast(const float* __restrict__ scores, int64_t score_stride,
                       const int64_t* __restrict__ n_vis, int64_t max_len,
                       int32_t* __restrict__ out_idx, int32_t* __restrict__ out_cnt,
                       int32_t* __restrict__ need_full) {
  extern __shared__ __align__(16) uint8_t dyn[];
  constexpr int kWarps = kThreads / 32;
  uint32_t* wl_key = reinterpret_cast<uint32_t*>(dyn);           // [kWarps][kWarpCap]
  int32_t* wl_id = reinterpret_cast<int32_t*>(wl_key + kWarps * kWarpCap);
  uint32_t* buf_key = reinterpret_cast<uint32_t*>(wl_id + kWarps * kWarpCap);  // pad32(kCandCap)
  int32_t* buf_idx = reinterpret_cast<int32_t*>(buf_key + pad32(kCandCap));
  __shared__ int hist[kSelBins];
  __shared__ SelectSmem sm;
  __shared__ MergeSmem ms;
  __shared__ int wcnt[kWarps + 1], woff[kWarps + 1];
  __shared__ int s_b1, s_a1, s_b2, s_fail, s_abort;
  __shared__ __align__(8) uint64_t s_bar;
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int b = tid; b < kSelBins; b += kThreads) hist[b] = 0;
  if (tid == 0) {
    s_fail = 0;
    s_abort = 0;
    mbar_init(&s_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the scores come from the scoring kernel
  const int nblk = static_cast<int>(clamp_blocks(n_vis, r, max_len));
  int32_t* dst = out_idx + static_cast<int64_t>(r) * kTopK;
  const float* row = scores + static_cast<int64_t>(r) * score_stride;
  if (nblk <= kTopK) {  // uniform: every visible block
    for (int j = tid; j < kTopK; j += kThreads) dst[j] = j < nblk ? j : -1;
    if (tid == 0) {
      out_cnt[r] = nblk;
      need_full[r] = 0;
    }
    return;
  }
  // The row into shared memory with bulk copies (rows are padded to a
  // multiple of 4 scores: the copy may read <= 3 past nblk); longer rows than
  // the stage holds go to the full kernel.
  if (nblk > kFastRowCap) {  // uniform
    if (tid == 0) need_full[r] = 1;
    return;
  }
  const float* rs = reinterpret_cast<const float*>(buf_idx + pad32(kCandCap));
  {
    const uint32_t bytes = static_cast<uint32_t>((nblk + 3) & ~3) * 4u;
    if (tid == 0) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(row);
      mbar_arrive_expect_tx(&s_bar, bytes);
      for (uint32_t off = 0; off < bytes; off += 65536u) {
        const uint32_t n = bytes - off < 65536u ? bytes - off : 65536u;
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
            "[%3];" ::"r"(smem_u32(rs) + off),
            "l"(src + off), "r"(n), "r"(smem_u32(&s_bar))
            : "memory");
      }
    }
    const bool landed = mbar_wait(&s_bar, 0, &s_abort);
    if (__syncthreads_or(!landed)) {  // timed out: the error word is set
      if (tid == 0) need_full[r] = 0;
      return;
    }
  }
  // 1. theta from 2048 evenly spaced samples (every key when the row fits the
  //    buffer)
  uint32_t theta = 0;
  if (nblk > kCandCap) {  // uniform
    uint32_t sk[kSampPer];
#pragma unroll
    for (int u = 0; u < kSampPer; ++u) {
      const int i = tid + u * kThreads;
      sk[u] = order_key(rs[static_cast<int64_t>(i) * nblk / (kSampPer * kThreads)]);
      atomicAdd(&hist[sk[u] >> kSelShift], 1);
    }
    __syncthreads();
    constexpr int kS = kSampPer * kThreads;
    int m_t = static_cast<int>((static_cast<int64_t>(kS) * kTargetSurvivors + nblk - 1) / nblk);
    m_t = m_t < 1 ? 1 : (m_t > kS ? kS : m_t);
    {
      int hc[4], sum = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hc[j] = hist[kSelBins - 1 - (tid * 4 + j)];
        sum += hc[j];
      }
      int tot;
      int cum = group_excl_scan<kThreads, 0>(sum, tid, sm.scan, &tot);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (cum < m_t && m_t <= cum + hc[j]) {
          s_b1 = kSelBins - 1 - (tid * 4 + j);
          s_a1 = cum;
        }
        cum += hc[j];
      }
    }
    __syncthreads();
    const uint32_t b1 = static_cast<uint32_t>(s_b1);
    const int m2 = m_t - s_a1;
    for (int b = tid; b < kSelBins; b += kThreads) hist[b] = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kSampPer; ++u)
      if ((sk[u] >> kSelShift) == b1) atomicAdd(&hist[(sk[u] >> 10) & (kSelBins - 1)], 1);
    __syncthreads();
    {
      int hc[4], sum = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hc[j] = hist[kSelBins - 1 - (tid * 4 + j)];
        sum += hc[j];
      }
      int tot;
      int cum = group_excl_scan<kThreads, 0>(sum, tid, sm.scan, &tot);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (cum < m2 && m2 <= cum + hc[j]) s_b2 = kSelBins - 1 - (tid * 4 + j);
        cum += hc[j];
      }
    }
    __syncthreads();
    theta = (b1 << kSelShift) | (static_cast<uint32_t>(s_b2) << 10);
  }
  // 2. each warp keeps the keys >= theta of a contiguous range, in block
  //    order (a lane reads four consecutive scores of each 128; ballots of
  //    the four place them)
  {
    const int per = ((nblk + kWarps - 1) / kWarps + 127) & ~127;  // multiple of 128
    const int w0 = min(warp * per, nblk), w1 = min(w0 + per, nblk);
    uint32_t* lk = wl_key + warp * kWarpCap;
    int32_t* li = wl_id + warp * kWarpCap;
    const uint32_t lt_mask = (1u << lane) - 1u;
    // keys >= theta are the scores >= the float whose key is theta (order_key
    // is monotone; theta at or below the lowest finite key keeps every
    // score); a NaN passes here and the final choice's key bound settles it
    const float ft = theta <= 0x00800000u ? -INFINITY
                     : __uint_as_float(theta >= 0x80000000u ? (theta & 0x7FFFFFFFu) : ~theta);
    int wc = 0;
    bool over = false;
#pragma unroll 2
    for (int base = w0; base < w1; base += 128) {
      const int i = base + lane * 4;
      const float4 v4 = i < w1 ? *reinterpret_cast<const float4*>(rs + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      const float f[4] = {v4.x, v4.y, v4.z, v4.w};
      uint32_t bal[4];
      bool keep[4];
      int tot = 0, before = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        keep[j] = i + j < w1 && !(f[j] < ft);  // (a NaN is kept: its key decides below)
        bal[j] = __ballot_sync(0xffffffffu, keep[j]);
        tot += __popc(bal[j]);
        before += __popc(bal[j] & lt_mask);  // kept by lower lanes (they come first)
      }
      if (tot > 0) {  // uniform
        if (wc + tot > kWarpCap) {
          over = true;
        } else {
          int pos = wc + before;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (keep[j]) {
              lk[pos] = order_key(f[j]);
              li[pos] = i + j;
              ++pos;
            }
          }
        }
        wc += over ? 0 : tot;
      }
    }
    if (lane == 0) {
      wcnt[warp] = wc;
      if (over) s_fail = 1;
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int x = tid < kWarps ? wcnt[tid] : 0;
    const int xi = warp_incl_scan(x);
    if (tid < kWarps) woff[tid] = xi - x;
    if (tid == 31) woff[kWarps] = xi;
  }
  __syncthreads();
  const int c = woff[kWarps];
  if (s_fail || c < kTopK) {  // uniform: the full kernel selects this row
    if (tid == 0) need_full[r] = 1;
    return;
  }
  if (tid == 0) need_full[r] = 0;
  // 3. the survivors in block order, and the histogram of their keys
  for (int b = tid; b < kSelBins; b += kThreads) hist[b] = 0;
  for (int b = tid; b < 3 * 128; b += kThreads) (&ms.rh[0][0])[b] = 0;
  if (tid < 3) {
    ms.dig[tid] = 0;
    ms.abv[tid] = 0;
  }
  if (tid == 0) {
    ms.kmin = 0xFFFFFFFFu;
    ms.kmax = 0;
  }
  __syncthreads();
  {
    const uint32_t* lk = wl_key + warp * kWarpCap;
    const int32_t* li = wl_id + warp * kWarpCap;
    const int n = wcnt[warp], o = woff[warp];
    for (int e = lane; e < n; e += 32) {
      buf_key[pad32(o + e)] = lk[e];
      buf_idx[pad32(o + e)] = li[e];
      atomicAdd(&hist[lk[e] >> kSelShift], 1);
    }
  }
  __syncthreads();
  int cut_bin = -1, above = 0;
  {
    int hc[4], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      hc[j] = hist[kSelBins - 1 - (tid * 4 + j)];
      sum += hc[j];
    }
    int tot;
    int cum = group_excl_scan<kThreads, 0>(sum, tid, sm.scan, &tot);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (cum < kTopK && kTopK <= cum + hc[j]) {
        s_b1 = kSelBins - 1 - (tid * 4 + j);
        s_a1 = cum;
      }
      cum += hc[j];
    }
    __syncthreads();
    cut_bin = s_b1;
    above = s_a1;
  }
  merge_final<kThreads, 0>(buf_key, buf_idx, c, theta, cut_bin, above, sm, ms, dst, out_cnt + r,
                           tid);
}

// Prefill top-k for the rows k_select_rows_fast flagged (need_full[r] != 0;
// cleared here), persistent over the rows.  The row's scores (at most
// kRowCap) come into shared memory with bulk copies and turn into order keys
// in place; an exact radix select (an 11-bit digit, then three 7-bit digits,
// each counting the keys that share the prefix chosen so far) finds the key
// T of the 512th-best block and how many of the blocks equal to T are taken
// (the lowest).  An ordered compaction over contiguous per-thread ranges
// then writes the blocks above T and those taken at T in ascending order.
// Any distribution of scores, ties included, is handled.
__global__ void __launch_bounds__(kThreads, 1)
    k_select_rows_full(const float* __restrict__ scores, int64_t score_stride,
                       const int64_t* __restrict__ n_vis, int64_t max_len, int rows,
                       int32_t* __restrict__ out_idx, int32_t* __restrict__ out_cnt,
                       int32_t* __restrict__ need_full) {
  extern __shared__ __align__(16) uint8_t dyn[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn);
  __shared__ int hist[kSelBins];
  __shared__ int scan_s[33];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_dig, s_abv;
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the flags come from k_select_rows_fast
  uint32_t phase = 0;
#pragma unroll 1
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    if (need_full[r] == 0) continue;  // uniform
    const int nblk = static_cast<int>(clamp_blocks(n_vis, r, max_len));  // > 512, <= kRowCap
    int32_t* dst = out_idx + static_cast<int64_t>(r) * kTopK;
    for (int b = tid; b < kSelBins; b += kThreads) hist[b] = 0;
    __syncthreads();  // (also: the previous row is done with the keys)
    // rows are padded to a multiple of 4 scores: the copy may read <= 3 past nblk
    const uint32_t bytes = static_cast<uint32_t>((nblk + 3) & ~3) * 4u;
    if (tid == 0) {
      const uint8_t* src =
          reinterpret_cast<const uint8_t*>(scores + static_cast<int64_t>(r) * score_stride);
      mbar_arrive_expect_tx(&bar, bytes);
      for (uint32_t off = 0; off < bytes; off += 65536u) {
        const uint32_t n = bytes - off < 65536u ? bytes - off : 65536u;
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
            "[%3];" ::"r"(smem_u32(dyn) + off),
            "l"(src + off), "r"(n), "r"(smem_u32(&bar))
            : "memory");
      }
    }
    const bool landed = mbar_wait(&bar, phase, &s_abort);
    phase ^= 1;
    if (__syncthreads_or(!landed)) return;  // timed out: the error word is set

    // 1. keys in place, counted by their top 11 bits
#pragma unroll 4
    for (int b = tid; b < nblk; b += kThreads) {
      const uint32_t k = order_key(__uint_as_float(keys[b]));
      keys[b] = k;
      atomicAdd(&hist[k >> kSelShift], 1);
    }
    __syncthreads();
    int above = 0, cut = 0;
    {
      int hc[4], sum = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hc[j] = hist[kSelBins - 1 - (tid * 4 + j)];
        sum += hc[j];
      }
      int tot;
      int cum = group_excl_scan<kThreads, 0>(sum, tid, scan_s, &tot);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (cum < kTopK && kTopK <= cum + hc[j]) {
          s_dig = kSelBins - 1 - (tid * 4 + j);
          s_abv = cum;
        }
        cum += hc[j];
      }
      __syncthreads();
      cut = s_dig;
      above = s_abv;
    }
    // 2. three 7-bit digits of the keys in the cut bin
    uint32_t prefix = static_cast<uint32_t>(cut) << kSelShift;
    uint32_t pmask = ~((1u << kSelShift) - 1u);
    int rem = kTopK - above;
#pragma unroll 1
    for (int d = 0; d < 3; ++d) {
      const int shift = kSelShift - 7 * (d + 1);
      __syncthreads();  // s_dig of the previous digit has been read
      if (tid < 128) hist[tid] = 0;
      __syncthreads();
#pragma unroll 4
      for (int b = tid; b < nblk; b += kThreads) {
        const uint32_t k = keys[b];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 127u], 1);
      }
      __syncthreads();
      if (tid < 32) {
        int c[4], lsum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c[j] = hist[127 - (tid * 4 + j)];
          lsum += c[j];
        }
        int cum = warp_incl_scan(lsum) - lsum;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (cum < rem && rem <= cum + c[j]) {
            s_dig = 127 - (tid * 4 + j);
            s_abv = cum;
          }
          cum += c[j];
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(s_dig) << shift;
      pmask |= 127u << shift;
      rem -= s_abv;
    }
    // 3. blocks above T = prefix, then the first rem equal to it, in order
    const uint32_t T = prefix;
    const int per = (nblk + kThreads - 1) / kThreads;
    const int q0 = min(tid * per, nblk), q1 = min(q0 + per, nblk);
    int cg = 0, ce = 0;
#pragma unroll 1
    for (int q = q0; q < q1; ++q) {
      const uint32_t k = keys[q];
      cg += k > T;
      ce += k == T;
    }
    int tot;
    const int ex = group_excl_scan<kThreads, 0>((cg << 16) | ce, tid, scan_s, &tot);
    int eq_seen = ex & 0xFFFF;
    int pos = (ex >> 16) + min(rem, eq_seen);
#pragma unroll 1
    for (int q = q0; q < q1; ++q) {
      const uint32_t k = keys[q];
      if (k > T || (k == T && eq_seen++ < rem)) dst[pos++] = q;
    }
    if (tid == 0) {
      out_cnt[r] = kTopK;
      need_full[r] = 0;
    }
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

cudaError_t launch_key_hist(const SelectBlocksArgs& a, cudaStream_t stream) {
  if (a.rows == 0 || a.nchunk == 0) return cudaSuccess;
  if ((a.score_stride & 3) != 0) return cudaErrorInvalidValue;
  cudaError_t e = launch_ex(k_key_hist, dim3(a.nchunk, a.rows), dim3(kThreads), 0, stream, a.pdl,
                            1, a.scores, a.score_stride, a.n_vis, a.max_len,
                            const_cast<uint32_t*>(a.ghist));
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_select_blocks(const SelectBlocksArgs& a, cudaStream_t stream) {
  if (a.rows == 0 || a.nchunk == 0) return cudaSuccess;
  if (a.nchunk > kThreads || (a.score_stride & 3) != 0) return cudaErrorInvalidValue;
  constexpr int kSmem = pad32(kMergeCap) * 8;
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64;  // devices beyond the cache: set every call
  if (!cached || !attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(k_select_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (cached) attr_set[dev] = true;
  }
  cudaError_t e = launch_ex(k_select_blocks, dim3(a.nchunk, a.rows), dim3(kThreads), kSmem,
                            stream, a.pdl, 1, a.scores, a.score_stride, a.n_vis, a.max_len,
                            a.ghist, a.nchunk, a.list_key, a.list_idx, a.list_cnt, a.done,
                            a.out_idx, a.out_cnt);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

bool select_rows_fits(int64_t max_len) { return max_len / kPool <= kRowCap; }

cudaError_t launch_select_rows(const SelectBlocksArgs& a, int num_sms, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (!select_rows_fits(a.max_len) || (a.score_stride & 3) != 0 || !a.done)
    return cudaErrorInvalidValue;
  constexpr int kFastSmem =
      2 * (kThreads / 32) * kWarpCap * 4 + 2 * pad32(kCandCap) * 4 + kFastRowCap * 4;
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64;  // devices beyond the cache: set every call
  if (!cached || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_select_rows_fast,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kFastSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_select_rows_full, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kRowCap * 4);
    if (e != cudaSuccess) return e;
    if (cached) attr_set[dev] = true;
  }
  cudaError_t e = launch_ex(k_select_rows_fast, dim3(a.rows), dim3(kThreads), kFastSmem, stream,
                            a.pdl, 1, a.scores, a.score_stride, a.n_vis, a.max_len, a.out_idx,
                            a.out_cnt, a.done);
  count_launches(1);
  if (e != cudaSuccess) return e;
  // the rows the fast path could not settle; shared memory for the longest
  const int64_t nb = a.max_len / kPool;
  const int smem = static_cast<int>(((nb + 3) & ~int64_t(3)) * 4);
  const int grid = a.rows < num_sms ? a.rows : num_sms;
  e = launch_ex(k_select_rows_full, dim3(grid), dim3(kThreads), smem > 0 ? smem : 16, stream,
                true, 1, a.scores, a.score_stride, a.n_vis, a.max_len, a.rows, a.out_idx,
                a.out_cnt, a.done);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

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
