// Device working set of latent rows for a latent cache kept in host memory.
//
// [W3] "GLM-5.3 Sparse Attention은 연산량을 줄이지만 HBM 수요는 지속된다", section
// "HiSparse는 전체 이력을 GPU 밖으로 옮긴다": the full history lives in host
// memory, a working set of recently used entries stays on the GPU, and only
// the entries a step selects that are not resident are fetched.  The result is
// exactly the attention over the host cache: the rows are the same bf16 rows.
//
// The working set of a sequence is a pool of `nslots` slots of one 4-token
// block each (4 KiB of latent rows) in device memory, plus one more slot that
// holds the partial tail block of the step.  Maps: slot -> block (slot_blk,
// -1 empty) and block -> slot (blk_slot, -1 not resident); slot_stamp is the
// last step that used a slot.  Policy: a block selected in this step stays
// resident; a missing block takes the next slot, in ring order from the
// sequence's hand, that this step does not use (first in, first out among
// the slots not in use; a block that keeps being selected keeps its slot).
//
// k_ws_update (one CTA of 512 threads per sequence): marks the hits, picks
// one victim per miss, updates the maps and the hand, and writes for the
// attention the selected ids remapped to slots (same order, -1 kept for ids
// out of range), their count and the pool length nslots*4 + tail; the blocks
// to fetch go to a per-sequence fill list.  k_ws_fill: one warp per block to
// fetch (4 KiB read from host memory through the device's mapping of it) and
// per tail token; then the attention kernel runs on the pool.
#include "select.cuh"
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kWsThreads = 512;

__global__ void __launch_bounds__(kWsThreads)
    k_ws_update(const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                const int64_t* __restrict__ n_vis, int64_t len_cap, int64_t cap_blk, int nslots,
                int32_t* __restrict__ slot_blk, int32_t* __restrict__ blk_slot,
                int32_t* __restrict__ slot_stamp, int32_t* __restrict__ hand, int32_t step,
                int64_t* __restrict__ stats, int32_t* __restrict__ r_idx, int32_t* __restrict__ r_cnt,
                int64_t* __restrict__ r_nvis, int32_t* __restrict__ fill_blk,
                int32_t* __restrict__ fill_slot, int32_t* __restrict__ fill_n) {
  __shared__ int scan[33];
  __shared__ int s_victim[kTopK];    // victim slot of each miss, in order
  __shared__ int s_found, s_hand;
  const int r = blockIdx.x, tid = threadIdx.x;
  int64_t n = n_vis[r];
  n = n < 0 ? 0 : (n > len_cap ? len_cap : n);
  const int64_t nblk = n / kPool;
  int cnt = count[r];
  cnt = cnt < 0 ? 0 : (cnt > kTopK ? kTopK : cnt);
  if (cnt > nblk) cnt = static_cast<int>(nblk);
  int32_t* sb = slot_blk + static_cast<int64_t>(r) * nslots;
  int32_t* bs = blk_slot + static_cast<int64_t>(r) * cap_blk;
  int32_t* ss = slot_stamp + static_cast<int64_t>(r) * nslots;
  // 1. hits: the block's slot is used by this step; misses are listed
  const int j = tid;  // one list entry per thread (kWsThreads == kTopK)
  int b = j < cnt ? idx[static_cast<int64_t>(r) * kTopK + j] : -1;
  const bool valid = b >= 0 && b < nblk;
  int slot = valid ? bs[b] : -1;
  const bool hit = slot >= 0;
  if (hit) ss[slot] = step;
  const bool miss = valid && !hit;
  int nmiss;
  const int mpos = group_excl_scan<kWsThreads, 0>(miss ? 1 : 0, tid, scan, &nmiss);
  if (tid == 0) {
    s_found = 0;
    s_hand = hand[r];
  }
  __syncthreads();  // (the hits' stamps are written before the victims are chosen)
  // 2. victims: the first nmiss slots, in ring order from the hand, that this
  //    step does not use
  int h = s_hand;
  int last = -1;
#pragma unroll 1
  for (int base = 0; base < nslots && s_found < nmiss; base += kWsThreads) {
    const int k = base + tid;
    const int sl = (h + k) % nslots;
    const bool elig = k < nslots && ss[sl] != step;
    int tot;
    const int pos = group_excl_scan<kWsThreads, 0>(elig ? 1 : 0, tid, scan, &tot);
    const int found = s_found;
    if (elig && found + pos < nmiss) {
      s_victim[found + pos] = sl;
      if (found + pos == nmiss - 1) last = k;
    }
    __syncthreads();
    if (tid == 0) s_found = found + tot;
    __syncthreads();
  }
  if (last >= 0) hand[r] = (h + last + 1) % nslots;  // one thread holds the last victim
  // 3. the misses take their victims (distinct slots, distinct blocks)
  int32_t* fb = fill_blk + static_cast<int64_t>(r) * kTopK;
  int32_t* fs = fill_slot + static_cast<int64_t>(r) * kTopK;
  if (miss && mpos < s_found) {
    const int v = s_victim[mpos];
    const int old = sb[v];
    if (old >= 0 && old < cap_blk) bs[old] = -1;
    sb[v] = b;
    ss[v] = step;
    fb[mpos] = b;
    fs[mpos] = v;
    slot = v;
  }
  __syncthreads();
  if (miss) bs[b] = slot;  // after every eviction above
  // 4. the remapped selection for the attention, and the counters
  r_idx[static_cast<int64_t>(r) * kTopK + j] = j < cnt ? (valid ? slot : -1) : -1;
  if (tid == 0) {
    r_cnt[r] = cnt;
    r_nvis[r] = static_cast<int64_t>(nslots) * kPool + (n - nblk * kPool);
    fill_n[r] = min(nmiss, s_found);
    stats[2 * r] += cnt - nmiss;  // hits (ids out of range count as hits: nothing to fetch)
    stats[2 * r + 1] += nmiss;
  }
}

// Fills the fetched blocks and the tail slot: one warp per 4 KiB block or
// per 1 KiB tail token; lane l copies 16-byte pieces l, l+32, ...
__global__ void __launch_bounds__(256)
    k_ws_fill(const __nv_bfloat16* __restrict__ host_lat, int64_t seq_stride, int64_t len_cap,
              const int64_t* __restrict__ n_vis, int nslots, __nv_bfloat16* __restrict__ pool,
              const int32_t* __restrict__ fill_blk, const int32_t* __restrict__ fill_slot,
              const int32_t* __restrict__ fill_n) {
  const int r = blockIdx.y, lane = threadIdx.x & 31;
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int nf = fill_n[r];
  int64_t n = n_vis[r];
  n = n < 0 ? 0 : (n > len_cap ? len_cap : n);
  const int64_t nblk = n / kPool;
  const int tail = static_cast<int>(n - nblk * kPool);
  const __nv_bfloat16* hl = host_lat + static_cast<int64_t>(r) * seq_stride;
  __nv_bfloat16* pr = pool + static_cast<int64_t>(r) * (nslots + 1) * kPool * kLatent;
  if (w < nf) {
    const int64_t b = fill_blk[static_cast<int64_t>(r) * kTopK + w];
    const int64_t s = fill_slot[static_cast<int64_t>(r) * kTopK + w];
    const uint4* src = reinterpret_cast<const uint4*>(hl + b * kPool * kLatent);
    uint4* dst = reinterpret_cast<uint4*>(pr + s * kPool * kLatent);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i * 32 + lane] = src[i * 32 + lane];
  } else if (w < nf + tail) {
    const int64_t t = nblk * kPool + (w - nf);
    const uint4* src = reinterpret_cast<const uint4*>(hl + t * kLatent);
    uint4* dst = reinterpret_cast<uint4*>(pr + (static_cast<int64_t>(nslots) * kPool + (w - nf)) *
                                          kLatent);
#pragma unroll
    for (int i = 0; i < 2; ++i) dst[i * 32 + lane] = src[i * 32 + lane];
  }
}

}  // namespace

cudaError_t launch_ws_update(const WsArgs& a, cudaStream_t stream) {
  k_ws_update<<<a.rows, kWsThreads, 0, stream>>>(
      a.idx, a.count, a.n_vis, a.len_cap, a.cap_blk, a.nslots, a.slot_blk, a.blk_slot,
      a.slot_stamp, a.hand, a.step, a.stats, a.r_idx, a.r_cnt, a.r_nvis, a.fill_blk, a.fill_slot,
      a.fill_n);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 512 blocks + 3 tail tokens per sequence at most: 65 CTAs of 8 warps
  k_ws_fill<<<dim3((kTopK + kPool + 7) / 8, a.rows), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.host_latent), a.seq_stride, a.len_cap, a.n_vis, a.nslots,
      static_cast<__nv_bfloat16*>(a.pool), a.fill_blk, a.fill_slot, a.fill_n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
