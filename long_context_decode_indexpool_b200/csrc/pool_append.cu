// IndexPool cache write.
//
// [W1] "GLM-5.3-Flash: 하이브리드 희소·선형 어텐션과 IndexPool·EPD로 1M 컨텍스트를
// 오픈 소스로 서빙하는 방법", section "IndexPool: 인덱서 KV 캐시를 4배 압축":
// the indexer keys of 4 consecutive positions are merged by a learned
// weighted mean, k_pool = sum_i w_i k_i with sum_i w_i = 1.
//
// Block b holds tokens 4b..4b+3 in time order; w_i weighs the i-th of them.
// A block is pooled when its last token is appended; until then its raw keys
// wait in a 3-slot tail per sequence.  The pooled value is the fp32 sum
// rounded once to bf16 (round-to-nearest-even).
//
// Work split: grid (x, B).  CTA x of sequence b pools blocks
// blk_lo + x*kBlocksPerCta ..; 16 threads per block, 8 dims (16 bytes) per
// thread.  Only the first block of an append can read the tail, and only CTA
// x = 0 handles it; that CTA also writes the new tail after a barrier, so no
// tail slot is overwritten before it has been read.
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kPoolThreads = 128;
constexpr int kChunksPerRow = kIdxDim / 8;                          // 16
constexpr int kBlocksPerPass = kPoolThreads / kChunksPerRow;        // 8
constexpr int kBlocksPerCta = 8 * kBlocksPerPass;                   // 64

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__global__ void __launch_bounds__(kPoolThreads)
    k_pool_append(const __nv_bfloat16* __restrict__ raw_k, int n_new, float w0, float w1,
                  float w2, float w3, __nv_bfloat16* __restrict__ tail,
                  __nv_bfloat16* __restrict__ pooled, int64_t cap_blk,
                  const int64_t* __restrict__ len_dev, int64_t len_host, int64_t max_len,
                  int64_t* __restrict__ nvis_out, uint32_t* __restrict__ init_hist,
                  int32_t* __restrict__ init_done) {
  pdl_trigger();
  const int b = blockIdx.y;
  int64_t len = len_dev ? len_dev[b] : len_host;
  // Clamp so that every access stays inside the caches whatever the device
  // lengths hold.
  if (len < 0) len = 0;
  if (len > max_len - n_new) len = max_len - n_new;
  const int64_t end = len + n_new;
  if (blockIdx.x == 0) {
    if (nvis_out && threadIdx.x == 0) nvis_out[b] = end;
    if (init_hist) {
      for (int i = threadIdx.x; i < kSelHistBins; i += kPoolThreads)
        init_hist[static_cast<int64_t>(b) * kSelHistBins + i] = 0u;
      if (threadIdx.x == 0) init_done[b] = 0;
      if (threadIdx.x == 0 && b == 0) init_done[gridDim.y] = 0;  // the scoring work counter
    }
  }
  if (n_new <= 0) return;

  const int64_t blk_lo = len / kPool;
  const int64_t blk_done = end / kPool;  // blocks [blk_lo, blk_done) complete now
  const int chunk = threadIdx.x % kChunksPerRow;
  const int sub = threadIdx.x / kChunksPerRow;
  const float w[4] = {w0, w1, w2, w3};
  const __nv_bfloat16* raw_b = raw_k + static_cast<int64_t>(b) * n_new * kIdxDim;
  __nv_bfloat16* tail_b = tail + static_cast<int64_t>(b) * (kPool - 1) * kIdxDim;
  __nv_bfloat16* pooled_b = pooled + static_cast<int64_t>(b) * cap_blk * kIdxDim;

  const int64_t first = blk_lo + static_cast<int64_t>(blockIdx.x) * kBlocksPerCta;
  for (int pass = 0; pass < kBlocksPerCta / kBlocksPerPass; ++pass) {
    const int64_t blk = first + pass * kBlocksPerPass + sub;
    if (blk >= blk_done) break;
    float acc[8];
#pragma unroll
    for (int i = 0; i < kPool; ++i) {
      const int64_t p = blk * kPool + i;
      const __nv_bfloat16* src = (p < len) ? tail_b + (p % kPool) * kIdxDim
                                           : raw_b + (p - len) * kIdxDim;
      float f[8];
      load8(src + chunk * 8, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = (i == 0) ? f[e] * w[0] : __fmaf_rn(f[e], w[i], acc[e]);
    }
    uint4 o;
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) oh[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    *reinterpret_cast<uint4*>(pooled_b + blk * kIdxDim + chunk * 8) = o;
  }

  // New keys of the still-incomplete last block go to the tail (CTA 0 only,
  // after every read of the old tail above).
  if (blockIdx.x == 0 && (end % kPool) != 0) {
    __syncthreads();
    const int64_t p0 = (end / kPool) * kPool;
    for (int64_t p = (p0 > len ? p0 : len) + sub; p < end; p += kBlocksPerPass) {
      const uint4 v = *reinterpret_cast<const uint4*>(raw_b + (p - len) * kIdxDim + chunk * 8);
      *reinterpret_cast<uint4*>(tail_b + (p % kPool) * kIdxDim + chunk * 8) = v;
    }
  }
}

// n_vis of the prefill queries: query t sees pos0 + t + 1 tokens.
__global__ void k_prefill_nvis(int64_t* __restrict__ n_vis, int T, int64_t pos0) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) n_vis[t] = pos0 + t + 1;
}

}  // namespace

cudaError_t launch_pool_append(const PoolAppendArgs& a, cudaStream_t stream) {
  if (a.n_new <= 0 && a.nvis_out == nullptr && a.init_hist == nullptr) return cudaSuccess;
  // Blocks an append can touch: at most ceil((n_new + 3) / 4) + 1.
  const int64_t blocks = (static_cast<int64_t>(a.n_new) + 2 * kPool) / kPool;
  dim3 grid(static_cast<unsigned>((blocks + kBlocksPerCta - 1) / kBlocksPerCta), a.B);
  if (grid.x == 0) grid.x = 1;
  k_pool_append<<<grid, kPoolThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.raw_k), a.n_new, a.w[0], a.w[1], a.w[2], a.w[3],
      static_cast<__nv_bfloat16*>(a.tail), static_cast<__nv_bfloat16*>(a.pooled_k), a.cap_blk,
      a.len_dev, a.len_host, a.max_len, a.nvis_out, a.init_hist, a.init_done);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_prefill_nvis(int64_t* n_vis, int T, int64_t pos0, cudaStream_t stream) {
  k_prefill_nvis<<<(T + 255) / 256, 256, 0, stream>>>(n_vis, T, pos0);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
