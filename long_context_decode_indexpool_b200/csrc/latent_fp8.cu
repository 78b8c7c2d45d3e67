// FP8 (E4M3) latent cache.
//
// [W1] "GLM-5.3-Flash: 하이브리드 희소·선형 어텐션과 IndexPool·EPD로 1M 컨텍스트를
// 오픈 소스로 서빙하는 방법", section "양자화: W8A8와 혼합 캐시": recent,
// important cache entries are kept in FP8.  The page gives no format or scale;
// the reading here: a 512-wide MLA latent row x is stored as E4M3 codes
// (4 exponent bits with bias 7, 3 mantissa bits, largest 448, subnormal step
// 2^-9) of x / 2^e, with one power-of-two scale per row, e the smallest
// integer with max |x| <= 448 * 2^e (not below -149; 0 for an all-zero row),
// rounded to nearest, ties to even.  A dequantised row (code value * 2^e) is
// exact in bf16, so attention over the FP8 cache is attention over those
// bf16 rows.
//
// k_latent_quant_fp8: one warp per row; lane l holds dims 8l..8l+7 and
//   256+8l..256+8l+7 (two 16-byte loads), finds max |x| by shuffles, and
//   converts two values per instruction (cvt.rn.satfinite.e4m3x2.f32).
// k_gather_fp8: the attention's token list of a row (selected blocks in
//   order, block ids outside [0, n/4) left out, then the partial tail),
//   dequantised into a compact bf16 buffer [row, 2052, 512] with one warp per
//   token, plus the ids 0..c-1, count c and length 4c + tail that make the
//   existing attention kernel walk exactly those rows.
#include <cuda_fp8.h>

#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kQuantThreads = 256;  // 8 rows per CTA
constexpr int kGatherThreads = 256;  // 8 tokens per CTA

// the smallest e with amax <= 448 * 2^e (amax = m 2^E, m in [0.5, 1)):
// E - 9 when m <= 7/8, else E - 8; not below -149; 0 for amax = 0
__device__ __forceinline__ int e4m3_row_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int E = 0;
  const float m = frexpf(amax, &E);
  const int e = m <= 0.875f ? E - 9 : E - 8;
  return e < -149 ? -149 : e;
}

__global__ void __launch_bounds__(kQuantThreads)
    k_latent_quant_fp8(const __nv_bfloat16* __restrict__ lat, int64_t n, uint8_t* __restrict__ codes,
                       int32_t* __restrict__ exps) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + (threadIdx.x >> 5);
  if (row >= n) return;  // uniform per warp
  const __nv_bfloat16* x = lat + row * kLatent;
  float v[16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + h * 256 + lane * 8);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(b[i]);
      v[8 * h + 2 * i] = f.x;
      v[8 * h + 2 * i + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = e4m3_row_exponent(amax);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t pk = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int k = 8 * h + 4 * q + 2 * i;
        // x / 2^e is exact (|x| / 2^e <= 448); one nearest-even rounding to E4M3
        const float2 f = make_float2(ldexpf(v[k], -e), ldexpf(v[k + 1], -e));
        pk |= static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3))
              << (16 * i);
      }
      w[q] = pk;
    }
    *reinterpret_cast<uint2*>(codes + row * kLatent + h * 256 + lane * 8) = make_uint2(w[0], w[1]);
  }
  if (lane == 0) exps[row] = e;
}

// bf16 bits of an E4M3 pair times 2^e (exact: 4 significant bits).
__device__ __forceinline__ uint32_t fp8x2_to_bf16x2(uint16_t pair, float scale) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void __launch_bounds__(kGatherThreads)
    k_gather_fp8(const uint8_t* __restrict__ codes, const int32_t* __restrict__ exps,
                 int64_t seq_stride, int64_t len_cap, const int32_t* __restrict__ idx,
                 const int32_t* __restrict__ count, const int64_t* __restrict__ n_vis,
                 __nv_bfloat16* __restrict__ dense, int64_t dense_stride, int32_t* __restrict__ c_idx,
                 int32_t* __restrict__ c_cnt, int64_t* __restrict__ c_nvis) {
  __shared__ int s_off[kTopK / 32 + 1];  // valid ids before each group of 32
  const int r = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t n = n_vis[r];
  n = n < 0 ? 0 : (n > len_cap ? len_cap : n);
  const int64_t nblk = n / kPool;
  int cnt = count[r];
  cnt = cnt < 0 ? 0 : (cnt > kTopK ? kTopK : cnt);
  if (cnt > nblk) cnt = static_cast<int>(nblk);
  const int32_t* ir = idx + static_cast<int64_t>(r) * kTopK;
  // valid ids (in [0, nblk)), compacted in order: warp w counts groups w, w+8
  for (int g = warp; g < kTopK / 32; g += kGatherThreads / 32) {
    const int j = g * 32 + lane;
    const int b = j < cnt ? ir[j] : -1;
    const uint32_t ball = __ballot_sync(0xffffffffu, b >= 0 && b < nblk);
    if (lane == 0) s_off[g + 1] = __popc(ball);
  }
  __syncthreads();
  if (tid == 0) {
    s_off[0] = 0;
    for (int g = 1; g <= kTopK / 32; ++g) s_off[g] += s_off[g - 1];
  }
  __syncthreads();
  const int valid = s_off[kTopK / 32];
  const int tail = static_cast<int>(n - nblk * kPool);
  const int S = valid * kPool + tail;
  if (blockIdx.x == 0) {
    // the compact list: valid blocks 0..valid-1, then the tail
    for (int j = tid; j < kTopK; j += kGatherThreads)
      c_idx[static_cast<int64_t>(r) * kTopK + j] = j < valid ? j : -1;
    if (tid == 0) {
      c_cnt[r] = valid;
      c_nvis[r] = S;
    }
  }
  const uint8_t* cr = codes + static_cast<int64_t>(r) * seq_stride;
  const int32_t* er = exps + static_cast<int64_t>(r) * (seq_stride / kLatent);
  __nv_bfloat16* dr = dense + static_cast<int64_t>(r) * dense_stride;
  // token k of the compact list: one warp, 16 codes (16 bytes) per lane
  for (int k = blockIdx.x * (kGatherThreads / 32) + warp; k < S;
       k += gridDim.x * (kGatherThreads / 32)) {
    int64_t pos;
    if (k < valid * kPool) {
      // the (k / 4)-th valid id: find its group by the prefix, then its lane
      const int want = k / kPool;
      int g = 0;
      while (s_off[g + 1] <= want) ++g;
      const int j = g * 32 + lane;
      const int b = j < cnt ? ir[j] : -1;
      const bool ok = b >= 0 && b < nblk;
      const uint32_t ball = __ballot_sync(0xffffffffu, ok);
      const int rank = want - s_off[g];  // the rank-th set bit of ball
      const int src = __fns(ball, 0, rank + 1);
      const int bsel = __shfl_sync(0xffffffffu, b, src);
      pos = static_cast<int64_t>(bsel) * kPool + (k & 3);
    } else {
      pos = nblk * kPool + (k - valid * kPool);
    }
    const uint4 u = *reinterpret_cast<const uint4*>(cr + pos * kLatent + lane * 16);
    const float scale = ldexpf(1.f, er[pos]);
    const uint32_t c4[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = fp8x2_to_bf16x2(static_cast<uint16_t>(c4[i] & 0xffffu), scale);
      o[2 * i + 1] = fp8x2_to_bf16x2(static_cast<uint16_t>(c4[i] >> 16), scale);
    }
    uint4* dst = reinterpret_cast<uint4*>(dr + static_cast<int64_t>(k) * kLatent + lane * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_latent_quant_fp8(const void* lat, int64_t n, uint8_t* codes, int32_t* exps,
                                    cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t per = kQuantThreads / 32;
  const int64_t blocks = (n + per - 1) / per;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  k_latent_quant_fp8<<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(lat), n, codes, exps);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gather_fp8(int rows, const uint8_t* codes, const int32_t* exps,
                              int64_t seq_stride, int64_t len_cap, const int32_t* idx,
                              const int32_t* count, const int64_t* n_vis, void* dense,
                              int64_t dense_stride, int32_t* c_idx, int32_t* c_cnt,
                              int64_t* c_nvis, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  // 2051 tokens at most per row, 8 per CTA: 32 CTAs of 64 tokens
  dim3 grid(32, rows);
  k_gather_fp8<<<grid, kGatherThreads, 0, stream>>>(codes, exps, seq_stride, len_cap, idx, count,
                                                    n_vis, static_cast<__nv_bfloat16*>(dense),
                                                    dense_stride, c_idx, c_cnt, c_nvis);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
