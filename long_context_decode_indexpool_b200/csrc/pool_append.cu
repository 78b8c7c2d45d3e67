// IndexPool cache write.
//
// [W1] "GLM-5.3-Flash: 하이브리드 희소·선형 어텐션과 IndexPool·EPD로 1M 컨텍스트를
// 오픈 소스로 서빙하는 방법", section "IndexPool: 인덱서 KV 캐시를 4배 압축":
// the indexer keys of 4 consecutive positions are merged by a learned
// weighted mean, k_pool = sum_i w_i k_i with sum_i w_i = 1.
//
// Block b holds tokens 4b..4b+3 in time order; w_i weighs the i-th of them.
// A block is pooled when its last token is appended; until then its raw keys
// wait in a 3-slot tail per sequence.  The pooled value is formed in fp64
// (each product of a bf16 key and an fp32 weight is exact there; the four
// are added in time order, starting from +0) and rounded once: to bf16
// (round-to-nearest-even), or, in the INT8 cache ([W1] section "양자화:
// W8A8와 혼합 캐시": far, compressed indexer entries in INT8), to int8 codes
// with one power-of-two scale per block; the 16 threads of a block find its
// max |x| by shuffles.  With learned (non-dyadic) weights an fp32 sum would
// round twice and could land one bf16 step away from the single rounding of
// the exact value; the fp64 sum does not.
//
// Per-token weights (spx_pool_append_tok): instead of four weights per
// layer, token p brings its own weight (a learned gate's output; the four
// weights of a block sum to 1), and the weights of a still-incomplete block
// wait in a 3-slot weight tail beside the key tail.
//
// Work split: grid (x, B).  CTA x of sequence b pools blocks
// blk_lo + x*kBlocksPerCta ..; 16 threads per block, 8 dims (16 bytes) per
// thread.  Only the first block of an append can read the tail, and only CTA
// x = 0 handles it; that CTA also writes the new tail after a barrier, so no
// tail slot is overwritten before it has been read.
#include "spx_device.cuh"
#include "spx_internal.h"
#include "spx_launch.cuh"

namespace spx {

namespace {

constexpr int kPoolThreads = 128;
constexpr int kChunksPerRow = kIdxDim / 8;                          // 16
constexpr int kBlocksPerPass = kPoolThreads / kChunksPerRow;        // 8
constexpr int kBlocksPerCta = 8 * kBlocksPerPass;                   // 64

// bf16 bits of the nearest-even rounding of a double: 8 significant bits
// from 2^-126 up, a fixed spacing of 2^-133 below (the bf16 subnormals).
__device__ __forceinline__ uint16_t bf16_rne_f64(double v) {
  const double a = fabs(v);
  double r;
  if (a >= 0x1p-126) {
    // keep 7 of the 52 stored fraction bits: add just under half of the
    // dropped weight (plus one on a tie with an odd kept part), then clear
    uint64_t u = static_cast<uint64_t>(__double_as_longlong(a));
    u += ((1ull << 44) - 1ull) + ((u >> 45) & 1ull);
    u &= ~((1ull << 45) - 1ull);
    r = __longlong_as_double(static_cast<long long>(u));
  } else {
    r = rint(a * 0x1p133) * 0x1p-133;  // exact scalings around one rounding
  }
  // r has at most 8 significant bits: its fp32 conversion is exact (or inf
  // above the fp32 range), and bf16 is the fp32 pattern's top half
  const uint32_t f = __float_as_uint(__double2float_rn(r));
  return static_cast<uint16_t>((f >> 16) | (signbit(v) ? 0x8000u : 0u));
}

// INT8 code exponent of an fp64 vector maximum (as i8_exponent): the
// smallest e with amax <= 127 * 2^e, not below -149, 0 for amax = 0.
__device__ __forceinline__ int i8_exponent_f64(double amax) {
  if (!(amax > 0.0)) return 0;
  int E = 0;
  const double m = frexp(amax, &E);
  const int e = m <= 127.0 / 128.0 ? E - 7 : E - 6;
  return e < -149 ? -149 : e;
}

__device__ __forceinline__ uint32_t i8_code_f64(double x, int e) {
  return static_cast<uint32_t>(__double2int_rn(ldexp(x, -e))) & 0xffu;
}

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

// INT8 codes of the query heads of row b (the scoring kernel's B operand):
// warp w quantises heads w, w+4, ..; lane l holds dims 4l..4l+3.  The
// head's scale is folded into its weight: wq = w_head * 2^e.  Every load
// is issued before the first head is worked on (one round trip, not one a
// head: this runs on the decode step's critical path).
__device__ void quant_q_row(const __nv_bfloat16* __restrict__ q_idx,
                            const float* __restrict__ w_head, int8_t* __restrict__ q8,
                            float* __restrict__ wq, int b) {
  constexpr int kWarps = kPoolThreads / 32;
  constexpr int kPer = kIdxHeads / kWarps;  // heads of one warp
  static_assert(kIdxHeads % kWarps == 0, "whole heads per warp");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint2 u[kPer];
  float wh[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t row = static_cast<int64_t>(b) * kIdxHeads + warp + kWarps * i;
    u[i] = *reinterpret_cast<const uint2*>(q_idx + row * kIdxDim + 4 * lane);
    wh[i] = lane == 0 ? w_head[row] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t row = static_cast<int64_t>(b) * kIdxHeads + warp + kWarps * i;
    const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i].x));
    const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i].y));
    float amax = fmaxf(fmaxf(fabsf(x01.x), fabsf(x01.y)), fmaxf(fabsf(x23.x), fabsf(x23.y)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int e = i8_exponent(amax);
    const uint32_t packed = (static_cast<uint32_t>(i8_code(x01.x, e)) & 0xffu) |
                            ((static_cast<uint32_t>(i8_code(x01.y, e)) & 0xffu) << 8) |
                            ((static_cast<uint32_t>(i8_code(x23.x, e)) & 0xffu) << 16) |
                            (static_cast<uint32_t>(i8_code(x23.y, e)) << 24);
    *reinterpret_cast<uint32_t*>(q8 + row * kIdxDim + 4 * lane) = packed;
    if (lane == 0) wq[row] = wh[i] * ldexpf(1.f, e);
  }
}

struct PoolKParams {
  const __nv_bfloat16* raw_k;
  int n_new;
  float w[4];
  const float* raw_w;  // per-token weights [B, n_new] (or NULL: w)
  float* tail_w;       // per-token weights of the tail [B, pool-1]
  __nv_bfloat16* tail;
  void* pooled;        // bf16 rows, or int8 code rows
  float* k_scale;      // int8 cache: per-block scale
  int64_t cap_blk;
  const int64_t* len_dev;
  int64_t len_host;
  int64_t max_len;
  int64_t* nvis_out;
  uint32_t* init_hist;
  int32_t* init_done;
  const __nv_bfloat16* q_idx;  // optional query quantisation (int8 cache)
  const float* w_head;
  int8_t* q8;
  float* wq;
};

template <bool I8>
__global__ void __launch_bounds__(kPoolThreads) k_pool_append(const PoolKParams p) {
  pdl_trigger();
  // Launched early (after the previous step's last kernel started), it waits
  // for that kernel to finish before touching anything: the previous step's
  // selection state and lengths are rewritten here.
  pdl_wait();
  const int b = blockIdx.y;
  int64_t len = p.len_dev ? p.len_dev[b] : p.len_host;
  // Clamp so that every access stays inside the caches whatever the device
  // lengths hold.
  if (len < 0) len = 0;
  if (len > p.max_len - p.n_new) len = p.max_len - p.n_new;
  const int64_t end = len + p.n_new;
  if (blockIdx.x == 0) {
    if (p.nvis_out && threadIdx.x == 0) p.nvis_out[b] = end;
    if (p.init_hist) {
      for (int i = threadIdx.x; i < kSelHistBins; i += kPoolThreads)
        p.init_hist[static_cast<int64_t>(b) * kSelHistBins + i] = 0u;
      if (threadIdx.x == 0) p.init_done[b] = 0;
      if (threadIdx.x == 0 && b == 0) p.init_done[gridDim.y] = 0;  // the scoring work counter
    }
    if constexpr (I8) {
      if (p.q_idx) quant_q_row(p.q_idx, p.w_head, p.q8, p.wq, b);
    }
  }
  if (p.n_new <= 0) return;

  const int64_t blk_lo = len / kPool;
  const int64_t blk_done = end / kPool;  // blocks [blk_lo, blk_done) complete now
  const int chunk = threadIdx.x % kChunksPerRow;
  const int sub = threadIdx.x / kChunksPerRow;
  const __nv_bfloat16* raw_b = p.raw_k + static_cast<int64_t>(b) * p.n_new * kIdxDim;
  __nv_bfloat16* tail_b = p.tail + static_cast<int64_t>(b) * (kPool - 1) * kIdxDim;

  const int64_t first = blk_lo + static_cast<int64_t>(blockIdx.x) * kBlocksPerCta;
  for (int pass = 0; pass < kBlocksPerCta / kBlocksPerPass; ++pass) {
    const int64_t blk0 = first + pass * kBlocksPerPass;
    if (blk0 >= blk_done) break;  // uniform
    const int64_t blk = blk0 + sub;
    const bool active = blk < blk_done;
    // fp64 sum from +0 in time order (each product is exact)
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    if (active) {
#pragma unroll
      for (int i = 0; i < kPool; ++i) {
        const int64_t t = blk * kPool + i;
        const __nv_bfloat16* src = (t < len) ? tail_b + (t % kPool) * kIdxDim
                                             : raw_b + (t - len) * kIdxDim;
        float f[8];
        load8(src + chunk * 8, f);
        const double wi = static_cast<double>(
            !p.raw_w ? p.w[i]
                     : (t < len ? p.tail_w[static_cast<int64_t>(b) * (kPool - 1) + t % kPool]
                                : p.raw_w[static_cast<int64_t>(b) * p.n_new + (t - len)]));
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = __fma_rn(static_cast<double>(f[e]), wi, acc[e]);
      }
    }
    if constexpr (I8) {
      // the block's 16 threads are lanes 0-15 or 16-31 of one warp
      double amax = 0.0;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmax(amax, fabs(acc[e]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const int ex = i8_exponent_f64(amax);
      uint32_t w2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        w2[h] = i8_code_f64(acc[4 * h], ex) | (i8_code_f64(acc[4 * h + 1], ex) << 8) |
                (i8_code_f64(acc[4 * h + 2], ex) << 16) | (i8_code_f64(acc[4 * h + 3], ex) << 24);
      if (active) {
        int8_t* row = static_cast<int8_t*>(p.pooled) +
                      (static_cast<int64_t>(b) * p.cap_blk + blk) * kIdxDim;
        *reinterpret_cast<uint2*>(row + chunk * 8) = make_uint2(w2[0], w2[1]);
        if (chunk == 0) p.k_scale[static_cast<int64_t>(b) * p.cap_blk + blk] = ldexpf(1.f, ex);
      }
    } else {
      if (active) {
        uint32_t h2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          h2[e] = static_cast<uint32_t>(bf16_rne_f64(acc[2 * e])) |
                  (static_cast<uint32_t>(bf16_rne_f64(acc[2 * e + 1])) << 16);
        const uint4 o = make_uint4(h2[0], h2[1], h2[2], h2[3]);
        __nv_bfloat16* row = static_cast<__nv_bfloat16*>(p.pooled) +
                             (static_cast<int64_t>(b) * p.cap_blk + blk) * kIdxDim;
        *reinterpret_cast<uint4*>(row + chunk * 8) = o;
      }
    }
  }

  // New keys of the still-incomplete last block go to the tail (CTA 0 only,
  // after every read of the old tail above).
  if (blockIdx.x == 0 && (end % kPool) != 0) {
    __syncthreads();
    const int64_t p0 = (end / kPool) * kPool;
    for (int64_t t = (p0 > len ? p0 : len) + sub; t < end; t += kBlocksPerPass) {
      const uint4 v = *reinterpret_cast<const uint4*>(raw_b + (t - len) * kIdxDim + chunk * 8);
      *reinterpret_cast<uint4*>(tail_b + (t % kPool) * kIdxDim + chunk * 8) = v;
      if (p.raw_w && chunk == 0)
        p.tail_w[static_cast<int64_t>(b) * (kPool - 1) + t % kPool] =
            p.raw_w[static_cast<int64_t>(b) * p.n_new + (t - len)];
    }
  }
}

// Query quantisation alone (standalone INT8 scoring call): one CTA per row.
__global__ void __launch_bounds__(kPoolThreads)
    k_quant_q(const __nv_bfloat16* __restrict__ q_idx, const float* __restrict__ w_head,
              int8_t* __restrict__ q8, float* __restrict__ wq) {
  quant_q_row(q_idx, w_head, q8, wq, blockIdx.x);
}

// n_vis of the prefill queries: query t sees pos0 + t + 1 tokens.
__global__ void k_prefill_nvis(int64_t* __restrict__ n_vis, int T, int64_t pos0) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) n_vis[t] = pos0 + t + 1;
}

}  // namespace

cudaError_t launch_pool_append(const PoolAppendArgs& a, cudaStream_t stream) {
  if (a.n_new <= 0 && a.nvis_out == nullptr && a.init_hist == nullptr && a.q_idx == nullptr)
    return cudaSuccess;
  // Blocks an append can touch: at most ceil((n_new + 3) / 4) + 1.
  const int64_t blocks = (static_cast<int64_t>(a.n_new) + 2 * kPool) / kPool;
  dim3 grid(static_cast<unsigned>((blocks + kBlocksPerCta - 1) / kBlocksPerCta), a.B);
  if (grid.x == 0) grid.x = 1;
  PoolKParams p{};
  p.raw_k = static_cast<const __nv_bfloat16*>(a.raw_k);
  p.n_new = a.n_new;
  for (int i = 0; i < 4; ++i) p.w[i] = a.w[i];
  p.raw_w = a.raw_w;
  p.tail_w = a.tail_w;
  p.tail = static_cast<__nv_bfloat16*>(a.tail);
  p.pooled = a.pooled_k;
  p.k_scale = a.k_scale;
  p.cap_blk = a.cap_blk;
  p.len_dev = a.len_dev;
  p.len_host = a.len_host;
  p.max_len = a.max_len;
  p.nvis_out = a.nvis_out;
  p.init_hist = a.init_hist;
  p.init_done = a.init_done;
  p.q_idx = static_cast<const __nv_bfloat16*>(a.q_idx);
  p.w_head = a.w_head;
  p.q8 = a.q8;
  p.wq = a.wq;
  cudaError_t e = a.i8 ? launch_ex(k_pool_append<true>, grid, dim3(kPoolThreads), 0, stream,
                                   a.pdl, 1, p)
                       : launch_ex(k_pool_append<false>, grid, dim3(kPoolThreads), 0, stream,
                                   a.pdl, 1, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quant_q(int B, const void* q_idx, const float* w_head, int8_t* q8, float* wq,
                           cudaStream_t stream) {
  k_quant_q<<<B, kPoolThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(q_idx), w_head, q8,
                                            wq);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_prefill_nvis(int64_t* n_vis, int T, int64_t pos0, cudaStream_t stream) {
  k_prefill_nvis<<<(T + 255) / 256, 256, 0, stream>>>(n_vis, T, pos0);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
