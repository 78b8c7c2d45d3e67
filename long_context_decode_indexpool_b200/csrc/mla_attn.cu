// Sparse MLA attention over the gathered latent rows of the selected tokens.
//
// [W3] "GLM-5.3 Sparse Attention은 연산량을 줄이지만 HBM 수요는 지속된다", section
// "GLM-5.3 Sparse Attention이 실제로 바꾸는 것": the core multi-head latent
// attention runs only on the positions the indexer selected; with no more
// positions than the budget it stays dense.  [W4] "GLM-5.3-Flash vs
// Qwen3.8-Flash-Next: ...", section "의견이 갈리는 지점 — 위치 인코딩": the
// sparse MLA layers carry no rotary part (NoPE), so in the absorbed form the
// 512-wide latent row c_t is both the key and the value of every head.
//
//   out[h] = sum_t softmax_t(sm_scale * q_h . c_t) c_t   over the token set S
//   S = tokens of the selected blocks  U  the query's partial tail block.
//
// Kernel (one CTA = one query row, 16 heads, one split of the token list):
// 64-token sub-tiles of latent rows are gathered with 16-byte cp.async into
// a double-buffered, XOR-swizzled shared-memory tile (each selected block is
// 4 KiB contiguous in HBM).  QK^T and PV run on bf16 tensor-core MMAs with
// fp32 accumulation; the softmax is online in base 2 (exp2 of
// sm_scale*log2(e)-scaled logits).  Splits of one (row, head group) write
// unnormalised partial outputs with their running max and sum; a merge
// kernel combines them with the log-sum-exp rule.
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSub = 64;                       // tokens per sub-tile
constexpr int kRowBytes = kLatent * 2;         // 1024
constexpr int kQSmem = kHeadGroup * kRowBytes; // 16 KiB
constexpr int kKVSmem = kSub * kRowBytes;      // 64 KiB
constexpr int kPSmem = kHeadGroup * kSub * 2;  // 2 KiB
constexpr int kSmemBytes = 128 + kQSmem + 2 * kKVSmem + kPSmem + 2 * kSub * 8 +
                           2 * kWarps * kHeadGroup * 4;
constexpr float kLn2 = 0.69314718055994530942f;

struct KParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* latent;
  int64_t seq_stride;
  int64_t len_cap;  // min(max_len, cap_tok)
  const int32_t* idx;
  const int32_t* count;
  const int64_t* n_vis;
  int heads;
  int groups;
  int nsplit;
  int split_tokens;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;   // [rows, groups, nsplit, 16, 512]
  float* part_ml;  // [rows, groups, nsplit, 16, 2]
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// byte offset of 16-byte chunk `c` of row `r` in a swizzled tile with
// `row_bytes` per row (chunk index XOR row mod 8)
__device__ __forceinline__ uint32_t swz(int r, int c, int row_bytes) {
  return static_cast<uint32_t>(r * row_bytes + ((c ^ (r & 7)) << 4));
}

struct RowInfo {
  int64_t nblk;  // complete blocks visible
  int cnt;       // selected blocks
  int S;         // tokens in the list
};

__device__ __forceinline__ RowInfo row_info(const KParams& p, int r) {
  RowInfo ri;
  int64_t n = p.n_vis[r];
  n = n < 0 ? 0 : (n > p.len_cap ? p.len_cap : n);
  ri.nblk = n / kPool;
  int c = p.count[r];
  c = c < 0 ? 0 : (c > kTopK ? kTopK : c);
  if (c > ri.nblk) c = static_cast<int>(ri.nblk);
  ri.cnt = c;
  ri.S = c * kPool + static_cast<int>(n - ri.nblk * kPool);
  return ri;
}

// token position of entry j of row r's list, or -1 (skipped block)
__device__ __forceinline__ int64_t token_pos(const KParams& p, int r, const RowInfo& ri, int j) {
  if (j < ri.cnt * kPool) {
    const int b = p.idx[static_cast<int64_t>(r) * kTopK + (j >> 2)];
    if (b < 0 || b >= ri.nblk) return -1;
    return static_cast<int64_t>(b) * kPool + (j & 3);
  }
  return ri.nblk * kPool + (j - ri.cnt * kPool);
}

__global__ void __launch_bounds__(kThreads, 1) k_sparse_attn(const KParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 127) &
                                           ~static_cast<uintptr_t>(127));
  uint8_t* q_s = sm;
  uint8_t* kv_s = q_s + kQSmem;
  uint8_t* p_s = kv_s + 2 * kKVSmem;
  int64_t* pos_s = reinterpret_cast<int64_t*>(p_s + kPSmem);  // [2][64]
  float* red_max = reinterpret_cast<float*>(pos_s + 2 * kSub);  // [8][16]
  float* red_sum = red_max + kWarps * kHeadGroup;             // [8][16]

  const int split = blockIdx.x, r = blockIdx.y, g = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const RowInfo ri = row_info(p, r);
  const int j_begin = split * p.split_tokens;
  const int j_end = min(ri.S, j_begin + p.split_tokens);
  const int nsub = j_end > j_begin ? (j_end - j_begin + kSub - 1) / kSub : 0;
  const int h0 = lane >> 2;  // rows h0 and h0 + 8 of the accumulator fragments
  const int64_t unit = (static_cast<int64_t>(r) * p.groups + g);

  if (nsub == 0) {
    if (p.nsplit == 1) {
      for (int i = tid; i < kHeadGroup * kLatent; i += kThreads)
        p.out[(static_cast<int64_t>(r) * p.heads + g * kHeadGroup) * kLatent + i] =
            __float2bfloat16_rn(0.f);
      if (p.lse && tid < kHeadGroup)
        p.lse[static_cast<int64_t>(r) * p.heads + g * kHeadGroup + tid] = -INFINITY;
    } else {
      const int64_t base = (unit * p.nsplit + split) * kHeadGroup;
      for (int i = tid; i < kHeadGroup * kLatent; i += kThreads) p.part_o[base * kLatent + i] = 0.f;
      if (tid < kHeadGroup) {
        p.part_ml[(base + tid) * 2] = -INFINITY;
        p.part_ml[(base + tid) * 2 + 1] = 0.f;
      }
    }
    return;
  }

  const __nv_bfloat16* lat = p.latent + static_cast<int64_t>(r) * p.seq_stride;
  const uint32_t q_u = smem_u32(q_s), kv_u = smem_u32(kv_s), p_u = smem_u32(p_s);

  // Q tile [16 heads x 512] -> shared (part of the first cp.async group)
  {
    const __nv_bfloat16* qg =
        p.q + (static_cast<int64_t>(r) * p.heads + g * kHeadGroup) * kLatent;
    for (int c = tid; c < kHeadGroup * (kLatent / 8); c += kThreads) {
      const int h = c >> 6, ch = c & 63;
      cp_async16(q_u + swz(h, ch, kRowBytes), qg + h * kLatent + ch * 8, true);
    }
  }

  auto fill_pos = [&](int sub, int buf) {
    if (tid < kSub) {
      const int j = j_begin + sub * kSub + tid;
      pos_s[buf * kSub + tid] = j < j_end ? token_pos(p, r, ri, j) : -1;
    }
  };
  auto issue_kv = [&](int buf) {
    const uint32_t dst = kv_u + buf * kKVSmem;
    const int64_t* ps = pos_s + buf * kSub;
#pragma unroll 4
    for (int i = 0; i < (kSub * (kLatent / 8)) / kThreads; ++i) {
      const int c = i * kThreads + tid;
      const int t = c >> 6, ch = c & 63;
      const int64_t pos = ps[t];
      const __nv_bfloat16* src = lat + (pos >= 0 ? pos : 0) * kLatent + ch * 8;
      cp_async16(dst + swz(t, ch, kRowBytes), src, pos >= 0);
    }
  };

  fill_pos(0, 0);
  __syncthreads();
  issue_kv(0);
  cp_async_commit();

  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  for (int sub = 0; sub < nsub; ++sub) {
    const int buf = sub & 1;
    if (sub + 1 < nsub) {
      fill_pos(sub + 1, buf ^ 1);
      __syncthreads();
      issue_kv(buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const uint32_t kvb = kv_u + buf * kKVSmem;
    const int64_t* ps = pos_s + buf * kSub;

    // ---- S = Q K^T for this warp's 8 tokens ------------------------------
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int kk = 0; kk < kLatent / 16; kk += 2) {
      uint32_t b0, b1, b2, b3;
      {
        const int t = warp * 8 + (lane & 7);
        const int ch = kk * 2 + (lane >> 3);
        ldsm_x4(kvb + swz(t, ch, kRowBytes), b0, b1, b2, b3);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t a0, a1, a2, a3;
        const int row = lane & 15;
        const int ch = (kk + u) * 2 + (lane >> 4);
        ldsm_x4(q_u + swz(row, ch, kRowBytes), a0, a1, a2, a3);
        if (u == 0)
          mma_bf16(sacc, a0, a1, a2, a3, b0, b1);
        else
          mma_bf16(sacc, a0, a1, a2, a3, b2, b3);
      }
    }

    // ---- online softmax ---------------------------------------------------
    const int tcol = warp * 8 + 2 * (lane & 3);
    const bool v0 = ps[tcol] >= 0, v1 = ps[tcol + 1] >= 0;
    float x[4];
    x[0] = v0 ? sacc[0] * p.scale_log2 : -INFINITY;
    x[1] = v1 ? sacc[1] * p.scale_log2 : -INFINITY;
    x[2] = v0 ? sacc[2] * p.scale_log2 : -INFINITY;
    x[3] = v1 ? sacc[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
    }
    if ((lane & 3) == 0) {
      red_max[warp * kHeadGroup + h0] = mx0;
      red_max[warp * kHeadGroup + h0 + 8] = mx1;
    }
    __syncthreads();
    float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      tm0 = fmaxf(tm0, red_max[w * kHeadGroup + h0]);
      tm1 = fmaxf(tm1, red_max[w * kHeadGroup + h0 + 8]);
    }
    const float mn0 = fmaxf(m_run[0], tm0), mn1 = fmaxf(m_run[1], tm1);
    const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m_run[0] - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m_run[1] - mn1);
    float pv[4];
    pv[0] = x[0] == -INFINITY ? 0.f : exp2f(x[0] - mn0);
    pv[1] = x[1] == -INFINITY ? 0.f : exp2f(x[1] - mn0);
    pv[2] = x[2] == -INFINITY ? 0.f : exp2f(x[2] - mn1);
    pv[3] = x[3] == -INFINITY ? 0.f : exp2f(x[3] - mn1);
    l_run[0] = l_run[0] * al0 + pv[0] + pv[1];
    l_run[1] = l_run[1] * al1 + pv[2] + pv[3];
    m_run[0] = mn0;
    m_run[1] = mn1;
    {
      const uint32_t off = static_cast<uint32_t>((lane & 3) * 4);
      __nv_bfloat162 w0 = __floats2bfloat162_rn(pv[0], pv[1]);
      __nv_bfloat162 w1 = __floats2bfloat162_rn(pv[2], pv[3]);
      *reinterpret_cast<__nv_bfloat162*>(p_s + swz(h0, warp, kSub * 2) + off) = w0;
      *reinterpret_cast<__nv_bfloat162*>(p_s + swz(h0 + 8, warp, kSub * 2) + off) = w1;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
    __syncthreads();

    // ---- O += P V for this warp's 64 dims -------------------------------------
#pragma unroll
    for (int kk = 0; kk < kSub / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      {
        const int row = lane & 15;
        const int ch = kk * 2 + (lane >> 4);
        ldsm_x4(p_u + swz(row, ch, kSub * 2), a0, a1, a2, a3);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int t = kk * 16 + (lane & 15);
        const int ch = warp * 8 + np * 2 + (lane >> 4);
        ldsm_x4_t(kvb + swz(t, ch, kRowBytes), b0, b1, b2, b3);
        mma_bf16(o[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }

  // ---- row sums over the quad and the warps ----------------------------------
  float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
  for (int o2 = 1; o2 < 4; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
  }
  if ((lane & 3) == 0) {
    red_sum[warp * kHeadGroup + h0] = l0;
    red_sum[warp * kHeadGroup + h0 + 8] = l1;
  }
  __syncthreads();
  float L0 = 0.f, L1 = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    L0 += red_sum[w * kHeadGroup + h0];
    L1 += red_sum[w * kHeadGroup + h0 + 8];
  }

  const int dcol = warp * 64 + 2 * (lane & 3);
  if (p.nsplit == 1) {
    const float inv0 = L0 > 0.f ? 1.f / L0 : 0.f, inv1 = L1 > 0.f ? 1.f / L1 : 0.f;
    __nv_bfloat16* o0 = p.out + (static_cast<int64_t>(r) * p.heads + g * kHeadGroup + h0) * kLatent;
    __nv_bfloat16* o1 = o0 + 8 * kLatent;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      *reinterpret_cast<__nv_bfloat162*>(o0 + dcol + 8 * i) =
          __floats2bfloat162_rn(o[i][0] * inv0, o[i][1] * inv0);
      *reinterpret_cast<__nv_bfloat162*>(o1 + dcol + 8 * i) =
          __floats2bfloat162_rn(o[i][2] * inv1, o[i][3] * inv1);
    }
    if (p.lse && warp == 0 && (lane & 3) == 0) {
      float* ls = p.lse + static_cast<int64_t>(r) * p.heads + g * kHeadGroup;
      ls[h0] = L0 > 0.f ? (m_run[0] + __log2f(L0)) * kLn2 : -INFINITY;
      ls[h0 + 8] = L1 > 0.f ? (m_run[1] + __log2f(L1)) * kLn2 : -INFINITY;
    }
  } else {
    const int64_t base = (unit * p.nsplit + split) * kHeadGroup;
    float* po0 = p.part_o + (base + h0) * kLatent;
    float* po1 = po0 + 8 * kLatent;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      *reinterpret_cast<float2*>(po0 + dcol + 8 * i) = make_float2(o[i][0], o[i][1]);
      *reinterpret_cast<float2*>(po1 + dcol + 8 * i) = make_float2(o[i][2], o[i][3]);
    }
    if (warp == 0 && (lane & 3) == 0) {
      p.part_ml[(base + h0) * 2] = m_run[0];
      p.part_ml[(base + h0) * 2 + 1] = L0;
      p.part_ml[(base + h0 + 8) * 2] = m_run[1];
      p.part_ml[(base + h0 + 8) * 2 + 1] = L1;
    }
  }
}

// Combines the split partials of one (row, head group):
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  out = sum_s O_s 2^(m_s - M) / L.
__global__ void __launch_bounds__(256) k_attn_merge(const float* __restrict__ part_o,
                                                    const float* __restrict__ part_ml,
                                                    int nsplit, int heads, int groups,
                                                    __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse) {
  const int r = blockIdx.x, g = blockIdx.y;
  const int64_t unit = static_cast<int64_t>(r) * groups + g;
  for (int e = threadIdx.x; e < kHeadGroup * (kLatent / 4); e += blockDim.x) {
    const int h = e / (kLatent / 4), d4 = e % (kLatent / 4);
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s)
      M = fmaxf(M, part_ml[((unit * nsplit + s) * kHeadGroup + h) * 2]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const int64_t base = (unit * nsplit + s) * kHeadGroup + h;
        const float m = part_ml[base * 2];
        if (m == -INFINITY) continue;
        const float wgt = exp2f(m - M);
        L += part_ml[base * 2 + 1] * wgt;
        const float4 v = *reinterpret_cast<const float4*>(part_o + base * kLatent + d4 * 4);
        acc.x += v.x * wgt;
        acc.y += v.y * wgt;
        acc.z += v.z * wgt;
        acc.w += v.w * wgt;
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* o = out + (static_cast<int64_t>(r) * heads + g * kHeadGroup + h) * kLatent + d4 * 4;
    reinterpret_cast<__nv_bfloat162*>(o)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    reinterpret_cast<__nv_bfloat162*>(o)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    if (lse && d4 == 0)
      lse[static_cast<int64_t>(r) * heads + g * kHeadGroup + h] =
          L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
  }
}

}  // namespace

AttnPlan plan_attn(int rows, int heads, int64_t max_len, int num_sms) {
  AttnPlan p{};
  p.rows = rows;
  p.heads = heads;
  p.groups = heads / kHeadGroup;
  const int64_t max_blk = max_len / kPool;
  int64_t s_max = (max_blk > kTopK ? kTopK : max_blk) * kPool + kPool - 1;
  if (s_max > max_len) s_max = max_len;
  if (s_max < 1) s_max = 1;
  const int64_t units = static_cast<int64_t>(rows) * p.groups;
  int nsplit = 1;
  if (units < num_sms) nsplit = static_cast<int>((num_sms + units - 1) / units);
  int64_t ts = (s_max + nsplit - 1) / nsplit;
  ts = (ts + kSub - 1) / kSub * kSub;
  p.split_tokens = static_cast<int>(ts);
  p.nsplit = static_cast<int>((s_max + ts - 1) / ts);
  p.ws_bytes = 0;
  if (p.nsplit > 1) {
    const size_t n = static_cast<size_t>(units) * p.nsplit * kHeadGroup;
    p.ws_bytes = ((n * kLatent * 4 + 255) & ~static_cast<size_t>(255)) + n * 2 * 4;
  }
  return p;
}

cudaError_t launch_attn(const AttnPlan& pl, const AttnArgs& a, cudaStream_t stream) {
  if (pl.rows == 0) return cudaSuccess;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  KParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.latent = static_cast<const __nv_bfloat16*>(a.latent);
  p.seq_stride = a.seq_stride;
  p.len_cap = a.max_len < a.cap_tok ? a.max_len : a.cap_tok;
  p.idx = a.idx;
  p.count = a.count;
  p.n_vis = a.n_vis;
  p.heads = pl.heads;
  p.groups = pl.groups;
  p.nsplit = pl.nsplit;
  p.split_tokens = pl.split_tokens;
  p.scale_log2 = a.sm_scale * 1.44269504088896340736f;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  const size_t n = static_cast<size_t>(pl.rows) * pl.groups * pl.nsplit * kHeadGroup;
  p.part_o = static_cast<float*>(a.ws);
  p.part_ml = pl.nsplit > 1
                  ? reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) +
                                             ((n * kLatent * 4 + 255) & ~static_cast<size_t>(255)))
                  : nullptr;
  dim3 grid(pl.nsplit, pl.rows, pl.groups);
  k_sparse_attn<<<grid, kThreads, kSmemBytes, stream>>>(p);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || pl.nsplit == 1) return e;
  k_attn_merge<<<dim3(pl.rows, pl.groups), 256, 0, stream>>>(p.part_o, p.part_ml, pl.nsplit,
                                                             pl.heads, pl.groups, p.out, p.lse);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
