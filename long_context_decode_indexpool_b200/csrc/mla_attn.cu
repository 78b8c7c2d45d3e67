// Sparse MLA attention over the gathered latent rows of the selected tokens,
// on the 5th-generation tensor cores.
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
// One CTA = one query row, 64 heads, one split of the row's token list.
// The list is walked in tiles of 64 tokens:
//   * gather: 128 threads copy the tile's latent rows (each selected block is
//     4 KiB contiguous in HBM) with 16-byte cp.async into shared memory in the
//     128-byte-swizzle K-major layout (8 regions of 64 dims), double-buffered;
//   * S = Q C^T: 32 tcgen05.mma (M = 64 heads, N = 64 tokens, K = 16) into
//     TMEM lanes 16-31 of each 32-lane quarter (an M = 64 accumulator uses
//     lanes 0-15 of each quarter, so the other half is free);
//   * softmax: the thread that owns TMEM lane 16+i of warp w holds the logits
//     of head 16w+i for the tile, masks skipped/absent tokens, keeps the
//     running max m (base 2) and sum l, writes P (bf16) to shared memory.  The
//     running max is raised lazily: only when a tile's max exceeds it by more
//     than 8 (so p <= 2^8) is O rescaled, by the partner thread that owns
//     lane i (the O row of the same head);
//   * O += P C: 8 tcgen05.mma (M = 64, N = 256, K = 16; C is read in its
//     MN-major form from the same shared-memory tile) into TMEM lanes 0-15,
//     columns 0-511.
// A split writes out/lse directly (one split) or an unnormalised partial with
// its (m, l) for the merge kernel (log-sum-exp rule).
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kThreads = 128;
constexpr int kTT = 64;                         // tokens per tile
constexpr int kHG = 64;                         // heads per CTA (MMA M)
constexpr int kRegion = 64 * 128;               // [64 rows x 128 B] = 8 KiB
constexpr int kQBytes = 8 * kRegion;            // 64 KiB
constexpr int kKVBytes = 8 * kRegion;           // 64 KiB per tile
constexpr int kPBytes = kRegion;                // [64 heads x 64 tokens] bf16
constexpr int kSmemBytes = 1024 + kQBytes + 2 * kKVBytes + kPBytes + 2 * kTT * 8 + 64;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLazy = 8.f;                    // rescale threshold (log2 units)
constexpr uint32_t kIdescQK = idesc_bf16_f32(64, kTT);
// PV: B (the latent tile) is MN-major: set the "transpose B" bit.
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256) | (1u << 16);

struct KParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* latent;
  int64_t seq_stride;
  int64_t len_cap;  // min(max_len, cap_tok)
  const int32_t* idx;
  const int32_t* count;
  const int64_t* n_vis;
  int heads;
  int nsplit;
  int split_tokens;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;   // [rows, nsplit, heads, 512]
  float* part_ml;  // [rows, nsplit, heads, 2]
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
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte piece `c` (0..63) of row `r` in a tile stored as 8
// regions of [64 rows x 128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzle
// layout: 64-element groups along MN `lbo` bytes apart, 8-row groups along K
// `sbo` bytes apart.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = sm;
  uint8_t* kv_s = q_s + kQBytes;
  uint8_t* p_s = kv_s + 2 * kKVBytes;
  int64_t* pos_s = reinterpret_cast<int64_t*>(p_s + kPBytes);  // [2][64]
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(pos_s + 2 * kTT);
  uint64_t* bar_pv = bar_qk + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_pv + 1);

  const int split = blockIdx.x, r = blockIdx.y, hg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h0 = hg * kHG;
  const RowInfo ri = row_info(p, r);
  const int j_begin = split * p.split_tokens;
  const int j_end = min(ri.S, j_begin + p.split_tokens);
  const int ntiles = j_end > j_begin ? (j_end - j_begin + kTT - 1) / kTT : 0;
  // head owned by this thread: lanes 0-15 hold O rows, lanes 16-31 S rows
  const int hloc = warp * 16 + (lane & 15);
  const int head = h0 + hloc;
  const bool head_ok = head < p.heads;

  if (ntiles == 0) {
    for (int i = tid; i < kHG * kLatent; i += kThreads) {
      const int hh = h0 + i / kLatent;
      if (hh >= p.heads) continue;
      if (p.nsplit == 1)
        p.out[(static_cast<int64_t>(r) * p.heads + hh) * kLatent + i % kLatent] =
            __float2bfloat16_rn(0.f);
      else
        p.part_o[((static_cast<int64_t>(r) * p.nsplit + split) * p.heads + hh) * kLatent +
                 i % kLatent] = 0.f;
    }
    if (tid < kHG && h0 + tid < p.heads) {
      const int hh = h0 + tid;
      if (p.nsplit == 1) {
        if (p.lse) p.lse[static_cast<int64_t>(r) * p.heads + hh] = -INFINITY;
      } else {
        const int64_t b = (static_cast<int64_t>(r) * p.nsplit + split) * p.heads + hh;
        p.part_ml[b * 2] = -INFINITY;
        p.part_ml[b * 2 + 1] = 0.f;
      }
    }
    return;
  }

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_pv, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }

  const __nv_bfloat16* lat = p.latent + static_cast<int64_t>(r) * p.seq_stride;
  const uint32_t q_u = smem_u32(q_s), kv_u = smem_u32(kv_s), p_u = smem_u32(p_s);

  // Q [64 heads x 512] (heads beyond H zero-filled): part of the first group
  {
    const __nv_bfloat16* qr = p.q + (static_cast<int64_t>(r) * p.heads) * kLatent;
    for (int c = tid; c < kHG * 64; c += kThreads) {
      const int h = c >> 6, piece = c & 63;
      const bool ok = h0 + h < p.heads;
      cp_async16(q_u + sw_off(h, piece),
                 qr + static_cast<int64_t>(ok ? h0 + h : 0) * kLatent + piece * 8, ok);
    }
  }
  auto fill_pos = [&](int tile, int buf) {
    if (tid < kTT) {
      const int j = j_begin + tile * kTT + tid;
      pos_s[buf * kTT + tid] = j < j_end ? token_pos(p, r, ri, j) : -1;
    }
  };
  auto gather = [&](int buf) {
    const uint32_t dst = kv_u + buf * kKVBytes;
    const int64_t* ps = pos_s + buf * kTT;
#pragma unroll 4
    for (int i = 0; i < (kTT * 64) / kThreads; ++i) {
      const int c = i * kThreads + tid;
      const int t = c >> 6, piece = c & 63;
      const int64_t pos = ps[t];
      cp_async16(dst + sw_off(t, piece), lat + (pos >= 0 ? pos : 0) * kLatent + piece * 8,
                 pos >= 0);
    }
    cp_async_commit();
  };

  fill_pos(0, 0);
  __syncthreads();
  gather(0);  // group: Q + tile 0
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // MMA destinations: O in the lower half of each 32-lane quarter (lanes
  // 0-15, columns 0-511), S in the upper half (lanes 16-31, columns 0-63).
  const uint32_t t_o = tmem;
  const uint32_t t_s = tmem + (16u << 16);
  const uint32_t my_lane_base = static_cast<uint32_t>(warp * 32) << 16;

  float m_run = -INFINITY, l_run = 0.f;  // meaningful in the S-lane threads
  bool ok_all = true;

  for (int j = 0; j < ntiles; ++j) {
    const int buf = j & 1;
    cp_async_wait<0>();
    fence_proxy_async();
    __syncthreads();

    // ---- S = Q C^T --------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kvb = kv_u + buf * kKVBytes;
#pragma unroll
      for (int k = 0; k < kLatent / 16; ++k) {
        const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
        umma_bf16(t_s, sdesc_kmajor_sw128(q_u + off), sdesc_kmajor_sw128(kvb + off), kIdescQK,
                  k > 0 ? 1u : 0u);
      }
      umma_commit(bar_qk);
    }
    // the previous PV must be done before its buffer is refilled and before
    // P or O are touched again
    if (j > 0) {
      volatile int no_abort = 0;
      ok_all &= mbar_wait(bar_pv, (j - 1) & 1, &no_abort);
    }
    if (j + 1 < ntiles) {
      fill_pos(j + 1, buf ^ 1);
      __syncthreads();
      gather(buf ^ 1);
    }
    {
      volatile int no_abort = 0;
      ok_all &= mbar_wait(bar_qk, j & 1, &no_abort);
    }
    tc_fence_after();

    // ---- softmax -----------------------------------------------------------
    // A warp reads its own 32-lane quarter: lanes 16-31 receive the S rows
    // (lanes 0-15 receive O columns 0-63, unused here).
    float s[kTT];
    {
      uint32_t* sr = reinterpret_cast<uint32_t*>(s);
      tmem_ld_x32_async(tmem + my_lane_base, sr);
      tmem_ld_x32_async(tmem + my_lane_base + 32, sr + 32);
      tmem_ld_wait_regs<kTT>(sr);
    }
    const int64_t* ps = pos_s + buf * kTT;
    float mt = -INFINITY;
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
      s[t] = ps[t] >= 0 ? s[t] * p.scale_log2 : -INFINITY;
      mt = fmaxf(mt, s[t]);
    }
    float alpha = 1.f;
    if (lane >= 16) {
      if (m_run == -INFINITY) {
        m_run = mt;
      } else if (mt > m_run + kLazy) {
        alpha = exp2f(m_run - mt);
        m_run = mt;
      }
    }
    // O rows live in the partner lane (lane - 16): rescale there if needed
    const float alpha_o = __shfl_sync(0xffffffffu, alpha, (lane & 15) + 16);
    if (__any_sync(0xffffffffu, alpha_o != 1.f) && j > 0) {
      // whole warp: lanes 0-15 scale their O rows, lanes 16-31 rewrite what they read
      const float f = lane < 16 ? alpha_o : 1.f;
#pragma unroll 1
      for (int c = 0; c < kLatent; c += 32) {
        float v[32];
        tmem_ld_32x32b_x32(t_o + my_lane_base + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= f;
        tmem_st_32x32b_x32(t_o + my_lane_base + c, v);
      }
    }
    if (lane >= 16) {
      float lsum = 0.f;
      uint32_t packed[kTT / 2];
#pragma unroll
      for (int t = 0; t < kTT; t += 2) {
        const float a = s[t] == -INFINITY ? 0.f : exp2f(s[t] - m_run);
        const float b = s[t + 1] == -INFINITY ? 0.f : exp2f(s[t + 1] - m_run);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
        lsum += __low2float(h2) + __high2float(h2);
        packed[t / 2] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      l_run = l_run * alpha + lsum;
      // row hloc of P: 8 pieces of 16 B
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t a = p_u + hloc * 128 + ((c ^ (hloc & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(packed[4 * c]),
                     "r"(packed[4 * c + 1]), "r"(packed[4 * c + 2]), "r"(packed[4 * c + 3])
                     : "memory");
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- O += P C ----------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kvb = kv_u + buf * kKVBytes;
#pragma unroll
      for (int k = 0; k < kTT / 16; ++k) {
        const uint64_t ad = sdesc_kmajor_sw128(p_u + k * 32);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
          const uint64_t bd =
              sdesc_mn_sw128(kvb + nh * 4 * kRegion + k * 16 * 128, kRegion, 1024);
          umma_bf16(t_o + nh * 256, ad, bd, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
        }
      }
      umma_commit(bar_pv);
    }
  }
  {
    volatile int no_abort = 0;
    ok_all &= mbar_wait(bar_pv, (ntiles - 1) & 1, &no_abort);
  }
  tc_fence_after();

  // ---- epilogue: lanes 0-15 own the O rows ----------------------------------
  // The rows go through shared memory (the latent tiles are free now) so that
  // all 128 threads store them to global memory in coalesced 16-byte pieces.
  const float m_h = __shfl_sync(0xffffffffu, m_run, (lane & 15) + 16);
  const float l_h = __shfl_sync(0xffffffffu, l_run, (lane & 15) + 16);
  const bool single = p.nsplit == 1;
  const float scale_o = single ? (l_h > 0.f ? 1.f / l_h : 0.f) : 1.f;
  // staging: single split -> bf16 rows of 1 KiB; partial -> fp32 rows of 2 KiB
  // (64 rows x 2 KiB = 128 KiB = both latent buffers).  16-byte pieces are
  // rotated by the row index to spread the banks.
  uint8_t* stage = kv_s;
  const int row_bytes = single ? kLatent * 2 : kLatent * 4;
  const int pieces = row_bytes / 16;
#pragma unroll 1
  for (int c0 = 0; c0 < kLatent; c0 += 128) {
    float vv[128];
    uint32_t* vr = reinterpret_cast<uint32_t*>(vv);
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld_x32_async(t_o + my_lane_base + c0 + 32 * q, vr + 32 * q);
    tmem_ld_wait_regs<128>(vr);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = c0 + 32 * q;
    const float* v = vv + 32 * q;
    if (lane < 16) {
      if (single) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * i] * scale_o, v[2 * i + 1] * scale_o);
          w[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int piece = (c * 2 / 16 + i + hloc) % pieces;
          *reinterpret_cast<uint4*>(stage + hloc * row_bytes + piece * 16) =
              make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int piece = (c * 4 / 16 + i + hloc) % pieces;
          *reinterpret_cast<float4*>(stage + hloc * row_bytes + piece * 16) =
              make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    }
  }
  }
  if (lane < 16 && head_ok && ok_all) {
    if (single) {
      if (p.lse)
        p.lse[static_cast<int64_t>(r) * p.heads + head] =
            l_h > 0.f ? (m_h + __log2f(l_h)) * kLn2 : -INFINITY;
    } else {
      const int64_t b = (static_cast<int64_t>(r) * p.nsplit + split) * p.heads + head;
      p.part_ml[b * 2] = l_h > 0.f ? m_h : -INFINITY;
      p.part_ml[b * 2 + 1] = l_h;
    }
  }
  __syncthreads();
  if (ok_all) {
    const int nrows = min(kHG, p.heads - h0);
    uint8_t* gbase = single ? reinterpret_cast<uint8_t*>(p.out + (static_cast<int64_t>(r) * p.heads + h0) * kLatent)
                            : reinterpret_cast<uint8_t*>(p.part_o + ((static_cast<int64_t>(r) * p.nsplit + split) * p.heads + h0) * kLatent);
    for (int e = tid; e < nrows * pieces; e += kThreads) {
      const int row = e / pieces, piece = e % pieces;
      const int sp = (piece + row) % pieces;
      *reinterpret_cast<uint4*>(gbase + static_cast<int64_t>(row) * row_bytes + piece * 16) =
          *reinterpret_cast<const uint4*>(stage + row * row_bytes + sp * 16);
    }
  }
  if (!ok_all && tid == 0) atomicExch(&g_device_error, kErrWaitTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Combines the split partials of one (row, head):
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  out = sum_s O_s 2^(m_s - M) / L.
__global__ void __launch_bounds__(128) k_attn_merge(const float* __restrict__ part_o,
                                                    const float* __restrict__ part_ml,
                                                    int nsplit, int heads,
                                                    __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse) {
  __shared__ float s_w[64];
  __shared__ float s_inv, s_lse;
  const int r = blockIdx.x, hh = blockIdx.y;
  auto base_of = [&](int s) { return (static_cast<int64_t>(r) * nsplit + s) * heads + hh; };
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, part_ml[base_of(s) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < nsplit; s += 32) {
      const float m = part_ml[base_of(s) * 2];
      const float wgt = (M == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M);
      s_w[s] = wgt;
      L += part_ml[base_of(s) * 2 + 1] * wgt;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      s_inv = L > 0.f ? 1.f / L : 0.f;
      s_lse = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  const int d4 = threadIdx.x;  // 128 threads x 4 dims
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < nsplit; s0 += 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // independent loads in flight
      const int s = s0 + u;
      v[u] = s < nsplit && s_w[s] != 0.f
                 ? *reinterpret_cast<const float4*>(part_o + base_of(s) * kLatent + d4 * 4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float wgt = s0 + u < nsplit ? s_w[s0 + u] : 0.f;
      acc.x += v[u].x * wgt;
      acc.y += v[u].y * wgt;
      acc.z += v[u].z * wgt;
      acc.w += v[u].w * wgt;
    }
  }
  const float inv = s_inv;
  __nv_bfloat16* o = out + (static_cast<int64_t>(r) * heads + hh) * kLatent + d4 * 4;
  reinterpret_cast<__nv_bfloat162*>(o)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  reinterpret_cast<__nv_bfloat162*>(o)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  if (lse && threadIdx.x == 0) lse[static_cast<int64_t>(r) * heads + hh] = s_lse;
}

}  // namespace

AttnPlan plan_attn(int rows, int heads, int64_t max_len, int num_sms) {
  AttnPlan p{};
  p.rows = rows;
  p.heads = heads;
  p.groups = (heads + kHG - 1) / kHG;
  const int64_t max_blk = max_len / kPool;
  int64_t s_max = (max_blk > kTopK ? kTopK : max_blk) * kPool + kPool - 1;
  if (s_max > max_len) s_max = max_len;
  if (s_max < 1) s_max = 1;
  const int64_t units = static_cast<int64_t>(rows) * p.groups;
  int nsplit = 1;
  if (units < num_sms) nsplit = static_cast<int>((num_sms + units - 1) / units);
  int64_t ts = (s_max + nsplit - 1) / nsplit;
  ts = (ts + kTT - 1) / kTT * kTT;
  if (ts < 2 * kTT) ts = 2 * kTT;  // at least two tiles per split: fewer partials
  p.split_tokens = static_cast<int>(ts);
  p.nsplit = static_cast<int>((s_max + ts - 1) / ts);
  if (p.nsplit > 64) {  // the merge keeps at most 64 split weights
    ts = ((s_max + 63) / 64 + kTT - 1) / kTT * kTT;
    p.split_tokens = static_cast<int>(ts);
    p.nsplit = static_cast<int>((s_max + ts - 1) / ts);
  }
  p.ws_bytes = 0;
  if (p.nsplit > 1) {
    const size_t n = static_cast<size_t>(rows) * p.nsplit * heads;
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
  p.nsplit = pl.nsplit;
  p.split_tokens = pl.split_tokens;
  p.scale_log2 = a.sm_scale * 1.44269504088896340736f;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  const size_t n = static_cast<size_t>(pl.rows) * pl.nsplit * pl.heads;
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
  k_attn_merge<<<dim3(pl.rows, pl.heads), 128, 0, stream>>>(p.part_o, p.part_ml, pl.nsplit,
                                                            pl.heads, p.out, p.lse);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
