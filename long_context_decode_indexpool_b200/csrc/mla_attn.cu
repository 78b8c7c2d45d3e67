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
// One CTA = one query row, 64 heads, one split of the row's token list.  The
// token positions of the split (and a validity bit per token) are computed
// once into shared memory; the list is then walked in tiles of 64 tokens.
//
// TMEM (128 lanes x 512 columns; an M = 64 accumulator puts row 16w+i of
// the tile in lane 32w+i, or 32w+16+i with the lane offset 16):
//   O dims   0-255: lanes 32w+i,    columns 0-255
//   O dims 256-511: lanes 32w+16+i, columns 0-255
//   S (64 tokens):  lanes 32w+16+i, columns 256+64b .. (b = S buffer 0/1)
// Worker warps w and w+4 (w < 4) both reach lanes 32w .. 32w+31.  Warp w
// takes tokens 0-31 of each tile and columns 0-127 of O, warp w+4 tokens
// 32-63 and columns 128-255.  In each, the two threads of TMEM lanes i and
// 16+i share head 16w+i: the thread of lane 16+i hands the logits of the
// first 16 tokens to its partner (one shuffle each), so a thread works on 16
// logits; the two warps exchange their tile maxima per head through shared
// memory (a barrier of the pair) and keep partial row sums.
//
// Per tile: 16-byte cp.async gather of the latent rows into the
// 128-byte-swizzle K-major layout by seven gather warps (double-buffered; a
// buffer is refilled as soon as the PV of its previous tile is done, the
// first two tiles load at once; the cache may be device memory or mapped
// pinned host memory).  S = Q C^T as 32
// tcgen05.mma (M = 64, N = 64, K = 16); softmax in registers (running max in
// base 2, raised lazily: O is rescaled only when a tile's max exceeds it by
// more than 8); P (bf16) to shared memory; O += P C as 8 tcgen05.mma
// (M = 64, N = 256, K = 16, C read MN-major from the same tile).  While the
// first tile's softmax runs, the tensor core already computes the second
// tile's logits.
//
// A row with a single split writes its normalised output directly.  The n
// splits of one (row, head group) otherwise form a thread-block cluster: each
// CTA writes its output rows normalised by its own l (bf16, like P) to L2
// (one bulk copy per TMEM lane quarter of 16 rows) and its per-head (m, l)
// (fp32) with plain stores, the cluster barrier publishes them, and CTA k
// reads back heads [k*64/n, (k+1)*64/n) of all splits with bulk copies and
// combines them with the log-sum-exp rule (weights 2^(m_s - M) l_s / L) into
// the bf16 output and the log-sum-exp.  No second kernel runs.  (Moving the
// partials through distributed shared memory instead, by loads or by bulk
// copies between the CTAs, measured slower.)
#include <atomic>

#include "spx_device.cuh"
#include "spx_internal.h"
#include "spx_launch.cuh"

namespace spx {

namespace {

constexpr int kWork = 256;                      // worker threads (warps 0-7)
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;                   // gather warps 9 ..
// gather threads (7 warps): 16 warps in all leave 128 registers a thread
// (registers are granted in groups of 4 warps: 17 warps would get 96)
constexpr int kProd = 224;
// 8 worker warps, the MMA warp, the gather warps
constexpr int kThreads = kProdWarp0 * 32 + kProd;
constexpr int kTT = 64;                         // tokens per tile
constexpr int kHG = 64;                         // heads per CTA (MMA M)
constexpr int kRegion = 64 * 128;               // [64 rows x 128 B] = 8 KiB
constexpr int kQBytes = 8 * kRegion;            // 64 KiB
constexpr int kKVBytes = 8 * kRegion;           // 64 KiB per tile
// The two latent tiles share 8 regions of [128 rows x 128 B] (tile b in rows
// 64b..64b+63), so that both together also form one N = 128 operand.
constexpr int kKVRegion = 2 * kRegion;          // 16 KiB
constexpr int kPBytes = kRegion;                // [64 heads x 64 tokens] bf16 (two buffers)
constexpr int kMaxList = kTopK * kPool + kPool - 1;             // tokens in a list, at most
constexpr int kPosCap = (kMaxList + kTT - 1) / kTT * kTT;       // position slots
constexpr int kMaxCluster = 16;                 // splits per (row, head group)
constexpr int kSmemBytes = 1024 + kQBytes + 2 * kKVBytes + 2 * kPBytes + kPosCap * 4 +
                           (kPosCap / 32) * 4 + 128;
static_assert(((kPosCap * 4 + (kPosCap / 32) * 4) & 7) == 0, "barriers 8-byte aligned");
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLazy = 8.f;                    // rescale threshold (log2 units)
constexpr uint32_t kIdescQK = idesc_bf16_f32(64, kTT);
constexpr uint32_t kIdescQK2 = idesc_bf16_f32(64, 2 * kTT);  // both tiles at once
// PV: B (the latent tile) is MN-major: set the "transpose B" bit.
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256) | (1u << 16);
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct KParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* latent;
  int64_t seq_stride;
  int64_t len_cap;  // min(max_len, cap_tok)
  const int32_t* idx;
  const int32_t* count;
  const int64_t* n_vis;
  int heads;
  int nsplit;        // = cluster size
  int split_tokens;  // list entries per split (the last split takes the rest)
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  __nv_bfloat16* part_o;  // [rows, groups, nsplit, 64, 512] O / l of each split (nsplit > 1)
  float* part_ml;         // [rows, groups, nsplit, 64, 2]   (m, l)
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

// Barrier of the two worker warps that share TMEM lane quarter qd (ids 1-4).
__device__ __forceinline__ void pair_sync(int qd) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + qd) : "memory");
}

// Thread-block cluster helpers.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Bulk copies (TMA engine, no tensor map): shared -> global and
// global -> shared (completing on an mbarrier); 16-byte aligned, sizes a
// multiple of 16.
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t sdst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sdst),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Byte offset of 16-byte piece `c` (0..63) of row `r` in a tile stored as 8
// regions of [64 rows x 128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
// The same for row r (0..127) of the latent tile pair (regions of 16 KiB).
__device__ __forceinline__ uint32_t kv_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kKVRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4));
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

// cnt: the row's selected-block count (from p.count, or chosen in the kernel)
__device__ __forceinline__ RowInfo row_info(const KParams& p, int r, int cnt) {
  RowInfo ri;
  int64_t n = p.n_vis[r];
  n = n < 0 ? 0 : (n > p.len_cap ? p.len_cap : n);
  ri.nblk = n / kPool;
  int c = cnt;
  c = c < 0 ? 0 : (c > kTopK ? kTopK : c);
  if (c > ri.nblk) c = static_cast<int>(ri.nblk);
  ri.cnt = c;
  ri.S = c * kPool + static_cast<int>(n - ri.nblk * kPool);
  return ri;
}

// token position of entry j of row r's list, or -1 (skipped block); b is
// the selected block id idx[r][j / 4] when j is in the selected part
__device__ __forceinline__ int64_t token_pos_of(const RowInfo& ri, int j, int b) {
  if (j < ri.cnt * kPool) {
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
  uint8_t* kv_s = q_s + kQBytes;  // two latent tiles; afterwards the combine rows
  uint8_t* p_s = kv_s + 2 * kKVBytes;                               // [2] P buffers
  int32_t* pos_s = reinterpret_cast<int32_t*>(p_s + 2 * kPBytes);   // [kPosCap]
  uint32_t* vm_s = reinterpret_cast<uint32_t*>(pos_s + kPosCap);    // [kPosCap / 32] valid bits
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(vm_s + kPosCap / 32);  // [2]: S(t) in buffer t&1
  uint64_t* bar_pv = bar_qk + 2;   // [2]: PV(t) done, t & 1
  uint64_t* bar_kv = bar_qk + 4;   // [2]: tile t in latent buffer t & 1
  uint64_t* bar_p = bar_qk + 6;    // [2]: P(t) written, t & 1
  uint64_t* bar_q = bar_qk + 8;    // Q landed
  uint64_t* bar_red = bar_qk + 9;  // combine: rows of the other splits
  uint64_t* bar_drain = bar_qk + 10;  // every MMA of the CTA done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_qk + 11);
  __shared__ float red_m[2][2][kHG];  // [tile parity][token half][head]: tile maxima
  __shared__ float red_l[2][kHG];     // [token half][head]: row sums

  const int split = blockIdx.x, r = blockIdx.y, hg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool worker = tid < kWork;  // warps 0-7; warp 8 issues the MMAs, warps 9-15 gather
  const int h0 = hg * kHG;
  const int n_cl = p.nsplit;
  // head of this thread; lanes i and 16+i of a worker warp share it
  const int hloc = (warp & 3) * 16 + (lane & 15);
  const int half = lane >> 4;  // 0: dims 0-255, 1: dims 256-511 (and a token sub-half)
  const int qd = warp & 3;      // workers: TMEM lane quarter
  const int th = (warp >> 2) & 1;  // workers: half of a tile's tokens, of O's columns
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t q_u = smem_u32(q_s), kv_u = smem_u32(kv_s), p_u = smem_u32(p_s);

  // ---- set-up that needs nothing from the previous kernel -------------------
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_qk[i], 1);
      mbar_init(&bar_pv[i], 1);
      mbar_init(&bar_kv[i], kProd / 32);  // one arrive per gather warp
      mbar_init(&bar_p[i], kWork / 32);  // one arrive per worker warp
    }
    mbar_init(bar_q, kWork / 32);
    mbar_init(bar_red, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // Q [64 heads x 512] (heads beyond H zero-filled): part of the first group
  if (worker) {
    const __nv_bfloat16* qr = p.q + (static_cast<int64_t>(r) * p.heads) * kLatent;
#pragma unroll 4
    for (int c = tid; c < kHG * 64; c += kWork) {
      const int h = c >> 6, piece = c & 63;
      const bool ok = h0 + h < p.heads;
      cp_async16(q_u + sw_off(h, piece),
                 qr + static_cast<int64_t>(ok ? h0 + h : 0) * kLatent + piece * 8, ok);
    }
  }
  pdl_trigger();
  pdl_wait();  // the selected blocks come from the previous kernel
  bool ok_all = true;

  const int32_t* idx_row = p.idx + static_cast<int64_t>(r) * kTopK;
  const int row_cnt = p.count[r];

  // the block id of this thread's first list entry goes out with the row's
  // length and count (one round trip instead of two)
  const int j_first = split * p.split_tokens + tid;
  const int b_first = (worker && j_first < kTopK * kPool) ? idx_row[j_first >> 2] : -1;
  const RowInfo ri = row_info(p, r, row_cnt);
  const int j_begin = split * p.split_tokens;
  const int j_end = split == n_cl - 1 ? ri.S : min(ri.S, j_begin + p.split_tokens);
  const int nlist = j_end > j_begin ? j_end - j_begin : 0;
  const int ntiles = (nlist + kTT - 1) / kTT;
  float m_run = -INFINITY, l_run = 0.f;  // of head hloc (both threads)
  uint32_t tmem = 0;

  if (ntiles > 0) {  // uniform
    const __nv_bfloat16* lat = p.latent + static_cast<int64_t>(r) * p.seq_stride;
    if (worker) {
      // every token position of the split, once, with a validity bit per token
#pragma unroll 1
      for (int i0 = 0; i0 < ntiles * kTT; i0 += kWork) {
        const int i = i0 + tid;
        int64_t pos = -1;
        if (i < nlist) {
          const int j = j_begin + i;
          const int b = i0 == 0 ? b_first : (j < ri.cnt * kPool ? idx_row[j >> 2] : -1);
          pos = token_pos_of(ri, j, b);
        }
        if (i < ntiles * kTT) pos_s[i] = static_cast<int32_t>(pos);
        const uint32_t bits = __ballot_sync(0xffffffffu, pos >= 0);
        if (lane == 0 && i < ntiles * kTT) vm_s[i >> 5] = bits;
      }
      // Q has landed (the workers' only cp.async group)
      cp_async_wait<0>();
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = *tmem_holder;

    if (warp >= kProdWarp0) {
      // ======================= gather warps =================================
      // Tile t goes into latent buffer t & 1 as soon as PV(t-2) has released
      // it: 64 tokens x 64 pieces of 16 bytes, spread over all gather
      // threads; token slots with nothing to load are zero-filled by the
      // same copies.  Tiles 0 and 1 go out at once as two cp.async groups.
      const int gt = tid - kProdWarp0 * 32;
      auto issue_tile = [&](int t) {
        const int row0 = (t & 1) * kTT;
        const int32_t* ps = pos_s + t * kTT;
#pragma unroll 8
        for (int i = 0; i < (kTT * 64 + kProd - 1) / kProd; ++i) {
          const int c = i * kProd + gt;
          if (c < kTT * 64) {
            const int tk = c >> 6, piece = c & 63;
            const int pos = ps[tk];
            cp_async16(kv_u + kv_off(row0 + tk, piece),
                       lat + static_cast<int64_t>(pos >= 0 ? pos : 0) * kLatent + piece * 8,
                       pos >= 0);
          }
        }
        cp_async_commit();
      };
      auto publish = [&](int t) {  // this warp's part of tile t is in place
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_kv[t & 1]);
      };
      issue_tile(0);
      if (ntiles > 1) {
        issue_tile(1);
        cp_async_wait<1>();
        publish(0);
        cp_async_wait<0>();
        publish(1);
      } else {
        cp_async_wait<0>();
        publish(0);
      }
#pragma unroll 1
      for (int t = 2; t < ntiles; ++t) {
        {
          volatile int no_abort = 0;
          ok_all &= mbar_wait(&bar_pv[t & 1], ((t - 2) >> 1) & 1, &no_abort);
        }
        issue_tile(t);
        cp_async_wait<0>();
        publish(t);
      }
    } else if (warp == kMmaWarp) {
      // ======================= MMA issuer (warp 8) ===========================
      // Issues whichever is ready first: S = Q C^T of the next tile (its data
      // landed, and the softmax of the tile that last used its S buffer is
      // done), or O += P C of the oldest tile whose P is written.  Tiles 0
      // and 1 go as one N = 128 product (their S buffers are adjacent).  The
      // whole warp runs the loop (lane 0 polls the barriers and broadcasts
      // the decision), so the descriptors are warp-uniform and one elected
      // lane issues each MMA.
      volatile int no_abort = 0;
      {
        int okq = 1;
        if (lane == 0) okq = mbar_wait(bar_q, 0, &no_abort) ? 1 : 0;
        ok_all &= __shfl_sync(0xffffffffu, okq, 0) != 0;
      }
      const uint32_t aq = smem_u32(&bar_kv[0]), aq1 = smem_u32(&bar_kv[1]);
      const uint32_t ap0 = smem_u32(&bar_p[0]), ap1 = smem_u32(&bar_p[1]);
      int nq = 0, np = 0;
      uint64_t t_last = globaltimer_ns();
      while (np < ntiles && ok_all) {
        const bool pair = nq == 0 && ntiles > 1;
        int ready = 0;  // 1: QK(nq), 2: PV(np), 3: waited too long
        if (lane == 0) {
          // test_wait, not try_wait: a try_wait suspended on one barrier
          // would miss the other completing (measured: QK started up to
          // 0.5 us after its tile landed)
          if (nq < ntiles && nq <= np + 1) {
            bool r = mbar_test_wait((nq & 1) ? aq1 : aq, (nq >> 1) & 1);
            if (r && pair) r = mbar_test_wait(aq1, 0);
            if (r) ready = 1;
          }
          if (ready == 0 && np < nq && mbar_test_wait((np & 1) ? ap1 : ap0, (np >> 1) & 1))
            ready = 2;
          if (ready == 0 && globaltimer_ns() - t_last > kWaitLimitNs) ready = 3;
        }
        ready = __shfl_sync(0xffffffffu, ready, 0);
        // O += P C of tile np (its P written)
        auto issue_pv = [&]() {
          tc_fence_after();
          const uint32_t kvb = kv_u + (np & 1) * kTT * 128;
          const uint32_t pb = p_u + (np & 1) * kPBytes;
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
            for (int k = 0; k < kTT / 16; ++k) {
              const uint64_t ad = sdesc_kmajor_sw128(pb + k * 32);
              const uint64_t bd =
                  sdesc_mn_sw128(kvb + nh * 4 * kKVRegion + k * 16 * 128, kKVRegion, 1024);
              umma_bf16_elect(tmem + (static_cast<uint32_t>(16 * nh) << 16), ad, bd, kIdescPV,
                              (np > 0 || k > 0) ? 1u : 0u);
            }
          }
          umma_commit_elect(&bar_pv[np & 1]);
          ++np;
        };
        if (ready == 1) {
          tc_fence_after();
          const uint32_t kvb = kv_u + (nq & 1) * kTT * 128;
          const uint32_t d = tmem + (16u << 16) + 256 + 64 * (nq & 1);
          const uint32_t idesc = pair ? kIdescQK2 : kIdescQK;
#pragma unroll
          for (int k = 0; k < kLatent / 16; ++k) {
            const uint32_t qoff = (k >> 2) * kRegion + (k & 3) * 32;
            const uint32_t koff = (k >> 2) * kKVRegion + (k & 3) * 32;
            umma_bf16_elect(d, sdesc_kmajor_sw128(q_u + qoff), sdesc_kmajor_sw128(kvb + koff),
                            idesc, k > 0 ? 1u : 0u);
          }
          umma_commit_elect(&bar_qk[nq & 1]);
          if (pair) umma_commit_elect(&bar_qk[1]);
          nq += pair ? 2 : 1;
          t_last = globaltimer_ns();
        } else if (ready == 2) {
          issue_pv();
          t_last = globaltimer_ns();
        } else if (ready == 3) {
          ok_all = false;
          if (lane == 0) atomicExch(&g_device_error, kErrWaitTimeout);
        }
      }
      // every MMA issued here completes before TMEM is read or released
      umma_commit_elect(bar_drain);
      if (lane == 0) mbar_wait(bar_drain, 0, &no_abort);
      __syncwarp();
    } else if (worker) {
      // ======================= workers (warps 0-7) ==========================
      // Warps w and w + 4 share TMEM lane quarter w & 3 (heads 16(w&3) ..
      // +15): warp w takes tokens 0-31 of each tile, warp w + 4 tokens 32-63,
      // so a thread works on 16 logits.  The tile's maximum per head is
      // exchanged between the two through shared memory, so both raise the
      // running maximum alike; each keeps a partial row sum.
#pragma unroll 1
      for (int j = 0; j < ntiles; ++j) {
        const int buf = j & 1;
        {
          volatile int no_abort = 0;
          ok_all &= mbar_wait(&bar_qk[buf], (j >> 1) & 1, &no_abort);
        }
        tc_fence_after();

        // ---- softmax: 16 logits of head hloc per thread --------------------
        float s[16];
        {
          // lanes 16-31 receive the 32 logits of their head in this warp's
          // half of the tile; tokens 0-15 of it go to the partner lane
          uint32_t a[32];
          tmem_ld_x32_async(tmem + lane_base + 256 + 64 * buf + 32 * th, a);
          tmem_ld_wait_regs<32>(a);
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const uint32_t x = __shfl_xor_sync(0xffffffffu, a[t], 16);
            s[t] = __uint_as_float(half ? a[16 + t] : x);
          }
        }
        const uint32_t vm = (vm_s[j * 2 + th] >> (16 * half)) & 0xFFFFu;
#pragma unroll
        for (int t = 0; t < 16; ++t) s[t] = ((vm >> t) & 1u) ? s[t] * p.scale_log2 : -INFINITY;
        float mx[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          mx[u] = fmaxf(fmaxf(s[4 * u], s[4 * u + 1]), fmaxf(s[4 * u + 2], s[4 * u + 3]));
        float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        // the other half of the tile (double-buffered by tile parity: a slot
        // is rewritten only after the partner passed the next exchange)
        if (half == 0) red_m[buf][th][hloc] = mt;
        pair_sync(qd);
        mt = fmaxf(mt, red_m[buf][th ^ 1][hloc]);
        float alpha = 1.f;
        if (m_run == -INFINITY) {
          m_run = mt;
        } else if (mt > m_run + kLazy) {
          alpha = exp2f(m_run - mt);
          m_run = mt;
        }
        if (__any_sync(0xffffffffu, alpha != 1.f) && j > 0) {
          // O holds tiles up to j-1: let PV(j-1) finish, then each thread
          // scales its half of the O row of its head, this warp's columns
          {
            volatile int no_abort = 0;
            ok_all &= mbar_wait(&bar_pv[(j - 1) & 1], ((j - 1) >> 1) & 1, &no_abort);
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 128 * th; c < 128 * th + 128; c += 32) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + lane_base + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st_32x32b_x32(tmem + lane_base + c, v);
          }
        }
        uint32_t packed[8];
        float ps[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float e[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            e[i] = s[4 * u + i] == -INFINITY ? 0.f : exp2f(s[4 * u + i] - m_run);
          const __nv_bfloat162 a = __floats2bfloat162_rn(e[0], e[1]);
          const __nv_bfloat162 b = __floats2bfloat162_rn(e[2], e[3]);
          packed[2 * u] = *reinterpret_cast<const uint32_t*>(&a);
          packed[2 * u + 1] = *reinterpret_cast<const uint32_t*>(&b);
          ps[u] = (__low2float(a) + __high2float(a)) + (__low2float(b) + __high2float(b));
        }
        float lsum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        l_run = l_run * alpha + lsum;  // this warp's half of the tokens
        // P buffer j & 1 is free once PV(j-2) is done
        if (j >= 2) {
          volatile int no_abort = 0;
          ok_all &= mbar_wait(&bar_pv[buf], ((j - 2) >> 1) & 1, &no_abort);
        }
        // row hloc of P, pieces 4 th + 2 half .. +1 (16 B each)
        const uint32_t pb = p_u + buf * kPBytes;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int piece = 4 * th + 2 * half + c;
          const uint32_t a = pb + hloc * 128 + ((piece ^ (hloc & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(packed[4 * c]),
                       "r"(packed[4 * c + 1]), "r"(packed[4 * c + 2]), "r"(packed[4 * c + 3])
                       : "memory");
        }
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p[buf]);  // the MMA warp issues O += P C
      }
      {
        volatile int no_abort = 0;
        ok_all &= mbar_wait(&bar_pv[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, &no_abort);
      }
      tc_fence_after();
      // the row sum over both halves of the tokens
      if (half == 0) red_l[th][hloc] = l_run;
      pair_sync(qd);
      l_run += red_l[th ^ 1][hloc];
    }
    __syncwarp();
  }

  // ---- output ----------------------------------------------------------------
  cp_async_wait<0>();  // (a split without tokens still has Q copies in flight)
  const bool have = ntiles > 0 && ok_all && l_run > 0.f;
  const int64_t unit = static_cast<int64_t>(r) * gridDim.z + hg;  // (row, head group)
  // This split's output rows, normalised by its own l, as bf16 rows of 1 KiB
  // staged in the latent buffers (16-byte pieces rotated by the row to spread
  // the banks).
  uint8_t* stage = kv_s;
  const uint32_t stage_u = smem_u32(stage);
  if (ntiles > 0 && worker) {
    const float inv = have ? 1.f / l_run : 0.f;
#pragma unroll 1
    for (int c0 = 128 * th; c0 < 128 * th + 128; c0 += 32) {
      float v[32];
      tmem_ld_32x32b_x32(tmem + lane_base + c0, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat162 h2 =
              __floats2bfloat162_rn(v[8 * i + 2 * u] * inv, v[8 * i + 2 * u + 1] * inv);
          w[u] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        const int piece = ((256 * half + c0) / 8 + i + hloc) & 63;
        *reinterpret_cast<uint4*>(stage + hloc * 1024 + piece * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (n_cl > 1) {
      // this quarter's 16 rows (16 KiB, contiguous) go to L2 at once, while
      // the other quarters are still staging theirs
      const int64_t first_row = (unit * n_cl + split) * kHG;
      fence_proxy_async();
      pair_sync(qd);  // both warps' columns are staged
      if (th == 0 && lane == 0) {
        bulk_store(p.part_o + (first_row + qd * 16) * kLatent, stage_u + qd * 16 * 1024,
                   16 * kLatent * 2);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
  }
  if (n_cl == 1) {
    if (worker && half == 0 && th == 0 && h0 + hloc < p.heads && p.lse)
      p.lse[static_cast<int64_t>(r) * p.heads + h0 + hloc] =
          have ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    __syncthreads();
    const int nrows = min(kHG, p.heads - h0);
    uint8_t* gbase =
        reinterpret_cast<uint8_t*>(p.out + (static_cast<int64_t>(r) * p.heads + h0) * kLatent);
#pragma unroll 1
    for (int e = tid; worker && e < nrows * 64; e += kWork) {
      const int row = e >> 6, piece = e & 63;
      const uint4 val =
          ntiles > 0 ? *reinterpret_cast<const uint4*>(stage + row * 1024 + ((piece + row) & 63) * 16)
                     : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(gbase + static_cast<int64_t>(row) * 1024 + piece * 16) = val;
    }
  } else {
    // The staged rows (same layout in L2, one bulk copy) and (m, l) of this
    // split go to L2; the cluster barrier publishes them.
    const int64_t first_row = (unit * n_cl + split) * kHG;
    if (ntiles > 0 && worker && lane == 0) {
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // this warp's rows are in L2
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    if (worker && half == 0 && th == 0) {
      float* pm = p.part_ml + (first_row + hloc) * 2;
      pm[0] = have ? m_run : -INFINITY;
      pm[1] = have ? l_run : 0.f;
    }
    cluster_sync_all();
    // CTA k combines heads [k*rows_per, (k+1)*rows_per) of the group: the
    // rows of split c come back with one bulk copy (they are contiguous in
    // L2) into the latent buffers (slot c*nh + hh); weights 2^(m_c - M) l_c /
    // L from the (m, l).
    const int k = static_cast<int>(cluster_rank());
    const int rows_per = kHG / n_cl;
    const int hk = k * rows_per;
    int nh = p.heads - h0 - hk;
    nh = nh < 0 ? 0 : (nh > rows_per ? rows_per : nh);
    const float* pm_all = p.part_ml + (unit * n_cl) * kHG * 2;
    const __nv_bfloat16* po_all = p.part_o + (unit * n_cl) * kHG * kLatent;
    float* w_s = reinterpret_cast<float*>(p_s);  // [64] combine weights
    if (nh > 0) {  // uniform
      const int nrows = nh * n_cl;
      if (tid == 0) mbar_arrive_expect_tx(bar_red, static_cast<uint32_t>(nrows) * 1024u);
      if (tid < n_cl) {  // split c's rows of heads hk .. hk+nh-1: contiguous, one copy
        const int c = tid;
        bulk_load(stage_u + c * nh * 1024, po_all + (static_cast<int64_t>(c) * kHG + hk) * kLatent,
                  static_cast<uint32_t>(nh) * 1024u, bar_red);
      }
      if (tid < kHG) {  // warps 0-1: groups of n_cl lanes, one group per head
        const int hh = tid / n_cl, c = tid % n_cl;
        float2 ml = make_float2(-INFINITY, 0.f);
        if (tid < nrows) ml = __ldcg(reinterpret_cast<const float2*>(pm_all + (c * kHG + hk + hh) * 2));
        float M = ml.x;
        for (int o = n_cl >> 1; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float e = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M) * ml.y;
        float L = e;
        for (int o = n_cl >> 1; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        w_s[tid] = L > 0.f ? e / L : 0.f;
        if (c == 0 && tid < nrows && p.lse)
          p.lse[static_cast<int64_t>(r) * p.heads + h0 + hk + hh] =
              L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      }
      __syncthreads();
      {
        volatile int no_abort = 0;
        ok_all &= mbar_wait(bar_red, 0, &no_abort);
      }
      // thread t: 8 dims (one 16-byte piece) of one head, two heads per pass
#pragma unroll 1
      for (int e = tid; worker && e < nh * 64; e += kWork) {
        const int hh = e >> 6, piece = e & 63;
        const int h = hk + hh;
        float wc[kMaxCluster];
        uint4 v[kMaxCluster];
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c) {
          wc[c] = c < n_cl ? w_s[hh * n_cl + c] : 0.f;
          v[c] = wc[c] != 0.f ? *reinterpret_cast<const uint4*>(
                                    stage + (c * nh + hh) * 1024 + ((piece + h) & 63) * 16)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c) {
          const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&u[q]);
            acc[2 * q] += __low2float(b2) * wc[c];
            acc[2 * q + 1] += __high2float(b2) * wc[c];
          }
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
          o[q] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(r) * p.heads + h0 + h) * kLatent +
                                  piece * 8) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  if (!ok_all && tid == 0) atomicExch(&g_device_error, kErrWaitTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(*tmem_holder, 512);
}

// Number of clusters of n CTAs of the attention kernel the device can hold
// at once (cached per device).
int active_clusters(int n) {
  static std::atomic<int> cache[64][5];  // count + 1; 0: not queried yet
  int dev = 0;
  cudaGetDevice(&dev);
  int lg = 0;
  while ((1 << lg) < n) ++lg;
  if (dev < 64 && cache[dev][lg].load() > 0) return cache[dev][lg].load() - 1;
  // both instantiations have the same launch shape and shared memory
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = n;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int num = 0;
  if (cudaOccupancyMaxActiveClusters(&num, k_sparse_attn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    num = 0;
  }
  if (dev < 64) cache[dev][lg].store(num + 1);
  return num;
}

// Cluster size for `units` (row, head group) pairs, at most `want` (a power
// of two): the largest size whose clusters all fit on the device at once (a
// second wave of clusters would double the time), else the largest that fits
// at all.
int pick_cluster(int want, int64_t units) {
  int fits_at_all = 1;
  for (int n = want; n > 1; n >>= 1) {
    const int num = active_clusters(n);
    if (num >= units) return n;
    if (num > 0 && fits_at_all == 1) fits_at_all = n;
  }
  return fits_at_all;
}

bool set_attrs() {
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && attr_set[dev]) return true;
  if (cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return false;
  if (dev >= 0 && dev < 64) attr_set[dev] = true;
  return true;
}


}  // namespace

AttnPlan plan_attn(int rows, int heads, int64_t max_len, int num_sms) {
  AttnPlan p{};
  p.rows = rows;
  p.heads = heads;
  p.groups = (heads + kHG - 1) / kHG;
  const int64_t max_blk = max_len / kPool;
  const int64_t bt = (max_blk > kTopK ? kTopK : max_blk) * kPool;  // block tokens in a list
  const int64_t units = static_cast<int64_t>(rows) * p.groups;
  // splits per (row, group): a power of two up to 16 that keeps every SM
  // busy at most once and every split at least one tile long
  int n = 1;
  while (n < kMaxCluster && units * (2 * n) <= num_sms && bt / (2 * n) >= kTT) n *= 2;
  p.nsplit = n;
  int64_t ts = (bt + n - 1) / n;
  ts = (ts + kTT - 1) / kTT * kTT;
  if (ts < kTT) ts = kTT;
  p.split_tokens = static_cast<int>(ts);
  p.ws_bytes = 0;
  if (n > 1) {
    const size_t units_n = static_cast<size_t>(units) * n * kHG;
    p.ws_bytes = ((units_n * kLatent * 2 + 255) & ~static_cast<size_t>(255)) + units_n * 2 * 4;
  }
  return p;
}

cudaError_t launch_attn(const AttnPlan& pl0, const AttnArgs& a, cudaStream_t stream) {
  if (pl0.rows == 0) return cudaSuccess;
  if (!set_attrs()) return cudaGetLastError();
  AttnPlan pl = pl0;
  if (pl.nsplit > 1) {
    const int n = pick_cluster(pl.nsplit, static_cast<int64_t>(pl.rows) * pl.groups);
    if (n != pl.nsplit) {  // fewer, longer splits
      const int64_t total = static_cast<int64_t>(pl.split_tokens) * pl.nsplit;
      int64_t ts = (total + n - 1) / n;
      pl.split_tokens = static_cast<int>((ts + kTT - 1) / kTT * kTT);
      pl.nsplit = n;
    }
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
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (pl.nsplit > 1) {
    const size_t units_n = static_cast<size_t>(pl.rows) * pl.groups * pl.nsplit * kHG;
    p.part_o = static_cast<__nv_bfloat16*>(a.ws);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) +
                                         ((units_n * kLatent * 2 + 255) & ~static_cast<size_t>(255)));
  }
  cudaError_t e = launch_ex(k_sparse_attn, dim3(pl.nsplit, pl.rows, pl.groups), dim3(kThreads),
                            kSmemBytes, stream, a.pdl, pl.nsplit, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace spx
