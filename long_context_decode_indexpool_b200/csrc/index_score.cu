// Lightning-indexer scoring on the 5th-generation tensor cores; on the
// decode path the epilogue also keeps the key histogram that the top-k
// block selection starts from.
//
// [W4] "GLM-5.3-Flash vs Qwen3.8-Flash-Next: 두 중국 AI 연구소가 독립적으로 같은
// 모델 설계로 수렴한 이유", section "수렴점 2 — 4배 압축 후 2,048 토큰만 유지":
// a 32-head lightning indexer scores the pooled keys and the 512 best 4-token
// blocks are kept.  The score of block b for query t is
// s = sum_h w_{t,h} ReLU(q_{t,h} . k_pool[b]) (the DeepSeek indexer form
// named by [W3] "GLM-5.3 Sparse Attention은 연산량을 줄이지만 HBM 수요는
// 지속된다", section "GLM-5.3 Sparse Attention이 실제로 바꾸는 것").
//
// The dot products form a GEMM with the keys as the M side:
//   D[128 keys x N] = K_tile[128 x 128] * Qg[N x 128]^T,  N = 32 * NQ,
// where Qg stacks the 32 heads of NQ queries that share the key tiles (decode:
// NQ = 1, one query per sequence, its own keys; prefill: NQ = 8 consecutive
// queries of one sequence).  With the keys on M, TMEM lane i holds key i and
// its N head dot products sit in that lane's columns, so the ReLU-weighted
// sum over heads is a per-thread loop in the epilogue: no cross-thread
// reduction at all.
//
// Roles (320 threads, or 576 for eight queries per group; one CTA per SM,
// persistent over a contiguous range of (query group, key tile) work items):
//   warp 0      TMA producer: key tiles into a kStages ring (two 16 KiB
//               boxes of 64 dims, 128-byte swizzle), query groups into
//               kQSlots slots.
//   warp 1      allocates TMEM; issues 8 tcgen05.mma (K = 16 each) per tile
//               into a ring of TMEM accumulators (4 slots for one query per
//               group, 2 for eight), the whole warp running the loop and one
//               elected lane issuing (warp-uniform descriptors).
//   warps 2-9   epilogue: tcgen05.ld of the accumulator row, ReLU, weighted
//               head sum in fp32, length mask; then either a store of the
//               fp32 scores (and, with SELECT, a histogram of their keys).
//               Warps 2-5 take the even tiles, 6-9 the odd ones (4 warps,
//               one per scheduler, left the epilogue latency-bound).
//               With eight queries per group (256 accumulator columns a
//               tile) warps 2-17: the four warps of a TMEM lane quarter take
//               two queries each, so that enough warps hide the latency of
//               the loads and of the head sums to keep up with the MMAs.
//
// SELECT (decode): besides the scores, the epilogue counts the row's keys
// (scores mapped to order-preserving 32-bit keys) in a 2048-bin shared-memory
// histogram of their top 11 bits and adds it into a global per-row histogram
// when it leaves the row.  Once the launch is complete that histogram locates
// the bin of the row's 512th-largest key exactly; the selection kernel
// (topk.cu) then only keeps blocks at or above that bin.
//
// INT8 cache (decode and prefill, [W1] section "양자화: W8A8와 혼합 캐시"):
// the keys are int8 codes with one power-of-two scale per block and the
// query heads come quantised the same way, their scales folded into w.  A
// tile is then one 16 KiB box of 128-byte rows (half the bytes), the MMA is
// 4 tcgen05.mma kind::i8 (K = 32 each) into exact s32 accumulators, and the
// epilogue takes ReLU on the integer dot, sums w_h * dot over the heads in
// fp32 and multiplies by the block's scale.
//
// Before its wait on the previous kernel a CTA sets up its barriers and
// TMEM and, on the decode path, plans its work from the lengths before the
// append and sends its first key tiles to L2; after the wait the plan is
// checked against the lengths the append wrote.
//
// Every wait is bounded; on a timeout the CTA drains and exits with the
// device error word set.
#include "select.cuh"
#include <atomic>

#include "spx_device.cuh"
#include "spx_internal.h"
#include "spx_launch.cuh"

namespace spx {

__device__ int g_device_error = 0;

namespace {

constexpr int kTileM = 128;
constexpr int kHalfBytes = kTileM * 64 * 2;  // 128 rows x 128 bytes: one TMA box
constexpr int kHistBins = 2048;              // top 11 key bits
constexpr int kHistShift = 21;
// Decode work split: each CTA first takes an equal static range of 7/8 of the
// tiles, then the rest in chunks of kDynChunk tiles from an atomic counter,
// so that CTAs that stream faster take more and all finish together.
constexpr int kDynChunk = 4;
constexpr int kMaxDynGroups = 512;
constexpr int kRing = 4;  // chunk indices handed from the TMA warp to the others
constexpr int kPrefetchTiles = 6;  // decode: first tiles of a CTA sent to L2 before the wait

// I8: the INT8 cache: 128-byte key rows (one box per tile), int8 query
// codes, kind::i8 MMAs into s32 accumulators (N = 32 heads for one query,
// 256 for eight).
template <int NQ, bool SELECT, bool I8>
struct Cfg {
  static_assert(!I8 || !SELECT || NQ == 1, "the key histogram is kept for one query per group");
  static constexpr int kN = 32 * NQ;
  static constexpr int kEpiWarps = NQ == 8 ? 16 : 8;
  // one query: two groups of 4 warps take alternate tiles (accumulator
  // slots 0, 2 and 1, 3); eight queries: every warp takes every tile
  static constexpr int kEpiGroups = NQ == 8 ? 1 : 2;
  static constexpr int kEpi = 32 * kEpiWarps;        // epilogue threads
  static constexpr int kThreads = 64 + kEpi;
  static constexpr int kQPerWarp = NQ * 4 * kEpiGroups / kEpiWarps;  // queries of one thread
  static constexpr int kTileBytes = I8 ? kHalfBytes : 2 * kHalfBytes;  // 128 keys
  // I8 with one query: the tile's 128 block scales (512 B) follow it in the
  // stage; with eight (keys shared by the queries, L2-resident) each
  // epilogue thread loads its key's scale while the MMA runs, so the MMA's
  // commit alone releases the stage
  static constexpr bool kScaleInStage = I8 && NQ == 1;
  static constexpr int kStageBytes = kScaleInStage ? kTileBytes + 1024 : kTileBytes;
  static constexpr int kStages = I8 ? 10 : (NQ == 1 ? 6 : 4);
  static constexpr int kQSlots = NQ == 1 ? 2 : 1;
  static constexpr int kQHalf = kN * 128;  // one 128-byte-wide box of Q
  static constexpr int kQBytes = I8 ? kQHalf : 2 * kQHalf;
  // TMEM accumulator ring: 4 slots of 32 columns for one query (the MMA of
  // tile t+4 waits for the epilogue of tile t), 2 of 256 for eight
  static constexpr int kAcc = NQ == 1 ? 4 : 2;
  static constexpr int kTmemCols = kAcc * kN;
  static constexpr int kQOff = kStages * kStageBytes;
  static constexpr int kWOff = kQOff + kQSlots * kQBytes;
  static constexpr int kNbOff = kWOff + kN * 4;
  static constexpr int kSelOff = (kNbOff + NQ * 8 + 15) & ~15;
  static constexpr int kSelBytes =
      SELECT ? kHistBins * 4 : 0;
  static constexpr int kBarOff = (kSelOff + kSelBytes + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * kQSlots + 2 * kAcc + 1;
  static constexpr int kSmem = 1024 + kBarOff + kNumBars * 8 + 16;
  static constexpr uint32_t kIdesc = I8 ? idesc_s8_s32(kTileM, kN) : idesc_bf16_f32(kTileM, kN);
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct KParams {
  const float* w_head;
  const float* k_scale;  // I8: [key batches, cap_blk] block scales
  int64_t cap_blk;
  const int64_t* n_vis;
  const int64_t* len_spec;  // optional: lengths before the append (planning only)
  int n_add;
  float* scores;
  int64_t score_stride;
  int64_t max_len;
  int rows;
  int groups;
  int shared_keys;
  uint32_t* ghist;     // SELECT: [rows, kHistBins] key histogram, zero on entry
  int* work_counter;   // zero on entry; NULL: static split only
};

// (a0, a1) += (w0 x0, w1 x1): one fma.rn.f32x2, each lane rounded once like
// a scalar fma.rn.f32.
__device__ __forceinline__ void ffma2(float& a0, float& a1, float w0, float w1, float x0,
                                      float x1) {
  asm("{\n\t.reg .b64 a, w, x;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 w, {%2, %3};\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "fma.rn.f32x2 a, w, x, a;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(w0), "f"(w1), "f"(x0), "f"(x1));
}

// Pooled blocks of a row: from n_vis or, with `spec`, from the lengths
// before the append the way the pool kernel turns them into n_vis.
template <int NQ>
__device__ __forceinline__ int64_t row_blocks(const KParams& p, int row, bool spec = false) {
  int64_t n;
  if (spec) {
    int64_t len = p.len_spec[row];
    if (len < 0) len = 0;
    if (len > p.max_len - p.n_add) len = p.max_len - p.n_add;
    n = len + p.n_add;
  } else {
    n = p.n_vis[row];
  }
  n = n < 0 ? 0 : (n > p.max_len ? p.max_len : n);
  return n / kPool;
}

template <int NQ>
__device__ __forceinline__ int group_tiles(const KParams& p, int g, bool spec = false) {
  int64_t nb = 0;
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    const int r = g * NQ + j;
    if (r < p.rows) {
      const int64_t v = row_blocks<NQ>(p, r, spec);
      nb = v > nb ? v : nb;
    }
  }
  return static_cast<int>((nb + kTileM - 1) / kTileM);
}

// Walks (group, tile) work items in order; `gstart` is the global index of
// tile 0 of the current group.  `tab` (shared memory, or NULL) holds the
// first flat tile of every group and the total, [groups + 1].
template <int NQ>
struct Walker {
  int g, t, nt;
  int64_t gstart;
  const int* tab;
  __device__ int tiles(const KParams& p, int gg) const {
    return tab ? tab[gg + 1] - tab[gg] : group_tiles<NQ>(p, gg);
  }
  __device__ void init(const KParams& p, int g0, int t0, int64_t lo, const int* tab_) {
    tab = tab_;
    g = g0;
    t = t0;
    nt = tiles(p, g0);
    gstart = lo - t0;
  }
  __device__ void advance(const KParams& p) {
    if (++t >= nt) {
      gstart += nt;
      t = 0;
      do {
        ++g;
        nt = (g < p.groups) ? tiles(p, g) : 1;
      } while (nt == 0);
    }
  }
};

// Shared description of the CTA's work: the static range, then (if enabled)
// chunks of the dynamic pool taken by the TMA warp and posted in a ring.
struct Sched {
  int64_t lo;      // first static item
  int n_static;    // static items
  int g0, t0;      // (group, tile) of item lo
  bool dyn;
  int64_t dyn_begin, total;
  int nchunk;
  const int* pre;  // smem [groups + 1]: first flat tile of each group
  const int* gt;   // the same table when the Walker may use it, or NULL
  int* ring;       // smem [kRing]
  uint64_t* ring_full;
  uint64_t* ring_empty;
  int* counter;
};

enum Role { kProducer, kMmaRole, kEpiRole };

// Yields the CTA's work items in order, the same sequence in every role.
template <int NQ>
struct WorkSrc {
  Walker<NQ> w;
  int left = 0;
  bool started = false;
  int slot = 0;
  uint32_t ph = 0;

  __device__ bool next(const KParams& p, const Sched& sc, Role role, int lane,
                       volatile int* abort) {
    if (!started) {
      started = true;
      if (sc.n_static > 0) {
        w.init(p, sc.g0, sc.t0, sc.lo, sc.gt);
        left = sc.n_static - 1;
        return true;
      }
    } else if (left > 0) {
      w.advance(p);
      --left;
      return true;
    }
    if (!sc.dyn) return false;
    int k;
    if (role == kProducer) {
      // a whole warp: lane 0 takes the chunk and posts it, the warp follows
      int ok = 1, kk = -1;
      if (lane == 0) {
        ok = mbar_wait(&sc.ring_empty[slot], ph ^ 1, abort) ? 1 : 0;
        if (ok) {
          kk = atomicAdd(sc.counter, 1);
          if (kk >= sc.nchunk) kk = -1;
          sc.ring[slot] = kk;
          mbar_arrive(&sc.ring_full[slot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      k = __shfl_sync(0xffffffffu, kk, 0);
      if (!ok) return false;
    } else if (role == kMmaRole) {
      // a whole warp: lane 0 waits and reads the slot, the warp follows
      int ok = 1, kk = -1;
      if (lane == 0) {
        ok = mbar_wait(&sc.ring_full[slot], ph, abort) ? 1 : 0;
        if (ok) kk = sc.ring[slot];
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      k = __shfl_sync(0xffffffffu, kk, 0);
      if (!ok) return false;
      if (lane == 0) mbar_arrive(&sc.ring_empty[slot]);
    } else {
      if (!mbar_wait(&sc.ring_full[slot], ph, abort)) return false;
      k = sc.ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc.ring_empty[slot]);
    }
    if (++slot == kRing) {
      slot = 0;
      ph ^= 1;
    }
    if (k < 0) return false;
    const int64_t f = sc.dyn_begin + static_cast<int64_t>(k) * kDynChunk;
    const int64_t n = sc.total - f < kDynChunk ? sc.total - f : kDynChunk;
    int lo_g = 0, hi_g = p.groups - 1;  // the group g with pre[g] <= f < pre[g+1]
    while (lo_g < hi_g) {
      const int mid = (lo_g + hi_g + 1) >> 1;
      if (sc.pre[mid] <= f) lo_g = mid; else hi_g = mid - 1;
    }
    while (sc.pre[lo_g + 1] <= f) ++lo_g;  // skip groups without tiles
    w.init(p, lo_g, static_cast<int>(f - sc.pre[lo_g]), f, sc.gt);
    left = static_cast<int>(n) - 1;
    return true;
  }
};

}  // namespace

template <int NQ, bool SELECT, bool I8>
__global__ void __launch_bounds__(Cfg<NQ, SELECT, I8>::kThreads, 1)
    k_index_score(const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_q, const KParams p) {
  using C = Cfg<NQ, SELECT, I8>;
  constexpr int kThreads = C::kThreads;
  constexpr int kEpi = C::kEpi;
  auto epi_sync = [] { group_sync<C::kEpi, 1>(); };
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_smem = smem;
  uint8_t* q_smem = smem + C::kQOff;
  float* w_smem = reinterpret_cast<float*>(smem + C::kWOff);
  int64_t* nb_smem = reinterpret_cast<int64_t*>(smem + C::kNbOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + C::kStages;
  uint64_t* qfull = empty + C::kStages;
  uint64_t* qempty = qfull + C::kQSlots;
  uint64_t* accfull = qempty + C::kQSlots;
  uint64_t* accempty = accfull + C::kAcc;
  uint64_t* drain = accempty + C::kAcc;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  __shared__ int s_scan[33];
  __shared__ int s_g0, s_t0;
  __shared__ int s_pre[kMaxDynGroups + 1];
  __shared__ int s_ring[kRing];
  __shared__ __align__(8) uint64_t ring_bars[2 * kRing];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_q);
  }
  pdl_trigger();  // the next kernel's CTAs may be scheduled as SMs free up

  // ---- barriers and TMEM (nothing here depends on the previous kernel) ---
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // I8: full also counts the producer lanes' scale copies, empty the
      // epilogue group that reads the scales
      mbar_init(&full[s], C::kScaleInStage ? 1 + 32 : 1);
      mbar_init(&empty[s], C::kScaleInStage ? 1 + C::kEpiWarps / C::kEpiGroups : 1);
    }
    for (int s = 0; s < C::kQSlots; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
    }
    for (int s = 0; s < C::kAcc; ++s) {
      mbar_init(&accfull[s], 1);
      mbar_init(&accempty[s], C::kEpiWarps / C::kEpiGroups);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&ring_bars[s], 1);  // full: the TMA warp posted a chunk
      mbar_init(&ring_bars[kRing + s], 1 + C::kEpiWarps);  // empty: MMA thread + epilogue warps
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // ---- this CTA's work: a contiguous static range, then dynamic chunks ----
  const bool tab = p.groups <= kMaxDynGroups;         // uniform: tile counts in shared memory
  const bool dyn = p.work_counter != nullptr && tab;  // uniform
  const int64_t G = gridDim.x;
  Sched sc;
  sc.dyn = dyn;
  sc.pre = s_pre;
  sc.gt = tab ? s_pre : nullptr;
  sc.ring = s_ring;
  sc.ring_full = ring_bars;
  sc.ring_empty = ring_bars + kRing;
  sc.counter = p.work_counter;
  // the split of the tiles over the CTAs, from n_vis or (spec) from the
  // lengths before the append
  auto plan = [&](bool spec) {
    int64_t total = 0;
    for (int base = 0; base < p.groups; base += kThreads) {
      const int g = base + tid;
      const int c = g < p.groups ? group_tiles<NQ>(p, g, spec) : 0;
      int sum;
      const int ex = block_excl_scan(c, s_scan, &sum);
      if (tab && g < p.groups) s_pre[g] = static_cast<int>(total + ex);
      total += sum;
    }
    if (tab && tid == 0) s_pre[p.groups] = static_cast<int>(total);
    __syncthreads();
    sc.total = total;
    if (dyn) {
      const int64_t per = total * 7 / (8 * G);
      sc.lo = per * blockIdx.x;
      sc.n_static = static_cast<int>(per);
      sc.dyn_begin = per * G;
      sc.nchunk = static_cast<int>((total - sc.dyn_begin + kDynChunk - 1) / kDynChunk);
    } else {
      sc.lo = total * blockIdx.x / G;
      sc.n_static = static_cast<int>(total * (blockIdx.x + 1) / G - sc.lo);
      sc.dyn_begin = total;
      sc.nchunk = 0;
    }
    sc.g0 = 0;
    sc.t0 = 0;
    if (sc.n_static > 0) {  // uniform
      int64_t run = 0;
      for (int base = 0; base < p.groups; base += kThreads) {
        const int g = base + tid;
        const int c = g < p.groups ? (tab ? s_pre[g + 1] - s_pre[g] : group_tiles<NQ>(p, g, spec)) : 0;
        int sum;
        const int ex = block_excl_scan(c, s_scan, &sum);
        if (c > 0 && run + ex <= sc.lo && sc.lo < run + ex + c) {
          s_g0 = g;
          s_t0 = static_cast<int>(sc.lo - run - ex);
        }
        run += sum;
        if (run > sc.lo) break;  // uniform
      }
      __syncthreads();
      sc.g0 = s_g0;
      sc.t0 = s_t0;
    }
  };
  // Decode plans from the caller's lengths while the previous kernel (the
  // append) still runs, and keeps the plan if n_vis agrees after the wait.
  const bool spec = tab && p.len_spec != nullptr;  // uniform
  if (spec) plan(true);
  if (spec && tid == 0 && sc.n_static > 0) {
    // the first tiles of the static range head for L2 while the append runs
    // (a prefetch reads no data into the CTA, so a plan that turns out
    // wrong costs only the traffic)
    Walker<NQ> pw;
    pw.init(p, sc.g0, sc.t0, sc.lo, sc.gt);
    const int n = sc.n_static < kPrefetchTiles ? sc.n_static : kPrefetchTiles;
    for (int i = 0; i < n; ++i) {
      if (i) pw.advance(p);
      const int kb = p.shared_keys ? 0 : pw.g;
      tma_prefetch_3d(&map_k, 0, pw.t * kTileM, kb);
      if constexpr (!I8) tma_prefetch_3d(&map_k, 64, pw.t * kTileM, kb);
    }
  }
  pdl_wait();  // lengths, keys and the histogram come from the previous kernel
  if (spec) {
    int bad = 0;
    for (int g = tid; g < p.groups; g += kThreads)
      bad |= s_pre[g + 1] - s_pre[g] != group_tiles<NQ>(p, g);
    if (__syncthreads_or(bad)) plan(false);  // uniform
  } else {
    plan(false);
  }
  if (!dyn && sc.n_static <= 0) {  // uniform: no tiles for this CTA
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
    return;
  }

  if (warp == 0) {
    // ======================= TMA producer =================================
    // The whole warp runs the loop (lane 0 waits and issues the TMA copies;
    // with the INT8 cache every lane also copies four block scales).
    auto wait0 = [&](uint64_t* bar, uint32_t parity) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    // per-row keys are read once (decode); keys shared by every query
    // group (prefill) are re-read from L2
    const uint64_t stream_pol = p.shared_keys ? l2_evict_normal_policy() : l2_evict_first_policy();
    WorkSrc<NQ> src;
    const Walker<NQ>& w = src.w;
    int stage = 0, cur_g = -1, qs = C::kQSlots - 1;
    uint32_t ph = 0, qe_ph[2] = {0, 0};
    int issued = 0, q_issued_slot = -1;
    uint32_t q_issued_ph = 0;
    while (src.next(p, sc, kProducer, lane, abort_flag)) {
      if (w.g != cur_g) {
        qs = (qs + 1) % C::kQSlots;
        if (!wait0(&qempty[qs], qe_ph[qs] ^ 1)) break;
        qe_ph[qs] ^= 1;
        if (lane == 0) {
          uint8_t* dst = q_smem + qs * C::kQBytes;
          mbar_arrive_expect_tx(&qfull[qs], C::kQBytes);
          tma_load_2d(dst, &map_q, &qfull[qs], 0, w.g * C::kN);
          if constexpr (!I8) tma_load_2d(dst + C::kQHalf, &map_q, &qfull[qs], 64, w.g * C::kN);
        }
        q_issued_slot = qs;
        q_issued_ph = qe_ph[qs] ^ 1;
        cur_g = w.g;
      }
      if (!wait0(&empty[stage], ph ^ 1)) break;
      uint8_t* dst = a_smem + stage * C::kStageBytes;
      const int kb = p.shared_keys ? 0 : w.g;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[stage], C::kTileBytes);
        tma_load_3d_hint(dst, &map_k, &full[stage], 0, w.t * kTileM, kb, stream_pol);
        if constexpr (!I8)
          tma_load_3d_hint(dst + kHalfBytes, &map_k, &full[stage], 64, w.t * kTileM, kb, stream_pol);
      }
      if constexpr (C::kScaleInStage) {
        // the tile's 128 block scales into the stage behind the codes (zeros
        // past the cache); each lane's copies arrive on the stage's barrier
        // when they land, so the epilogue reads them from shared memory
        const int64_t base = static_cast<int64_t>(kb) * p.cap_blk + static_cast<int64_t>(w.t) * kTileM;
        const int64_t left = p.cap_blk - static_cast<int64_t>(w.t) * kTileM;
        const uint32_t sdst = smem_u32(dst + C::kTileBytes);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = lane * 4 + u;
          const bool v = j < left;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(sdst + j * 4),
                       "l"(v ? p.k_scale + base + j : p.k_scale), "r"(v ? 4 : 0)
                       : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                         smem_u32(&full[stage]))
                     : "memory");
      }
      ++issued;
      if (++stage == C::kStages) {
        stage = 0;
        ph ^= 1;
      }
    }
    if (*abort_flag) {
      // Let the copies already issued land before the CTA exits.
      if constexpr (C::kScaleInStage) asm volatile("cp.async.wait_all;" ::: "memory");
      if (lane == 0) {
        const int first = issued > C::kStages ? issued - C::kStages : 0;
        for (int i = first; i < issued; ++i) {
          volatile int no_abort = 0;
          mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1, &no_abort);
        }
        if (q_issued_slot >= 0) {
          volatile int no_abort = 0;
          mbar_wait(&qfull[q_issued_slot], q_issued_ph, &no_abort);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer ====================================
    // The whole warp runs the loop (lane 0 waits on the barriers and the warp
    // follows its result), so the descriptors are warp-uniform and one
    // elected lane issues each MMA.
    auto wait0 = [&](uint64_t* bar, uint32_t parity) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    WorkSrc<NQ> src;
    const Walker<NQ>& w = src.w;
    int stage = 0, acc = 0, cur_g = -1, qs = C::kQSlots - 1;
    uint32_t ph = 0, acc_ph = 0, qf_ph[2] = {0, 0};
    const uint32_t a_base = smem_u32(a_smem);
    const uint32_t q_base = smem_u32(q_smem);
    while (src.next(p, sc, kMmaRole, lane, abort_flag)) {
      if (w.g != cur_g) {
        if (cur_g >= 0) umma_commit_elect(&qempty[qs]);
        qs = (qs + 1) % C::kQSlots;
        if (!wait0(&qfull[qs], qf_ph[qs])) break;
        qf_ph[qs] ^= 1;
        cur_g = w.g;
      }
      if (!wait0(&accempty[acc], acc_ph ^ 1)) break;
      if (!wait0(&full[stage], ph)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::kN);
      const uint32_t a0 = a_base + stage * C::kStageBytes;
      const uint32_t b0 = q_base + qs * C::kQBytes;
      if constexpr (I8) {
        // K = 32 int8 per MMA: four 32-byte steps along the 128-byte rows
#pragma unroll
        for (int k = 0; k < kIdxDim / 32; ++k) {
          const uint64_t ad = sdesc_kmajor_sw128(a0 + k * 32);
          const uint64_t bd = sdesc_kmajor_sw128(b0 + k * 32);
          umma_s8_elect(d, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
        }
      } else {
#pragma unroll
        for (int k = 0; k < kIdxDim / 16; ++k) {
          const uint32_t koff = (k & 3) * 32;
          const uint64_t ad = sdesc_kmajor_sw128(a0 + (k >> 2) * kHalfBytes + koff);
          const uint64_t bd = sdesc_kmajor_sw128(b0 + (k >> 2) * C::kQHalf + koff);
          umma_bf16_elect(d, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
        }
      }
      umma_commit_elect(&empty[stage]);
      umma_commit_elect(&accfull[acc]);
      if (++stage == C::kStages) {
        stage = 0;
        ph ^= 1;
      }
      if (++acc == C::kAcc) {
        acc = 0;
        acc_ph ^= 1;
      }
    }
    // Wait for every MMA issued by this warp before TMEM is released.
    umma_commit_elect(drain);
    if (lane == 0) {
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
    __syncwarp();
  } else {
    // ======================= epilogue =====================================
    const int quarter = warp & 3;  // TMEM lanes quarter*32 .. +31
    const int et = tid - 64;       // 0 .. kEpi-1
    const int row_in_tile = quarter * 32 + lane;
    const int wq = (warp - 2) >> 2;                  // this warp's set of 4
    const int grp = wq % C::kEpiGroups;              // tiles with seq % groups == grp
    const int q0 = (wq / C::kEpiGroups) * C::kQPerWarp;  // first query of this thread
    static_assert(C::kAcc % C::kEpiGroups == 0, "a group owns whole accumulator slots");
    int seq = 0, est = 0;  // tile sequence number; its key stage (I8 scales)
    uint32_t est_ph = 0;
    WorkSrc<NQ> src;
    const Walker<NQ>& w = src.w;
    int acc = 0, cur_g = -1;
    uint32_t acc_ph = 0;
    bool aborted = false;

    uint32_t* lhist = reinterpret_cast<uint32_t*>(smem + C::kSelOff);  // SELECT
    if constexpr (SELECT) {
      for (int b = et; b < kHistBins; b += kEpi) lhist[b] = 0;
      epi_sync();
    }
    // Leaves row r (SELECT): adds the CTA's counts into the row's histogram.
    auto flush_hist = [&](int r) {
      uint32_t* gh = p.ghist + static_cast<int64_t>(r) * kHistBins;
      epi_sync();
#pragma unroll 4
      for (int b = et; b < kHistBins; b += kEpi) {
        const uint32_t c = lhist[b];
        if (c) {
          atomicAdd(gh + b, c);
          lhist[b] = 0;
        }
      }
      epi_sync();
    };

    while (src.next(p, sc, kEpiRole, lane, abort_flag)) {
      if (w.g != cur_g) {
        if constexpr (SELECT) {
          if (cur_g >= 0) flush_hist(cur_g);
        }
        epi_sync();
        for (int j = et; j < C::kN; j += kEpi) {
          const int r = w.g * NQ + j / kIdxHeads;
          w_smem[j] = r < p.rows ? p.w_head[static_cast<int64_t>(r) * kIdxHeads + (j % kIdxHeads)] : 0.f;
        }
        if (et < NQ) {
          const int r = w.g * NQ + et;
          nb_smem[et] = r < p.rows ? row_blocks<NQ>(p, r) : 0;
        }
        epi_sync();
        cur_g = w.g;
      }
      const int my_st = est;
      const uint32_t my_st_ph = est_ph;
      if (++est == C::kStages) {
        est = 0;
        est_ph ^= 1;
      }
      if ((seq++ % C::kEpiGroups) != grp) {  // the other group's tile
        if (++acc == C::kAcc) {
          acc = 0;
          acc_ph ^= 1;
        }
        continue;
      }
      const int64_t blk = static_cast<int64_t>(w.t) * kTileM + row_in_tile;
      float ksc = 1.f;  // I8: the block's scale
      if constexpr (I8 && !C::kScaleInStage) {
        const int kb = p.shared_keys ? 0 : w.g;
        if (blk < p.cap_blk) ksc = __ldg(p.k_scale + static_cast<int64_t>(kb) * p.cap_blk + blk);
      }
      if (!mbar_wait(&accfull[acc], acc_ph, abort_flag)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      if constexpr (C::kScaleInStage) {
        // (the stage's barrier completed before the MMA ran; waiting on it
        // again orders the scale copies before these reads)
        if (!mbar_wait(&full[my_st], my_st_ph, abort_flag)) {
          aborted = true;
          break;
        }
        ksc = reinterpret_cast<const float*>(a_smem + my_st * C::kStageBytes +
                                             C::kTileBytes)[row_in_tile];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[my_st]);  // this warp is done with the stage
      }
      constexpr int kQ = C::kQPerWarp;
      float scv[kQ];
      // ReLU-weighted head sum of one query's 32 accumulator columns; four
      // interleaved partial sums over the heads (short dependency chains)
      auto head_sum = [&](const uint32_t* v, int j) {
        const float* wj = w_smem + j * kIdxHeads;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        auto relu = [&](int h) {
          if constexpr (I8) {
            const int dot = static_cast<int>(v[h]);  // exact s32 dot product
            return static_cast<float>(dot > 0 ? dot : 0);
          } else {
            const float f = __uint_as_float(v[h]);
            return f > 0.f ? f : 0.f;
          }
        };
        // heads h and h+1 go to partial sums h & 3 and (h & 3) + 1 with one
        // paired fp32 FMA (each lane rounds as a scalar FMA would)
#pragma unroll
        for (int h = 0; h < kIdxHeads; h += 2)
          ffma2(s4[h & 3], s4[(h & 3) + 1], wj[h], wj[h + 1], relu(h), relu(h + 1));
        float sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        if constexpr (I8) sc *= ksc;
        return sc;
      };
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(acc * C::kN);
#pragma unroll
      for (int j = 0; j < kQ; ++j) {
        uint32_t v[32];
        tmem_ld_x32_async(trow + (q0 + j) * 32, v);
        tmem_ld_wait_regs<32>(v);
        scv[j] = head_sum(v, q0 + j);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
      if (++acc == C::kAcc) {
        acc = 0;
        acc_ph ^= 1;
      }

#pragma unroll
      for (int j = 0; j < kQ; ++j) {
        const int r = w.g * NQ + q0 + j;
        if (r < p.rows && blk < nb_smem[q0 + j]) {
          p.scores[static_cast<int64_t>(r) * p.score_stride + blk] = scv[j];
          if constexpr (SELECT) atomicAdd(&lhist[order_key(scv[j]) >> kHistShift], 1u);
        }
      }
    }
    if constexpr (SELECT) {
      if (!aborted && cur_g >= 0) flush_hist(cur_g);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

namespace {

template <int NQ, bool SELECT, bool I8>
cudaError_t launch_cfg(const ScoreArgs& a, cudaStream_t stream) {
  using C = Cfg<NQ, SELECT, I8>;
  CUtensorMap map_k, map_q;
  if constexpr (I8) {
    // one 128-byte row per key and per query head
    const uint64_t dims[3] = {static_cast<uint64_t>(kIdxDim), static_cast<uint64_t>(a.cap_blk),
                              static_cast<uint64_t>(a.key_batches)};
    const uint64_t strides[2] = {kIdxDim * 1ull, static_cast<uint64_t>(a.cap_blk) * kIdxDim};
    const uint32_t box[3] = {kIdxDim, kTileM, 1};
    if (!encode_tensor_map(&map_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.pooled_k, dims, strides,
                           box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const uint64_t qdims[2] = {static_cast<uint64_t>(kIdxDim),
                               static_cast<uint64_t>(a.rows) * kIdxHeads};
    const uint64_t qstrides[1] = {kIdxDim * 1ull};
    const uint32_t qbox[2] = {kIdxDim, static_cast<uint32_t>(C::kN)};
    if (!encode_tensor_map(&map_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q_idx, qdims, qstrides,
                           qbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {static_cast<uint64_t>(kIdxDim), static_cast<uint64_t>(a.cap_blk),
                              static_cast<uint64_t>(a.key_batches)};
    const uint64_t strides[2] = {kIdxDim * 2ull, static_cast<uint64_t>(a.cap_blk) * kIdxDim * 2ull};
    const uint32_t box[3] = {64, kTileM, 1};
    if (!encode_tensor_map(&map_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.pooled_k, dims,
                           strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const uint64_t qdims[2] = {static_cast<uint64_t>(kIdxDim),
                               static_cast<uint64_t>(a.rows) * kIdxHeads};
    const uint64_t qstrides[1] = {kIdxDim * 2ull};
    const uint32_t qbox[2] = {64, static_cast<uint32_t>(C::kN)};
    if (!encode_tensor_map(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q_idx, qdims, qstrides,
                           qbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64;  // devices beyond the cache: set every call
  if (!cached || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_index_score<NQ, SELECT, I8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    if (cached) attr_set[dev] = true;
  }
  KParams p{};
  p.w_head = a.w_head;
  p.k_scale = a.k_scale;
  p.cap_blk = a.cap_blk;
  p.n_vis = a.n_vis;
  p.len_spec = a.len_spec;
  p.n_add = a.n_add;
  p.scores = a.scores;
  p.score_stride = a.score_stride;
  p.max_len = a.max_len;
  p.rows = a.rows;
  p.groups = (a.rows + NQ - 1) / NQ;
  p.shared_keys = a.key_batches == 1 ? 1 : 0;
  p.ghist = a.sel_ghist;
  p.work_counter = a.work_counter;
  const int grid = score_grid(a.nq, a.rows, a.max_len, a.num_sms);
  if (grid == 0) return cudaSuccess;
  cudaError_t e = launch_ex(k_index_score<NQ, SELECT, I8>, dim3(grid), dim3(C::kThreads), C::kSmem,
                            stream, a.pdl, 1, map_k, map_q, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int score_grid(int nq, int rows, int64_t max_len, int num_sms) {
  const int groups = (rows + nq - 1) / nq;
  const int64_t max_blk = max_len / kPool;
  const int64_t tiles_ub = static_cast<int64_t>(groups) * ((max_blk + kTileM - 1) / kTileM);
  return static_cast<int>(tiles_ub < num_sms ? tiles_ub : num_sms);
}

cudaError_t launch_index_score(const ScoreArgs& a, cudaStream_t stream) {
  if (a.nq == 1) {
    if (a.i8) {
      if (a.sel_ghist) return launch_cfg<1, true, true>(a, stream);
      return launch_cfg<1, false, true>(a, stream);
    }
    if (a.sel_ghist) return launch_cfg<1, true, false>(a, stream);
    return launch_cfg<1, false, false>(a, stream);
  }
  if (a.nq == 8) {
    if (a.i8) return launch_cfg<8, false, true>(a, stream);
    return launch_cfg<8, false, false>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace spx
