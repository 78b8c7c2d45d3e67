// Lightning-indexer scoring on the 5th-generation tensor cores, with the
// top-k block selection fused into the epilogue on the decode path.
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
// Roles (192 threads, one CTA per SM, persistent over a contiguous range of
// (query group, key tile) work items):
//   warp 0      TMA producer: key tiles into a kStages ring (two 16 KiB
//               boxes of 64 dims, 128-byte swizzle), query groups into
//               kQSlots slots.
//   warp 1      allocates TMEM; one lane issues 8 tcgen05.mma (K = 16 each)
//               per tile into one of two TMEM accumulators.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator row, ReLU, weighted
//               head sum in fp32, length mask; then either a store of the
//               fp32 scores, or (SELECT) the fused top-k below.
//
// Fused top-k, first stage (SELECT, decode): the epilogue keeps, per row, an
// index-ordered buffer of candidate blocks in shared memory.  A candidate
// enters only if its key is >= theta, a lower bound of the row's final
// 512th-largest key:
//   * from time to time the CTA adds its 2048-bin histogram of the row's keys
//     (top 11 key bits) into a global per-row histogram and takes an
//     asynchronous snapshot of it (cp.async); at the next flush the highest
//     bin b with at least 512 keys at or above it in the snapshot gives
//     theta >= b's lower edge (any snapshot of monotone counts is a valid
//     lower bound);
//   * when the buffer fills, an exact in-place top-512 of the buffer raises
//     the admission bound to its 512th key + 1 (a later, higher-index
//     candidate equal to it loses the tie), while the buffered ties at that
//     key stay eligible (they are filtered with the key itself).
// When the CTA leaves a row it publishes its list (<= 512 entries, index
// order) and, if it holds the row's first or last tile, its own index.  The
// second stage (k_select_merge in topk.cu, the next launch) reads the
// complete histogram, filters the lists of the row's CTAs (CTA order = index
// order) and selects the 512 block ids.  The union of per-chunk exact top-512
// lists contains the row's top-512, so the result is exact.
//
// Every wait is bounded; on a timeout the CTA drains and exits with the
// device error word set.
#include "select.cuh"
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

__device__ int g_device_error = 0;

namespace {

constexpr int kTileM = 128;
constexpr int kHalfBytes = kTileM * 64 * 2;  // 128 rows x 128 bytes
constexpr int kTileBytes = 2 * kHalfBytes;   // 32 KiB: one tile of 128 keys
constexpr int kThreads = 192;
constexpr int kEpi = 128;                    // epilogue threads
constexpr int kHistBins = 2048;              // top 11 key bits
constexpr int kHistShift = 21;
constexpr int kBufCap = 2048;                // candidate buffer entries
constexpr int kEarlyFlush = 4;               // tiles between the first two flushes
constexpr int kFlushTiles = 16;              // tiles between later flushes

template <int NQ, bool SELECT>
struct Cfg {
  static constexpr int kN = 32 * NQ;
  static constexpr int kStages = SELECT ? 5 : (NQ == 1 ? 6 : 4);
  static constexpr int kQSlots = NQ == 1 ? 2 : 1;
  static constexpr int kQHalf = kN * 128;
  static constexpr int kQBytes = 2 * kQHalf;
  static constexpr int kTmemCols = 2 * kN;
  static constexpr int kQOff = kStages * kTileBytes;
  static constexpr int kWOff = kQOff + kQSlots * kQBytes;
  static constexpr int kNbOff = kWOff + kN * 4;
  static constexpr int kSelOff = (kNbOff + NQ * 8 + 15) & ~15;
  static constexpr int kSelBytes =
      SELECT ? (2 * kHistBins * 4 + pad32(kBufCap) * 8 + static_cast<int>(sizeof(SelectSmem)) + 64 +
                (kEpi + 1) * 4)
             : 0;
  static constexpr int kBarOff = (kSelOff + kSelBytes + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * kQSlots + 4 + 1;
  static constexpr int kSmem = 1024 + kBarOff + kNumBars * 8 + 16;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, kN);
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct KParams {
  const float* w_head;
  const int64_t* n_vis;
  float* scores;
  int64_t score_stride;
  int64_t max_len;
  int rows;
  int groups;
  int shared_keys;
  // fused selection, first stage (decode)
  uint32_t* ghist;     // [rows, kHistBins]  zero on entry
  uint32_t* list_key;  // [grid + rows, 512]
  int32_t* list_idx;   // [grid + rows, 512]
  int32_t* list_cnt;   // [grid + rows]
  int32_t* row_first;  // [rows] CTA holding the row's first tile (-1 on entry)
  int32_t* row_last;   // [rows] CTA holding the row's last tile (-1 on entry)
  int64_t* total_out;  // [1] total tiles of the launch
};

template <int NQ>
__device__ __forceinline__ int64_t row_blocks(const KParams& p, int row) {
  int64_t n = p.n_vis[row];
  n = n < 0 ? 0 : (n > p.max_len ? p.max_len : n);
  return n / kPool;
}

template <int NQ>
__device__ __forceinline__ int group_tiles(const KParams& p, int g) {
  int64_t nb = 0;
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    const int r = g * NQ + j;
    if (r < p.rows) {
      const int64_t v = row_blocks<NQ>(p, r);
      nb = v > nb ? v : nb;
    }
  }
  return static_cast<int>((nb + kTileM - 1) / kTileM);
}

// Walks (group, tile) work items in order; `gstart` is the global index of
// tile 0 of the current group.
template <int NQ>
struct Walker {
  int g, t, nt;
  int64_t gstart;
  __device__ void init(const KParams& p, int g0, int t0, int64_t lo) {
    g = g0;
    t = t0;
    nt = group_tiles<NQ>(p, g0);
    gstart = lo - t0;
  }
  __device__ void advance(const KParams& p) {
    if (++t >= nt) {
      gstart += nt;
      t = 0;
      do {
        ++g;
        nt = (g < p.groups) ? group_tiles<NQ>(p, g) : 1;
      } while (nt == 0);
    }
  }
};

__device__ __forceinline__ void epi_sync() { group_sync<kEpi, 1>(); }

// ---------------------------------------------------------------------------
// Fused selection state of the epilogue warps (SELECT only).
// ---------------------------------------------------------------------------
struct SelState {
  uint32_t* lhist;     // smem [kHistBins]: this CTA's counts since the last flush
  uint32_t* snap;      // smem [kHistBins]: snapshot of the global histogram
  uint32_t* buf_key;   // smem [kBufCap]
  int32_t* buf_idx;    // smem [kBufCap]
  SelectSmem* ss;      // smem
  int* wcnt;           // smem [2][4]
  int* misc;           // smem [8]: threshold broadcast
  int* seg_off;        // smem [kEpi + 1]: list offsets during a merge
  int nbuf;
  int par;
  int since_flush;
  bool snap_pending;   // a snapshot copy is in flight (cp.async group)
  int flushes;         // flushes done in the current row
  uint32_t theta;      // admission bound for new (higher-index) candidates
  uint32_t tkeep;      // bound for candidates already in the buffer (<= theta)
};

// Appends the passing elements of the 128 epilogue threads to the buffer in
// the order (slot, lane), slot in [0, 4).
__device__ __forceinline__ void sel_append(SelState& S, bool pass, uint32_t key, int32_t idx,
                                           int slot, int lane) {
  const unsigned bal = __ballot_sync(0xffffffffu, pass);
  if (lane == 0) S.wcnt[S.par * 4 + slot] = __popc(bal);
  epi_sync();
  int off = 0, tot = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = S.wcnt[S.par * 4 + q];
    off += q < slot ? c : 0;
    tot += c;
  }
  if (pass) {
    const int pos = S.nbuf + off + __popc(bal & ((1u << lane) - 1u));
    S.buf_key[pad32(pos)] = key;
    S.buf_idx[pad32(pos)] = idx;
  }
  S.nbuf += tot;
  S.par ^= 1;
}

// Exact in-place top-K of the buffer among keys >= tkeep; raises the bounds.
__device__ __forceinline__ void sel_compact(SelState& S, int et) {
  epi_sync();
  uint32_t key[16];
  int32_t idx[16];
  uint32_t valid = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int j = et * 16 + i;
    key[i] = 0;
    idx[i] = 0;
    if (j < S.nbuf) {
      key[i] = S.buf_key[pad32(j)];
      idx[i] = S.buf_idx[pad32(j)];
      if (key[i] >= S.tkeep) valid |= 1u << i;
    }
  }
  epi_sync();
  uint32_t thr;
  const int n = group_select<16, kEpi, 1>(key, valid, kTopK, et, *S.ss, &thr, [&](int i, int pos) {
    S.buf_key[pad32(pos)] = key[i];
    S.buf_idx[pad32(pos)] = idx[i];
  });
  if (thr != 0) {
    // Later arrivals have higher block ids, so one equal to thr loses to the
    // kept ties: admit only keys above thr.  Kept entries equal to thr stay.
    const uint32_t t1 = thr == 0xFFFFFFFFu ? thr : thr + 1;
    S.theta = t1 > S.theta ? t1 : S.theta;
    S.tkeep = thr > S.tkeep ? thr : S.tkeep;
  }
  S.nbuf = n;
  epi_sync();
}

// Lower bound of the row's K-th largest key from a histogram `h` (shared
// or global memory, kHistBins counts).  Thread et reads bins
// kHistBins-1 - (j*128 + et): chunk j holds 128 consecutive bins in
// descending order.  Chunk totals locate the chunk where the count from the
// top reaches K, a scan inside it the bin.
template <bool kGlobal>
__device__ __forceinline__ uint32_t hist_threshold(const SelState& S, const uint32_t* h, int et) {
  constexpr int kChunks = kHistBins / kEpi;
  const int lane = et & 31, wid = et >> 5;
  int c[kChunks];
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    const uint32_t* a = h + (kHistBins - 1 - (j * kEpi + et));
    c[j] = static_cast<int>(kGlobal ? __ldcg(a) : *a);
  }
  int mine = 0;
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    int v = c[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == j) mine = v;
  }
  int* tmp = S.ss->hist;  // [4][32]; no selection runs concurrently
  tmp[wid * 32 + lane] = lane < kChunks ? mine : 0;
  epi_sync();
  if (wid == 0) {
    const int tj = tmp[lane] + tmp[32 + lane] + tmp[64 + lane] + tmp[96 + lane];
    const int incl = warp_incl_scan(tj);
    const int excl = incl - tj;
    const unsigned m = __ballot_sync(0xffffffffu, excl < kTopK && kTopK <= incl);
    const int J = m ? __ffs(m) - 1 : -1;
    const int before = __shfl_sync(0xffffffffu, excl, J < 0 ? 0 : J);
    if (lane == 0) {
      S.misc[2] = J;
      S.misc[3] = before;
      S.misc[1] = 0;
    }
  }
  epi_sync();
  const int J = S.misc[2];
  if (J >= 0) {  // uniform
    const int before = S.misc[3];
    int v = 0;
#pragma unroll
    for (int j = 0; j < kChunks; ++j) v = (j == J) ? c[j] : v;
    int tot;
    const int ex = group_excl_scan<kEpi, 1>(v, et, S.ss->scan, &tot);
    if (before + ex < kTopK && kTopK <= before + ex + v)
      S.misc[1] = static_cast<int>(static_cast<uint32_t>(kHistBins - 1 - (J * kEpi + et)) << kHistShift);
    epi_sync();
  }
  const uint32_t t = static_cast<uint32_t>(S.misc[1]);
  epi_sync();
  return t;
}

// Snapshot of the row's global histogram into shared memory, in flight
// until the next flush (16-byte cp.async through L2).
__device__ __forceinline__ void snap_issue(SelState& S, const uint32_t* gh, int et) {
  const uint32_t dst = smem_u32(S.snap);
#pragma unroll
  for (int i = 0; i < (kHistBins * 4) / (16 * kEpi); ++i) {
    const int c = i * kEpi + et;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + c * 16),
                 "l"(reinterpret_cast<const uint8_t*>(gh) + c * 16)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  S.snap_pending = true;
}

__device__ __forceinline__ void snap_wait(SelState& S) {
  if (S.snap_pending) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    S.snap_pending = false;
  }
}

// Adds the CTA's local counts into the row's global histogram (bins
// j*128 + et: no shared-memory bank conflicts), tightens theta from the
// snapshot taken at the previous flush, and starts the next snapshot.
__device__ __forceinline__ void sel_flush(SelState& S, uint32_t* gh, int et, bool have_snap) {
  snap_wait(S);
  epi_sync();
#pragma unroll 8
  for (int j = 0; j < kHistBins / kEpi; ++j) {
    const int b = j * kEpi + et;
    const uint32_t c = S.lhist[b];
    if (c) {
      atomicAdd(gh + b, c);
      S.lhist[b] = 0;
    }
  }
  if (have_snap) {
    const uint32_t t = hist_threshold<false>(S, S.snap, et);
    S.theta = t > S.theta ? t : S.theta;
    S.tkeep = t > S.tkeep ? t : S.tkeep;
  }
  epi_sync();  // every thread is done with the old snapshot
  snap_issue(S, gh, et);
  S.since_flush = 0;
}

}  // namespace

template <int NQ, bool SELECT>
__global__ void __launch_bounds__(kThreads, 1)
    k_index_score(const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_q, const KParams p) {
  using C = Cfg<NQ, SELECT>;
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
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  __shared__ int s_scan[33];
  __shared__ int s_g0, s_t0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- locate this CTA's contiguous range of work items -------------------
  int64_t total = 0;
  for (int base = 0; base < p.groups; base += kThreads) {
    const int g = base + tid;
    int sum;
    block_excl_scan(g < p.groups ? group_tiles<NQ>(p, g) : 0, s_scan, &sum);
    total += sum;
  }
  const int64_t G = gridDim.x;
  const int64_t lo = total * blockIdx.x / G;
  const int64_t hi = total * (blockIdx.x + 1) / G;
  if (lo >= hi) return;  // uniform
  {
    int64_t run = 0;
    for (int base = 0; base < p.groups; base += kThreads) {
      const int g = base + tid;
      const int c = g < p.groups ? group_tiles<NQ>(p, g) : 0;
      int sum;
      const int ex = block_excl_scan(c, s_scan, &sum);
      if (c > 0 && run + ex <= lo && lo < run + ex + c) {
        s_g0 = g;
        s_t0 = static_cast<int>(lo - run - ex);
      }
      run += sum;
      if (run > lo) break;  // uniform
    }
  }
  const int n_items = static_cast<int>(hi - lo);

  // ---- barriers and TMEM ---------------------------------------------------
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::kQSlots; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&accfull[s], 1);
      mbar_init(&accempty[s], 4);
    }
    mbar_init(drain, 1);
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

  if (warp == 0) {
    // ======================= TMA producer =================================
    if (lane == 0) {
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_q);
      // per-row keys are read once (decode); keys shared by every query
      // group (prefill) are re-read from L2
      const uint64_t stream_pol = p.shared_keys ? l2_evict_normal_policy() : l2_evict_first_policy();
      Walker<NQ> w;
      w.init(p, s_g0, s_t0, lo);
      int stage = 0, cur_g = -1, qs = C::kQSlots - 1;
      uint32_t ph = 0, qe_ph[2] = {0, 0};
      int issued = 0, q_issued_slot = -1;
      uint32_t q_issued_ph = 0;
      for (int i = 0; i < n_items; ++i) {
        if (w.g != cur_g) {
          qs = (qs + 1) % C::kQSlots;
          if (!mbar_wait(&qempty[qs], qe_ph[qs] ^ 1, abort_flag)) break;
          qe_ph[qs] ^= 1;
          uint8_t* dst = q_smem + qs * C::kQBytes;
          mbar_arrive_expect_tx(&qfull[qs], C::kQBytes);
          tma_load_2d(dst, &map_q, &qfull[qs], 0, w.g * C::kN);
          tma_load_2d(dst + C::kQHalf, &map_q, &qfull[qs], 64, w.g * C::kN);
          q_issued_slot = qs;
          q_issued_ph = qe_ph[qs] ^ 1;
          cur_g = w.g;
        }
        if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag)) break;
        uint8_t* dst = a_smem + stage * kTileBytes;
        const int kb = p.shared_keys ? 0 : w.g;
        mbar_arrive_expect_tx(&full[stage], kTileBytes);
        tma_load_3d_hint(dst, &map_k, &full[stage], 0, w.t * kTileM, kb, stream_pol);
        tma_load_3d_hint(dst + kHalfBytes, &map_k, &full[stage], 64, w.t * kTileM, kb, stream_pol);
        ++issued;
        if (++stage == C::kStages) {
          stage = 0;
          ph ^= 1;
        }
        w.advance(p);
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA exits.
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
  } else if (warp == 1) {
    // ======================= MMA issuer ====================================
    if (lane == 0) {
      Walker<NQ> w;
      w.init(p, s_g0, s_t0, lo);
      int stage = 0, acc = 0, cur_g = -1, qs = C::kQSlots - 1;
      uint32_t ph = 0, acc_ph = 0, qf_ph[2] = {0, 0};
      const uint32_t a_base = smem_u32(a_smem);
      const uint32_t q_base = smem_u32(q_smem);
      for (int i = 0; i < n_items; ++i) {
        if (w.g != cur_g) {
          if (cur_g >= 0) umma_commit(&qempty[qs]);
          qs = (qs + 1) % C::kQSlots;
          if (!mbar_wait(&qfull[qs], qf_ph[qs], abort_flag)) break;
          qf_ph[qs] ^= 1;
          cur_g = w.g;
        }
        if (!mbar_wait(&accempty[acc], acc_ph ^ 1, abort_flag)) break;
        if (!mbar_wait(&full[stage], ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::kN);
        const uint32_t a0 = a_base + stage * kTileBytes;
        const uint32_t b0 = q_base + qs * C::kQBytes;
#pragma unroll
        for (int k = 0; k < kIdxDim / 16; ++k) {
          const uint32_t koff = (k & 3) * 32;
          const uint64_t ad = sdesc_kmajor_sw128(a0 + (k >> 2) * kHalfBytes + koff);
          const uint64_t bd = sdesc_kmajor_sw128(b0 + (k >> 2) * C::kQHalf + koff);
          umma_bf16(d, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        umma_commit(&accfull[acc]);
        if (++stage == C::kStages) {
          stage = 0;
          ph ^= 1;
        }
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
        w.advance(p);
      }
      // Wait for every MMA issued by this thread before TMEM is released.
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ======================= epilogue =====================================
    const int quarter = warp & 3;  // TMEM lanes quarter*32 .. +31
    const int et = tid - 64;       // 0..127
    const int row_in_tile = quarter * 32 + lane;
    Walker<NQ> w;
    w.init(p, s_g0, s_t0, lo);
    int acc = 0, cur_g = -1, cur_nt = 0;
    int64_t cur_gstart = 0;
    uint32_t acc_ph = 0;
    bool aborted = false;

    SelState S;
    if constexpr (SELECT) {
      uint8_t* sel = smem + C::kSelOff;
      S.lhist = reinterpret_cast<uint32_t*>(sel);
      S.snap = S.lhist + kHistBins;
      S.buf_key = S.snap + kHistBins;
      S.buf_idx = reinterpret_cast<int32_t*>(S.buf_key + pad32(kBufCap));
      S.ss = reinterpret_cast<SelectSmem*>(S.buf_idx + pad32(kBufCap));
      S.wcnt = reinterpret_cast<int*>(S.ss + 1);
      S.misc = S.wcnt + 8;
      S.seg_off = S.misc + 8;
      S.nbuf = 0;
      S.par = 0;
      S.since_flush = 0;
      S.snap_pending = false;
      S.flushes = 0;
      S.theta = 0;
      S.tkeep = 0;
      for (int b = et; b < kHistBins; b += kEpi) S.lhist[b] = 0;
      epi_sync();
    }

    // Leaves row r: flush the counts, filter with the freshest snapshot,
    // publish this CTA's list (and its index if it holds an end of the row).
    auto finish_row = [&](int r, int64_t gstart, int nt) {
      uint32_t* gh = p.ghist + static_cast<int64_t>(r) * kHistBins;
      sel_flush(S, gh, et, S.snap_pending);
      snap_wait(S);
      epi_sync();
      {
        const uint32_t t = hist_threshold<false>(S, S.snap, et);
        S.theta = t > S.theta ? t : S.theta;
        S.tkeep = t > S.tkeep ? t : S.tkeep;
      }
      sel_compact(S, et);
      const int64_t slot = static_cast<int64_t>(blockIdx.x) + r;
      for (int i = et; i < S.nbuf; i += kEpi) {
        p.list_key[slot * kTopK + i] = S.buf_key[pad32(i)];
        p.list_idx[slot * kTopK + i] = S.buf_idx[pad32(i)];
      }
      if (et == 0) {
        p.list_cnt[slot] = S.nbuf;
        if (gstart >= lo) p.row_first[r] = static_cast<int>(blockIdx.x);
        if (gstart + nt <= hi) p.row_last[r] = static_cast<int>(blockIdx.x);
        if (lo == 0) p.total_out[0] = total;
      }
      epi_sync();
      S.nbuf = 0;
      S.theta = 0;
      S.tkeep = 0;
      S.since_flush = 0;
      S.flushes = 0;
    };

    for (int i = 0; i < n_items; ++i) {
      if (w.g != cur_g) {
        if constexpr (SELECT) {
          if (cur_g >= 0) finish_row(cur_g, cur_gstart, cur_nt);
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
        cur_nt = w.nt;
        cur_gstart = w.gstart;
      }
      if (!mbar_wait(&accfull[acc], acc_ph, abort_flag)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const int64_t blk = static_cast<int64_t>(w.t) * kTileM + row_in_tile;
      float sc[NQ];
#pragma unroll 1
      for (int j = 0; j < NQ; ++j) {
        const int r = w.g * NQ + j;
        if (r >= p.rows) break;  // uniform
        float v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * C::kN + j * 32),
                           v);
        const float* wj = w_smem + j * kIdxHeads;
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) s = __fmaf_rn(wj[h], v[h] > 0.f ? v[h] : 0.f, s);
        sc[j] = s;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;

      if constexpr (SELECT) {
        const bool valid = blk < nb_smem[0];
        const uint32_t key = order_key(sc[0]);
        if (valid) atomicAdd(&S.lhist[key >> kHistShift], 1u);
        sel_append(S, valid && key >= S.theta, key, static_cast<int32_t>(blk), quarter, lane);
        if (++S.since_flush >= (S.flushes >= 2 ? kFlushTiles : kEarlyFlush)) {
          sel_flush(S, p.ghist + static_cast<int64_t>(w.g) * kHistBins, et, S.snap_pending);
          ++S.flushes;
        }
        if (S.nbuf > kBufCap - kEpi) sel_compact(S, et);
      } else {
#pragma unroll 1
        for (int j = 0; j < NQ; ++j) {
          const int r = w.g * NQ + j;
          if (r >= p.rows) break;
          if (blk < nb_smem[j]) p.scores[static_cast<int64_t>(r) * p.score_stride + blk] = sc[j];
        }
      }
      w.advance(p);
    }
    if constexpr (SELECT) {
      if (!aborted && cur_g >= 0) finish_row(cur_g, cur_gstart, cur_nt);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

namespace {

template <int NQ, bool SELECT>
cudaError_t launch_cfg(const ScoreArgs& a, cudaStream_t stream) {
  using C = Cfg<NQ, SELECT>;
  CUtensorMap map_k, map_q;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kIdxDim), static_cast<uint64_t>(a.cap_blk),
                              static_cast<uint64_t>(a.key_batches)};
    const uint64_t strides[2] = {kIdxDim * 2ull, static_cast<uint64_t>(a.cap_blk) * kIdxDim * 2ull};
    const uint32_t box[3] = {64, kTileM, 1};
    if (!encode_tensor_map(&map_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.pooled_k, dims,
                           strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(kIdxDim),
                              static_cast<uint64_t>(a.rows) * kIdxHeads};
    const uint64_t strides[1] = {kIdxDim * 2ull};
    const uint32_t box[2] = {64, static_cast<uint32_t>(C::kN)};
    if (!encode_tensor_map(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q_idx, dims, strides,
                           box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_index_score<NQ, SELECT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  KParams p{};
  p.w_head = a.w_head;
  p.n_vis = a.n_vis;
  p.scores = a.scores;
  p.score_stride = a.score_stride;
  p.max_len = a.max_len;
  p.rows = a.rows;
  p.groups = (a.rows + NQ - 1) / NQ;
  p.shared_keys = a.key_batches == 1 ? 1 : 0;
  p.ghist = a.sel_ghist;
  p.list_key = a.sel_list_key;
  p.list_idx = a.sel_list_idx;
  p.list_cnt = a.sel_list_cnt;
  p.row_first = a.sel_row_first;
  p.row_last = a.sel_row_last;
  p.total_out = a.sel_total;
  const int grid = score_grid(a.nq, a.rows, a.max_len, a.num_sms);
  if (grid == 0) return cudaSuccess;
  k_index_score<NQ, SELECT><<<grid, kThreads, C::kSmem, stream>>>(map_k, map_q, p);
  count_launches(1);
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
    if (a.sel_ghist) return launch_cfg<1, true>(a, stream);
    return launch_cfg<1, false>(a, stream);
  }
  if (a.nq == 8) return launch_cfg<8, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace spx
