// Exact top-K selection by a group of NT threads (a whole CTA, or a named
// subset such as the epilogue warps of a warp-specialised kernel).
//
// Ordering: 32-bit keys whose unsigned order is the score order; among
// equal keys the lower position (= lower block index, since candidates are
// held in index order) wins, so the selection is the first K elements of a
// strict total order and is unique.  Used by the top-k kernels and by the
// fused scoring kernel of the decode path.
#pragma once

#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

// Monotone map from fp32 to uint32 (-0 folded onto +0).  Finite inputs give
// keys >= 0x007FFFFF, so 0 never names a real score.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Shared-memory candidate buffers are padded by one word per 32 entries: a
// thread that owns 16 consecutive entries then reads them without bank
// conflicts (entry p lives at word p + p/32).
__host__ __device__ constexpr int pad32(int p) { return p + (p >> 5); }

template <int NT, int BAR>
__device__ __forceinline__ void group_sync() {
  if constexpr (BAR == 0) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
  }
}

// Exclusive prefix sum over the NT threads of the group (gtid in [0, NT)).
// `scratch` holds 33 ints.
template <int NT, int BAR>
__device__ __forceinline__ int group_excl_scan(int v, int gtid, int* scratch, int* total) {
  constexpr int kWarps = NT / 32;
  const int lane = gtid & 31, warp = gtid >> 5;
  const int inc = warp_incl_scan(v);
  if (lane == 31) scratch[warp] = inc;
  group_sync<NT, BAR>();
  if (warp == 0) {
    const int x = lane < kWarps ? scratch[lane] : 0;
    const int xi = warp_incl_scan(x);
    if (lane < kWarps) scratch[lane] = xi - x;
    if (lane == 31) scratch[32] = xi;
  }
  group_sync<NT, BAR>();
  const int res = scratch[warp] + inc - v;
  *total = scratch[32];
  group_sync<NT, BAR>();
  return res;
}

struct SelectSmem {
  int hist[256];
  int scan[33];
  int digit;
  int above;
};

// Selects the best min(K, n_valid) candidates of the group: thread g holds E
// candidates at positions g*E .. g*E+E-1 (bit i of `valid` set if present).
// emit(i, out_pos) is called for every survivor; out_pos increases with the
// position.  *thr receives the K-th largest key when a cut was needed (0
// when every valid candidate was kept).  Returns the survivor count.
template <int E, int NT, int BAR, typename Emit>
__device__ __forceinline__ int group_select(const uint32_t (&key)[E], uint32_t valid, int K,
                                            int gtid, SelectSmem& sm, uint32_t* thr, Emit emit) {
  const int lane = gtid & 31;
  {
    int n_all;
    int pos = group_excl_scan<NT, BAR>(__popc(valid), gtid, sm.scan, &n_all);
    if (n_all <= K) {
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((valid >> i) & 1u) emit(i, pos++);
      *thr = 0;
      return n_all;
    }
  }
  // Bits shared by every valid key need no histogram: find them from the
  // group-wide min and max first (this also avoids the worst same-address
  // atomic contention, on the leading digits).
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      kmin = key[i] < kmin ? key[i] : kmin;
      kmax = key[i] > kmax ? key[i] : kmax;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t a = __shfl_xor_sync(0xffffffffu, kmin, o);
    const uint32_t b = __shfl_xor_sync(0xffffffffu, kmax, o);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (lane == 0) {
    sm.hist[(gtid >> 5) * 2] = static_cast<int>(kmin);
    sm.hist[(gtid >> 5) * 2 + 1] = static_cast<int>(kmax);
  }
  group_sync<NT, BAR>();
  kmin = 0xFFFFFFFFu;
  kmax = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t a = static_cast<uint32_t>(sm.hist[2 * w]);
    const uint32_t b = static_cast<uint32_t>(sm.hist[2 * w + 1]);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  group_sync<NT, BAR>();
  // All valid keys lie in [kmin, kmax], so they share every bit above the
  // highest bit where kmin and kmax differ.
  const uint32_t diff = kmin ^ kmax;
  uint32_t prefix = 0, pmask = 0;
  int remaining = K;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    if ((diff >> shift) == 0) {  // uniform: this digit is common to all keys
      prefix |= kmin & (255u << shift);
      pmask |= 255u << shift;
      continue;
    }
    for (int b = gtid; b < 256; b += NT) sm.hist[b] = 0;
    group_sync<NT, BAR>();
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if (((valid >> i) & 1u) && (key[i] & pmask) == prefix)
        atomicAdd(&sm.hist[(key[i] >> shift) & 255u], 1);
    }
    group_sync<NT, BAR>();
    if (gtid < 32) {
      // lane L owns bins 255-8L .. 248-8L (descending)
      int local[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        local[j] = sm.hist[255 - (lane * 8 + j)];
        lsum += local[j];
      }
      int incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      int cum = incl - lsum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (cum < remaining && remaining <= cum + local[j]) {
          sm.digit = 255 - (lane * 8 + j);
          sm.above = cum;
        }
        cum += local[j];
      }
    }
    group_sync<NT, BAR>();
    prefix |= static_cast<uint32_t>(sm.digit) << shift;
    pmask |= 255u << shift;
    remaining -= sm.above;
    group_sync<NT, BAR>();
  }
  int ngt = 0, neq = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      ngt += key[i] > prefix;
      neq += key[i] == prefix;
    }
  }
  int eq_tot, total;
  const int eq_before = group_excl_scan<NT, BAR>(neq, gtid, sm.scan, &eq_tot);
  int take = remaining - eq_before;
  take = take < 0 ? 0 : (take > neq ? neq : take);
  int pos = group_excl_scan<NT, BAR>(ngt + take, gtid, sm.scan, &total);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      if (key[i] > prefix) {
        emit(i, pos++);
      } else if (key[i] == prefix && take > 0) {
        --take;
        emit(i, pos++);
      }
    }
  }
  *thr = prefix;
  return total;
}

// Scores are counted by their top 11 key bits (sign, exponent, 2 mantissa
// bits) in 2048-bin histograms; the bin of a key is key >> kSelKeyShift.
constexpr int kSelKeyShift = 32 - 11;

// Shared state of the final choice.
struct MergeSmem {
  int rh[3][128];  // radix histograms of the three 7-bit digits below the cut bin
  int dig[3], abv[3];
  uint32_t kmin, kmax;
};

// The row's result from the n buffered (key, block) pairs, in block order;
// entries below lo_key are not candidates.  Every candidate above the cut
// bin is selected; the (K - above) best of the cut bin (ties: lower block)
// complete the set.  Writes the ascending block ids, -1 padded, and the
// count.  This code runs once per row: its loops stay rolled, so that it is
// short (instruction fetch, not arithmetic, bounds a one-pass kernel).
template <int NT, int BAR>
__device__ __noinline__ void merge_final(const uint32_t* bk, const int32_t* bi, int n_in,
                                         uint32_t lo_key, int cut_bin, int above, SelectSmem& sm,
                                         MergeSmem& ms, int32_t* dst, int32_t* cnt_out,
                                         int gtid) {
  const int tid = gtid;
  const int per = (n_in + NT - 1) / NT;
  const int q0 = min(tid * per, n_in), q1 = min(q0 + per, n_in);
  const bool cut = cut_bin >= 0;  // uniform
  const uint32_t cut_lo = cut ? static_cast<uint32_t>(cut_bin) << kSelKeyShift : 0u;
  const uint32_t cut_hi = cut ? cut_lo | ((1u << kSelKeyShift) - 1u) : 0xFFFFFFFFu;
  const uint32_t in_lo = lo_key > cut_lo ? lo_key : cut_lo;
  // candidate classes: sure (above the cut bin, or every candidate when no
  // cut is needed) and in-cut
  uint32_t T = 0xFFFFFFFFu;
  int need_eq = 0;
  if (cut) {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0;
#pragma unroll 1
    for (int q = q0; q < q1; ++q) {
      const uint32_t k = bk[pad32(q)];
      if (k >= in_lo && k <= cut_hi) {
        kmin = k < kmin ? k : kmin;
        kmax = k > kmax ? k : kmax;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t x = __shfl_xor_sync(0xffffffffu, kmin, o);
      const uint32_t y = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = x < kmin ? x : kmin;
      kmax = y > kmax ? y : kmax;
    }
    if ((tid & 31) == 0 && kmin <= kmax) {
      atomicMin(&ms.kmin, kmin);
      atomicMax(&ms.kmax, kmax);
    }
    group_sync<NT, BAR>();
    // the candidates of the cut bin share every bit above the highest one
    // where their min and max differ; the rest comes from radix passes
    kmin = ms.kmin;
    const uint32_t diff = kmin ^ ms.kmax;
    uint32_t prefix = 0, pmask = 0;
    int rem = kTopK - above;
#pragma unroll 1
    for (int d = 0; d < 3; ++d) {
      const int shift = 14 - 7 * d;
      if ((diff >> shift) == 0) {  // uniform
        prefix |= kmin & (127u << shift);
        pmask |= 127u << shift;
        continue;
      }
#pragma unroll 1
      for (int q = q0; q < q1; ++q) {
        const uint32_t k = bk[pad32(q)];
        if (k >= in_lo && k <= cut_hi && (k & pmask) == prefix)
          atomicAdd(&ms.rh[d][(k >> shift) & 127u], 1);
      }
      group_sync<NT, BAR>();
      if (tid < 32) {
        int c[4], lsum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c[j] = ms.rh[d][127 - (tid * 4 + j)];
          lsum += c[j];
        }
        int cum = warp_incl_scan(lsum) - lsum;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (cum < rem && rem <= cum + c[j]) {
            ms.dig[d] = 127 - (tid * 4 + j);
            ms.abv[d] = cum;
          }
          cum += c[j];
        }
      }
      group_sync<NT, BAR>();
      prefix |= static_cast<uint32_t>(ms.dig[d]) << shift;
      pmask |= 127u << shift;
      rem -= ms.abv[d];
    }
    T = cut_lo | (prefix & ((1u << kSelKeyShift) - 1u));
    need_eq = rem;
  }
  // chosen: every sure candidate, the in-cut ones above T and the first
  // need_eq equal to T.  One scan of (above, equal) counts packed in 16-bit
  // halves (at most 8192 each) places them.
  auto sure = [&](uint32_t k) { return cut ? k > cut_hi : k >= lo_key; };
  int ca = 0, ce = 0;
#pragma unroll 1
  for (int q = q0; q < q1; ++q) {
    const uint32_t k = bk[pad32(q)];
    if (sure(k)) ++ca;
    else if (cut && k >= in_lo && k <= cut_hi) {
      ca += k > T;
      ce += k == T;
    }
  }
  int tot;
  const int ex = group_excl_scan<NT, BAR>((ca << 16) | ce, tid, sm.scan, &tot);
  int eq_seen = ex & 0xFFFF;
  int pos = (ex >> 16) + min(need_eq, eq_seen);
#pragma unroll 1
  for (int q = q0; q < q1; ++q) {
    const uint32_t k = bk[pad32(q)];
    bool take = sure(k);
    if (!take && cut && k >= in_lo && k <= cut_hi) {
      if (k > T) take = true;
      else if (k == T) take = eq_seen++ < need_eq;
    }
    if (take && pos < kTopK) dst[pos++] = bi[pad32(q)];
  }
  int n = (tot >> 16) + min(need_eq, tot & 0xFFFF);
  if (n > kTopK) n = kTopK;  // cannot happen for consistent inputs
  for (int j = n + tid; j < kTopK; j += NT) dst[j] = -1;
  if (tid == 0) *cnt_out = n;
}


}  // namespace spx
