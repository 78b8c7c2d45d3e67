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

}  // namespace spx
