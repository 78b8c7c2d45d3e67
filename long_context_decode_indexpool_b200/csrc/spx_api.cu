// C ABI of libspx: host-side validation, workspace layout and launch
// sequencing.  Every check runs before the first launch of a call, so a call
// that returns an error has enqueued nothing.  No allocation, no
// synchronisation (except spx_device_error, which says so).
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "spx.h"
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded tensor maps of recent calls.  A decode loop passes the same
// caches and query buffers on every step, so the maps are encoded once and
// copied afterwards.  The key is everything the encoding depends on; a map
// is a pure function of it (the device is part of the key only because the
// same address may name memory of another device).
struct MapKey {
  int dev, dtype, rank, swizzle;
  const void* base;
  uint64_t dims[5], strides[4];
  uint32_t box[5];
};
constexpr int kMapCacheSize = 32;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
};
MapCache& map_cache() {
  static MapCache c;
  return c;
}

}  // namespace

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
  if (rank < 1 || rank > 5) return false;
  MapKey k;
  std::memset(&k, 0, sizeof(k));
  if (cudaGetDevice(&k.dev) != cudaSuccess) return false;
  k.dtype = static_cast<int>(dtype);
  k.rank = rank;
  k.swizzle = static_cast<int>(swizzle);
  k.base = base;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides_bytes[i];
  MapCache& c = map_cache();
  {
    std::lock_guard<std::mutex> g(c.mu);
    for (int i = 0; i < kMapCacheSize; ++i) {
      if (c.used[i] && std::memcmp(&c.key[i], &k, sizeof(k)) == 0) {
        *map = c.map[i];
        return true;
      }
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  const bool ok = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs,
                     bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  if (ok) {
    std::lock_guard<std::mutex> g(c.mu);
    const int i = c.next;
    c.next = (c.next + 1) % kMapCacheSize;
    c.key[i] = k;
    c.map[i] = *map;
    c.used[i] = true;
  }
  return ok;
}

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

spx_status check_dims(const spx_dims* d) {
  if (!d) return SPX_ERR_INVALID_ARG;
  if (d->idx_heads != kIdxHeads || d->idx_dim != kIdxDim || d->pool != kPool ||
      d->topk_blocks != kTopK || d->latent != kLatent)
    return SPX_ERR_UNSUPPORTED;
  if (d->heads < kHeadGroup || d->heads > kMaxHeads || d->heads % kHeadGroup != 0)
    return SPX_ERR_UNSUPPORTED;
  if (!std::isfinite(d->sm_scale) || !(d->sm_scale > 0.f)) return SPX_ERR_INVALID_ARG;
  return SPX_OK;
}

int device_sm_count() {
  static std::atomic<int> cache[64];  // zero-initialised: not queried yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev].load()) return cache[dev].load();
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace spx

using namespace spx;

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

spx_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SPX_OK : SPX_ERR_CUDA; }

// Score row stride used inside the fused calls: max_blk rounded up to 64.
inline int64_t score_stride_for(int64_t max_len) {
  const int64_t mb = max_len / kPool;
  return (mb + 63) / 64 * 64;
}

// Workspace of the prefill call:
//   n_vis [rows] int64 | scores [rows, stride] f32 | idx [rows, 512] | count [rows]
//   | key histograms [rows, 2048] | chunk counters [rows] | list keys, list
//   ids [rows*nchunk, 512] | list counts [rows*nchunk] | attention scratch
//   | INT8 cache: query codes [rows, 32, 128] int8, head weights [rows, 32]
struct FusedLayout {
  size_t nvis, scores, idx, count, hist, done, lkey, lidx, lcnt, attn, q8, wq, total;
  int64_t stride;
  int nchunk;
  AttnPlan ap;
};

FusedLayout fused_layout(int rows, int heads, int64_t max_len) {
  FusedLayout L{};
  L.stride = score_stride_for(max_len);
  const int64_t max_blk = max_len / kPool;
  L.nchunk = static_cast<int>((max_blk + kSelChunk - 1) / kSelChunk);
  if (L.nchunk < 1) L.nchunk = 1;
  L.ap = plan_attn(rows, heads, max_len, device_sm_count());
  const size_t lists = static_cast<size_t>(rows) * L.nchunk;
  size_t o = 0;
  L.nvis = o;
  o += up(static_cast<size_t>(rows) * 8);
  L.scores = o;
  o += up(static_cast<size_t>(rows) * L.stride * 4);
  L.idx = o;
  o += up(static_cast<size_t>(rows) * kTopK * 4);
  L.count = o;
  o += up(static_cast<size_t>(rows) * 4);
  L.hist = o;
  o += up(static_cast<size_t>(rows) * kSelHistBins * 4);
  L.done = o;
  o += up(static_cast<size_t>(rows) * 4);
  L.lkey = o;
  o += up(lists * kTopK * 4);
  L.lidx = o;
  o += up(lists * kTopK * 4);
  L.lcnt = o;
  o += up(lists * 4);
  L.attn = o;
  o += up(L.ap.ws_bytes);
  L.q8 = o;  // INT8 cache: query codes [rows, 32, 128] and scaled head weights [rows, 32]
  o += up(static_cast<size_t>(rows) * kIdxHeads * kIdxDim);
  L.wq = o;
  o += up(static_cast<size_t>(rows) * kIdxHeads * 4);
  L.total = o;
  return L;
}

// Workspace of the fused decode call:
//   n_vis [B] | idx [B,512] | count [B] | key histogram [B,2048] | done [B+1]
//   | scores [B, stride] | list keys, list ids [B*nchunk, 512]
//   | list counts [B*nchunk] | attention scratch | INT8 cache: query codes
//   [B,32,128] int8 and head weights [B,32] with the query scales folded in
struct DecodeLayout {
  size_t nvis, idx, count, hist, done, scores, lkey, lidx, lcnt, attn, q8, wq, total;
  int64_t stride;  // scores per row, a multiple of 4
  int nchunk;
  AttnPlan ap;
};

DecodeLayout decode_layout(int B, int heads, int64_t max_len) {
  DecodeLayout L{};
  const int sms = device_sm_count();
  const int64_t max_blk = max_len / kPool;
  L.stride = (max_blk + 3) / 4 * 4;
  if (L.stride < 4) L.stride = 4;
  L.nchunk = static_cast<int>((max_blk + kSelChunk - 1) / kSelChunk);
  if (L.nchunk < 1) L.nchunk = 1;
  L.ap = plan_attn(B, heads, max_len, sms);
  const size_t lists = static_cast<size_t>(B) * L.nchunk;
  size_t o = 0;
  L.nvis = o;
  o += up(static_cast<size_t>(B) * 8);
  L.idx = o;
  o += up(static_cast<size_t>(B) * kTopK * 4);
  L.count = o;
  o += up(static_cast<size_t>(B) * 4);
  L.hist = o;
  o += up(static_cast<size_t>(B) * kSelHistBins * 4);
  L.done = o;  // B chunk counters of the selection + the scoring work counter
  o += up(static_cast<size_t>(B + 1) * 4);
  L.scores = o;
  o += up(static_cast<size_t>(B) * L.stride * 4);
  L.lkey = o;
  o += up(lists * kTopK * 4);
  L.lidx = o;
  o += up(lists * kTopK * 4);
  L.lcnt = o;
  o += up(lists * 4);
  L.attn = o;
  o += up(L.ap.ws_bytes);
  L.q8 = o;
  o += up(static_cast<size_t>(B) * kIdxHeads * kIdxDim);
  L.wq = o;
  o += up(static_cast<size_t>(B) * kIdxHeads * 4);
  L.total = o;
  return L;
}

// Workspace of the standalone INT8 scoring call: query codes | head weights.
size_t score_i8_ws(int B) {
  return up(static_cast<size_t>(B) * kIdxHeads * kIdxDim) + up(static_cast<size_t>(B) * kIdxHeads * 4);
}

spx_status check_pool_w(const float* w, float out[4]) {
  if (!w) return SPX_ERR_INVALID_ARG;
  double s = 0.0;
  for (int i = 0; i < kPool; ++i) {
    if (!std::isfinite(w[i])) return SPX_ERR_INVALID_ARG;
    out[i] = w[i];
    s += w[i];
  }
  if (std::fabs(s - 1.0) > 1e-6) return SPX_ERR_INVALID_ARG;
  return SPX_OK;
}

}  // namespace

extern "C" {

const char* spx_status_string(spx_status s) {
  switch (s) {
    case SPX_OK: return "SPX_OK";
    case SPX_ERR_INVALID_ARG: return "SPX_ERR_INVALID_ARG";
    case SPX_ERR_SHAPE: return "SPX_ERR_SHAPE";
    case SPX_ERR_UNSUPPORTED: return "SPX_ERR_UNSUPPORTED";
    case SPX_ERR_WORKSPACE: return "SPX_ERR_WORKSPACE";
    case SPX_ERR_CUDA: return "SPX_ERR_CUDA";
    case SPX_ERR_DEVICE: return "SPX_ERR_DEVICE";
  }
  return "SPX_ERR_UNKNOWN";
}

const char* spx_version(void) { return "libspx 0.1.0 (sm_100a)"; }

uint64_t spx_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

spx_status spx_dims_init(spx_dims* d, int32_t heads, float sm_scale) {
  if (!d) return SPX_ERR_INVALID_ARG;
  d->idx_heads = kIdxHeads;
  d->idx_dim = kIdxDim;
  d->pool = kPool;
  d->topk_blocks = kTopK;
  d->heads = heads;
  d->latent = kLatent;
  d->sm_scale = sm_scale;
  return check_dims(d);
}

spx_status spx_device_error(int32_t* code, spx_stream stream) {
  if (!code) return SPX_ERR_INVALID_ARG;
  int v = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return SPX_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SPX_ERR_CUDA;
  const int zero = 0;
  if (v != 0) {
    if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return SPX_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPX_ERR_CUDA;
  }
  *code = v;
  return SPX_OK;
}

spx_status spx_selftest_wait_timeout(int64_t limit_ns, int64_t* result, spx_stream stream) {
  if (!result || !al4(result)) return SPX_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 1000000000) return SPX_ERR_INVALID_ARG;
  return cuda_status(launch_wait_selftest(static_cast<uint64_t>(limit_ns), result,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

spx_status pool_append_impl(const spx_dims* d, int32_t B, const void* raw_k, int32_t n_new,
                            const float* pool_w, void* tail, void* pooled_k, float* k_scale,
                            bool i8, int64_t cap_blk, const int64_t* len_dev, int64_t max_len,
                            spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  float w[4];
  if ((st = check_pool_w(pool_w, w)) != SPX_OK) return st;
  if (B < 1 || B > 65535 || n_new < 0 || cap_blk < 1) return SPX_ERR_SHAPE;
  if (max_len < n_new || max_len > kPool * cap_blk) return SPX_ERR_SHAPE;
  if (!tail || !pooled_k || !len_dev || (n_new > 0 && !raw_k)) return SPX_ERR_INVALID_ARG;
  if (!al16(tail) || !al16(pooled_k) || (raw_k && !al16(raw_k)) || (len_dev && !al4(len_dev)))
    return SPX_ERR_INVALID_ARG;
  if (i8 && (!k_scale || !al4(k_scale))) return SPX_ERR_INVALID_ARG;
  if (n_new == 0) return SPX_OK;
  PoolAppendArgs a{};
  a.i8 = i8;
  a.k_scale = k_scale;
  a.B = B;
  a.raw_k = raw_k;
  a.n_new = n_new;
  for (int i = 0; i < 4; ++i) a.w[i] = w[i];
  a.tail = tail;
  a.pooled_k = pooled_k;
  a.cap_blk = cap_blk;
  a.len_dev = len_dev;
  a.len_host = 0;
  a.max_len = max_len;
  a.nvis_out = nullptr;
  return cuda_status(launch_pool_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

// Host checks shared by the bf16 and INT8 scoring calls.
spx_status check_score_args(const spx_dims* d, int32_t B, const void* q_idx, const float* w_head,
                            const void* pooled_k, int64_t cap_blk, const int64_t* n_vis,
                            int64_t max_len, float* scores, int64_t score_stride) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (B < 1 || cap_blk < 1 || max_len < 0 || max_len > kPool * cap_blk) return SPX_ERR_SHAPE;
  if (cap_blk > (int64_t(1) << 31) - 1 || static_cast<int64_t>(B) * kIdxHeads > (1ll << 31) - 1)
    return SPX_ERR_SHAPE;
  if (score_stride < max_len / kPool) return SPX_ERR_SHAPE;
  if (!q_idx || !w_head || !pooled_k || !n_vis || !scores) return SPX_ERR_INVALID_ARG;
  if (!al16(q_idx) || !al16(pooled_k) || !al4(w_head) || !al4(scores)) return SPX_ERR_INVALID_ARG;
  return SPX_OK;
}

}  // namespace

extern "C" {

spx_status spx_pool_append(const spx_dims* d, int32_t B, const void* raw_k, int32_t n_new,
                           const float* pool_w, void* tail, void* pooled_k, int64_t cap_blk,
                           const int64_t* len_dev, int64_t max_len, spx_stream stream) {
  return pool_append_impl(d, B, raw_k, n_new, pool_w, tail, pooled_k, nullptr, false, cap_blk,
                          len_dev, max_len, stream);
}

spx_status spx_pool_append_tok(const spx_dims* d, int32_t B, const void* raw_k, const float* raw_w,
                               int32_t n_new, void* tail, float* tail_w, void* pooled_k,
                               int64_t cap_blk, const int64_t* len_dev, int64_t max_len,
                               spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (B < 1 || B > 65535 || n_new < 0 || cap_blk < 1) return SPX_ERR_SHAPE;
  if (max_len < n_new || max_len > kPool * cap_blk) return SPX_ERR_SHAPE;
  if (!tail || !tail_w || !pooled_k || !len_dev || (n_new > 0 && (!raw_k || !raw_w)))
    return SPX_ERR_INVALID_ARG;
  if (!al16(tail) || !al16(pooled_k) || (raw_k && !al16(raw_k)) || !al4(len_dev) ||
      !al4(tail_w) || (raw_w && !al4(raw_w)))
    return SPX_ERR_INVALID_ARG;
  if (n_new == 0) return SPX_OK;
  PoolAppendArgs a{};
  a.B = B;
  a.raw_k = raw_k;
  a.n_new = n_new;
  a.raw_w = raw_w;
  a.tail_w = tail_w;
  a.tail = tail;
  a.pooled_k = pooled_k;
  a.cap_blk = cap_blk;
  a.len_dev = len_dev;
  a.max_len = max_len;
  return cuda_status(launch_pool_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

spx_status spx_pool_append_i8(const spx_dims* d, int32_t B, const void* raw_k, int32_t n_new,
                              const float* pool_w, void* tail, void* pooled_k8, float* k_scale,
                              int64_t cap_blk, const int64_t* len_dev, int64_t max_len,
                              spx_stream stream) {
  return pool_append_impl(d, B, raw_k, n_new, pool_w, tail, pooled_k8, k_scale, true, cap_blk,
                          len_dev, max_len, stream);
}

spx_status spx_index_score(const spx_dims* d, int32_t B, const void* q_idx, const float* w_head,
                           const void* pooled_k, int64_t cap_blk, const int64_t* n_vis,
                           int64_t max_len, float* scores, int64_t score_stride,
                           spx_stream stream) {
  spx_status st =
      check_score_args(d, B, q_idx, w_head, pooled_k, cap_blk, n_vis, max_len, scores, score_stride);
  if (st != SPX_OK) return st;
  ScoreArgs a{};
  a.nq = 1;
  a.rows = B;
  a.key_batches = B;
  a.q_idx = q_idx;
  a.w_head = w_head;
  a.pooled_k = pooled_k;
  a.cap_blk = cap_blk;
  a.n_vis = n_vis;
  a.max_len = max_len;
  a.scores = scores;
  a.score_stride = score_stride;
  a.num_sms = device_sm_count();
  return cuda_status(launch_index_score(a, reinterpret_cast<cudaStream_t>(stream)));
}

spx_status spx_index_score_i8_workspace_size(const spx_dims* d, int32_t B, size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (B < 1 || B > 65535) return SPX_ERR_SHAPE;
  *bytes = score_i8_ws(B);
  return SPX_OK;
}

spx_status spx_index_score_i8(const spx_dims* d, int32_t B, const void* q_idx,
                              const float* w_head, const void* pooled_k8, const float* k_scale,
                              int64_t cap_blk, const int64_t* n_vis, int64_t max_len,
                              float* scores, int64_t score_stride, void* ws, size_t ws_bytes,
                              spx_stream stream) {
  spx_status st = check_score_args(d, B, q_idx, w_head, pooled_k8, cap_blk, n_vis, max_len,
                                   scores, score_stride);
  if (st != SPX_OK) return st;
  if (B > 65535) return SPX_ERR_SHAPE;
  if (!k_scale) return SPX_ERR_INVALID_ARG;
  if (!al4(k_scale)) return SPX_ERR_INVALID_ARG;
  if (!ws || ws_bytes < score_i8_ws(B) || !al16(ws)) return SPX_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int8_t* q8 = static_cast<int8_t*>(ws);
  float* wq = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       up(static_cast<size_t>(B) * kIdxHeads * kIdxDim));
  cudaError_t e = launch_quant_q(B, q_idx, w_head, q8, wq, s);
  if (e != cudaSuccess) return SPX_ERR_CUDA;
  ScoreArgs a{};
  a.nq = 1;
  a.i8 = true;
  a.k_scale = k_scale;
  a.rows = B;
  a.key_batches = B;
  a.q_idx = q8;
  a.w_head = wq;
  a.pooled_k = pooled_k8;
  a.cap_blk = cap_blk;
  a.n_vis = n_vis;
  a.max_len = max_len;
  a.scores = scores;
  a.score_stride = score_stride;
  a.num_sms = device_sm_count();
  return cuda_status(launch_index_score(a, s));
}

spx_status spx_topk_workspace_size(const spx_dims* d, int32_t rows, int64_t max_len,
                                   size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (rows < 1 || rows > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  *bytes = plan_topk(rows, max_len).ws_bytes;
  return SPX_OK;
}

spx_status spx_topk_blocks(const spx_dims* d, int32_t rows, const float* scores,
                           int64_t score_stride, const int64_t* n_vis, int64_t max_len,
                           int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                           spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (rows < 1 || rows > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  if (max_len / kPool > (int64_t(1) << 31) - 1) return SPX_ERR_SHAPE;
  if (score_stride < max_len / kPool) return SPX_ERR_SHAPE;
  if (!scores || !n_vis || !idx || !count) return SPX_ERR_INVALID_ARG;
  if (!al4(scores) || !al4(idx) || !al4(count)) return SPX_ERR_INVALID_ARG;
  const TopkPlan p = plan_topk(rows, max_len);
  if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes || !al16(ws))) return SPX_ERR_WORKSPACE;
  return cuda_status(launch_topk(p, scores, score_stride, n_vis, max_len, idx, count, ws,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

spx_status spx_attn_workspace_size(const spx_dims* d, int32_t rows, int64_t max_len,
                                   size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (rows < 1 || rows > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  *bytes = plan_attn(rows, d->heads, max_len, device_sm_count()).ws_bytes;
  return SPX_OK;
}

spx_status spx_sparse_mla_attn(const spx_dims* d, int32_t rows, const void* q, const void* latent,
                               int64_t seq_stride, int64_t cap_tok, const int32_t* idx,
                               const int32_t* count, const int64_t* n_vis, int64_t max_len,
                               void* out, float* lse, void* ws, size_t ws_bytes,
                               spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (rows < 1 || rows > 65535 || max_len < 0 || cap_tok < 1 || seq_stride < 0)
    return SPX_ERR_SHAPE;
  if (seq_stride != 0 && seq_stride < cap_tok * kLatent) return SPX_ERR_SHAPE;
  if (!q || !latent || !idx || !count || !n_vis || !out) return SPX_ERR_INVALID_ARG;
  if (!al16(q) || !al16(latent) || !al16(out) || !al4(idx) || !al4(count) || (lse && !al4(lse)))
    return SPX_ERR_INVALID_ARG;
  const AttnPlan p = plan_attn(rows, d->heads, max_len, device_sm_count());
  if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes || !al16(ws))) return SPX_ERR_WORKSPACE;
  AttnArgs a{};
  a.q = q;
  a.latent = latent;
  a.seq_stride = seq_stride;
  a.cap_tok = cap_tok;
  a.idx = idx;
  a.count = count;
  a.n_vis = n_vis;
  a.max_len = max_len;
  a.sm_scale = d->sm_scale;
  a.out = out;
  a.lse = lse;
  a.ws = ws;
  return cuda_status(launch_attn(p, a, reinterpret_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
spx_status spx_latent_quant_fp8(const void* latent, int64_t n, void* codes, int32_t* exps,
                                spx_stream stream) {
  if (n < 0) return SPX_ERR_SHAPE;
  if (n == 0) return SPX_OK;
  if (!latent || !codes || !exps) return SPX_ERR_INVALID_ARG;
  if (!al16(latent) || !al16(codes) || !al4(exps)) return SPX_ERR_INVALID_ARG;
  return cuda_status(launch_latent_quant_fp8(latent, n, static_cast<uint8_t*>(codes), exps,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Workspace of spx_sparse_mla_attn_fp8: compact bf16 rows [rows, 2052, 512]
// | ids [rows, 512] | counts [rows] | lengths [rows] | attention scratch
struct Fp8Layout {
  size_t dense, cidx, ccnt, cnvis, attn, total;
  AttnPlan ap;
};

Fp8Layout fp8_layout(int rows, int heads) {
  Fp8Layout L{};
  L.ap = plan_attn(rows, heads, kFp8Dense, device_sm_count());
  size_t o = 0;
  L.dense = o;
  o += up(static_cast<size_t>(rows) * kFp8Dense * kLatent * 2);
  L.cidx = o;
  o += up(static_cast<size_t>(rows) * kTopK * 4);
  L.ccnt = o;
  o += up(static_cast<size_t>(rows) * 4);
  L.cnvis = o;
  o += up(static_cast<size_t>(rows) * 8);
  L.attn = o;
  o += up(L.ap.ws_bytes);
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

spx_status spx_attn_fp8_workspace_size(const spx_dims* d, int32_t rows, int64_t max_len,
                                       size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (rows < 1 || rows > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  *bytes = fp8_layout(rows, d->heads).total;
  return SPX_OK;
}

spx_status spx_sparse_mla_attn_fp8(const spx_dims* d, int32_t rows, const void* q,
                                   const void* codes, const int32_t* exps, int64_t seq_stride,
                                   int64_t cap_tok, const int32_t* idx, const int32_t* count,
                                   const int64_t* n_vis, int64_t max_len, void* out, float* lse,
                                   void* ws, size_t ws_bytes, spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (rows < 1 || rows > 65535 || max_len < 0 || cap_tok < 1 || seq_stride < 0)
    return SPX_ERR_SHAPE;
  if (seq_stride != 0 && seq_stride < cap_tok * kLatent) return SPX_ERR_SHAPE;
  if (seq_stride % kLatent != 0) return SPX_ERR_SHAPE;
  if (!q || !codes || !exps || !idx || !count || !n_vis || !out) return SPX_ERR_INVALID_ARG;
  if (!al16(q) || !al16(codes) || !al4(exps) || !al16(out) || !al4(idx) || !al4(count) ||
      (lse && !al4(lse)))
    return SPX_ERR_INVALID_ARG;
  const Fp8Layout L = fp8_layout(rows, d->heads);
  if (!ws || ws_bytes < L.total || !al16(ws)) return SPX_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* cidx = reinterpret_cast<int32_t*>(base + L.cidx);
  int32_t* ccnt = reinterpret_cast<int32_t*>(base + L.ccnt);
  int64_t* cnvis = reinterpret_cast<int64_t*>(base + L.cnvis);
  const int64_t len_cap = max_len < cap_tok ? max_len : cap_tok;
  cudaError_t e = launch_gather_fp8(rows, static_cast<const uint8_t*>(codes), exps, seq_stride,
                                    len_cap, idx, count, n_vis, base + L.dense,
                                    static_cast<int64_t>(kFp8Dense) * kLatent, cidx, ccnt, cnvis,
                                    s);
  if (e != cudaSuccess) return SPX_ERR_CUDA;
  AttnArgs a{};
  a.q = q;
  a.latent = base + L.dense;
  a.seq_stride = static_cast<int64_t>(kFp8Dense) * kLatent;
  a.cap_tok = kFp8Dense;
  a.idx = cidx;
  a.count = ccnt;
  a.n_vis = cnvis;
  a.max_len = kFp8Dense;
  a.sm_scale = d->sm_scale;
  a.out = out;
  a.lse = lse;
  a.ws = base + L.attn;
  return cuda_status(launch_attn(L.ap, a, s));
}

}  // extern "C"

namespace {

// Workspace of spx_sparse_mla_attn_ws: remapped ids [rows, 512] | counts |
// lengths | fill blocks, fill slots [rows, 512] | fill counts | attention
struct WsLayout {
  size_t ridx, rcnt, rnvis, fblk, fslot, fn, attn, total;
  AttnPlan ap;
};

WsLayout ws_layout(int rows, int heads, int nslots) {
  WsLayout L{};
  L.ap = plan_attn(rows, heads, static_cast<int64_t>(nslots + 1) * kPool, device_sm_count());
  size_t o = 0;
  L.ridx = o;
  o += up(static_cast<size_t>(rows) * kTopK * 4);
  L.rcnt = o;
  o += up(static_cast<size_t>(rows) * 4);
  L.rnvis = o;
  o += up(static_cast<size_t>(rows) * 8);
  L.fblk = o;
  o += up(static_cast<size_t>(rows) * kTopK * 4);
  L.fslot = o;
  o += up(static_cast<size_t>(rows) * kTopK * 4);
  L.fn = o;
  o += up(static_cast<size_t>(rows) * 4);
  L.attn = o;
  o += up(L.ap.ws_bytes);
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

spx_status spx_ws_workspace_size(const spx_dims* d, int32_t rows, int32_t nslots, size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (rows < 1 || rows > 65535 || nslots < kTopK || nslots > (1 << 26)) return SPX_ERR_SHAPE;
  *bytes = ws_layout(rows, d->heads, nslots).total;
  return SPX_OK;
}

spx_status spx_sparse_mla_attn_ws(const spx_dims* d, int32_t rows, const void* q,
                                  const void* host_latent, int64_t seq_stride, int64_t cap_tok,
                                  const int32_t* idx, const int32_t* count, const int64_t* n_vis,
                                  int64_t max_len, void* pool, int32_t nslots, int32_t* slot_blk,
                                  int32_t* blk_slot, int32_t* slot_stamp, int32_t* hand,
                                  int32_t step, int64_t* stats, void* out, float* lse, void* ws,
                                  size_t ws_bytes, spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (rows < 1 || rows > 65535 || max_len < 0 || cap_tok < 1 || seq_stride < 0)
    return SPX_ERR_SHAPE;
  if (seq_stride != 0 && seq_stride < cap_tok * kLatent) return SPX_ERR_SHAPE;
  if (nslots < kTopK || nslots > (1 << 26)) return SPX_ERR_SHAPE;
  if (!q || !host_latent || !idx || !count || !n_vis || !pool || !slot_blk || !blk_slot ||
      !slot_stamp || !hand || !stats || !out)
    return SPX_ERR_INVALID_ARG;
  if (!al16(q) || !al16(host_latent) || !al16(pool) || !al16(out) || !al4(idx) || !al4(count) ||
      !al4(slot_blk) || !al4(blk_slot) || !al4(slot_stamp) || !al4(hand) || (lse && !al4(lse)) ||
      (reinterpret_cast<uintptr_t>(stats) & 7u) || (reinterpret_cast<uintptr_t>(n_vis) & 7u))
    return SPX_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(rows, d->heads, nslots);
  if (!ws || ws_bytes < L.total || !al16(ws)) return SPX_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  WsArgs w{};
  w.rows = rows;
  w.idx = idx;
  w.count = count;
  w.n_vis = n_vis;
  w.len_cap = max_len < cap_tok ? max_len : cap_tok;
  w.cap_blk = cap_tok / kPool;
  w.nslots = nslots;
  w.slot_blk = slot_blk;
  w.blk_slot = blk_slot;
  w.slot_stamp = slot_stamp;
  w.hand = hand;
  w.step = step;
  w.stats = stats;
  w.host_latent = host_latent;
  w.seq_stride = seq_stride;
  w.pool = pool;
  w.r_idx = reinterpret_cast<int32_t*>(base + L.ridx);
  w.r_cnt = reinterpret_cast<int32_t*>(base + L.rcnt);
  w.r_nvis = reinterpret_cast<int64_t*>(base + L.rnvis);
  w.fill_blk = reinterpret_cast<int32_t*>(base + L.fblk);
  w.fill_slot = reinterpret_cast<int32_t*>(base + L.fslot);
  w.fill_n = reinterpret_cast<int32_t*>(base + L.fn);
  cudaError_t e = launch_ws_update(w, s);
  if (e != cudaSuccess) return SPX_ERR_CUDA;
  const int64_t pool_tok = static_cast<int64_t>(nslots + 1) * kPool;
  AttnArgs a{};
  a.q = q;
  a.latent = pool;
  a.seq_stride = pool_tok * kLatent;
  a.cap_tok = pool_tok;
  a.idx = w.r_idx;
  a.count = w.r_cnt;
  a.n_vis = w.r_nvis;
  a.max_len = pool_tok;
  a.sm_scale = d->sm_scale;
  a.out = out;
  a.lse = lse;
  a.ws = base + L.attn;
  return cuda_status(launch_attn(L.ap, a, s));
}

// ---------------------------------------------------------------------------
spx_status spx_decode_workspace_size(const spx_dims* d, int32_t B, int64_t max_len,
                                     size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  *bytes = decode_layout(B, d->heads, max_len).total;
  return SPX_OK;
}

}  // extern "C"

namespace {

// The fused decode step for either pooled-key format (i8: int8 codes in
// pooled_k plus block scales in k_scale).
spx_status decode_impl(const spx_dims* d, int32_t B, const void* raw_k, const float* pool_w,
                       void* tail, void* pooled_k, float* k_scale, bool i8, int64_t cap_blk,
                       const int64_t* len_dev, const void* q_idx, const float* w_head,
                       const void* q, const void* latent, int64_t cap_tok, int64_t max_len,
                       void* out, float* lse, int32_t* idx_out, int32_t* count_out, void* ws,
                       size_t ws_bytes, const spx_timing* timing, spx_stream stream) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  float w[4] = {0.f, 0.f, 0.f, 0.f};
  if (raw_k && (st = check_pool_w(pool_w, w)) != SPX_OK) return st;
  if (B < 1 || B > 65535 || cap_blk < 1 || cap_tok < 1 || max_len < 1) return SPX_ERR_SHAPE;
  if (max_len > kPool * cap_blk || max_len > cap_tok) return SPX_ERR_SHAPE;
  if (cap_blk > (int64_t(1) << 31) - 1 || static_cast<int64_t>(B) * kIdxHeads > (1ll << 31) - 1)
    return SPX_ERR_SHAPE;
  if (!pooled_k || !len_dev || !q_idx || !w_head || !q || !latent || !out)
    return SPX_ERR_INVALID_ARG;
  if (raw_k && !tail) return SPX_ERR_INVALID_ARG;
  if (i8 && (!k_scale || !al4(k_scale))) return SPX_ERR_INVALID_ARG;
  if (!al16(pooled_k) || !al16(q_idx) || !al16(q) || !al16(latent) || !al16(out) ||
      !al4(w_head) || !al4(len_dev) || (raw_k && (!al16(raw_k) || !al16(tail))) ||
      (lse && !al4(lse)) || (idx_out && !al4(idx_out)) || (count_out && !al4(count_out)))
    return SPX_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(B, d->heads, max_len);
  if (L.nchunk > kMaxSelChunks) return SPX_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < L.total || !al16(ws)) return SPX_ERR_WORKSPACE;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int64_t* n_vis = reinterpret_cast<int64_t*>(base + L.nvis);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + L.idx);
  int32_t* count = count_out ? count_out : reinterpret_cast<int32_t*>(base + L.count);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.hist);
  int32_t* done = reinterpret_cast<int32_t*>(base + L.done);
  float* scores = reinterpret_cast<float*>(base + L.scores);

  // 1. append (or just copy the lengths) -> n_vis; reset the selection state
  PoolAppendArgs pa{};
  pa.B = B;
  pa.raw_k = raw_k;
  pa.n_new = raw_k ? 1 : 0;
  for (int i = 0; i < 4; ++i) pa.w[i] = w[i];
  pa.tail = tail;
  pa.pooled_k = pooled_k;
  pa.cap_blk = cap_blk;
  pa.len_dev = len_dev;
  pa.len_host = 0;
  pa.max_len = max_len;
  pa.nvis_out = n_vis;
  pa.init_hist = hist;
  pa.init_done = done;
  pa.pdl = true;
  int8_t* q8 = reinterpret_cast<int8_t*>(base + L.q8);
  float* wq = reinterpret_cast<float*>(base + L.wq);
  if (i8) {
    pa.i8 = true;
    pa.k_scale = k_scale;
    pa.q_idx = q_idx;  // quantised here for the scoring kernel
    pa.w_head = w_head;
    pa.q8 = q8;
    pa.wq = wq;
  }
  cudaError_t e = launch_pool_append(pa, s);
  if (e != cudaSuccess) return SPX_ERR_CUDA;

  // 2. indexer scores and their key histogram
  if (timing && timing->score_begin &&
      cudaEventRecord(static_cast<cudaEvent_t>(timing->score_begin), s) != cudaSuccess)
    return SPX_ERR_CUDA;
  ScoreArgs sa{};
  sa.nq = 1;
  sa.i8 = i8;
  sa.k_scale = k_scale;
  sa.rows = B;
  sa.key_batches = B;
  sa.q_idx = i8 ? static_cast<const void*>(q8) : q_idx;
  sa.w_head = i8 ? wq : w_head;
  sa.pooled_k = pooled_k;
  sa.cap_blk = cap_blk;
  sa.n_vis = n_vis;
  sa.len_spec = len_dev;  // plans the work before the append finishes
  sa.n_add = pa.n_new;
  sa.max_len = max_len;
  sa.scores = scores;
  sa.score_stride = L.stride;
  sa.num_sms = device_sm_count();
  sa.sel_ghist = hist;
  sa.work_counter = done + B;
  // Each kernel of the chain may start while its predecessor finishes (its
  // set-up overlaps; it waits before reading the predecessor's output),
  // except across a timing event.
  sa.pdl = !(timing && timing->score_begin);
  if ((e = launch_index_score(sa, s)) != cudaSuccess) return SPX_ERR_CUDA;
  if (timing && timing->score_end &&
      cudaEventRecord(static_cast<cudaEvent_t>(timing->score_end), s) != cudaSuccess)
    return SPX_ERR_CUDA;
  // 3. top-512 blocks per row: chunks of the scores filtered at the exact
  // cut bin of the scoring kernel's key histogram, the last chunk's CTA
  // making the final choice
  SelectBlocksArgs ma{};
  ma.rows = B;
  ma.scores = scores;
  ma.score_stride = L.stride;
  ma.n_vis = n_vis;
  ma.max_len = max_len;
  ma.ghist = hist;
  ma.nchunk = L.nchunk;
  ma.list_key = reinterpret_cast<uint32_t*>(base + L.lkey);
  ma.list_idx = reinterpret_cast<int32_t*>(base + L.lidx);
  ma.list_cnt = reinterpret_cast<int32_t*>(base + L.lcnt);
  ma.done = done;
  ma.out_idx = idx;
  ma.out_cnt = count;
  ma.pdl = !(timing && timing->score_end);
  if ((e = launch_select_blocks(ma, s)) != cudaSuccess) return SPX_ERR_CUDA;

  // 4. attention over the selected blocks' tokens and the partial tail
  AttnArgs aa{};
  aa.q = q;
  aa.latent = latent;
  aa.seq_stride = cap_tok * kLatent;
  aa.cap_tok = cap_tok;
  aa.idx = idx;
  aa.count = count;
  aa.n_vis = n_vis;
  aa.max_len = max_len;
  aa.sm_scale = d->sm_scale;
  aa.out = out;
  aa.lse = lse;
  aa.ws = base + L.attn;
  aa.pdl = !(timing && timing->score_end);
  return cuda_status(launch_attn(L.ap, aa, s));
}

}  // namespace

extern "C" {

spx_status spx_decode_fused(const spx_dims* d, int32_t B, const void* raw_k, const float* pool_w,
                            void* tail, void* pooled_k, int64_t cap_blk, const int64_t* len_dev,
                            const void* q_idx, const float* w_head, const void* q,
                            const void* latent, int64_t cap_tok, int64_t max_len, void* out,
                            float* lse, int32_t* idx_out, int32_t* count_out, void* ws,
                            size_t ws_bytes, const spx_timing* timing, spx_stream stream) {
  return decode_impl(d, B, raw_k, pool_w, tail, pooled_k, nullptr, false, cap_blk, len_dev, q_idx,
                     w_head, q, latent, cap_tok, max_len, out, lse, idx_out, count_out, ws,
                     ws_bytes, timing, stream);
}

spx_status spx_decode_fused_i8(const spx_dims* d, int32_t B, const void* raw_k,
                               const float* pool_w, void* tail, void* pooled_k8, float* k_scale,
                               int64_t cap_blk, const int64_t* len_dev, const void* q_idx,
                               const float* w_head, const void* q, const void* latent,
                               int64_t cap_tok, int64_t max_len, void* out, float* lse,
                               int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                               const spx_timing* timing, spx_stream stream) {
  return decode_impl(d, B, raw_k, pool_w, tail, pooled_k8, k_scale, true, cap_blk, len_dev, q_idx,
                     w_head, q, latent, cap_tok, max_len, out, lse, idx_out, count_out, ws,
                     ws_bytes, timing, stream);
}

// ---------------------------------------------------------------------------
spx_status spx_prefill_workspace_size(const spx_dims* d, int32_t T, int64_t pos0,
                                      size_t* bytes) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  if (!bytes) return SPX_ERR_INVALID_ARG;
  if (T < 1 || T > 65535 || pos0 < 0) return SPX_ERR_SHAPE;
  *bytes = fused_layout(T, d->heads, pos0 + T).total;
  return SPX_OK;
}

// Chunked prefill, bf16 or INT8 (k_scale set) pooled-key cache.
static spx_status prefill_impl(const spx_dims* d, int32_t T, const void* raw_k, const float* pool_w,
                        void* tail, void* pooled_k, float* k_scale, int64_t cap_blk,
                        int64_t pos0, const void* q_idx, const float* w_head, const void* q,
                        const void* latent, int64_t cap_tok, void* out, float* lse,
                        int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                        const spx_timing* timing, spx_stream stream, bool i8) {
  spx_status st = check_dims(d);
  if (st != SPX_OK) return st;
  float w[4];
  if ((st = check_pool_w(pool_w, w)) != SPX_OK) return st;
  if (T < 1 || T > 65535 || pos0 < 0 || cap_blk < 1 || cap_tok < 1) return SPX_ERR_SHAPE;
  const int64_t max_len = pos0 + T;
  if (max_len > kPool * cap_blk || max_len > cap_tok) return SPX_ERR_SHAPE;
  if (cap_blk > (int64_t(1) << 31) - 1) return SPX_ERR_SHAPE;
  if (!raw_k || !tail || !pooled_k || !q_idx || !w_head || !q || !latent || !out)
    return SPX_ERR_INVALID_ARG;
  if (i8 && (!k_scale || !al4(k_scale))) return SPX_ERR_INVALID_ARG;
  if (!al16(raw_k) || !al16(tail) || !al16(pooled_k) || !al16(q_idx) || !al16(q) ||
      !al16(latent) || !al16(out) || !al4(w_head) || (lse && !al4(lse)) ||
      (idx_out && !al4(idx_out)) || (count_out && !al4(count_out)))
    return SPX_ERR_INVALID_ARG;
  const FusedLayout L = fused_layout(T, d->heads, max_len);
  if (L.nchunk > kMaxSelChunks) return SPX_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < L.total || !al16(ws)) return SPX_ERR_WORKSPACE;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  // rows short enough are selected by one CTA each (scores staged in shared
  // memory); longer ones by key histograms and chunk lists, whose
  // histograms and chunk counters start at zero
  const bool rows_sel = select_rows_fits(max_len);
  if (!rows_sel && cudaMemsetAsync(base + L.hist, 0, L.lkey - L.hist, s) != cudaSuccess)
    return SPX_ERR_CUDA;
  int64_t* n_vis = reinterpret_cast<int64_t*>(base + L.nvis);
  float* scores = reinterpret_cast<float*>(base + L.scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + L.idx);
  int32_t* count = count_out ? count_out : reinterpret_cast<int32_t*>(base + L.count);

  PoolAppendArgs pa{};
  pa.B = 1;
  pa.raw_k = raw_k;
  pa.n_new = T;
  for (int i = 0; i < 4; ++i) pa.w[i] = w[i];
  pa.tail = tail;
  pa.pooled_k = pooled_k;
  pa.cap_blk = cap_blk;
  pa.len_dev = nullptr;
  pa.len_host = pos0;
  pa.max_len = max_len;
  pa.nvis_out = nullptr;
  pa.i8 = i8;
  pa.k_scale = k_scale;
  cudaError_t e = launch_pool_append(pa, s);
  if (e != cudaSuccess) return SPX_ERR_CUDA;
  if ((e = launch_prefill_nvis(n_vis, T, pos0, s)) != cudaSuccess) return SPX_ERR_CUDA;
  int8_t* q8 = reinterpret_cast<int8_t*>(base + L.q8);
  float* wq = reinterpret_cast<float*>(base + L.wq);
  if (i8 && (e = launch_quant_q(T, q_idx, w_head, q8, wq, s)) != cudaSuccess) return SPX_ERR_CUDA;

  if (timing && timing->score_begin &&
      cudaEventRecord(static_cast<cudaEvent_t>(timing->score_begin), s) != cudaSuccess)
    return SPX_ERR_CUDA;
  ScoreArgs sa{};
  sa.nq = 8;
  sa.i8 = i8;
  sa.k_scale = k_scale;
  sa.rows = T;
  sa.key_batches = 1;
  sa.q_idx = i8 ? static_cast<const void*>(q8) : q_idx;
  sa.w_head = i8 ? wq : w_head;
  sa.pooled_k = pooled_k;
  sa.cap_blk = cap_blk;
  sa.n_vis = n_vis;
  sa.max_len = max_len;
  sa.scores = scores;
  sa.score_stride = L.stride;
  sa.num_sms = device_sm_count();
  if ((e = launch_index_score(sa, s)) != cudaSuccess) return SPX_ERR_CUDA;
  if (timing && timing->score_end &&
      cudaEventRecord(static_cast<cudaEvent_t>(timing->score_end), s) != cudaSuccess)
    return SPX_ERR_CUDA;

  // top-512 per query
  SelectBlocksArgs ma{};
  ma.rows = T;
  ma.scores = scores;
  ma.score_stride = L.stride;
  ma.n_vis = n_vis;
  ma.max_len = max_len;
  ma.ghist = reinterpret_cast<uint32_t*>(base + L.hist);
  ma.nchunk = L.nchunk;
  ma.list_key = reinterpret_cast<uint32_t*>(base + L.lkey);
  ma.list_idx = reinterpret_cast<int32_t*>(base + L.lidx);
  ma.list_cnt = reinterpret_cast<int32_t*>(base + L.lcnt);
  ma.done = reinterpret_cast<int32_t*>(base + L.done);
  ma.out_idx = idx;
  ma.out_cnt = count;
  // the selection may start while scoring finishes (except across a timing
  // event); it waits before reading the scores
  ma.pdl = rows_sel && !(timing && timing->score_end);
  if (rows_sel) {
    if ((e = launch_select_rows(ma, device_sm_count(), s)) != cudaSuccess)
      return SPX_ERR_CUDA;
  } else {
    if ((e = launch_key_hist(ma, s)) != cudaSuccess) return SPX_ERR_CUDA;
    if ((e = launch_select_blocks(ma, s)) != cudaSuccess) return SPX_ERR_CUDA;
  }

  AttnArgs aa{};
  aa.q = q;
  aa.latent = latent;
  aa.seq_stride = 0;
  aa.cap_tok = cap_tok;
  aa.idx = idx;
  aa.count = count;
  aa.n_vis = n_vis;
  aa.max_len = max_len;
  aa.sm_scale = d->sm_scale;
  aa.out = out;
  aa.lse = lse;
  aa.ws = base + L.attn;
  aa.pdl = true;  // set-up overlaps the selection; the ids are read after the wait
  return cuda_status(launch_attn(L.ap, aa, s));
}

spx_status spx_prefill_chunk(const spx_dims* d, int32_t T, const void* raw_k, const float* pool_w,
                             void* tail, void* pooled_k, int64_t cap_blk, int64_t pos0,
                             const void* q_idx, const float* w_head, const void* q,
                             const void* latent, int64_t cap_tok, void* out, float* lse,
                             int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                             const spx_timing* timing, spx_stream stream) {
  return prefill_impl(d, T, raw_k, pool_w, tail, pooled_k, nullptr, cap_blk, pos0, q_idx, w_head,
                      q, latent, cap_tok, out, lse, idx_out, count_out, ws, ws_bytes, timing,
                      stream, false);
}

spx_status spx_prefill_chunk_i8(const spx_dims* d, int32_t T, const void* raw_k,
                                const float* pool_w, void* tail, void* pooled_k8, float* k_scale,
                                int64_t cap_blk, int64_t pos0, const void* q_idx,
                                const float* w_head, const void* q, const void* latent,
                                int64_t cap_tok, void* out, float* lse, int32_t* idx_out,
                                int32_t* count_out, void* ws, size_t ws_bytes,
                                const spx_timing* timing, spx_stream stream) {
  return prefill_impl(d, T, raw_k, pool_w, tail, pooled_k8, k_scale, cap_blk, pos0, q_idx, w_head,
                      q, latent, cap_tok, out, lse, idx_out, count_out, ws, ws_bytes, timing,
                      stream, true);
}

}  // extern "C"
