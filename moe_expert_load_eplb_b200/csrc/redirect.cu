// redirect.cu -- S5: logical expert index -> physical replica index.
//
// A planner maps the router's logical indices to physical ones (page
// "DeepSeek开源LPLB...", usage example).  Replica rule: token t of the call
// (global token t0 + t) uses replica (t0 + t) mod logcnt[l, e] for all K
// slots:  out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]].
//
// HBM-bound gather, designed like the count kernel: a persistent grid
// streams 16 KB chunks of the index array through a 4-stage bulk-copy ring;
// the layer's tables (log2phy [E, X] and {logcnt, magic} [E]) sit in shared
// memory, reloaded only when a CTA crosses a layer boundary; results leave
// as 16-byte streaming stores.  Both divisions (position / K for the token,
// token mod logcnt for the slot) are multiply-high with per-divisor magic
// numbers.
#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 4096;  // int32 elements per stage (16 KB)
constexpr int kStages = 4;

struct RedirectArgs {
  const int32_t *idx;
  int32_t *out;
  int64_t per_layer;  // T * K  (< 2^31)
  int64_t cpl;
  int64_t nchunks;
  uint32_t K, k_magic;
  uint32_t t0;
  int32_t E, X;
  const int32_t *log2phy;
  const int32_t *logcnt;
  unsigned long long *bad;
  int32_t *status;
};

struct Chunk {
  int64_t layer, g0, g1, b0, b1;
};

__device__ __forceinline__ Chunk chunk_geometry(const RedirectArgs &a, int64_t c) {
  Chunk k;
  k.layer = c / a.cpl;
  const int64_t within = c - k.layer * a.cpl;
  k.g0 = k.layer * a.per_layer + within * kChunk;
  k.g1 = min(k.g0 + (int64_t)kChunk, (k.layer + 1) * a.per_layer);
  k.b0 = min((k.g0 + 3) & ~(int64_t)3, k.g1);
  k.b1 = max(k.g1 & ~(int64_t)3, k.b0);
  return k;
}

__global__ void __launch_bounds__(kThreads) redirect_kernel(RedirectArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  int32_t *stage = reinterpret_cast<int32_t *>(smem);
  uint2 *cm = reinterpret_cast<uint2 *>(smem + kStages * kChunk * sizeof(int32_t));
  int32_t *l2p = reinterpret_cast<int32_t *>(cm + a.E);
  __shared__ __align__(8) uint64_t full[kStages];

  const int tid = threadIdx.x;
  const int64_t c_begin = a.nchunks * blockIdx.x / gridDim.x;
  const int64_t c_end = a.nchunks * (blockIdx.x + 1) / gridDim.x;
  const int64_t n = c_end - c_begin;
  const uint32_t E = static_cast<uint32_t>(a.E);
  const int EX = a.E * a.X;

  uint64_t policy = 0;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    policy = l2_policy_evict_first();
  }
  __syncthreads();

  auto issue = [&](int64_t i) {
    const Chunk k = chunk_geometry(a, c_begin + i);
    const int s = static_cast<int>(i % kStages);
    const uint32_t bytes = static_cast<uint32_t>((k.b1 - k.b0) * sizeof(int32_t));
    mbar_arrive_expect_tx(&full[s], bytes);
    if (bytes) bulk_g2s_stream(stage + s * kChunk, a.idx + k.b0, bytes, &full[s], policy);
  };
  if (tid == 0)
    for (int64_t i = 0; i < n && i < kStages; ++i) issue(i);

  auto load_tables = [&](int64_t layer) {  // all threads; callers synchronise
    const int32_t *cnt = a.logcnt + layer * a.E;
    for (int e = tid; e < a.E; e += kThreads) {
      const int32_t c = __ldg(cnt + e);
      const bool valid = c >= 1 && c <= a.X;
      cm[e] = make_uint2(valid ? static_cast<uint32_t>(c) : 0u,
                         valid ? 0xffffffffu / static_cast<uint32_t>(c) : 0u);
    }
    const int32_t *src = a.log2phy + layer * EX;
    for (int i = tid; i < EX; i += kThreads) l2p[i] = __ldg(src + i);
  };

  uint32_t nbad = 0;
  bool range_err = false;
  // Physical index of the element at within-layer position pos with value e.
  auto map = [&](uint32_t pos, int32_t e) -> int32_t {
    if (static_cast<uint32_t>(e) >= E) {
      ++nbad;
      return -1;
    }
    const uint2 c = cm[e];
    if (c.x == 0) {
      range_err = true;
      return -1;
    }
    const uint32_t tok = a.t0 + div_magic(pos, a.K, a.k_magic);
    return l2p[e * a.X + static_cast<int>(mod_magic(tok, c.x, c.y))];
  };

  int64_t cur_layer = chunk_geometry(a, c_begin).layer;
  load_tables(cur_layer);
  __syncthreads();
  for (int64_t i = 0; i < n; ++i) {
    const Chunk k = chunk_geometry(a, c_begin + i);
    if (k.layer != cur_layer) {
      cur_layer = k.layer;
      load_tables(cur_layer);
      __syncthreads();
    }
    const int s = static_cast<int>(i % kStages);
    const bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>((i / kStages) & 1));
    if (ok) {
      const int64_t layer_base = k.layer * a.per_layer;
      const int4 *v = reinterpret_cast<const int4 *>(stage + s * kChunk);
      int4 *o = reinterpret_cast<int4 *>(a.out + k.b0);
      const uint32_t pos0 = static_cast<uint32_t>(k.b0 - layer_base);
      const int nv = static_cast<int>((k.b1 - k.b0) >> 2);
#pragma unroll 4
      for (int j = tid; j < nv; j += kThreads) {
        const int4 x = v[j];
        const uint32_t p = pos0 + 4u * static_cast<uint32_t>(j);
        int4 y;
        y.x = map(p, x.x);
        y.y = map(p + 1, x.y);
        y.z = map(p + 2, x.z);
        y.w = map(p + 3, x.w);
        __stcs(o + j, y);
      }
      const int head = static_cast<int>(k.b0 - k.g0);
      const int tail = static_cast<int>(k.g1 - k.b1);
      if (tid < head) {
        const int64_t g = k.g0 + tid;
        a.out[g] = map(static_cast<uint32_t>(g - layer_base), __ldg(a.idx + g));
      }
      if (tid >= 32 && tid - 32 < tail) {
        const int64_t g = k.b1 + (tid - 32);
        a.out[g] = map(static_cast<uint32_t>(g - layer_base), __ldg(a.idx + g));
      }
    }
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        for (int64_t j = i; j < n && j < i + kStages; ++j)
          mbar_wait_bounded(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
        report(a.status, EPLB_ERR_TIMEOUT);
      }
      return;
    }
    if (tid == 0 && i + kStages < n) issue(i + kStages);
  }

  if (range_err) report(a.status, EPLB_ERR_RANGE);
  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if ((tid & 31) == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}

size_t redirect_smem_bytes(int E, int X) {
  return static_cast<size_t>(kStages) * kChunk * sizeof(int32_t) + static_cast<size_t>(E) * 8 +
         static_cast<size_t>(E) * X * sizeof(int32_t);
}

}  // namespace

eplb_status launch_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, unsigned long long *bad, int32_t *status,
                            cudaStream_t stream) {
  DeviceInfo di;
  if (!device_info(&di)) return cuda_fail(cudaGetLastError());
  const size_t smem = redirect_smem_bytes(E, X);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  cudaError_t err = cudaFuncSetAttribute(redirect_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return cuda_fail(err);
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, redirect_kernel, kThreads, smem);
  if (err != cudaSuccess) return cuda_fail(err);
  if (per_sm < 1) per_sm = 1;
  RedirectArgs a;
  a.idx = idx;
  a.out = out;
  a.per_layer = T * K;
  a.cpl = (a.per_layer + kChunk - 1) / kChunk;
  a.nchunks = a.cpl * L;
  a.K = static_cast<uint32_t>(K);
  a.k_magic = 0xffffffffu / static_cast<uint32_t>(K);
  a.t0 = static_cast<uint32_t>(t0);
  a.E = E;
  a.X = X;
  a.log2phy = log2phy;
  a.logcnt = logcnt;
  a.bad = bad;
  a.status = status;
  const int64_t grid = std::min<int64_t>(a.nchunks, static_cast<int64_t>(di.sms) * per_sm);
  redirect_kernel<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(a);
  err = cudaGetLastError();
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
