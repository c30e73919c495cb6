// redirect.cu -- S5: logical expert index -> physical replica index.
//
// A planner maps the router's logical indices to physical ones (page
// "DeepSeek开源LPLB...", usage example).  Replica rule: token t of the call
// (global token t0 + t) uses replica (t0 + t) mod logcnt[l, e] for all K
// slots:  out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]].
//
// HBM-bound gather, streamed like the count kernel: each CTA owns a
// contiguous 16-byte aligned run of the flattened index array and walks it
// layer segment by layer segment; the segment's tables (log2phy [E, X] and
// {logcnt, magic} [E]) are loaded into shared memory once per segment;
// every thread keeps U = 4 independent 16-byte streaming loads in flight and
// writes 16-byte streaming stores.  Both divisions (position / K for the
// token, token mod logcnt for the slot) are multiply-high with per-divisor
// magic numbers; with K % 4 == 0 the four indices of a vector share a token.
//
// The same walker with kCount also builds the load histogram of S1 (the
// count kernel's lane-banked shared histogram, flushed per layer segment),
// so counting and redirecting one batch read its indices from HBM once:
// 8 bytes per index instead of 4 + 8.
#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 512;
constexpr int kU = 4;

struct RedirectArgs {
  const int32_t *idx;
  int64_t *counts;  // kCount only
  int32_t *out;
  int64_t per_layer;  // T * K  (< 2^31)
  int64_t total;
  uint32_t K, k_magic;
  uint32_t t0;
  int32_t E, X;
  const int32_t *log2phy;
  const int32_t *logcnt;
  unsigned long long *bad;
  int32_t *status;
};

template <bool kVecToken, bool kCount>
__global__ void __launch_bounds__(kThreads) redirect_kernel(RedirectArgs a) {
  // Tables carry a sentinel row E: an index outside [0, E) maps to it, so the
  // per-index path has no branch -- its log2phy entry is -1 and its histogram
  // bin (kCount) counts the bad indices.  An expert whose logcnt is outside
  // [1, X] gets logcnt 1 and a -1 entry in the shared copy (reported once).
  extern __shared__ __align__(16) unsigned char smem[];
  const int E1 = a.E + 1;
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem);  // [E+1][32], kCount only
  uint2 *cm = reinterpret_cast<uint2 *>(smem + (kCount ? E1 * 32 * sizeof(uint32_t) : 0));
  int32_t *l2p = reinterpret_cast<int32_t *>(cm + E1);  // [E+1][X]
  const int tid = threadIdx.x;
  const uint32_t lane = tid & 31;
  if (kCount) {
    for (int i = tid; i < E1 * 32; i += kThreads) hist[i] = 0;
  }
  const uint32_t E = static_cast<uint32_t>(a.E);
  const uint32_t X = static_cast<uint32_t>(a.X);
  const int EX = a.E * a.X;

  const int64_t r0 = (a.total * blockIdx.x / gridDim.x) & ~int64_t(3);
  const int64_t r1 = blockIdx.x + 1 == gridDim.x
                         ? a.total
                         : (a.total * (blockIdx.x + 1) / gridDim.x) & ~int64_t(3);
  uint32_t nbad = 0;
  bool range_err = false;
  // physical index of element value e whose token is tok (global)
  auto map = [&](int32_t e, uint32_t tok) -> int32_t {
    const bool ok = static_cast<uint32_t>(e) < E;
    const uint32_t ee = ok ? static_cast<uint32_t>(e) : E;
    if (kCount)
      atomicAdd(&hist[ee * 32u + lane], 1u);
    else
      nbad += ok ? 0u : 1u;
    const uint2 c = cm[ee];
    return l2p[ee * X + mod_magic(tok, c.x, c.y)];
  };

  int64_t g = r0;
  while (g < r1) {
    const int64_t layer = g / a.per_layer;
    const int64_t lbase = layer * a.per_layer;
    const int64_t g1 = min(r1, lbase + a.per_layer);
    __syncthreads();  // previous segment's table reads are done
    const int32_t *src = a.log2phy + layer * EX;
    for (int i = tid; i < EX; i += kThreads) l2p[i] = __ldg(src + i);
    if (tid < a.X) l2p[EX + tid] = -1;
    __syncthreads();
    const int32_t *cnt = a.logcnt + layer * a.E;
    for (int e = tid; e <= a.E; e += kThreads) {
      int32_t c = e < a.E ? __ldg(cnt + e) : 1;
      if (c < 1 || c > a.X) {
        range_err = true;
        c = 1;
        l2p[e * a.X] = -1;
      }
      cm[e] = make_uint2(static_cast<uint32_t>(c), 0xffffffffu / static_cast<uint32_t>(c));
    }
    __syncthreads();

    const int64_t b0 = min((g + 3) & ~int64_t(3), g1);
    const int64_t b1 = max(g1 & ~int64_t(3), b0);
    if (tid < b0 - g) {
      const int64_t p = g + tid;
      a.out[p] = map(__ldg(a.idx + p),
                     a.t0 + div_magic(static_cast<uint32_t>(p - lbase), a.K, a.k_magic));
    }
    if (tid >= 32 && tid - 32 < g1 - b1) {
      const int64_t p = b1 + (tid - 32);
      a.out[p] = map(__ldg(a.idx + p),
                     a.t0 + div_magic(static_cast<uint32_t>(p - lbase), a.K, a.k_magic));
    }
    // 16-byte vectors of this segment, indexed from its first one (32-bit)
    const int4 *pin = reinterpret_cast<const int4 *>(a.idx + b0);
    int4 *pout = reinterpret_cast<int4 *>(a.out + b0);
    const int nvec = static_cast<int>((b1 - b0) >> 2);
    const uint32_t pos0 = static_cast<uint32_t>(b0 - lbase);
    for (int i = tid; i < nvec; i += kThreads * kU) {
      int4 x[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        x[u] = i + u * kThreads < nvec ? __ldcs(pin + i + u * kThreads) : make_int4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int v = i + u * kThreads;
        if (v < nvec) {
          const uint32_t pos = pos0 + 4u * static_cast<uint32_t>(v);
          int4 y;
          if (kVecToken) {
            const uint32_t tok = a.t0 + div_magic(pos, a.K, a.k_magic);
            y.x = map(x[u].x, tok);
            y.y = map(x[u].y, tok);
            y.z = map(x[u].z, tok);
            y.w = map(x[u].w, tok);
          } else {
            y.x = map(x[u].x, a.t0 + div_magic(pos, a.K, a.k_magic));
            y.y = map(x[u].y, a.t0 + div_magic(pos + 1, a.K, a.k_magic));
            y.z = map(x[u].z, a.t0 + div_magic(pos + 2, a.K, a.k_magic));
            y.w = map(x[u].w, a.t0 + div_magic(pos + 3, a.K, a.k_magic));
          }
          __stcs(pout + v, y);
        }
      }
    }
    if (kCount) {
      __syncthreads();
      for (int b = tid; b <= a.E; b += kThreads) {
        uint32_t sum = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
          const int w = b * 32 + ((j + b) & 31);
          sum += hist[w];
          hist[w] = 0;
        }
        if (sum == 0) continue;
        if (b < a.E)
          atomicAdd(reinterpret_cast<unsigned long long *>(a.counts + layer * a.E + b),
                    static_cast<unsigned long long>(sum));
        else
          nbad += sum;
      }
    }
    g = g1;
  }

  if (range_err) report(a.status, EPLB_ERR_RANGE);
  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if (lane == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}

}  // namespace

eplb_status launch_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, int64_t *counts, unsigned long long *bad,
                            int32_t *status, cudaStream_t stream) {
  DeviceInfo di;
  if (!device_info(&di)) return cuda_fail(cudaGetLastError());
  const bool count = counts != nullptr;
  const size_t smem = (count ? static_cast<size_t>(E + 1) * 32 * sizeof(uint32_t) : 0) +
                      static_cast<size_t>(E + 1) * 8 + static_cast<size_t>(E + 1) * X * sizeof(int32_t);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  RedirectArgs a;
  a.idx = idx;
  a.counts = counts;
  a.out = out;
  a.per_layer = T * K;
  a.total = a.per_layer * L;
  a.K = static_cast<uint32_t>(K);
  a.k_magic = 0xffffffffu / static_cast<uint32_t>(K);
  a.t0 = static_cast<uint32_t>(t0);
  a.E = E;
  a.X = X;
  a.log2phy = log2phy;
  a.logcnt = logcnt;
  a.bad = bad;
  a.status = status;
  const bool vec_token = (K % 4) == 0;
  const void *fn;
  if (count)
    fn = vec_token ? reinterpret_cast<const void *>(redirect_kernel<true, true>)
                   : reinterpret_cast<const void *>(redirect_kernel<false, true>);
  else
    fn = vec_token ? reinterpret_cast<const void *>(redirect_kernel<true, false>)
                   : reinterpret_cast<const void *>(redirect_kernel<false, false>);
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return cuda_fail(err);
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
  if (err != cudaSuccess) return cuda_fail(err);
  per_sm = std::max(1, std::min(per_sm, 2));
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(static_cast<int64_t>(di.sms) * per_sm, (a.total + 4095) / 4096));
  void *args[] = {&a};
  err = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(grid)), dim3(kThreads), args, smem, stream);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
