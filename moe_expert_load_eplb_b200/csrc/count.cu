// count.cu -- S1: per-layer expert load histogram of routed top-k indices.
//
// The load of an expert is the number of tokens the router sent it (page
// "DualPipe и EPLB", Part 2, box "От переводчика: термины"):
//   counts[l, e] += #{(t, k) : idx[l, t, k] == e}.
//
// HBM-bound streaming design for B200:
//   * one 1024-thread CTA per SM; CTA b owns a contiguous, 16-byte aligned
//     run of the flattened [L, T*K] index array and walks it layer segment
//     by layer segment, so it meets at most a few layer boundaries;
//   * every thread keeps U = 4 independent 16-byte streaming loads
//     (ld.global.cs) in flight per iteration -- 64 KB per SM -- which on a
//     B200 measured faster than staging the same bytes through shared
//     memory with cp.async.bulk (4- to 12-stage rings, warp-specialised or
//     not);
//   * increments go to a lane-banked shared histogram: bin e of lane j is
//     word e*32 + j, so lane j always hits bank j and one warp-wide atomic
//     is conflict-free whatever the skew of the routing distribution; an
//     index outside [0, E) lands in a sentinel bin E, whose total is the
//     bad-index count (no branch per index);
//   * at each layer boundary and at the end the 32 lane copies of a bin are
//     summed (rotated reads, conflict-free) and added to the int64 output
//     with one global atomic per bin and CTA.
// Integer atomics make the result independent of scheduling.
#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 1024;
constexpr int kU = 4;

struct CountArgs {
  const int32_t *idx;
  int64_t per_layer;  // T * K
  int64_t total;      // L * T * K
  int32_t E;
  int64_t *counts;
  unsigned long long *bad;
};

__global__ void __launch_bounds__(kThreads, 1) count_loads_kernel(CountArgs a) {
  extern __shared__ __align__(16) uint32_t hist[];  // [E+1][32]; bin E counts bad indices
  const int tid = threadIdx.x;
  const uint32_t lane = tid & 31;
  const uint32_t E = static_cast<uint32_t>(a.E);
  const int E1 = a.E + 1;
  for (int i = tid; i < E1 * 32; i += kThreads) hist[i] = 0;
  __syncthreads();

  // this CTA's elements [r0, r1): boundaries rounded down to 4 elements
  const int64_t r0 = (a.total * blockIdx.x / gridDim.x) & ~int64_t(3);
  const int64_t r1 = blockIdx.x + 1 == gridDim.x
                         ? a.total
                         : (a.total * (blockIdx.x + 1) / gridDim.x) & ~int64_t(3);
  uint32_t nbad = 0;
  auto add = [&](int32_t e) {
    const uint32_t ee = static_cast<uint32_t>(e) < E ? static_cast<uint32_t>(e) : E;
    atomicAdd(&hist[ee * 32u + lane], 1u);
  };
  const int4 *vec = reinterpret_cast<const int4 *>(a.idx);

  int64_t g = r0;
  while (g < r1) {
    const int64_t layer = g / a.per_layer;
    const int64_t g1 = min(r1, (layer + 1) * a.per_layer);
    // [g, b0) head, [b0, b1) 16-byte aligned interior, [b1, g1) tail
    const int64_t b0 = min((g + 3) & ~int64_t(3), g1);
    const int64_t b1 = max(g1 & ~int64_t(3), b0);
    if (tid < b0 - g) add(__ldg(a.idx + g + tid));
    if (tid >= 32 && tid - 32 < g1 - b1) add(__ldg(a.idx + b1 + (tid - 32)));
    const int4 *pin = vec + (b0 >> 2);
    const int nvec = static_cast<int>((b1 - b0) >> 2);
    for (int i = tid; i < nvec; i += kThreads * kU) {
      int4 x[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        x[u] = i + u * kThreads < nvec ? __ldcs(pin + i + u * kThreads) : make_int4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (i + u * kThreads < nvec) {
          add(x[u].x);
          add(x[u].y);
          add(x[u].z);
          add(x[u].w);
        }
      }
    }
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
    __syncthreads();
    g = g1;
  }

  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if (lane == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}

}  // namespace

eplb_status launch_count_loads(const int32_t *idx, int64_t L, int64_t per_layer, int32_t E,
                               int64_t *counts, unsigned long long *bad, int32_t *status,
                               cudaStream_t stream) {
  (void)status;  // this kernel has no wait that could run out
  DeviceInfo di;
  if (!device_info(&di)) return cuda_fail(cudaGetLastError());
  const size_t smem = static_cast<size_t>(E + 1) * 32 * sizeof(uint32_t);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  cudaError_t err = cudaFuncSetAttribute(count_loads_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return cuda_fail(err);
  CountArgs a;
  a.idx = idx;
  a.per_layer = per_layer;
  a.total = per_layer * L;
  a.E = E;
  a.counts = counts;
  a.bad = bad;
  // one CTA per SM, fewer when there is too little work to share
  const int64_t grid =
      std::max<int64_t>(1, std::min<int64_t>(di.sms, (a.total + 4095) / 4096));
  count_loads_kernel<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(a);
  err = cudaGetLastError();
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
