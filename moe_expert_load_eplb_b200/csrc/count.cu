// count.cu -- S1: per-layer expert load histogram of routed top-k indices.
//
// The load of an expert is the number of tokens the router sent it (page
// "DualPipe и EPLB", Part 2, box "От переводчика: термины"):
//   counts[l, e] += #{(t, k) : idx[l, t, k] == e}.
//
// HBM-bound streaming design for B200:
//   * a layer's work is split over several 512-thread CTAs, which take its
//     blocks of 4096 vectors in turn (they sweep the layer side by side);
//     the grid is just under a whole number of waves (up to 8), so the
//     block scheduler gives the parts of slow SMs to fast ones and no thin
//     last wave is left;
//   * every thread keeps U independent 16-byte streaming loads
//     (ld.global.cs) in flight -- on a B200 this measured faster than
//     staging the same bytes through shared memory with cp.async.bulk (4- to
//     12-stage rings, warp-specialised or not);
//   * increments go to a lane-banked shared histogram: bin e of lane j is
//     word e*32 + j, so lane j always hits bank j and one warp-wide atomic
//     is conflict-free whatever the skew of the routing distribution; an
//     index outside [0, E) is clamped to a sentinel bin E (an unsigned min),
//     whose total is the bad-index count;
//   * at the end two threads per bin sum its 32 lane copies (rotated reads,
//     conflict-free) and add them to the int64 output with one global atomic
//     per bin and CTA.
// Integer atomics make the result independent of scheduling.
#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 512;
constexpr int kU = 8;
constexpr int64_t kChunk = 64 * 1024;  // indices per CTA aimed at
constexpr int64_t kMaxWaves = 8;

struct CountArgs {
  const int32_t *idx;
  int64_t per_layer;  // T * K
  int64_t chunks;     // CTAs per layer
  int32_t E;
  int64_t *counts;
  unsigned long long *bad;
};

__global__ void __launch_bounds__(kThreads) count_loads_kernel(CountArgs a) {
  extern __shared__ __align__(16) uint32_t hist[];  // [E+1][32]; bin E counts bad indices
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x;
  const uint32_t lane = tid & 31;
  const uint32_t E = static_cast<uint32_t>(a.E);
  const int E1 = a.E + 1;
  uint32_t *hist_lane = hist + lane;

  // part j of layer l: blocks j, j + chunks, ... of kThreads * kU vectors
  // of the layer's 16-byte aligned interior [b0, b1), so that the layer's
  // CTAs sweep it side by side (as in the redirect kernel); part 0 also
  // takes the up to 3 elements before b0 and after b1
  const int64_t layer = blockIdx.x / a.chunks;
  const int64_t j = blockIdx.x - layer * a.chunks;
  const int64_t lbase = layer * a.per_layer;
  const int64_t g = lbase, g1 = lbase + a.per_layer;
  const int64_t b0 = min((g + 3) & ~int64_t(3), g1);
  const int64_t b1 = max(g1 & ~int64_t(3), b0);
  const int4 *pin = reinterpret_cast<const int4 *>(a.idx) + (b0 >> 2);
  const int nvec = static_cast<int>((b1 - b0) >> 2);
  const int step = static_cast<int>(a.chunks) * (kThreads * kU);

  // first vectors in flight while the histogram is cleared
  int i = static_cast<int>(j) * (kThreads * kU) + tid;
  int4 x[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u)
    x[u] = i + u * kThreads < nvec ? __ldcs(pin + i + u * kThreads) : make_int4(0, 0, 0, 0);
  for (int q = tid; q < E1 * 32; q += kThreads) hist[q] = 0;
  __syncthreads();

  auto add = [&](int32_t e) { atomicAdd(hist_lane + min(static_cast<uint32_t>(e), E) * 32u, 1u); };
  if (j == 0 && tid < b0 - g) add(__ldg(a.idx + g + tid));
  if (j == 0 && tid >= 32 && tid - 32 < g1 - b1) add(__ldg(a.idx + b1 + (tid - 32)));
  while (i < nvec) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (i + u * kThreads < nvec) {
        add(x[u].x);
        add(x[u].y);
        add(x[u].z);
        add(x[u].w);
      }
    }
    i += step;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      x[u] = i + u * kThreads < nvec ? __ldcs(pin + i + u * kThreads) : make_int4(0, 0, 0, 0);
  }
  __syncthreads();

  // two threads per bin, 16 lane copies each (rotated: conflict-free)
  uint32_t nbad = 0;
  for (int t = tid; t - static_cast<int>(lane) < 2 * E1; t += kThreads) {  // warp-uniform
    const bool live = t < 2 * E1;
    const int b = t >> 1;
    const int h = (t & 1) * 16;
    uint32_t sum = 0;
    if (live) {
#pragma unroll 8
      for (int q = 0; q < 16; ++q) sum += hist[b * 32 + ((q + h + b) & 31)];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    if (!live || (t & 1) || sum == 0) continue;
    if (b < a.E)
      atomicAdd(reinterpret_cast<unsigned long long *>(a.counts + layer * a.E + b),
                static_cast<unsigned long long>(sum));
    else
      nbad += sum;
  }
  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if (lane == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}

}  // namespace

eplb_status launch_count_loads(const int32_t *idx, int64_t L, int64_t per_layer, int32_t E,
                               int64_t *counts, unsigned long long *bad, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  const size_t smem = static_cast<size_t>(E + 1) * 32 * sizeof(uint32_t);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  int per_sm = 0;
  const eplb_status st = prepare_kernel(reinterpret_cast<const void *>(count_loads_kernel),
                                        kThreads, smem, &per_sm);
  if (st != EPLB_OK) return st;
  per_sm = std::max(1, std::min(per_sm, 4));
  CountArgs a;
  a.idx = idx;
  a.per_layer = per_layer;
  a.E = E;
  a.counts = counts;
  a.bad = bad;
  // whole waves of layer chunks, as in the redirect kernel
  const int64_t total = per_layer * L;
  const int64_t slots = static_cast<int64_t>(di.sms) * per_sm;
  const int64_t waves = std::min(std::max<int64_t>(total / (kChunk * slots), 1), kMaxWaves);
  a.chunks = std::max<int64_t>(1, std::min(waves * slots / L, (per_layer + 4095) / 4096));
  const int64_t grid = L * a.chunks;
  if (grid > 0x7fffffffLL) return EPLB_ERR_LIMIT;  // one block per layer chunk
  void *args[] = {&a};
  const cudaError_t err = launch_pdl(reinterpret_cast<const void *>(count_loads_kernel), dim3(static_cast<unsigned>(grid)),
                   dim3(kThreads), smem, stream, args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
