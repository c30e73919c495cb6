// planutil.cu -- what a serving engine does around a plan, on the device:
//   * plan_stats: per-GPU load (sum of w / logcnt over the GPU's replicas)
//     and per-row min / max / mean / balancedness = mean / max -- the figures
//     page "DualPipe и EPLB", Part 2, quotes for its worked example (box
//     "От переводчика: что на рисунке", exercise 2 of "что сделать руками");
//   * fold_loads: loads recorded per physical expert -> per logical expert;
//   * initial_map: the plan before any load is known (routed experts first,
//     then the redundant slots cycling through the experts);
//   * plan_diff: which new physical slots must fetch their expert's weights
//     (the rearrangement step after a rebalance), and how many per row.
// One CTA per row everywhere; rows are small (P <= 2048).
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace eplb {
namespace {

constexpr int kThreads = 256;

// fp64 with explicit round-to-nearest operations in a fixed order (slot
// order per GPU, GPU order for the mean), so no contraction or reordering
// changes a bit.
__global__ void __launch_bounds__(kThreads) plan_stats_kernel(
    const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt, int E, int P, int gpus,
    double *gpu_load, double *stats, int32_t *status) {
  extern __shared__ double gl[];  // [gpus]
  const int64_t row = blockIdx.x;
  const int ppg = P / gpus;
  bool bad = false;
  for (int g = threadIdx.x; g < gpus; g += kThreads) {
    double acc = 0.0;
    for (int k = 0; k < ppg; ++k) {
      const int e = phy2log[row * P + g * ppg + k];
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      const int c = logcnt[row * E + e];
      if (c < 1) {
        bad = true;
        continue;
      }
      acc = __dadd_rn(acc, __ddiv_rn(static_cast<double>(loads[row * E + e]), static_cast<double>(c)));
    }
    gl[g] = acc;
    if (gpu_load) gpu_load[row * gpus + g] = acc;
  }
  if (bad) report(status, EPLB_ERR_RANGE);
  __syncthreads();
  if (threadIdx.x == 0 && stats) {
    double mn = gl[0], mx = gl[0], sum = 0.0;
    for (int g = 0; g < gpus; ++g) {
      mn = fmin(mn, gl[g]);
      mx = fmax(mx, gl[g]);
      sum = __dadd_rn(sum, gl[g]);
    }
    const double mean = __ddiv_rn(sum, static_cast<double>(gpus));
    stats[row * 4 + 0] = mn;
    stats[row * 4 + 1] = mx;
    stats[row * 4 + 2] = mean;
    stats[row * 4 + 3] = mx > 0.0 ? __ddiv_rn(mean, mx) : 1.0;
  }
}

__global__ void __launch_bounds__(kThreads) fold_loads_kernel(const int64_t *phys,
                                                              const int32_t *phy2log, int E, int P,
                                                              int64_t *logical, int32_t *status) {
  extern __shared__ unsigned long long acc[];  // [E]
  const int64_t row = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += kThreads) acc[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = threadIdx.x; p < P; p += kThreads) {
    const int e = phy2log[row * P + p];
    if (e < 0 || e >= E) {
      bad = true;
      continue;
    }
    atomicAdd(&acc[e], static_cast<unsigned long long>(phys[row * P + p]));
  }
  if (bad) report(status, EPLB_ERR_RANGE);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    logical[row * E + e] = static_cast<int64_t>(acc[e]);
}

__global__ void initial_map_kernel(int64_t total, int E, int P, int32_t *phy2log,
                                   int32_t *phyrank) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i % P);
    phy2log[i] = p % E;
    if (phyrank) phyrank[i] = p / E;
  }
}

// New slot p of GPU g keeps its expert e in place when fewer earlier new
// slots of g hold e than old slots of g did (the kept replicas are used up
// in slot order); otherwise it copies from the lowest old slot holding e.
__global__ void __launch_bounds__(kThreads) plan_diff_kernel(const int32_t *old_p2l,
                                                             const int32_t *new_p2l, int E, int P,
                                                             int gpus, int32_t *src,
                                                             int32_t *moves, int32_t *status) {
  extern __shared__ int first_old[];  // [E]
  __shared__ int nmoves;
  const int64_t row = blockIdx.x;
  const int32_t *o = old_p2l + row * P;
  const int32_t *n = new_p2l + row * P;
  const int ppg = P / gpus;
  for (int e = threadIdx.x; e < E; e += kThreads) first_old[e] = 0x7fffffff;
  if (threadIdx.x == 0) nmoves = 0;
  __syncthreads();
  bool bad = false;
  for (int p = threadIdx.x; p < P; p += kThreads) {
    const int e = o[p];
    if (e < 0 || e >= E)
      bad = true;
    else
      atomicMin(&first_old[e], p);
  }
  __syncthreads();
  int mine = 0;
  for (int p = threadIdx.x; p < P; p += kThreads) {
    const int e = n[p];
    if (e < 0 || e >= E) {
      bad = true;
      src[row * P + p] = -2;
      continue;
    }
    const int g0 = (p / ppg) * ppg;
    int old_here = 0, new_before = 0;
    for (int k = g0; k < g0 + ppg; ++k) {
      old_here += o[k] == e ? 1 : 0;
      new_before += (k < p && n[k] == e) ? 1 : 0;
    }
    const bool kept = new_before < old_here;
    const int from = first_old[e];
    src[row * P + p] = kept ? -1 : (from == 0x7fffffff ? -2 : from);
    mine += kept ? 0 : 1;
  }
  if (bad) report(status, EPLB_ERR_RANGE);
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if ((threadIdx.x & 31) == 0 && mine) atomicAdd(&nmoves, mine);
  __syncthreads();
  if (threadIdx.x == 0 && moves) moves[row] = nmoves;
}

eplb_status launched(cudaError_t err) { return err == cudaSuccess ? EPLB_OK : cuda_fail(err); }

}  // namespace

eplb_status launch_plan_stats(const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt,
                              int64_t R, int32_t E, int32_t P, int32_t gpus, double *gpu_load,
                              double *stats, int32_t *status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(gpus) * sizeof(double);
  cudaError_t err = cudaFuncSetAttribute(plan_stats_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return cuda_fail(err);
  plan_stats_kernel<<<static_cast<unsigned>(R), kThreads, smem, stream>>>(
      loads, phy2log, logcnt, E, P, gpus, gpu_load, stats, status);
  return launched(cudaGetLastError());
}

eplb_status launch_fold_loads(const int64_t *phys, const int32_t *phy2log, int64_t R, int32_t E,
                              int32_t P, int64_t *logical, int32_t *status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(E) * sizeof(unsigned long long);
  fold_loads_kernel<<<static_cast<unsigned>(R), kThreads, smem, stream>>>(phys, phy2log, E, P,
                                                                          logical, status);
  return launched(cudaGetLastError());
}

eplb_status launch_initial_map(int64_t R, int32_t E, int32_t P, int32_t *phy2log,
                               int32_t *phyrank, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  const int64_t total = R * P;
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(di.sms) * 8);
  initial_map_kernel<<<static_cast<unsigned>(std::max<int64_t>(blocks, 1)), 256, 0, stream>>>(
      total, E, P, phy2log, phyrank);
  return launched(cudaGetLastError());
}

eplb_status launch_plan_diff(const int32_t *old_p2l, const int32_t *new_p2l, int64_t R, int32_t E,
                             int32_t P, int32_t gpus, int32_t *src, int32_t *moves,
                             int32_t *status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(E) * sizeof(int);
  plan_diff_kernel<<<static_cast<unsigned>(R), kThreads, smem, stream>>>(
      old_p2l, new_p2l, E, P, gpus, src, moves, status);
  return launched(cudaGetLastError());
}

}  // namespace eplb
