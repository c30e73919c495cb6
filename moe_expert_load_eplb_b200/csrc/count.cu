// count.cu -- S1: per-layer expert load histogram of routed top-k indices.
//
// The load of an expert is the number of tokens the router sent it (page
// "DualPipe и EPLB", Part 2, box "От переводчика: термины"):
//   counts[l, e] += #{(t, k) : idx[l, t, k] == e}.
//
// HBM-bound design for B200:
//   * persistent grid (SMs x resident CTAs); CTA b owns a contiguous run of
//     16 KB chunks of the flattened [L, T*K] index array (a chunk never
//     crosses a layer), so a CTA meets at most a few layer boundaries;
//   * one elected thread streams chunks into a 4-stage shared-memory ring
//     with 1-D cp.async.bulk copies completing on mbarriers (evict-first
//     L2 policy: every index is read once);
//   * consumers read the stage as 16-byte vectors and increment a
//     lane-banked histogram: bin e of lane j is word e*32 + j, i.e. lane j
//     always hits bank j, so one warp-wide atomic is conflict-free whatever
//     the skew of the routing distribution (no same-address or bank
//     conflicts inside an instruction);
//   * at a layer boundary and at the end the 32 lane copies of every bin
//     are summed (rotated reads, conflict-free) and added to the int64
//     output with one global atomic per bin.
#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 4096;  // int32 elements per stage (16 KB)
constexpr int kStages = 4;

struct CountArgs {
  const int32_t *idx;
  int64_t L;
  int64_t per_layer;  // T * K
  int64_t cpl;        // chunks per layer
  int64_t nchunks;
  int32_t E;
  int64_t *counts;
  unsigned long long *bad;
  int32_t *status;
};

struct Chunk {
  int64_t layer, g0, g1, b0, b1;  // [g0,g1) elements; [b0,b1) 16-byte aligned interior
};

__device__ __forceinline__ Chunk chunk_geometry(const CountArgs &a, int64_t c) {
  Chunk k;
  k.layer = c / a.cpl;
  const int64_t within = c - k.layer * a.cpl;
  k.g0 = k.layer * a.per_layer + within * kChunk;
  k.g1 = min(k.g0 + (int64_t)kChunk, (k.layer + 1) * a.per_layer);
  k.b0 = min((k.g0 + 3) & ~(int64_t)3, k.g1);
  k.b1 = max(k.g1 & ~(int64_t)3, k.b0);
  return k;
}

__global__ void __launch_bounds__(kThreads) count_loads_kernel(CountArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  int32_t *stage = reinterpret_cast<int32_t *>(smem);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + kStages * kChunk * sizeof(int32_t));
  __shared__ __align__(8) uint64_t full[kStages];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int64_t c_begin = a.nchunks * blockIdx.x / gridDim.x;
  const int64_t c_end = a.nchunks * (blockIdx.x + 1) / gridDim.x;
  const int64_t n = c_end - c_begin;
  const uint32_t E = static_cast<uint32_t>(a.E);

  for (int i = tid; i < a.E * 32; i += kThreads) hist[i] = 0;
  uint64_t policy = 0;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    policy = l2_policy_evict_first();
  }
  __syncthreads();

  auto issue = [&](int64_t i) {  // thread 0 only
    const Chunk k = chunk_geometry(a, c_begin + i);
    const int s = static_cast<int>(i % kStages);
    const uint32_t bytes = static_cast<uint32_t>((k.b1 - k.b0) * sizeof(int32_t));
    mbar_arrive_expect_tx(&full[s], bytes);
    if (bytes) bulk_g2s_stream(stage + s * kChunk, a.idx + k.b0, bytes, &full[s], policy);
  };
  if (tid == 0)
    for (int64_t i = 0; i < n && i < kStages; ++i) issue(i);

  auto flush = [&](int64_t layer) {  // all threads; callers synchronise around it
    for (int b = tid; b < a.E; b += kThreads) {
      uint32_t sum = 0;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const int w = b * 32 + ((j + b) & 31);
        sum += hist[w];
        hist[w] = 0;
      }
      if (sum) atomicAdd(reinterpret_cast<unsigned long long *>(a.counts + layer * a.E + b),
                         static_cast<unsigned long long>(sum));
    }
  };

  uint32_t nbad = 0;
  auto add = [&](int32_t e) {
    if (static_cast<uint32_t>(e) < E)
      atomicAdd(&hist[static_cast<uint32_t>(e) * 32u + lane], 1u);
    else
      ++nbad;
  };

  int64_t cur_layer = chunk_geometry(a, c_begin).layer;
  for (int64_t i = 0; i < n; ++i) {
    const Chunk k = chunk_geometry(a, c_begin + i);
    if (k.layer != cur_layer) {  // uniform: every thread computes the same k
      flush(cur_layer);
      __syncthreads();
      cur_layer = k.layer;
    }
    const int s = static_cast<int>(i % kStages);
    const bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>((i / kStages) & 1));
    if (ok) {
      const int4 *v = reinterpret_cast<const int4 *>(stage + s * kChunk);
      const int nv = static_cast<int>((k.b1 - k.b0) >> 2);
#pragma unroll 4
      for (int j = tid; j < nv; j += kThreads) {
        const int4 x = v[j];
        add(x.x);
        add(x.y);
        add(x.z);
        add(x.w);
      }
      const int head = static_cast<int>(k.b0 - k.g0);
      const int tail = static_cast<int>(k.g1 - k.b1);
      if (tid < head) add(__ldg(a.idx + k.g0 + tid));
      if (tid >= 32 && tid - 32 < tail) add(__ldg(a.idx + k.b1 + (tid - 32)));
    }
    if (__syncthreads_or(!ok)) {
      // A copy did not land in time: wait (bounded) for the copies this CTA
      // still has in flight so none writes into freed shared memory, report.
      if (tid == 0) {
        for (int64_t j = i; j < n && j < i + kStages; ++j)
          mbar_wait_bounded(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
        report(a.status, EPLB_ERR_TIMEOUT);
      }
      return;
    }
    if (tid == 0 && i + kStages < n) issue(i + kStages);
  }
  flush(cur_layer);

  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if (lane == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}

size_t count_smem_bytes(int E) {
  return static_cast<size_t>(kStages) * kChunk * sizeof(int32_t) +
         static_cast<size_t>(E) * 32 * sizeof(uint32_t);
}

}  // namespace

eplb_status launch_count_loads(const int32_t *idx, int64_t L, int64_t per_layer, int32_t E,
                               int64_t *counts, unsigned long long *bad, int32_t *status,
                               cudaStream_t stream) {
  DeviceInfo di;
  if (!device_info(&di)) return cuda_fail(cudaGetLastError());
  const size_t smem = count_smem_bytes(E);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  cudaError_t err = cudaFuncSetAttribute(count_loads_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return cuda_fail(err);
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, count_loads_kernel, kThreads, smem);
  if (err != cudaSuccess) return cuda_fail(err);
  if (per_sm < 1) per_sm = 1;
  CountArgs a;
  a.idx = idx;
  a.L = L;
  a.per_layer = per_layer;
  a.cpl = (per_layer + kChunk - 1) / kChunk;
  a.nchunks = a.cpl * L;
  a.E = E;
  a.counts = counts;
  a.bad = bad;
  a.status = status;
  const int64_t grid = std::min<int64_t>(a.nchunks, static_cast<int64_t>(di.sms) * per_sm);
  count_loads_kernel<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(a);
  err = cudaGetLastError();
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
