// internal.h -- launchers behind the C ABI (host side, not exported).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/eplb.h"

namespace eplb {

// Raises fn's dynamic shared-memory limit to `smem` bytes if it is lower
// (once per device and size) and, with per_sm, returns how many
// `threads`-thread CTAs of fn fit on one SM with that much shared memory
// (cached per device, kernel, CTA size and bytes): no per-launch driver
// queries.
eplb_status prepare_kernel(const void *fn, int threads, size_t smem, int *per_sm);

// Launches fn with programmatic stream serialisation (see pdl_trigger /
// pdl_wait in common.cuh); args as for cudaLaunchKernel.
inline cudaError_t launch_pdl(const void *fn, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}


// Devices this library keeps per-device state for (indices 0 .. kMaxDevices-1).
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
};

// Cached per device (queried once); EPLB_ERR_CUDA with the query's own error
// when it failed, EPLB_ERR_LIMIT for a device index of kMaxDevices or more.
eplb_status device_info(DeviceInfo *out);

// Records a CUDA error message for eplb_last_cuda_error() and maps it.
eplb_status cuda_fail(cudaError_t err);

eplb_status launch_count_loads(const int32_t *idx, int64_t L, int64_t per_layer, int32_t E,
                               int64_t *counts, unsigned long long *bad, cudaStream_t stream);

eplb_status launch_window(int64_t *steps, int64_t S, int64_t C, int64_t W, int64_t s_first,
                          int64_t *snaps, int64_t zero_row, cudaStream_t stream);

// Segments up to this many keys are sorted by rank counting; longer ones by
// a bitonic network over a power-of-two padding.
constexpr int kRankSortMax = 512;

struct RebalanceShape {
  int32_t E, P, G, N, gpus, X;   // G, N after the policy choice
  int32_t gs, gpn, lpn, ppn, ppg, mpn;
  int32_t npad;                  // step 3's key stride per node: ppn, or next_pow2(ppn) above kRankSortMax
  int32_t gpad;
  int32_t ibits, qbits, gibits, nqbits;
  int32_t cmax;                  // most replicas one expert can get: ppn - lpn + 1
  uint64_t lam_fixed;            // lcm(1..cmax) when <= 2^62, else 0
};

// Rows' loads are sums of ring_w ring rows of [R, E] (ring_w = 1: a plain
// load array); zero_slot >= 0 clears that ring row after reading it.
eplb_status launch_rebalance(int64_t *ring, int64_t ring_w, int64_t zero_slot, int64_t *loads_out,
                             int64_t R, const RebalanceShape &sh, int32_t *phy2log,
                             int32_t *phyrank, int32_t *logcnt, int32_t *log2phy, double *gpu_load,
                             double *stats, int32_t *status, cudaStream_t stream);

// Redirect; with counts != nullptr the same pass also adds the load histogram.
eplb_status launch_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, int64_t *counts, unsigned long long *bad,
                            int32_t *status, cudaStream_t stream);

// The serving step in one launch: count + redirect with the plan in force
// into ring[slot], then per layer, once its chunks are all counted, the window
// sum and rebalance into the next plan (zeroing ring[zero_slot] if >= 0).
eplb_status launch_serve(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                         const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                         int32_t *out, unsigned long long *bad, int64_t *ring, int64_t W,
                         int64_t slot, int64_t zero_slot, int64_t *loads_out,
                         const RebalanceShape &sh, int32_t *next_phy2log, int32_t *next_phyrank,
                         int32_t *next_logcnt, int32_t *next_log2phy, double *gpu_load,
                         double *stats, uint32_t *layer_done, int32_t *status,
                         cudaStream_t stream);

// Device address of the library-owned per-layer counters of
// eplb_serve_step_noalloc (kStaticLayers of them) on the current device,
// looked up once per device; EPLB_ERR_LIMIT for a device index of
// kMaxDevices or more, EPLB_ERR_CUDA with the look-up's own error otherwise.
constexpr int64_t kStaticLayers = 4096;
eplb_status static_layer_done(uint32_t **out);

eplb_status launch_plan_stats(const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt,
                              int64_t R, int32_t E, int32_t P, int32_t gpus, double *gpu_load,
                              double *stats, int32_t *status, cudaStream_t stream);
eplb_status launch_fold_loads(const int64_t *phys, const int32_t *phy2log, int64_t R, int32_t E,
                              int32_t P, int64_t *logical, int32_t *status, cudaStream_t stream);
eplb_status launch_initial_map(int64_t R, int32_t E, int32_t P, int32_t *phy2log,
                               int32_t *phyrank, cudaStream_t stream);
eplb_status launch_plan_diff(const int32_t *old_p2l, const int32_t *new_p2l, int64_t R, int32_t E,
                             int32_t P, int32_t gpus, int32_t *src, int32_t *moves,
                             int32_t *status, cudaStream_t stream);

}  // namespace eplb
