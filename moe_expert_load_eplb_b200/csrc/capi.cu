// capi.cu -- the exported C ABI of libeplb.so: argument checks, policy
// choice and launches.  Declarations and contracts are in include/eplb.h.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "internal.h"

namespace eplb {
namespace {

std::once_flag g_once[kMaxDevices];
DeviceInfo g_info[kMaxDevices];
cudaError_t g_err[kMaxDevices];

thread_local char g_last_error[256] = "no error";

int bit_width(int64_t v) {  // bits needed to write v >= 0 (0 -> 0)
  int b = 0;
  while (v > 0) {
    ++b;
    v >>= 1;
  }
  return b;
}

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace {
std::mutex g_kernel_mu;
std::map<std::pair<int, const void *>, size_t> g_smem_set;                 // (device, fn) -> bytes
std::map<std::tuple<int, const void *, int, size_t>, int> g_blocks_per_sm;  // occupancy
}  // namespace

eplb_status prepare_kernel(const void *fn, int threads, size_t smem, int *per_sm) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err);
  std::lock_guard<std::mutex> lock(g_kernel_mu);
  const auto key = std::make_pair(dev, fn);
  const auto it = g_smem_set.find(key);
  if (it == g_smem_set.end() || it->second < smem) {
    err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return cuda_fail(err);
    g_smem_set[key] = smem;
  }
  if (per_sm != nullptr) {
    const auto okey = std::make_tuple(dev, fn, threads, smem);
    const auto oit = g_blocks_per_sm.find(okey);
    if (oit != g_blocks_per_sm.end()) {
      *per_sm = oit->second;
    } else {
      int n = 0;
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem);
      if (err != cudaSuccess) return cuda_fail(err);
      g_blocks_per_sm[okey] = n;
      *per_sm = n;
    }
  }
  return EPLB_OK;
}

eplb_status device_info(DeviceInfo *out) {
  int dev = 0;
  const cudaError_t gerr = cudaGetDevice(&dev);
  if (gerr != cudaSuccess) return cuda_fail(gerr);
  if (dev < 0 || dev >= kMaxDevices) return EPLB_ERR_LIMIT;
  std::call_once(g_once[dev], [dev]() {
    DeviceInfo d;
    g_err[dev] = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_err[dev] == cudaSuccess)
      g_err[dev] = cudaDeviceGetAttribute(&d.max_smem_optin,
                                          cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    g_info[dev] = d;
  });
  // the queries' own error, kept for every later call on this device
  if (g_err[dev] != cudaSuccess) return cuda_fail(g_err[dev]);
  *out = g_info[dev];
  return EPLB_OK;
}

eplb_status cuda_fail(cudaError_t err) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(err),
                cudaGetErrorString(err));
  return EPLB_ERR_CUDA;
}

}  // namespace eplb

using namespace eplb;

extern "C" {

const char *eplb_status_string(int32_t status) {
  switch (status) {
    case EPLB_OK: return "EPLB_OK";
    case EPLB_ERR_NULL: return "EPLB_ERR_NULL";
    case EPLB_ERR_SHAPE: return "EPLB_ERR_SHAPE";
    case EPLB_ERR_DIVISIBILITY: return "EPLB_ERR_DIVISIBILITY";
    case EPLB_ERR_RANGE: return "EPLB_ERR_RANGE";
    case EPLB_ERR_SLOTS: return "EPLB_ERR_SLOTS";
    case EPLB_ERR_CUDA: return "EPLB_ERR_CUDA";
    case EPLB_ERR_TIMEOUT: return "EPLB_ERR_TIMEOUT";
    case EPLB_ERR_ALIGN: return "EPLB_ERR_ALIGN";
    case EPLB_ERR_LIMIT: return "EPLB_ERR_LIMIT";
    case EPLB_ERR_INTERNAL: return "EPLB_ERR_INTERNAL";
    default: return "EPLB_ERR_UNKNOWN";
  }
}

const char *eplb_last_cuda_error(void) { return g_last_error; }

int32_t eplb_abi_version(void) { return (2 << 16) | 0; }

int32_t eplb_checking_build(void) {
#ifdef EPLB_CHECKS
  return 1;
#else
  return 0;
#endif
}

eplb_status eplb_count_loads(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                             int64_t *counts, int32_t accumulate, unsigned long long *bad,
                             cudaStream_t stream) {
  if (L < 0 || T < 0 || K < 1 || E < 1) return EPLB_ERR_SHAPE;
  if (E > 1024 || T > (int64_t(1) << 31) / K) return EPLB_ERR_LIMIT;
  if (L == 0) return EPLB_OK;
  if (counts == nullptr) return EPLB_ERR_NULL;
  if (T > 0 && idx == nullptr) return EPLB_ERR_NULL;
  if (T > 0 && !aligned16(idx)) return EPLB_ERR_ALIGN;
  if (!accumulate) {
    const cudaError_t err =
        cudaMemsetAsync(counts, 0, static_cast<size_t>(L) * E * sizeof(int64_t), stream);
    if (err != cudaSuccess) return cuda_fail(err);
  }
  if (T == 0) return EPLB_OK;
  return launch_count_loads(idx, L, T * K, E, counts, bad, stream);
}

eplb_status eplb_window_accumulate(int64_t *steps, int64_t S, int64_t L, int32_t E,
                                   int64_t W, int64_t s_first, int64_t *snaps, int64_t zero_row,
                                   cudaStream_t stream) {
  if (S < 0 || L < 0 || E < 1 || W < 1 || s_first < 0) return EPLB_ERR_SHAPE;
  if (zero_row < -1 || (zero_row >= S && S > 0)) return EPLB_ERR_SHAPE;
  if (S == 0 || L == 0) return s_first == 0 ? EPLB_OK : EPLB_ERR_SHAPE;
  if (s_first >= S) return EPLB_ERR_SHAPE;
  if (steps == nullptr || snaps == nullptr) return EPLB_ERR_NULL;
  const int64_t C = L * E;
  if (C > (int64_t(1) << 34)) return EPLB_ERR_LIMIT;
  return launch_window(steps, S, C, W, s_first, snaps, zero_row, stream);
}

static eplb_status rebalance_shape(int64_t R, int32_t E, int32_t P, int32_t G, int32_t N,
                                   int32_t gpus, int32_t X, RebalanceShape *out) {
  if (R < 0 || E < 1 || P < 1 || G < 1 || N < 1 || gpus < 1 || X < 1) return EPLB_ERR_SHAPE;
  if (P < E) return EPLB_ERR_SHAPE;
  if (E > 1024 || P > 2048 || R > 0x7fffffffLL) return EPLB_ERR_LIMIT;
  if (E % G != 0 || P % gpus != 0) return EPLB_ERR_DIVISIBILITY;
  RebalanceShape sh;
  sh.E = E;
  sh.P = P;
  sh.gpus = gpus;
  sh.X = X;
  if (G % N == 0) {  // hierarchical policy
    if (gpus % N != 0) return EPLB_ERR_DIVISIBILITY;
    sh.G = G;
    sh.N = N;
  } else {  // global policy: one group on one node
    sh.G = 1;
    sh.N = 1;
  }
  if (static_cast<int64_t>(E) * X > (int64_t(1) << 26)) return EPLB_ERR_LIMIT;
  sh.gs = E / sh.G;
  sh.gpn = sh.G / sh.N;
  sh.lpn = E / sh.N;
  sh.ppn = P / sh.N;
  sh.ppg = P / gpus;
  sh.mpn = gpus / sh.N;
  // the rank sort needs no padding (the stride is ppn: the key areas, sized
  // by npad, hold 4 x 72 instead of 4 x 128 keys on the DeepSeek-V3 shape,
  // so 6 rows share an SM instead of 5); the bitonic network does
  sh.npad = sh.ppn <= kRankSortMax ? sh.ppn : next_pow2(sh.ppn);
  sh.gpad = next_pow2(sh.G);
  sh.ibits = bit_width(sh.ppn);
  sh.qbits = bit_width(sh.mpn - 1);
  sh.gibits = bit_width(sh.G);
  sh.nqbits = bit_width(sh.N - 1);
  sh.cmax = sh.ppn - sh.lpn + 1;
  {
    unsigned __int128 lam = 1;
    for (int c = 2; c <= sh.cmax && lam != 0; ++c) {
      unsigned __int128 a = lam, b = static_cast<unsigned __int128>(c);
      while (b != 0) {
        const unsigned __int128 t = a % b;
        a = b;
        b = t;
      }
      lam = lam / a * c;
      if (lam > (static_cast<unsigned __int128>(1) << 62)) lam = 0;
    }
    sh.lam_fixed = static_cast<uint64_t>(lam);
  }
  *out = sh;
  return EPLB_OK;
}

eplb_status eplb_rebalance(const int64_t *loads, int64_t R, int32_t E, int32_t P, int32_t G,
                           int32_t N, int32_t gpus, int32_t X, int32_t *phy2log,
                           int32_t *phyrank, int32_t *logcnt, int32_t *log2phy, double *gpu_load,
                           double *stats, int32_t *status, cudaStream_t stream) {
  RebalanceShape sh;
  const eplb_status st = rebalance_shape(R, E, P, G, N, gpus, X, &sh);
  if (st != EPLB_OK || R == 0) return st;
  if (!loads || !phy2log || !phyrank || !logcnt || !log2phy) return EPLB_ERR_NULL;
  // the kernel only reads the load array when no ring slot is cleared
  return launch_rebalance(const_cast<int64_t *>(loads), 1, -1, nullptr, R, sh, phy2log, phyrank,
                          logcnt, log2phy, gpu_load, stats, status, stream);
}

eplb_status eplb_rebalance_window(int64_t *ring, int64_t W, int64_t zero_slot, int64_t R,
                                  int32_t E, int32_t P, int32_t G, int32_t N, int32_t gpus,
                                  int32_t X, int64_t *loads_out, int32_t *phy2log,
                                  int32_t *phyrank, int32_t *logcnt, int32_t *log2phy,
                                  double *gpu_load, double *stats, int32_t *status,
                                  cudaStream_t stream) {
  if (W < 1 || zero_slot < -1 || zero_slot >= W) return EPLB_ERR_SHAPE;
  RebalanceShape sh;
  const eplb_status st = rebalance_shape(R, E, P, G, N, gpus, X, &sh);
  if (st != EPLB_OK || R == 0) return st;
  if (!ring || !phy2log || !phyrank || !logcnt || !log2phy) return EPLB_ERR_NULL;
  return launch_rebalance(ring, W, zero_slot, loads_out, R, sh, phy2log, phyrank, logcnt, log2phy,
                          gpu_load, stats, status, stream);
}

eplb_status eplb_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                          const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                          int32_t *out, unsigned long long *bad, int32_t *status,
                          cudaStream_t stream) {
  if (L < 0 || T < 0 || K < 1 || E < 1 || X < 1 || t0 < 0) return EPLB_ERR_SHAPE;
  if (E > 1024 || static_cast<int64_t>(E) * X > 32768) return EPLB_ERR_LIMIT;
  if (T >= (int64_t(1) << 31) / K || t0 + T >= (int64_t(1) << 31)) return EPLB_ERR_LIMIT;
  if (L == 0 || T == 0) return EPLB_OK;
  if (!idx || !log2phy || !logcnt || !out) return EPLB_ERR_NULL;
  if (!aligned16(idx) || !aligned16(out)) return EPLB_ERR_ALIGN;
  return launch_redirect(idx, L, T, K, E, log2phy, X, logcnt, t0, out, nullptr, bad, status,
                         stream);
}

eplb_status eplb_count_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                                int64_t *counts, int32_t accumulate, const int32_t *log2phy,
                                int32_t X, const int32_t *logcnt, int64_t t0, int32_t *out,
                                unsigned long long *bad, int32_t *status, cudaStream_t stream) {
  if (L < 0 || T < 0 || K < 1 || E < 1 || X < 1 || t0 < 0) return EPLB_ERR_SHAPE;
  if (E > 1024 || static_cast<int64_t>(E) * X > 32768) return EPLB_ERR_LIMIT;
  if (T >= (int64_t(1) << 31) / K || t0 + T >= (int64_t(1) << 31)) return EPLB_ERR_LIMIT;
  if (L == 0) return EPLB_OK;
  if (counts == nullptr) return EPLB_ERR_NULL;
  if (T > 0 && (!idx || !log2phy || !logcnt || !out)) return EPLB_ERR_NULL;
  if (T > 0 && (!aligned16(idx) || !aligned16(out))) return EPLB_ERR_ALIGN;
  if (!accumulate) {
    const cudaError_t err =
        cudaMemsetAsync(counts, 0, static_cast<size_t>(L) * E * sizeof(int64_t), stream);
    if (err != cudaSuccess) return cuda_fail(err);
  }
  if (T == 0) return EPLB_OK;
  return launch_redirect(idx, L, T, K, E, log2phy, X, logcnt, t0, out, counts, bad, status,
                         stream);
}

eplb_status eplb_serve_step(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, unsigned long long *bad, int64_t *ring, int64_t W,
                            int64_t slot, int64_t zero_slot, int32_t P, int32_t G, int32_t N,
                            int32_t gpus, int64_t *loads_out, int32_t *next_phy2log,
                            int32_t *next_phyrank, int32_t *next_logcnt, int32_t *next_log2phy,
                            double *gpu_load, double *stats, uint32_t *layer_done,
                            int32_t *status, cudaStream_t stream) {
  if (L < 0 || T < 0 || K < 1 || E < 1 || X < 1 || t0 < 0) return EPLB_ERR_SHAPE;
  if (W < 1 || slot < 0 || slot >= W || zero_slot < -1 || zero_slot >= W) return EPLB_ERR_SHAPE;
  if (E > 1024 || static_cast<int64_t>(E) * X > 32768) return EPLB_ERR_LIMIT;
  if (T >= (int64_t(1) << 31) / K || t0 + T >= (int64_t(1) << 31)) return EPLB_ERR_LIMIT;
  RebalanceShape sh;
  const eplb_status st = rebalance_shape(L, E, P, G, N, gpus, X, &sh);
  if (st != EPLB_OK || L == 0) return st;
  if (!log2phy || !logcnt || !ring || !next_phy2log || !next_phyrank || !next_logcnt ||
      !next_log2phy || !layer_done)
    return EPLB_ERR_NULL;
  if (T > 0 && (!idx || !out)) return EPLB_ERR_NULL;
  if (T > 0 && (!aligned16(idx) || !aligned16(out))) return EPLB_ERR_ALIGN;
  // the plan in force is read while the next one is written
  if (next_log2phy == log2phy || next_logcnt == logcnt) return EPLB_ERR_SHAPE;
  return launch_serve(idx, L, T, K, E, log2phy, X, logcnt, t0, out, bad, ring, W, slot, zero_slot,
                      loads_out, sh, next_phy2log, next_phyrank, next_logcnt, next_log2phy,
                      gpu_load, stats, layer_done, status, stream);
}

eplb_status eplb_serve_step_noalloc(const int32_t *idx, int64_t L, int64_t T, int32_t K,
                                    int32_t E, const int32_t *log2phy, int32_t X,
                                    const int32_t *logcnt, int64_t t0, int32_t *out,
                                    unsigned long long *bad, int64_t *ring, int64_t W,
                                    int64_t slot, int64_t zero_slot, int32_t P, int32_t G,
                                    int32_t N, int32_t gpus, int64_t *loads_out,
                                    int32_t *next_phy2log, int32_t *next_phyrank,
                                    int32_t *next_logcnt, int32_t *next_log2phy, double *gpu_load,
                                    double *stats, int32_t *status, cudaStream_t stream) {
  if (L > kStaticLayers) return EPLB_ERR_LIMIT;
  if (L <= 0) {
    return eplb_serve_step(idx, L, T, K, E, log2phy, X, logcnt, t0, out, bad, ring, W, slot,
                           zero_slot, P, G, N, gpus, loads_out, next_phy2log, next_phyrank,
                           next_logcnt, next_log2phy, gpu_load, stats, nullptr, status, stream);
  }
  uint32_t *counters = nullptr;
  const eplb_status cst = static_layer_done(&counters);
  if (cst != EPLB_OK) return cst;
  return eplb_serve_step(idx, L, T, K, E, log2phy, X, logcnt, t0, out, bad, ring, W, slot,
                         zero_slot, P, G, N, gpus, loads_out, next_phy2log, next_phyrank,
                         next_logcnt, next_log2phy, gpu_load, stats, counters, status, stream);
}

eplb_status eplb_plan_stats(const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt,
                            int64_t R, int32_t E, int32_t P, int32_t gpus, double *gpu_load,
                            double *stats, int32_t *status, cudaStream_t stream) {
  if (R < 0 || E < 1 || P < 1 || gpus < 1) return EPLB_ERR_SHAPE;
  if (P % gpus != 0) return EPLB_ERR_DIVISIBILITY;
  if (gpus > 16384 || R > 0x7fffffffLL) return EPLB_ERR_LIMIT;
  if (R == 0) return EPLB_OK;
  if (!loads || !phy2log || !logcnt || (!gpu_load && !stats)) return EPLB_ERR_NULL;
  return launch_plan_stats(loads, phy2log, logcnt, R, E, P, gpus, gpu_load, stats, status, stream);
}

eplb_status eplb_fold_loads(const int64_t *phys, const int32_t *phy2log, int64_t R, int32_t E,
                            int32_t P, int64_t *logical, int32_t *status, cudaStream_t stream) {
  if (R < 0 || E < 1 || P < 1) return EPLB_ERR_SHAPE;
  if (E > 4096 || R > 0x7fffffffLL) return EPLB_ERR_LIMIT;
  if (R == 0) return EPLB_OK;
  if (!phys || !phy2log || !logical) return EPLB_ERR_NULL;
  return launch_fold_loads(phys, phy2log, R, E, P, logical, status, stream);
}

eplb_status eplb_initial_map(int64_t R, int32_t E, int32_t P, int32_t *phy2log, int32_t *phyrank,
                             cudaStream_t stream) {
  if (R < 0 || E < 1 || P < E) return EPLB_ERR_SHAPE;
  if (R == 0) return EPLB_OK;
  if (!phy2log) return EPLB_ERR_NULL;
  return launch_initial_map(R, E, P, phy2log, phyrank, stream);
}

eplb_status eplb_plan_diff(const int32_t *old_phy2log, const int32_t *new_phy2log, int64_t R,
                           int32_t E, int32_t P, int32_t gpus, int32_t *src, int32_t *moves,
                           int32_t *status, cudaStream_t stream) {
  if (R < 0 || E < 1 || P < 1 || gpus < 1) return EPLB_ERR_SHAPE;
  if (P % gpus != 0) return EPLB_ERR_DIVISIBILITY;
  if (E > 8192 || R > 0x7fffffffLL) return EPLB_ERR_LIMIT;
  if (R == 0) return EPLB_OK;
  if (!old_phy2log || !new_phy2log || !src) return EPLB_ERR_NULL;
  return launch_plan_diff(old_phy2log, new_phy2log, R, E, P, gpus, src, moves, status, stream);
}

}  // extern "C"
