// window.cu -- S2: sliding-window sums of per-step expert loads.
//
// Load is commonly predicted by a moving average over historical statistics
// (page "DualPipe и EPLB", Part 2, section "Алгоритм").  With the columns
// c = (l, e) of a [S, L*E] int64 array,
//   snaps[s - s_first, c] = sum_{u=max(0,s-W+1)}^{s} steps[u, c],  s >= s_first,
// i.e. a prefix scan along s of d[u] = steps[u] - steps[u-W].
//
// HBM-streaming design: a CTA owns a strip of `cw` adjacent columns and walks
// all S rows in blocks of rg*U rows.  Thread (g, col) loads U rows of its
// column (U independent 8-byte loads in flight per thread, coalesced across
// the strip), scans them in registers, and the rg row-group totals are
// combined through shared memory into the strip's running carry.  The strip
// width is chosen on the host so the strip count fills the SMs evenly.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kU = 8;  // rows per thread per block

__global__ void window_kernel(const int64_t *__restrict__ steps, int64_t S, int64_t C, int64_t W,
                              int64_t s_first, int64_t *__restrict__ snaps, int cw, int rg) {
  extern __shared__ int64_t part[];  // [rg][cw]
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x;
  const int col = tid % cw;
  const int g = tid / cw;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * cw + col;
  const bool active = (g < rg) && (c < C);
  const int64_t rows_per_blk = static_cast<int64_t>(rg) * kU;

  int64_t carry = 0;
  for (int64_t blk = 0; blk < S; blk += rows_per_blk) {
    const int64_t r0 = blk + static_cast<int64_t>(g) * kU;
    int64_t add[kU], sub[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t r = r0 + u;
      add[u] = (active && r < S) ? __ldcs(steps + r * C + c) : 0;
      sub[u] = (active && r < S && r >= W) ? __ldg(steps + (r - W) * C + c) : 0;
    }
    int64_t acc = 0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      acc += add[u] - sub[u];
      add[u] = acc;  // inclusive prefix within this thread's rows
    }
    if (g < rg) part[g * cw + col] = acc;
    __syncthreads();
    int64_t pre = carry, tot = 0;
    for (int h = 0; h < rg; ++h) {
      const int64_t p = part[h * cw + col];
      pre += (h < g) ? p : 0;
      tot += p;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t r = r0 + u;
      if (active && r < S && r >= s_first) __stcs(snaps + (r - s_first) * C + c, pre + add[u]);
    }
    carry += tot;
    __syncthreads();
  }
}

}  // namespace

eplb_status launch_window(const int64_t *steps, int64_t S, int64_t C, int64_t W, int64_t s_first,
                          int64_t *snaps, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  // Pick the strip width cw and row groups rg: rg never exceeds the row
  // blocks there are (short rings), the strip count fills the SMs evenly
  // (strips per SM rounded up cost the tail), and enough threads per SM keep
  // loads in flight.
  const int64_t max_rg = std::max<int64_t>(1, (S + kU - 1) / kU);
  int best_cw = 32;
  double best_score = -1.0;
  for (int cw = 8; cw <= 256; ++cw) {
    const int rg = static_cast<int>(std::min<int64_t>(std::max(1, 256 / cw), max_rg));
    if (cw * rg > 1024) continue;
    const int64_t strips = (C + cw - 1) / cw;
    const int64_t waves = (strips + di.sms - 1) / di.sms;
    const double balance = static_cast<double>(strips) / static_cast<double>(waves * di.sms);
    const double per_sm_threads = static_cast<double>(std::min<int64_t>(strips, waves * di.sms)) /
                                  di.sms * cw * rg;
    const double inflight = std::min(1.0, per_sm_threads / 1024.0);
    const double score = balance * inflight;
    if (score > best_score + 1e-9) {
      best_score = score;
      best_cw = cw;
    }
  }
  const int cw = static_cast<int>(std::min<int64_t>(best_cw, C));
  const int rg = static_cast<int>(std::min<int64_t>(std::max(1, 256 / cw), max_rg));
  const int64_t strips = (C + cw - 1) / cw;
  const size_t smem = static_cast<size_t>(rg) * cw * sizeof(int64_t);
  void *args[] = {&steps, &S, &C, &W, &s_first, &snaps, const_cast<int *>(&cw), const_cast<int *>(&rg)};
  const cudaError_t err = launch_pdl(reinterpret_cast<const void *>(window_kernel),
                                     dim3(static_cast<unsigned>(strips)), dim3(cw * rg), smem, stream,
                                     args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
