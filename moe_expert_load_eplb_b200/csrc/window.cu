// window.cu -- S2: sliding-window sums of per-step expert loads.
//
// Load is commonly predicted by a moving average over historical statistics
// (page "DualPipe и EPLB", Part 2, section "Алгоритм").  With the columns
// c = (l, e) of a [S, L*E] int64 array,
//   snaps[s - s_first, c] = sum_{u=max(0,s-W+1)}^{s} steps[u, c],  s >= s_first,
// i.e. a prefix scan along s of d[u] = steps[u] - steps[u-W].
//
// HBM-streaming design: a CTA owns a strip of kCols = 32 adjacent columns
// (one warp reads one 256-byte row segment: coalesced) and walks all S rows
// in blocks of rg * kU rows (kU = 8, or 4 when rows s - W are read too).  Warp g of the CTA holds rows g*kU .. g*kU+kU-1
// of the block for its 32 columns; it scans them in registers, the rg warp
// totals are combined through shared memory into the strip's running carry.
// The next block's kU loads per thread are issued before the current block
// is scanned (two blocks in registers), so a thread keeps kU independent
// 8-byte loads in flight while it waits on the barrier and writes; rows
// s - W are loaded only in blocks that reach them (none when W >= S).  With
// up to 16 warps per CTA and several CTAs per SM this keeps 64-128 KB of
// reads in flight per SM, which HBM3e needs for its bandwidth.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kCols = 32;    // columns per strip: one warp-wide row segment
constexpr int kMaxRg = 16;   // row groups (warps) per CTA

// kU rows per thread per block; kSub: some row s has s - W >= 0 (W < S), so
// blocks that reach row W also load rows s - W.  Without it a block is kU
// loads per thread; with it 2 kU, so it takes half the rows per block.
template <int kU, bool kSub>
struct WinBlock {
  int64_t add[kU];
  int64_t sub[kSub ? kU : 1];

  // Rows r0 .. r0+kU-1 of column c: one pointer stepped by C through a
  // whole group of rows, per-row checks only where the group is cut.
  __device__ __forceinline__ void load(const int64_t *__restrict__ steps, int64_t S, int64_t C,
                                       int64_t W, int64_t r0, int64_t c, bool col_ok) {
    if (col_ok && r0 + kU <= S) {
      const int64_t *p = steps + r0 * C + c;
#pragma unroll
      for (int u = 0; u < kU; ++u, p += C) add[u] = __ldcs(p);
    } else {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t r = r0 + u;
        add[u] = (col_ok && r < S) ? __ldcs(steps + r * C + c) : 0;
      }
    }
    if (kSub) {
      if (col_ok && r0 >= W && r0 + kU <= S) {
        const int64_t *p = steps + (r0 - W) * C + c;
#pragma unroll
        for (int u = 0; u < kU; ++u, p += C) sub[kSub ? u : 0] = __ldg(p);
      } else {
        const bool any_sub = r0 + kU - 1 >= W;  // warp-uniform: r0 is the warp's first row
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int64_t r = r0 + u;
          sub[kSub ? u : 0] = (any_sub && col_ok && r < S && r >= W) ? __ldg(steps + (r - W) * C + c) : 0;
        }
      }
    }
  }
  __device__ __forceinline__ int64_t d(int u) const { return kSub ? add[u] - sub[kSub ? u : 0] : add[u]; }
};

template <int kU, bool kSub>
__global__ void __launch_bounds__(kCols * kMaxRg) window_kernel(
    int64_t *__restrict__ steps, int64_t S, int64_t C, int64_t W, int64_t s_first,
    int64_t *__restrict__ snaps, int64_t zero_row) {
  __shared__ int64_t part[kMaxRg][kCols];
  pdl_trigger();
  pdl_wait();
  const int col = threadIdx.x;  // blockDim = (kCols, rg)
  const int g = threadIdx.y;
  const int rg = blockDim.y;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kCols + col;
  const bool col_ok = c < C;
  const int64_t rows_per_blk = static_cast<int64_t>(rg) * kU;

  WinBlock<kU, kSub> cur, nxt;
  cur.load(steps, S, C, W, static_cast<int64_t>(g) * kU, c, col_ok);
  int64_t carry = 0;
  for (int64_t blk = 0; blk < S; blk += rows_per_blk) {
    const int64_t r0 = blk + static_cast<int64_t>(g) * kU;
    // the next block's loads go out before this block is scanned
    if (blk + rows_per_blk < S) nxt.load(steps, S, C, W, r0 + rows_per_blk, c, col_ok);
    int64_t acc = 0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      acc += cur.d(u);
      cur.add[u] = acc;  // inclusive prefix within this thread's rows
    }
    part[g][col] = acc;
    __syncthreads();
    int64_t before = carry, tot = 0;
    for (int h = 0; h < rg; ++h) {
      const int64_t p = part[h][col];
      before += (h < g) ? p : 0;
      tot += p;
    }
    if (col_ok && r0 >= s_first && r0 + kU <= S) {
      int64_t *p = snaps + (r0 - s_first) * C + c;
#pragma unroll
      for (int u = 0; u < kU; ++u, p += C) __stcs(p, before + cur.add[u]);
    } else if (col_ok && r0 + kU > s_first) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t r = r0 + u;
        if (r < S && r >= s_first) __stcs(snaps + (r - s_first) * C + c, before + cur.add[u]);
      }
    }
    carry += tot;
    __syncthreads();
    cur = nxt;
  }
  // every row of this strip's columns has been read (the last block's loads
  // were consumed above): clear the requested row of them
  if (zero_row >= 0 && g == 0 && col_ok) steps[zero_row * C + c] = 0;
}

}  // namespace

eplb_status launch_window(int64_t *steps, int64_t S, int64_t C, int64_t W, int64_t s_first,
                          int64_t *snaps, int64_t zero_row, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  const bool sub = W < S;
  const int u = sub ? 4 : 8;
  const int64_t strips = (C + kCols - 1) / kCols;
  if (strips > 0x7fffffffLL) return EPLB_ERR_LIMIT;
  const void *fn = sub ? reinterpret_cast<const void *>(window_kernel<4, true>)
                       : reinterpret_cast<const void *>(window_kernel<8, false>);
  // row groups: no more warps than the rows fill (up to kMaxRg), and the
  // most that still let every strip's CTA be resident at once (one wave:
  // a second, partial wave would leave SMs idle while it runs)
  const int rg_rows = static_cast<int>(std::min<int64_t>(kMaxRg, std::max<int64_t>(1, (S + u - 1) / u)));
  int rg = rg_rows;
  for (int cand = rg_rows; cand >= 1; --cand) {
    int per_sm = 0;
    const eplb_status pst = prepare_kernel(fn, kCols * cand, 0, &per_sm);
    if (pst != EPLB_OK) return pst;
    if (static_cast<int64_t>(per_sm) * di.sms >= strips) {
      rg = cand;
      break;
    }
  }
  void *args[] = {&steps, &S, &C, &W, &s_first, &snaps, &zero_row};
  const cudaError_t err = launch_pdl(fn, dim3(static_cast<unsigned>(strips)), dim3(kCols, rg), 0,
                                     stream, args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
