// rebalance.cu -- S3/S4 (and, in ring mode, S2): rebalance_experts over R
// rows, one CTA per row.  The row's work is rebalance_row (rebalance_row.cuh),
// shared with the serving-step kernel.
#define EPLB_RB_COLD __noinline__    // cold paths out of line (rebalance_row.cuh)
#define EPLB_RB_SHARED __noinline__  // one copy of the shared building blocks
#include "rebalance_row.cuh"

namespace eplb {
namespace {

// Instruction warm-up before the wait on the previous kernel.  The row's
// first calls of the out-of-line rank sort and packing greedy are chains on
// one warp; when another kernel with a large code body ran on the SM just
// before (the count+redirect pass, or a kernel of 360 KB of straight-line
// code), their code is no longer in the SM's instruction cache and each
// first call took 1.0-1.5 us longer while it was fetched (clock64 probes on
// the DeepSeek-V3 row; the row's inline code showed no such cost, nor did an
// empty kernel with 200 KB of shared memory).  Every warp runs one of the two
// once on scratch keys in shared memory -- even warps the sort (8 keys per
// warp), odd warps the greedy (4 items onto 4 packs per 4-lane slot) -- so
// their code is fetched side by side while the ring's prefetches are in
// flight, and under a programmatic launch behind the previous kernel's tail.
// The serving step's calls take it (a rotating ring, zero_slot >= 0: the
// count+redirect pass runs just before on the stream): its 58-layer
// DeepSeek-V3 step went from 67.6 to 64.6 us (measured).  Timed alone right
// after count+redirect the kernel is unchanged (the fetch moves from the
// row's first calls into the warm-up); a plain call, whose code is often
// still cached, would pay the warm-up's 1-2 us for nothing.
constexpr size_t kWarmScratch = 10240;

template <bool kCap2>
__device__ __forceinline__ void warm_row_code(unsigned char *smem) {
  const int wid = static_cast<int>(threadIdx.x) >> 5, lane = static_cast<int>(threadIdx.x) & 31;
  uint64_t *skeys = reinterpret_cast<uint64_t *>(smem);  // 8 keys per warp, 16 warps
  uint64_t *sout = skeys + 128;
  uint64_t *pkeys = sout + 128;  // 4 items per slot, 128 slots
  int32_t *ipack = reinterpret_cast<int32_t *>(pkeys + 512);
  int32_t *irank = ipack + 512;
  if (wid & 1) {
    const int j = lane & 3;  // item j of slot 8 * wid + lane / 4
    pkeys[wid * 32 + lane] = (uint64_t(4 - j) << kIdxBits) | (kIdxMask - j);
    __syncwarp();
    pack_segments<uint64_t, kCap2>(pkeys, 4, nthr() >> 2, 4, 4, 1, nullptr, nullptr, ipack, irank, 4);
  } else {
    if (lane < 8) skeys[wid * 8 + lane] = (uint64_t(8 - lane) << kIdxBits) | (kIdxMask - lane);
    __syncwarp();
    rank_sort<uint64_t>(skeys, 8, nwarps(), 8, sout);
  }
  __syncthreads();  // the row reuses the scratch
}

template <bool kCap2>
__global__ void __launch_bounds__(kMaxThreads) rebalance_kernel(RbArgs a, int warm) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_trigger();
  // warm L2 with this row's ring rows while the previous kernel finishes:
  // the row's first phase sums them (one 128-byte line per thread)
  {
    const int E = a.s.E;
    const int lines = (E + 15) >> 4;  // 16 int64 per line
    const int64_t *row = a.ring + static_cast<int64_t>(blockIdx.x) * E;
    for (int64_t w = 0; w < a.ring_w; ++w, row += a.ring_stride)
      for (int j = threadIdx.x; j < lines; j += blockDim.x) prefetch_l2(row + min(j << 4, E - 1));
  }
  if (warm) warm_row_code<kCap2>(smem);
  pdl_wait();
  rebalance_row<kCap2>(a, blockIdx.x, smem);
}

// The same row for launches with many rows per SM: 128 threads and at most
// 64 registers (36 bytes spilled), so that shared memory, not registers,
// bounds the CTAs an SM holds (5 instead of 4 on the DeepSeek-V3 shape; the
// 58,000-row window sweep 3.6% faster, measured).
template <bool kCap2>
__global__ void __launch_bounds__(kManyRowThreads, 8) rebalance_many_kernel(RbArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_trigger();
  pdl_wait();
  rebalance_row<kCap2>(a, blockIdx.x, smem);
}

}  // namespace

eplb_status launch_rebalance(int64_t *ring, int64_t ring_w, int64_t zero_slot, int64_t *loads_out,
                             int64_t R, const RebalanceShape &sh, int32_t *phy2log,
                             int32_t *phyrank, int32_t *logcnt, int32_t *log2phy, double *gpu_load,
                             double *stats, int32_t *status, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  const Layout lay(sh);
  if (lay.total > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  // few rows: one 512-thread CTA per row on its own SM; many rows: 128-thread
  // CTAs several to an SM
  const bool many = R > 2 * static_cast<int64_t>(di.sms);
  const bool c2 = cap2_shape(sh);
  const void *fn = many ? (c2 ? reinterpret_cast<const void *>(rebalance_many_kernel<true>)
                              : reinterpret_cast<const void *>(rebalance_many_kernel<false>))
                        : (c2 ? reinterpret_cast<const void *>(rebalance_kernel<true>)
                              : reinterpret_cast<const void *>(rebalance_kernel<false>));
  const eplb_status pst = prepare_kernel(fn, many ? kManyRowThreads : kMaxThreads, lay.total,
                                         nullptr);
  if (pst != EPLB_OK) return pst;
  RbArgs a;
  a.ring = ring;
  a.ring_w = ring_w;
  a.ring_stride = R * sh.E;
  a.zero_slot = zero_slot;
  a.loads_out = loads_out;
  a.phy2log = phy2log;
  a.phyrank = phyrank;
  a.logcnt = logcnt;
  a.log2phy = log2phy;
  a.status = status;
  a.gpu_load = gpu_load;
  a.stats = stats;
  a.s = sh;
  a.x_magic = 0xffffffffu / static_cast<uint32_t>(sh.X);
  set_row_magics(a);
  a.table_vec4 = ((static_cast<int64_t>(sh.E) * sh.X) % 4 == 0) &&
                 (reinterpret_cast<uintptr_t>(log2phy) % 16 == 0);
  const int threads = many ? kManyRowThreads : kFewRowThreads;
  int warm = zero_slot >= 0 && lay.total >= kWarmScratch ? 1 : 0;  // the few-row kernel only
  void *args_many[] = {&a};
  void *args_few[] = {&a, &warm};
  void **args = many ? args_many : args_few;
  const cudaError_t err =
      launch_pdl(fn, dim3(static_cast<unsigned>(R)), dim3(threads), lay.total, stream, args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
