// serve.cu -- the serving step in one launch.
//
// Every CTA redirects one chunk of one layer with the plan in force and adds
// the chunk's counts to the current ring slot (S1 + S5, redirect_chunk).  The
// CTA that completes a layer -- the last of the layer's chunks to bump the
// layer's counter -- then computes that layer's next plan: the window sum
// over the ring (S2) and rebalance_experts (S3/S4, rebalance_row), into the
// buffers of the next plan.  Blocks run chunk-major, so the layers complete
// together in the last wave and their plans are built side by side in the
// tail (one row's rebalance after the last chunk) with no grid-wide wait or
// second launch in between; a layer-major order, which lets early layers
// plan while later ones stream, measured slower -- the planning CTAs hold
// SM slots the streaming chunks wait for.
//
// Ordering: the CTA's count atomics are ordered before its counter increment
// by a CTA barrier and a device-scope fence in the incrementing thread (the
// fence is cumulative over the writes the barrier ordered before it); the
// completing CTA fences again and reads the ring through L2 (ld.global.cg)
// only after it has seen the final count, so it sums the whole layer.  It
// resets the layer's counter for the next call.
#include <mutex>

#include "rebalance_row.cuh"
#include "redirect_chunk.cuh"

namespace eplb {
namespace {

struct ServeArgs {
  RedirectArgs r;  // counts = the current ring slot
  RbArgs b;        // the ring, the next plan
  uint32_t *layer_done;
};

template <bool kVecToken, bool kCap2>
__global__ void __launch_bounds__(kThreads) serve_kernel(ServeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int last;
  pdl_trigger();
  pdl_wait();
  // blocks run chunk-major (block b: layer b mod L, chunk b div L), so every
  // layer is completed in the last wave and the layers' plans are built
  // together in the tail instead of holding slots the streaming chunks need
  const int64_t L = gridDim.x / a.r.chunks;
  const int64_t layer = blockIdx.x % L;
  const int64_t cta = layer * a.r.chunks + blockIdx.x / L;
  redirect_chunk<kVecToken, true>(a.r, smem, cta);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(a.layer_done + layer, 1u) + 1u == static_cast<uint32_t>(a.r.chunks);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x == 0) a.layer_done[layer] = 0;
  rebalance_row<kCap2>(a.b, layer, smem);
}

}  // namespace

eplb_status launch_serve(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                         const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                         int32_t *out, unsigned long long *bad, int64_t *ring, int64_t W,
                         int64_t slot, int64_t zero_slot, int64_t *loads_out,
                         const RebalanceShape &sh, int32_t *next_phy2log, int32_t *next_phyrank,
                         int32_t *next_logcnt, int32_t *next_log2phy, double *gpu_load,
                         double *stats, uint32_t *layer_done, int32_t *status,
                         cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  RedirectSmem sp;
  eplb_status st = redirect_plan(E, true, di, &sp);
  if (st != EPLB_OK) return st;
  const Layout lay(sh);
  const size_t smem = std::max(sp.bytes, lay.total);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  ServeArgs a;
  const int64_t stride = L * E;
  redirect_fill(a.r, sp, idx, T, K, E, log2phy, X, logcnt, t0, out, ring + slot * stride, bad,
                status);
  a.b.ring = ring;
  a.b.ring_w = W;
  a.b.ring_stride = stride;
  a.b.zero_slot = zero_slot;
  a.b.loads_out = loads_out;
  a.b.phy2log = next_phy2log;
  a.b.phyrank = next_phyrank;
  a.b.logcnt = next_logcnt;
  a.b.log2phy = next_log2phy;
  a.b.status = status;
  a.b.gpu_load = gpu_load;
  a.b.stats = stats;
  a.b.s = sh;
  a.b.x_magic = 0xffffffffu / static_cast<uint32_t>(sh.X);
  set_row_magics(a.b);
  a.b.table_vec4 = ((static_cast<int64_t>(sh.E) * sh.X) % 4 == 0) &&
                   (reinterpret_cast<uintptr_t>(next_log2phy) % 16 == 0);
  a.layer_done = layer_done;
  const bool vec = (K % 4) == 0, cap2 = cap2_shape(sh);
  const void *fn =
      vec ? (cap2 ? reinterpret_cast<const void *>(serve_kernel<true, true>)
                  : reinterpret_cast<const void *>(serve_kernel<true, false>))
          : (cap2 ? reinterpret_cast<const void *>(serve_kernel<false, true>)
                  : reinterpret_cast<const void *>(serve_kernel<false, false>));
  int per_sm = 0;
  st = prepare_kernel(fn, kThreads, smem, &per_sm);
  if (st != EPLB_OK) return st;
  per_sm = std::max(1, std::min(per_sm, 4));
  a.r.chunks = redirect_chunks(L, a.r.per_layer, static_cast<int64_t>(di.sms) * per_sm);
  const int64_t grid = L * a.r.chunks;
  if (grid > 0x7fffffffLL) return EPLB_ERR_LIMIT;  // one block per layer chunk
  void *args[] = {&a};
  const cudaError_t err =
      launch_pdl(fn, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, stream, args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

// Per-layer counters of eplb_serve_step_noalloc: one library-owned array per
// device, zero when the module loads and left zero by every call.  Calls of
// that entry point share it, so two of them must not be in flight at once on
// one device.
static __device__ __align__(256) uint32_t g_layer_done[kStaticLayers];

eplb_status static_layer_done(uint32_t **out) {
  static std::once_flag once[kMaxDevices];
  static void *addr[kMaxDevices];
  static cudaError_t err[kMaxDevices];
  int dev = 0;
  const cudaError_t gerr = cudaGetDevice(&dev);
  if (gerr != cudaSuccess) return cuda_fail(gerr);
  if (dev < 0 || dev >= kMaxDevices) return EPLB_ERR_LIMIT;
  std::call_once(once[dev], [dev] { err[dev] = cudaGetSymbolAddress(&addr[dev], g_layer_done); });
  // the look-up's own error, kept for every later call on this device
  if (err[dev] != cudaSuccess) return cuda_fail(err[dev]);
  *out = static_cast<uint32_t *>(addr[dev]);
  return EPLB_OK;
}

}  // namespace eplb
