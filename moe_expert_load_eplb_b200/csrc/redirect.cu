// redirect.cu -- S5 (and S1 + S5 fused): the redirect kernel, one CTA per
// layer chunk; the CTA's work is redirect_chunk (redirect_chunk.cuh), shared
// with the serving-step kernel.
#include "redirect_chunk.cuh"

namespace eplb {
namespace {

template <bool kVecToken, bool kCount>
__global__ void __launch_bounds__(kThreads) redirect_kernel(RedirectArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_trigger();
  pdl_wait();
  redirect_chunk<kVecToken, kCount>(a, smem, blockIdx.x);
}

}  // namespace

eplb_status launch_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, int64_t *counts, unsigned long long *bad,
                            int32_t *status, cudaStream_t stream) {
  DeviceInfo di;
  const eplb_status dst = device_info(&di);
  if (dst != EPLB_OK) return dst;
  const bool count = counts != nullptr;
  RedirectSmem sp;
  const eplb_status st = redirect_plan(E, count, di, &sp);
  if (st != EPLB_OK) return st;
  RedirectArgs a;
  redirect_fill(a, sp, idx, T, K, E, log2phy, X, logcnt, t0, out, counts, bad, status);
  const bool vec_token = (K % 4) == 0;
  const void *fn;
  if (count)
    fn = vec_token ? reinterpret_cast<const void *>(redirect_kernel<true, true>)
                   : reinterpret_cast<const void *>(redirect_kernel<false, true>);
  else
    fn = vec_token ? reinterpret_cast<const void *>(redirect_kernel<true, false>)
                   : reinterpret_cast<const void *>(redirect_kernel<false, false>);
  int per_sm = 0;
  const eplb_status pst = prepare_kernel(fn, kThreads, sp.bytes, &per_sm);
  if (pst != EPLB_OK) return pst;
  per_sm = std::max(1, std::min(per_sm, 4));
  a.chunks = redirect_chunks(L, a.per_layer, static_cast<int64_t>(di.sms) * per_sm);
  const int64_t grid = L * a.chunks;
  if (grid > 0x7fffffffLL) return EPLB_ERR_LIMIT;  // one block per layer chunk
  void *args[] = {&a};
  const cudaError_t err =
      launch_pdl(fn, dim3(static_cast<unsigned>(grid)), dim3(kThreads), sp.bytes, stream, args);
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
