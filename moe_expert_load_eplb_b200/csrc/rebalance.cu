// rebalance.cu -- S3/S4: rebalance_experts over R rows, one CTA per row.
//
// Follows page "DualPipe и EPLB", Part 2: section "Алгоритм" (hierarchical
// policy when num_groups % num_nodes == 0, else global = one group on one
// node) and the appendix functions balanced_packing, replicate_experts and
// rebalance_experts_hierarchical, with exact arithmetic:
//   step 1  group loads -> balanced_packing over nodes (G/N groups each);
//   step 2  replicate_experts per node: every extra replica goes to the
//           largest load per replica w/c (cross-multiplied, lowest index on
//           ties);
//   step 3  replica loads w/c -> balanced_packing over the node's GPUs
//           (P/gpus each); sums of w/c are held as integers w * (Lambda/c),
//           Lambda = lcm of the node's replica counts;
//   then the index bookkeeping and log2phy.
// balanced_packing visits items heaviest first with ties by ascending index
// and puts each into the lightest non-full pack (lowest pack index on ties).
//
// Latency-bound design: the row lives in shared memory; sorts are CTA-wide
// bitonic networks on composite keys (load << b | (mask - index)), which
// turns the stable (load desc, index asc) order into a plain descending sort
// of distinct integers; each node's serial greedy chains run in one warp
// (node n on warp n mod 4) as xor-butterfly argmax / argmin reductions with
// no block-wide barrier per step.  Keys are 64-bit when the row's magnitudes
// allow and 128-bit otherwise; both are exact, so the choice never changes
// the result.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int64_t kLoadLimit = int64_t(1) << 40;
constexpr uint32_t kNone = 0xffffffffu;

typedef unsigned __int128 u128;

struct RbArgs {
  const int64_t *loads;
  int32_t *phy2log, *phyrank, *logcnt, *log2phy, *status;
  RebalanceShape s;
  uint32_t x_magic;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Shared-memory carve-up of one row (byte offsets), identical on host and device.
struct Layout {
  size_t keys, pw, w, wm, gkey, npw, lam, mlog2log, cnt, lc, p2m, rrank, ipack, irank, outp, outr,
      gpack, grank, npc, pc, total;
  __host__ __device__ explicit Layout(const RebalanceShape &s) {
    size_t o = 0;
    keys = o; o += size_t(s.N) * s.npad * 16;  // u128 or u64 sort keys
    pw = o; o += size_t(s.gpus) * 16;          // pack weights of step 3 (N * mpn)
    o = align16(o);
    w = o; o += size_t(s.E) * 8;
    wm = o; o += size_t(s.E) * 8;
    gkey = o; o += size_t(s.gpad) * 8;
    npw = o; o += size_t(s.N) * 8;
    lam = o; o += size_t(s.N) * 8;
    mlog2log = o; o += size_t(s.E) * 4;
    cnt = o; o += size_t(s.E) * 4;
    lc = o; o += size_t(s.E) * 4;
    p2m = o; o += size_t(s.P) * 4;
    rrank = o; o += size_t(s.P) * 4;
    ipack = o; o += size_t(s.P) * 4;
    irank = o; o += size_t(s.P) * 4;
    outp = o; o += size_t(s.P) * 4;
    outr = o; o += size_t(s.P) * 4;
    gpack = o; o += size_t(s.G) * 4;
    grank = o; o += size_t(s.G) * 4;
    npc = o; o += size_t(s.N) * 4;
    pc = o; o += size_t(s.gpus) * 4;
    total = align16(o);
  }
};

__device__ __forceinline__ uint64_t shfl_xor(uint64_t v, int off) {
  return __shfl_xor_sync(0xffffffffu, static_cast<unsigned long long>(v), off);
}
__device__ __forceinline__ u128 shfl_xor(u128 v, int off) {
  const uint64_t lo = shfl_xor(static_cast<uint64_t>(v), off);
  const uint64_t hi = shfl_xor(static_cast<uint64_t>(v >> 64), off);
  return (static_cast<u128>(hi) << 64) | lo;
}

__device__ __forceinline__ uint64_t gcd_u64(uint64_t a, uint64_t b) {  // binary gcd
  if (a == 0) return b;
  if (b == 0) return a;
  const int shift = __ffsll(static_cast<long long>(a | b)) - 1;
  a >>= __ffsll(static_cast<long long>(a)) - 1;
  do {
    b >>= __ffsll(static_cast<long long>(b)) - 1;
    if (a > b) {
      const uint64_t t = a;
      a = b;
      b = t;
    }
    b -= a;
  } while (b != 0);
  return a << shift;
}

// lcm with overflow detection (results above 2^62 flag `ovf`).
__device__ __forceinline__ uint64_t lcm_u64(uint64_t a, uint64_t b, bool &ovf) {
  if (a == b || b <= 1) return a;
  if (a <= 1) return b;
  const uint64_t q = a / gcd_u64(a, b);
  const u128 r = static_cast<u128>(q) * b;
  if (r > (static_cast<u128>(1) << 62)) {
    ovf = true;
    return 1;
  }
  return static_cast<uint64_t>(r);
}

// CTA-wide bitonic sort, descending, of nseg independent segments of npad
// (power of two) keys each.  Ends with a barrier.
template <typename K>
__device__ void bitonic_desc(K *key, int npad, int nseg) {
  const int half = (npad * nseg) >> 1;
  for (int k = 2; k <= npad; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < half; t += kThreads) {
        const int i = ((t & ~(j - 1)) << 1) | (t & (j - 1));
        const int p = i | j;
        const bool desc = ((i & (npad - 1)) & k) == 0;
        const K x = key[i], y = key[p];
        if ((x < y) == desc) {
          key[i] = y;
          key[p] = x;
        }
      }
      __syncthreads();
    }
  }
}

// balanced_packing's greedy, run by one warp over items already sorted as
// composite keys (load << ibits | (imask - item)), descending.  Pack q is
// owned by lane q % 32; each lane caches the composite key
// (weight << qbits | q) of its lightest non-full pack and the warp takes
// the minimum with an xor butterfly, so ties go to the lowest pack index.
template <typename K>
__device__ void warp_pack(const K *skey, int n, int m, int cap, int ibits, int qbits, K *pw,
                          int32_t *pc, int32_t *ipack, int32_t *irank) {
  const int lane = threadIdx.x & 31;
  const K imask = (K(1) << ibits) - 1;
  const K qmask = (K(1) << qbits) - 1;
  const K kmax = ~K(0);
  for (int q = lane; q < m; q += 32) {
    pw[q] = 0;
    pc[q] = 0;
  }
  __syncwarp();
  K best = lane < m ? K(lane) : kmax;  // every pack empty: lowest owned index
  int rounds = 0;
  while ((1 << rounds) < min(m, 32)) ++rounds;
  for (int j = 0; j < n; ++j) {
    const K ck = skey[j];
    const K v = ck >> ibits;
    const int item = static_cast<int>(imask - (ck & imask));
    K b = best;
    for (int r = rounds - 1; r >= 0; --r) {
      const K o = shfl_xor(b, 1 << r);
      b = o < b ? o : b;
    }
    const int q = static_cast<int>(b & qmask);
    if (b != kmax && lane == (q & 31)) {
      const int rk = pc[q];
      pc[q] = rk + 1;
      pw[q] += v;
      ipack[item] = q;
      irank[item] = rk;
      K nb = kmax;
      for (int qq = lane; qq < m; qq += 32)
        if (pc[qq] < cap) {
          const K kk = (pw[qq] << qbits) | K(qq);
          nb = kk < nb ? kk : nb;
        }
      best = nb;
    }
    __syncwarp();
  }
}

// a beats b in replicate_experts' argmax: larger w/c, then lower index.
// ci packs (count << 16 | index); kNone marks "no candidate".
__device__ __forceinline__ bool rep_better(int64_t aw, uint32_t aci, int64_t bw, uint32_t bci) {
  if (aci == kNone) return false;
  if (bci == kNone) return true;
  const int64_t lhs = aw * static_cast<int64_t>(bci >> 16);
  const int64_t rhs = bw * static_cast<int64_t>(aci >> 16);
  return lhs > rhs || (lhs == rhs && (aci & 0xffffu) < (bci & 0xffffu));
}

__device__ void write_error_row(const RbArgs &a, int64_t row) {
  const RebalanceShape &s = a.s;
  for (int t = threadIdx.x; t < s.P; t += kThreads) {
    a.phy2log[row * s.P + t] = -1;
    a.phyrank[row * s.P + t] = -1;
  }
  for (int e = threadIdx.x; e < s.E; e += kThreads) a.logcnt[row * s.E + e] = 0;
  int32_t *gl = a.log2phy + row * static_cast<int64_t>(s.E) * s.X;
  for (int i = threadIdx.x; i < s.E * s.X; i += kThreads) gl[i] = -1;
}

template <typename K>
__device__ void step3_pack(const RbArgs &a, unsigned char *smem, const Layout &lay) {
  const RebalanceShape &s = a.s;
  K *keys = reinterpret_cast<K *>(smem + lay.keys);
  K *pw = reinterpret_cast<K *>(smem + lay.pw);
  const int64_t *wm = reinterpret_cast<const int64_t *>(smem + lay.wm);
  const uint64_t *lam = reinterpret_cast<const uint64_t *>(smem + lay.lam);
  const int32_t *cnt = reinterpret_cast<const int32_t *>(smem + lay.cnt);
  const int32_t *p2m = reinterpret_cast<const int32_t *>(smem + lay.p2m);
  int32_t *pc = reinterpret_cast<int32_t *>(smem + lay.pc);
  int32_t *ipack = reinterpret_cast<int32_t *>(smem + lay.ipack);
  int32_t *irank = reinterpret_cast<int32_t *>(smem + lay.irank);
  const K imask = (K(1) << s.ibits) - 1;
  for (int t = threadIdx.x; t < s.N * s.npad; t += kThreads) {
    const int n = t / s.npad;
    const int j = t - n * s.npad;
    K key = 0;
    if (j < s.ppn) {
      const int m = n * s.lpn + p2m[n * s.ppn + j];
      const K load = K(static_cast<uint64_t>(wm[m])) * K(lam[n] / static_cast<uint64_t>(cnt[m]));
      key = (load << s.ibits) | (imask - K(j));
    }
    keys[t] = key;
  }
  __syncthreads();
  bitonic_desc<K>(keys, s.npad, s.N);
  const int warp = threadIdx.x >> 5;
  for (int n = warp; n < s.N; n += kWarps)
    warp_pack<K>(keys + n * s.npad, s.ppn, s.mpn, s.ppg, s.ibits, s.qbits, pw + n * s.mpn,
                 pc + n * s.mpn, ipack + n * s.ppn, irank + n * s.ppn);
}

__global__ void __launch_bounds__(kThreads) rebalance_kernel(RbArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int flags[2];  // [0] 128-bit keys needed, [1] exact ratio too wide
  const RebalanceShape &s = a.s;
  const Layout lay(s);
  int64_t *w = reinterpret_cast<int64_t *>(smem + lay.w);
  int64_t *wm = reinterpret_cast<int64_t *>(smem + lay.wm);
  uint64_t *gkey = reinterpret_cast<uint64_t *>(smem + lay.gkey);
  uint64_t *npw = reinterpret_cast<uint64_t *>(smem + lay.npw);
  uint64_t *lam = reinterpret_cast<uint64_t *>(smem + lay.lam);
  int32_t *mlog2log = reinterpret_cast<int32_t *>(smem + lay.mlog2log);
  int32_t *cnt = reinterpret_cast<int32_t *>(smem + lay.cnt);
  int32_t *lc = reinterpret_cast<int32_t *>(smem + lay.lc);
  int32_t *p2m = reinterpret_cast<int32_t *>(smem + lay.p2m);
  int32_t *rrank = reinterpret_cast<int32_t *>(smem + lay.rrank);
  int32_t *ipack = reinterpret_cast<int32_t *>(smem + lay.ipack);
  int32_t *irank = reinterpret_cast<int32_t *>(smem + lay.irank);
  int32_t *outp = reinterpret_cast<int32_t *>(smem + lay.outp);
  int32_t *outr = reinterpret_cast<int32_t *>(smem + lay.outr);
  int32_t *gpack = reinterpret_cast<int32_t *>(smem + lay.gpack);
  int32_t *grank = reinterpret_cast<int32_t *>(smem + lay.grank);
  int32_t *npc = reinterpret_cast<int32_t *>(smem + lay.npc);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t row = blockIdx.x;
  if (tid == 0) {
    flags[0] = 0;
    flags[1] = 0;
  }

  // ---- load the row; loads must lie in [0, 2^40) -------------------------
  bool bad = false;
  for (int e = tid; e < s.E; e += kThreads) {
    const int64_t x = __ldg(a.loads + row * s.E + e);
    w[e] = x;
    bad |= (x < 0) | (x >= kLoadLimit);
  }
  if (__syncthreads_or(bad)) {
    write_error_row(a, row);
    if (tid == 0) report(a.status, EPLB_ERR_RANGE);
    return;
  }

  // ---- step 1: groups -> nodes ---------------------------------------------
  if (s.gpn == 1) {  // one group per node: the pages' identity short-cut
    for (int g = tid; g < s.G; g += kThreads) {
      gpack[g] = g;
      grank[g] = 0;
    }
  } else {
    const uint64_t gmask = (uint64_t(1) << s.gibits) - 1;
    for (int g = tid; g < s.gpad; g += kThreads) {
      uint64_t key = 0;
      if (g < s.G) {
        uint64_t sum = 0;
        for (int i = 0; i < s.gs; ++i) sum += static_cast<uint64_t>(w[g * s.gs + i]);
        key = (sum << s.gibits) | (gmask - g);
      }
      gkey[g] = key;
    }
    __syncthreads();
    bitonic_desc<uint64_t>(gkey, s.gpad, 1);
    if (warp == 0)
      warp_pack<uint64_t>(gkey, s.G, s.N, s.gpn, s.gibits, s.nqbits, npw, npc, gpack, grank);
  }
  __syncthreads();
  // mlog = logical order after the node permutation
  for (int e = tid; e < s.E; e += kThreads) {
    const int g = e / s.gs;
    const int m = (gpack[g] * s.gpn + grank[g]) * s.gs + (e - g * s.gs);
    mlog2log[m] = e;
    wm[m] = w[e];
  }
  __syncthreads();

  // ---- step 2: replicate_experts inside every node (warp n % 4) ----------
  const int kb = max(s.ibits, s.qbits);
  for (int n = warp; n < s.N; n += kWarps) {
    const int bm = n * s.lpn, bp = n * s.ppn;
    int64_t bw = 0;
    uint32_t bci = kNone;
    for (int i = lane; i < s.lpn; i += 32) {
      cnt[bm + i] = 1;
      p2m[bp + i] = i;
      rrank[bp + i] = 0;
      const uint32_t ci = (1u << 16) | static_cast<uint32_t>(i);
      if (rep_better(wm[bm + i], ci, bw, bci)) {
        bw = wm[bm + i];
        bci = ci;
      }
    }
    __syncwarp();
    int rounds = 0;
    while ((1 << rounds) < min(s.lpn, 32)) ++rounds;
    const int extra = s.ppn - s.lpn;
    for (int r = 0; r < extra; ++r) {
      int64_t mw = bw;
      uint32_t mci = bci;
      for (int k = rounds - 1; k >= 0; --k) {
        const int64_t ow = static_cast<int64_t>(shfl_xor(static_cast<uint64_t>(mw), 1 << k));
        const uint32_t oci = __shfl_xor_sync(0xffffffffu, mci, 1 << k);
        if (rep_better(ow, oci, mw, mci)) {
          mw = ow;
          mci = oci;
        }
      }
      const int b = static_cast<int>(mci & 0xffffu);
      if (mci != kNone && lane == (b & 31)) {
        const int old = cnt[bm + b];
        cnt[bm + b] = old + 1;
        p2m[bp + s.lpn + r] = b;
        rrank[bp + s.lpn + r] = old;
        bw = 0;
        bci = kNone;
        for (int i = lane; i < s.lpn; i += 32) {
          const uint32_t ci = (static_cast<uint32_t>(cnt[bm + i]) << 16) | static_cast<uint32_t>(i);
          if (rep_better(wm[bm + i], ci, bw, bci)) {
            bw = wm[bm + i];
            bci = ci;
          }
        }
      }
      __syncwarp();
    }
    // Lambda = lcm of this node's replica counts; choose the key width
    if (s.ppg > 1) {
      bool ovf = false;
      uint64_t lm = 1;
      int64_t wmax = 0;
      for (int i = lane; i < s.lpn; i += 32) {
        lm = lcm_u64(lm, static_cast<uint64_t>(cnt[bm + i]), ovf);
        wmax = max(wmax, wm[bm + i]);
      }
      for (int k = 16; k > 0; k >>= 1) {
        lm = lcm_u64(lm, shfl_xor(lm, k), ovf);
        wmax = max(wmax, static_cast<int64_t>(shfl_xor(static_cast<uint64_t>(wmax), k)));
      }
      ovf = __any_sync(0xffffffffu, ovf);
      if (lane == 0) {
        lam[n] = lm;
        const u128 maxsum = static_cast<u128>(static_cast<uint64_t>(wmax)) * lm * s.ppg;
        if (ovf || (maxsum >> (128 - kb - 1)) != 0)
          atomicOr(&flags[1], 1);
        else if ((maxsum >> (64 - kb - 1)) != 0)
          atomicOr(&flags[0], 1);
      }
    }
  }
  __syncthreads();
  if (flags[1]) {
    write_error_row(a, row);
    if (tid == 0) report(a.status, EPLB_ERR_RANGE);
    return;
  }

  // ---- step 3: replicas -> GPUs of each node ------------------------------
  if (s.ppg == 1) {  // one replica per GPU: identity short-cut
    for (int t = tid; t < s.P; t += kThreads) {
      const int n = t / s.ppn;
      ipack[t] = t - n * s.ppn;
      irank[t] = 0;
    }
  } else if (flags[0] == 0) {
    step3_pack<uint64_t>(a, smem, lay);
  } else {
    step3_pack<u128>(a, smem, lay);
  }
  __syncthreads();

  // ---- assembly: pphy = node*ppn + gpu*ppg + rank -------------------------
  for (int t = tid; t < s.P; t += kThreads) {
    const int n = t / s.ppn;
    const int pphy = n * s.ppn + ipack[t] * s.ppg + irank[t];
    outp[pphy] = mlog2log[n * s.lpn + p2m[t]];
    outr[pphy] = rrank[t];
  }
  for (int m = tid; m < s.E; m += kThreads) lc[mlog2log[m]] = cnt[m];
  __syncthreads();
  for (int t = tid; t < s.P; t += kThreads) {
    a.phy2log[row * s.P + t] = outp[t];
    a.phyrank[row * s.P + t] = outr[t];
  }
  for (int e = tid; e < s.E; e += kThreads) a.logcnt[row * s.E + e] = lc[e];
  int32_t *gl = a.log2phy + row * static_cast<int64_t>(s.E) * s.X;
  bool slots = false;
  for (int t = tid; t < s.P; t += kThreads) {
    const int k = outr[t];
    if (k < s.X)
      gl[outp[t] * s.X + k] = t;
    else
      slots = true;
  }
  const uint32_t X = static_cast<uint32_t>(s.X);
  for (int i = tid; i < s.E * s.X; i += kThreads) {
    const uint32_t e = div_magic(static_cast<uint32_t>(i), X, a.x_magic);
    if (static_cast<int>(i - e * X) >= lc[e]) gl[i] = -1;
  }
  if (slots) report(a.status, EPLB_ERR_SLOTS);
}

}  // namespace

eplb_status launch_rebalance(const int64_t *loads, int64_t R, const RebalanceShape &sh,
                             int32_t *phy2log, int32_t *phyrank, int32_t *logcnt,
                             int32_t *log2phy, int32_t *status, cudaStream_t stream) {
  DeviceInfo di;
  if (!device_info(&di)) return cuda_fail(cudaGetLastError());
  const Layout lay(sh);
  if (lay.total > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  cudaError_t err = cudaFuncSetAttribute(rebalance_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(lay.total));
  if (err != cudaSuccess) return cuda_fail(err);
  RbArgs a;
  a.loads = loads;
  a.phy2log = phy2log;
  a.phyrank = phyrank;
  a.logcnt = logcnt;
  a.log2phy = log2phy;
  a.status = status;
  a.s = sh;
  a.x_magic = 0xffffffffu / static_cast<uint32_t>(sh.X);
  rebalance_kernel<<<static_cast<unsigned>(R), kThreads, lay.total, stream>>>(a);
  err = cudaGetLastError();
  return err == cudaSuccess ? EPLB_OK : cuda_fail(err);
}

}  // namespace eplb
