// rebalance_row.cuh -- one row of S3/S4 (and the S2 ring sum) by one CTA:
// the device code behind rebalance.cu's kernel and the serving-step kernel.
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
//           Lambda a common multiple of the node's replica counts;
//   then the index bookkeeping and log2phy.
// balanced_packing visits items heaviest first with ties by ascending index
// and puts each into the lightest non-full pack (lowest pack index on ties).
//
// Latency-bound design, measured phase by phase with clock64 probes:
//   * the row lives in shared memory; every sort key is a composite integer
//     (load << b | (mask - index)), so the stable (load desc, index asc)
//     order is a plain descending order of distinct integers;
//   * sorts count ranks CTA-wide (a key's rank is the number of larger keys
//     in its segment); threads are grouped by segment and rank several keys
//     against each loaded key; segments longer than 512 use a bitonic network;
//   * replicate_experts: an expert outside the top R = P/N - E/N experts of
//     its node (by load, ties by index) has at least R quotients ahead of it,
//     so it never gets an extra replica; the R candidates are selected by
//     rank and the greedy runs on them alone -- as a ranking of (candidate,
//     divisor) pairs when there are few, else one candidate per lane with an
//     xor-butterfly argmax;
//   * balanced_packing keeps a node's packs sorted by composite key
//     (weight << 12 | pack) across the lanes of a segment (one position per
//     lane up to 32 packs, several per lane up to 256): each item takes the
//     first (lightest, lowest index) pack, and every position compares its
//     key and its right neighbour's with the updated pack's new key to shift
//     or take it; wider nodes use one warp per node and a butterfly argmin;
//   * Lambda is lcm(1..cmax) from the host when 64-bit keys can hold it, else
//     the lcm of the counts present in the node; keys are 64-bit when the
//     row's magnitudes allow and 128-bit otherwise.  All paths are exact, so
//     none changes the result.
#pragma once

#include <algorithm>

#include "common.cuh"
#include "internal.h"

// Paths the common shapes never take (128-entry packs, bitonic sorts, wide
// replication, the two-items-per-pack closed form) carry EPLB_RB_COLD.  The
// rebalance kernel defines it as __noinline__ before including this header:
// the row's code is then compact in the instruction cache, which made the
// 58-row DeepSeek-V3 rebalance about 2 us faster (measured).  The serving
// kernel keeps them inline: there the calls raised its register spills from
// 12 to 64 bytes a thread.
#ifndef EPLB_RB_COLD
#define EPLB_RB_COLD
#endif
// The building blocks several steps use (the rank sort, the packing greedy)
// carry EPLB_RB_SHARED: one out-of-line copy serves every call site in the
// rebalance kernel, so the instruction cache holds it after its first use
// (separate inlined copies are each fetched cold; sharing them made the
// 58-row DeepSeek-V3 rebalance 2 us faster, measured).
#ifndef EPLB_RB_SHARED
#define EPLB_RB_SHARED
#endif
// Loops strided by the CTA or a warp run once or twice per thread; they carry
// `#pragma unroll 1`, since the compiler's default unrolling only adds code
// that is fetched cold (the kernel 227 -> 171 KB of code; the 58-row
// DeepSeek-V3 rebalance with plan quality 28.8 -> 25.5 us and the 58,000-row
// sweep 4.6% faster, measured).

namespace eplb {
namespace {


// CTA size is chosen per launch: 512 threads when there are few rows (each
// row's parallel phases then spread over 4 warps per scheduler), 128 when
// many rows share every SM.
constexpr int kMaxThreads = 512;
constexpr int kFewRowThreads = 512;
constexpr int kManyRowThreads = 128;
__device__ __forceinline__ int nthr() { return static_cast<int>(blockDim.x); }
__device__ __forceinline__ int nwarps() { return static_cast<int>(blockDim.x) >> 5; }
constexpr int64_t kLoadLimit = int64_t(1) << 40;
constexpr int kTableMaxEntries = 16384;  // log2phy rows up to this size are built in smem
// Every composite key keeps an index (item, pack, group or expert, all < 4096)
// in its low kIdxBits bits, so keys are combined with constant shifts only.
constexpr int kIdxBits = 12;
constexpr uint64_t kIdxMask = (uint64_t(1) << kIdxBits) - 1;

typedef unsigned __int128 u128;

struct RbArgs {
  // A row's loads are the sum of W ring rows: loads[r, e] = sum_w ring[w, r, e]
  // (W = 1 for a plain load array).  zero_slot >= 0 clears that ring row's
  // part of each row after it was read; loads_out (nullable) gets the sums.
  int64_t *ring;
  int64_t ring_w, ring_stride, zero_slot;
  int64_t *loads_out;
  int32_t *phy2log, *phyrank, *logcnt, *log2phy, *status;
  // plan quality (nullable): per-GPU load [R, gpus] and {min, max, mean,
  // mean / max} [R, 4] of the plan just built, fp64
  double *gpu_load, *stats;
  RebalanceShape s;
  uint32_t x_magic;
  int table_vec4;  // log2phy rows may be written as 16-byte vectors
  // multiply-high divisors (floor((2^32 - 1) / d), 0 for d = 0) of the row's
  // index arithmetic: gs, lpn, ppn, the candidates nc, the extra replicas
  // R = ppn - lpn, nc * R, and step 3's keys per node; a 32-bit divide by a
  // run-time value is a long dependent sequence on the row's critical path
  uint32_t m_gs, m_lpn, m_ppn, m_nc, m_r, m_grid, m_per;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }
__host__ __device__ inline int bitmap_words(const RebalanceShape &s) { return (s.cmax + 32) / 32; }
__host__ __device__ inline bool table_in_smem(const RebalanceShape &s) {
  return static_cast<int64_t>(s.E) * s.X <= kTableMaxEntries;
}
// experts per node that can receive extra replicas
__host__ __device__ inline int num_cand(const RebalanceShape &s) {
  return min(s.ppn - s.lpn, s.lpn);
}

// x / d for 0 <= x < 2^31 by the magic m of d (common.cuh's div_magic)
__device__ __forceinline__ int qdivm(int x, int d, uint32_t m) {
  return static_cast<int>(div_magic(static_cast<uint32_t>(x), static_cast<uint32_t>(d), m));
}
inline uint32_t row_magic(int32_t d) { return d > 0 ? 0xffffffffu / static_cast<uint32_t>(d) : 0u; }
inline void set_row_magics(RbArgs &a) {
  const RebalanceShape &s = a.s;
  const int nc = num_cand(s), R = s.ppn - s.lpn;
  a.m_gs = row_magic(s.gs);
  a.m_lpn = row_magic(s.lpn);
  a.m_ppn = row_magic(s.ppn);
  a.m_nc = row_magic(nc);
  a.m_r = row_magic(R);
  a.m_grid = row_magic(nc * R);
  a.m_per = row_magic(s.npad <= kRankSortMax ? s.ppn : s.npad);  // step 3's keys per node
}

// Shared-memory carve-up of one row (byte offsets), identical on host and device.
struct Layout {
  size_t keys, sorted, pw, w, wm, gkey, gsorted, npw, lam, cand_w, table, mlog2log, cnt, lc, p2m,
      rrank, ipack, irank, outp, outr, gpack, grank, npc, pc, cand_i, cand_c, bitmap, total;
  __host__ __device__ explicit Layout(const RebalanceShape &s) {
    const int nc = num_cand(s);
    size_t o = 0;
    keys = o; o += size_t(s.N) * max(s.npad, s.lpn) * 16;  // u128/u64 keys, stride npad (or lpn)
    sorted = o; o += size_t(s.N) * s.npad * 16;
    pw = o; o += size_t(s.gpus) * 16;                       // pack weights of the warp fallback
    o = align16(o);
    w = o; o += size_t(s.E) * 8;
    wm = o; o += size_t(s.E) * 8;
    gkey = o; o += size_t(s.gpad) * 8;
    gsorted = o; o += size_t(s.gpad) * 8;
    npw = o; o += size_t(s.N) * 8;
    lam = o; o += size_t(s.N) * 8;
    cand_w = o; o += size_t(s.N) * nc * 8;
    o = align16(o);
    table = o; o += table_in_smem(s) ? size_t(s.E) * s.X * 4 : 0;
    o = align16(o);
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
    cand_i = o; o += size_t(s.N) * nc * 4;
    cand_c = o; o += size_t(s.N) * nc * 4;
    bitmap = o; o += size_t(s.N) * bitmap_words(s) * 4;
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
__device__ __forceinline__ uint64_t shfl_idx(uint64_t v, int src, int width) {
  return __shfl_sync(0xffffffffu, static_cast<unsigned long long>(v), src, width);
}
__device__ __forceinline__ u128 shfl_idx(u128 v, int src, int width) {
  const uint64_t lo = shfl_idx(static_cast<uint64_t>(v), src, width);
  const uint64_t hi = shfl_idx(static_cast<uint64_t>(v >> 64), src, width);
  return (static_cast<u128>(hi) << 64) | lo;
}
__device__ __forceinline__ uint64_t shfl_down_k(uint64_t v, int d, int width) {
  return __shfl_down_sync(0xffffffffu, static_cast<unsigned long long>(v), d, width);
}
__device__ __forceinline__ u128 shfl_down_k(u128 v, int d, int width) {
  const uint64_t lo = shfl_down_k(static_cast<uint64_t>(v), d, width);
  const uint64_t hi = shfl_down_k(static_cast<uint64_t>(v >> 64), d, width);
  return (static_cast<u128>(hi) << 64) | lo;
}
template <typename K>
__device__ __forceinline__ K kmin(K a, K b) {
  return b < a ? b : a;
}

__device__ __forceinline__ uint32_t gcd_u32(uint32_t a, uint32_t b) {  // binary gcd
  if (a == 0) return b;
  if (b == 0) return a;
  const int shift = __ffs(a | b) - 1;
  a >>= __ffs(a) - 1;
  do {
    b >>= __ffs(b) - 1;
    if (a > b) {
      const uint32_t t = a;
      a = b;
      b = t;
    }
    b -= a;
  } while (b != 0);
  return a << shift;
}

// lcm(lam, c) with lam <= 2^62; false when the result would exceed 2^62.
__device__ __forceinline__ bool lcm_into(uint64_t &lam, uint32_t c) {
  if (c < 2) return true;
  const uint32_t rem = lam >> 32 ? static_cast<uint32_t>(lam % c)
                                 : static_cast<uint32_t>(lam) % c;
  const uint32_t g = gcd_u32(rem, c);
  const u128 next = static_cast<u128>(lam) * (c / g);
  if (next > (static_cast<u128>(1) << 62)) return false;
  lam = static_cast<uint64_t>(next);
  return true;
}

// ---------------------------------------------------------------------------
// r[q] += the number of keys in [i0, i1) of a segment greater than me[q].
// 64-bit keys are read by 32-bit shared address, two per 16-byte load: the
// rank sort runs out of line, where the compiler cannot tell that the keys
// are in shared memory, and its generic single-key loads measured 1.6-2.3x
// slower on 8-288 keys.  128-bit keys (a rare path) keep the plain loop.
template <int Q, typename K>
__device__ __forceinline__ void count_greater(const K *seg, int i0, int i1, const K (&me)[Q],
                                              int (&r)[Q]) {
  if constexpr (sizeof(K) == 8) {
    const uint32_t base = smem_u32(seg);
    int i = i0;
    if (i < i1 && ((base + 8u * i) & 15u) != 0) {
      const uint64_t x = ld_shared_u64(base + 8u * i);
#pragma unroll
      for (int q = 0; q < Q; ++q) r[q] += x > me[q] ? 1 : 0;
      ++i;
    }
#pragma unroll 4
    for (; i + 1 < i1; i += 2) {
      uint64_t x, y;
      ld_shared_u64x2(base + 8u * i, x, y);
#pragma unroll
      for (int q = 0; q < Q; ++q) r[q] += (x > me[q] ? 1 : 0) + (y > me[q] ? 1 : 0);
    }
    if (i < i1) {
      const uint64_t x = ld_shared_u64(base + 8u * i);
#pragma unroll
      for (int q = 0; q < Q; ++q) r[q] += x > me[q] ? 1 : 0;
    }
  } else {
#pragma unroll 4
    for (int i = i0; i < i1; ++i) {
      const K kk = seg[i];
#pragma unroll
      for (int q = 0; q < Q; ++q) r[q] += kk > me[q] ? 1 : 0;
    }
  }
}

// Descending ranks of n distinct keys in each of nseg segments (segment g at
// key + g * stride).  Threads are grouped by segment (nthr() / nseg per
// segment); each ranks Q keys per pass (Q = 1, 2 or 4, the fewest that cover
// the segment) against every key it loads.  emit(g, j, rank, key) receives
// every key.
template <int Q, typename K, typename Emit>
__device__ void rank_pass(const K *key, int stride, int nseg, int n, int tps, Emit &emit) {
  const int segs_per_pass = nthr() / tps;
  const int sub = threadIdx.x % tps;
  for (int g0 = 0; g0 < nseg; g0 += segs_per_pass) {
    const int g = g0 + static_cast<int>(threadIdx.x) / tps;
    if (static_cast<int>(threadIdx.x) / tps >= segs_per_pass || g >= nseg) continue;
    const K *seg = key + g * stride;
    for (int j0 = sub; j0 < n; j0 += tps * Q) {
      K me[Q];
      int r[Q];
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const int j = j0 + q * tps;
        me[q] = j < n ? seg[j] : ~K(0);
        r[q] = 0;
      }
      count_greater<Q, K>(seg, 0, n, me, r);
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const int j = j0 + q * tps;
        if (j < n) emit(g, j, r[q], me[q]);
      }
    }
  }
}

// Same ranks with two threads per key when a segment has at least twice as
// many threads as keys: each compares the key with half the segment, and the
// pair adds its counts with one shuffle (the passes are warp-uniform).
template <typename K, typename Emit>
__device__ void rank_pass_split(const K *key, int stride, int nseg, int n, int tps, Emit &emit) {
  const int segs_per_pass = nthr() / tps;
  const int sub = threadIdx.x % tps;
  const int j = sub >> 1, half = sub & 1;
  const int h = (n + 1) >> 1;
  const int i0 = half * h, i1 = min(n, i0 + h);
  for (int g0 = 0; g0 < nseg; g0 += segs_per_pass) {
    const int gl = static_cast<int>(threadIdx.x) / tps;
    const int g = g0 + gl;
    const bool live = gl < segs_per_pass && g < nseg && j < n;
    const K *seg = key + (live ? g : 0) * stride;
    const K me[1] = {live ? seg[j] : K(0)};
    int r[1] = {0};
    if (live) count_greater<1, K>(seg, i0, i1, me, r);
    r[0] += __shfl_xor_sync(0xffffffffu, r[0], 1);
    if (live && half == 0) emit(g, j, r[0], me[0]);
  }
}

template <typename K, typename Emit>
__device__ void rank_segments(const K *key, int stride, int nseg, int n, Emit emit) {
  const int tps = nseg >= nthr() ? 1 : nthr() / nseg;
  if (2 * n <= tps && tps % 32 == 0)
    rank_pass_split<K>(key, stride, nseg, n, tps, emit);
  else if (n <= tps)
    rank_pass<1, K>(key, stride, nseg, n, tps, emit);
  else if (n <= 2 * tps)
    rank_pass<2, K>(key, stride, nseg, n, tps, emit);
  else
    rank_pass<4, K>(key, stride, nseg, n, tps, emit);
}

// The general passes, out of line: the common shapes below never fetch them.
template <typename K>
__device__ EPLB_RB_COLD void rank_sort_general(const K *key, int stride, int nseg, int n, K *out) {
  rank_segments<K>(key, stride, nseg, n, [&](int g, int, int r, K k) { out[g * stride + r] = k; });
}

// Descending ranks written out: out[g * stride + rank] = key (the stable
// (value desc, index asc) order of the composite keys).
template <typename K>
__device__ EPLB_RB_SHARED void rank_sort(const K *key, int stride, int nseg, int n, K *out) {
  if constexpr (sizeof(K) == 8) {
    // one key per thread: a warp per segment when it holds one (lanes are
    // keys, no index arithmetic), else nthr() / nseg threads per segment.
    // These two shapes cover the 8-, 64- and 72-key sorts of the DeepSeek-V3
    // row; the general passes cost 0.4-0.9 us more there in their index
    // arithmetic (measured).
    int g = -1, j = 0;
    if (n <= 32 && nseg <= nwarps()) {
      g = threadIdx.x >> 5;
      j = threadIdx.x & 31;
    } else if (nseg <= nthr() && n <= nthr() / nseg) {
      if ((nseg & (nseg - 1)) == 0) {  // nthr() is a power of two too: shifts
        const int ls = (__ffs(nthr()) - 1) - (__ffs(nseg) - 1);
        g = threadIdx.x >> ls;
        j = threadIdx.x - (g << ls);
      } else {
        const int tps = nthr() / nseg;
        g = threadIdx.x / tps;
        j = threadIdx.x - g * tps;
      }
    }
    if (g >= 0) {
      if (g < nseg && j < n) {
        const K *seg = key + g * stride;
        const K me[1] = {seg[j]};
        int r[1] = {0};
        count_greater<1, K>(seg, 0, n, me, r);
        out[g * stride + r[0]] = me[0];
      }
      return;
    }
  }
  rank_sort_general<K>(key, stride, nseg, n, out);
}

// CTA-wide bitonic sort, descending, of nseg segments of npad (power of two)
// keys each, in place; padding keys must be 0.
template <typename K>
__device__ EPLB_RB_COLD void bitonic_desc(K *key, int npad, int nseg) {
  const int half = (npad * nseg) >> 1;
  for (int k = 2; k <= npad; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll 1
      for (int t = threadIdx.x; t < half; t += nthr()) {
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

// ---------------------------------------------------------------------------
// balanced_packing's greedy over items sorted as composite keys
// (load << 12 | (4095 - item)), descending; the pack keys are
// weight << 12 | pack, so adding an item's load is one add of (key & ~4095).
//
// Same greedy with a node's packs spread over the lanes of a segment, in
// sorted order: for m <= 32 a segment is the next power of two >= m lanes
// with one position each; for larger m a segment is a whole warp and lane l
// holds positions l*PL .. l*PL+PL-1.  Per item: position 0 (the lightest,
// lowest index on ties) is broadcast, every position compares its key and
// its right neighbour's with the pack's new key, and takes the neighbour's
// key, the new key or its own -- one shuffle pair and a few selects per item
// (a ballot + popc for the insertion point measured 45 cycles on the chain).
// Counts move with keys.
template <typename K, int PL>
__device__ void pack_seg(const K *skey_base, int stride, int nseg, int n, int m, int cap,
                         int32_t *ipack, int32_t *irank, int out_stride) {
  const K imask = K(kIdxMask);
  const K kmax = ~K(0);
  int ms = 2;  // lanes per segment
  while (ms < m && ms < 32) ms <<= 1;
  if (PL > 1) ms = 32;
  const int lane = threadIdx.x & 31;
  const int li = lane & (ms - 1);            // lane within the segment
  const int lms = __ffs(ms) - 1;  // ms is a power of two
  const int slot = static_cast<int>(threadIdx.x) >> lms;
  const int slots = nthr() >> lms;
  const int warp_first_slot = (static_cast<int>(threadIdx.x) & ~31) >> lms;
  for (int g0 = 0; g0 < nseg; g0 += slots) {
    if (g0 + warp_first_slot >= nseg) continue;  // no segment of this warp is live: skip the chain
    const int g = g0 + slot;
    const bool active = g < nseg;
    const K *skey = skey_base + (active ? g : 0) * stride;
    K key[PL];
    int cnt[PL];
#pragma unroll
    for (int r = 0; r < PL; ++r) {
      const int pos = li * PL + r;
      key[r] = pos < m ? K(pos) : kmax;  // pack pos, weight 0
      cnt[r] = 0;
    }
    K nxt = skey[0];
    for (int j = 0; j < n; ++j) {
      const K c = nxt;
      if (j + 1 < n) nxt = skey[j + 1];
      const K best = shfl_idx(key[0], 0, ms);
      const int bc = __shfl_sync(0xffffffffu, cnt[0], 0, ms);
      const K up = shfl_down_k(key[0], 1, ms);  // position (li+1)*PL of the next lane
      const int upc = __shfl_down_sync(0xffffffffu, cnt[0], 1, ms);
      const K nk = bc + 1 < cap ? best + (c & ~imask) : kmax;
      // lt(q) = position q >= 1 holds a key below the new one; the lt
      // positions are a prefix 1..p.  Position q takes position q+1's key
      // when lt(q+1), the new key when lt(q) or q == 0 (and not lt(q+1)),
      // else keeps its own: no ballot needed, each lane sees q and q+1.
      bool ltk[PL];
#pragma unroll
      for (int r = 0; r < PL; ++r) ltk[r] = (li * PL + r) >= 1 && key[r] < nk;
      const bool lt_up = li + 1 < ms && up < nk;
#pragma unroll
      for (int r = 0; r < PL; ++r) {
        const bool next_lt = r + 1 < PL ? ltk[r + 1 < PL ? r + 1 : r] : lt_up;
        const K right = r + 1 < PL ? key[r + 1 < PL ? r + 1 : r] : up;
        const int rightc = r + 1 < PL ? cnt[r + 1 < PL ? r + 1 : r] : upc;
        const bool here = ltk[r] || (li * PL + r) == 0;
        key[r] = next_lt ? right : (here ? nk : key[r]);
        cnt[r] = next_lt ? rightc : (here ? bc + 1 : cnt[r]);
      }
      if (li == 0 && active) {
        const int item = static_cast<int>(imask - (c & imask));
        ipack[g * out_stride + item] = static_cast<int>(best & imask);
        irank[g * out_stride + item] = bc;
      }
    }
  }
}

// Same greedy for wide segments, one warp per segment: pack q is owned by
// lane q % 32 (state in shared memory); each lane caches the composite key
// of its lightest non-full pack; the warp takes the minimum with an xor
// butterfly.
template <typename K>
__device__ EPLB_RB_COLD void pack_warp(const K *skey, int n, int m, int cap, K *pw, int32_t *pc,
                          int32_t *ipack, int32_t *irank) {
  const int lane = threadIdx.x & 31;
  const K imask = K(kIdxMask);
  const K kmax = ~K(0);
#pragma unroll 1
  for (int q = lane; q < m; q += 32) {
    pw[q] = 0;
    pc[q] = 0;
  }
  __syncwarp();
  K best = lane < m ? K(lane) : kmax;
  int rounds = 0;
  while ((1 << rounds) < min(m, 32)) ++rounds;
  for (int j = 0; j < n; ++j) {
    const K ck = skey[j];
    K b = best;
    for (int r = rounds - 1; r >= 0; --r) b = kmin(b, shfl_xor(b, 1 << r));
    const int q = static_cast<int>(b & imask);
    if (b != kmax && lane == (q & 31)) {
      const int rk = pc[q];
      pc[q] = rk + 1;
      pw[q] += ck & ~imask;  // weights kept pre-shifted
      const int item = static_cast<int>(imask - (ck & imask));
      ipack[item] = q;
      irank[item] = rk;
      K nb = kmax;
#pragma unroll 1
      for (int qq = lane; qq < m; qq += 32)
        if (pc[qq] < cap) nb = kmin(nb, pw[qq] | K(qq));
      best = nb;
    }
    __syncwarp();
  }
}

// The greedy in closed form when every pack takes exactly two items
// (n == 2m) and the m heaviest items all weigh more than zero.  First items:
// item j (sorted, 0-based) finds packs 0..j-1 heavier than the empty ones,
// so it opens pack j.  Second items: no pack changes weight until it is full, so
// the packs take their second item lightest first -- ascending (weight,
// index) of their first item -- and pack p takes item m + pos(p).  One
// thread per pack, no dependent chain.
constexpr int kCap2MinPacks = 16;

// True when either packing step of rebalance_experts on shape s has two items
// per pack over at least kCap2MinPacks packs (the closed form may apply).
__host__ __device__ inline bool cap2_shape(const RebalanceShape &s) {
  return (s.ppg == 2 && s.ppn == 2 * s.mpn && s.mpn >= kCap2MinPacks) ||
         (s.gpn == 2 && s.G == 2 * s.N && s.N >= kCap2MinPacks);
}

template <typename K>
__device__ EPLB_RB_COLD void pack_cap2(const K *skey_base, int stride, int nseg, int m, int32_t *ipack,
                          int32_t *irank, int out_stride) {
  const K imask = K(kIdxMask);
#pragma unroll 1
  for (int t = threadIdx.x; t < nseg * m; t += nthr()) {
    const int g = t / m;
    const int p = t - g * m;
    const K *skey = skey_base + g * stride;
    const K kp = skey[p];
    const K wp = kp >> kIdxBits;
    int item = static_cast<int>(imask - (kp & imask));
    ipack[g * out_stride + item] = p;
    irank[g * out_stride + item] = 0;
    int pos = 0;
    for (int q = 0; q < m; ++q) {
      const K wq = skey[q] >> kIdxBits;
      pos += (wq < wp || (wq == wp && q < p)) ? 1 : 0;
    }
    const K k2 = skey[m + pos];
    item = static_cast<int>(imask - (k2 & imask));
    ipack[g * out_stride + item] = p;
    irank[g * out_stride + item] = 1;
  }
}

// Packs nseg segments (segment g: n sorted keys at skey + g * stride, results
// at ipack/irank + g * out_stride) into m packs of cap items each.  Called by
// every thread of the CTA (the lane-parallel variant needs whole warps).
// kCap2 compiles in the two-items-per-pack closed form; kernels for shapes
// that can never take it are built without it (its code alone, never run,
// slowed the row by about 2 us: the kernel is instruction-fetch bound).
template <typename K>
__device__ EPLB_RB_COLD void pack_segments_wide(const K *skey, int stride, int nseg, int n, int m,
                                                int cap, K *pw, int32_t *pc, int32_t *ipack,
                                                int32_t *irank, int out_stride);

template <typename K, bool kCap2>
__device__ EPLB_RB_SHARED void pack_segments(const K *skey, int stride, int nseg, int n, int m, int cap, K *pw,
                              int32_t *pc, int32_t *ipack, int32_t *irank, int out_stride) {
  if (n <= 0) return;
  if constexpr (kCap2) {
    // closed form only for long chains: on a few packs (8 groups onto 4
    // nodes) the vote cost more than the short greedy it replaces (measured)
    if (cap == 2 && n == 2 * m && m >= kCap2MinPacks) {  // every segment has this shape
      bool ok = true;
#pragma unroll 1
      for (int g = threadIdx.x; g < nseg; g += nthr())
        ok &= (skey[g * stride + m - 1] >> kIdxBits) != K(0);
      if (__syncthreads_and(ok)) {
        pack_cap2<K>(skey, stride, nseg, m, ipack, irank, out_stride);
        return;
      }
    }
  }
  if (m <= 32) {
    pack_seg<K, 1>(skey, stride, nseg, n, m, cap, ipack, irank, out_stride);
  } else {
    pack_segments_wide<K>(skey, stride, nseg, n, m, cap, pw, pc, ipack, irank, out_stride);
  }
}

template <typename K>
__device__ EPLB_RB_COLD void pack_segments_wide(const K *skey, int stride, int nseg, int n, int m,
                                                int cap, K *pw, int32_t *pc, int32_t *ipack,
                                                int32_t *irank, int out_stride) {
  if (m <= 64) {
    pack_seg<K, 2>(skey, stride, nseg, n, m, cap, ipack, irank, out_stride);
  } else if (m <= 128) {
    pack_seg<K, 4>(skey, stride, nseg, n, m, cap, ipack, irank, out_stride);
  } else if (m <= 256 && sizeof(K) == 8) {
    pack_seg<K, 8>(skey, stride, nseg, n, m, cap, ipack, irank, out_stride);
  } else {
#pragma unroll 1
    for (int g = threadIdx.x >> 5; g < nseg; g += nwarps())
      pack_warp<K>(skey + g * stride, n, m, cap, pw + g * m, pc + g * m, ipack + g * out_stride,
                   irank + g * out_stride);
  }
}

// ---------------------------------------------------------------------------
// replicate_experts.  a beats b on a larger w/c, then a lower index.
__device__ __forceinline__ bool rep_better(int64_t aw, int ac, int ai, int64_t bw, int bc, int bi) {
  const int64_t lhs = aw * static_cast<int64_t>(bc);
  const int64_t rhs = bw * static_cast<int64_t>(ac);
  return lhs > rhs || (lhs == rhs && ai < bi);
}

// D'Hondt form of the greedy: the extra replicas, in order, are the R best
// (candidate k, divisor d) pairs by w_k / d desc, expert index asc, d asc
// (each step takes the largest current quotient, and an expert's quotients
// w/1, w/2, ... only decrease).  Pair (k, d) has at least k + d - 1 pairs
// ahead of it (the k heavier candidates' first pairs and (k, 1 .. d-1)), so
// only pairs with d <= R - k can be picked and only those are ranked.  All
// pairs of all nodes are ranked in parallel; the picks need no serial chain.
__device__ void replicate_pairs(const RebalanceShape &s, const int64_t *cand_w,
                                const int32_t *cand_i, int32_t *cand_c, int32_t *p2m,
                                int32_t *rrank, uint32_t m_grid, uint32_t m_r) {
  // Pair (k, d) -- candidate k's d-th extra replica, value w_k / d -- ranks
  // after every pair of greater value, and after equal-valued pairs of a
  // lower expert index (same expert: lower d).  Candidate k2 has D2 = R - k2
  // pairs; those ahead of (k, d) are d2 < w_k2 * d / w_k, plus d2 equal to it
  // when the quotient is exact and id2 < id: one quotient per k2 instead of
  // D2 cross-multiplied compares.
  const int R = s.ppn - s.lpn, nc = num_cand(s);
  const int grid = nc * R;
#pragma unroll 1
  for (int t = threadIdx.x; t < s.N * grid; t += nthr()) {
    const int n = qdivm(t, grid, m_grid);
    const int p = t - n * grid;
    const int k = qdivm(p, R, m_r);
    const int d = p - k * R + 1;
    if (d > R - k) continue;
    const int64_t w = cand_w[n * nc + k];
    const int id = cand_i[n * nc + k];
    int rank = d - 1;  // the same expert's earlier replicas
    if (cand_w[n * nc] < (int64_t(1) << 31) / (R + 1)) {
      // the node's heaviest candidate times R + 1 is below 2^31, so every
      // product below is too: the same ranking in 32-bit integers (about
      // half the instructions of the 64-bit one; the estimate's error stays
      // within the fix-ups)
      const int32_t w32 = static_cast<int32_t>(w);
      const float rw = __frcp_rn(static_cast<float>(w32 > 0 ? w32 : 1));
#pragma unroll 4
      for (int k2 = 0; k2 < nc; ++k2) {
        const int32_t w2 = static_cast<int32_t>(cand_w[n * nc + k2]);
        const int id2 = cand_i[n * nc + k2];
        const int D2 = R - k2;
        const int32_t A = w2 * d;
        int ahead;
        if (w32 == 0) {
          ahead = (w2 > 0 || id2 < id) ? D2 : 0;
        } else if (A >= w32 * (D2 + 1)) {
          ahead = D2;
        } else {
          int32_t q = static_cast<int32_t>(__fmul_rn(static_cast<float>(A), rw));
          int32_t r = A - q * w32;
          if (r < 0) { --q; r += w32; }
          if (r < 0) { --q; r += w32; }
          if (r >= w32) { ++q; r -= w32; }
          if (r >= w32) { ++q; r -= w32; }
          ahead = min(max(r == 0 ? q - 1 + (id2 < id ? 1 : 0) : q, 0), D2);
        }
        rank += k2 == k ? 0 : ahead;
      }
      if (rank < R) {
        p2m[n * s.ppn + s.lpn + rank] = id;
        rrank[n * s.ppn + s.lpn + rank] = d;
        atomicAdd(&cand_c[n * nc + k], 1);
      }
      continue;
    }
    for (int k2 = 0; k2 < nc; ++k2) {
      if (k2 == k) continue;
      const int64_t w2 = cand_w[n * nc + k2];
      const int id2 = cand_i[n * nc + k2];
      const int D2 = R - k2;
      int ahead;
      if (w == 0) {  // every value is >= 0: ahead if larger, or equal with a lower index
        ahead = (w2 > 0 || id2 < id) ? D2 : 0;
      } else {
        const int64_t A = w2 * d;  // < 2^51
        if (A >= w * (D2 + 1)) {
          ahead = D2;  // even d2 = D2 is strictly ahead
        } else {
          // q = floor(A / w) <= D2: a float estimate, then exact integer fix-up
          int64_t q = static_cast<int64_t>(__fmul_rn(static_cast<float>(A),
                                                     __frcp_rn(static_cast<float>(w))));
          int64_t r = A - q * w;
          if (r < 0) { --q; r += w; }
          if (r < 0) { --q; r += w; }
          if (r >= w) { ++q; r -= w; }
          if (r >= w) { ++q; r -= w; }
          ahead = static_cast<int>(r == 0 ? q - 1 + (id2 < id ? 1 : 0) : q);
          ahead = min(max(ahead, 0), D2);
        }
      }
      rank += ahead;
    }
    if (rank < R) {
      p2m[n * s.ppn + s.lpn + rank] = id;
      rrank[n * s.ppn + s.lpn + rank] = d;
      atomicAdd(&cand_c[n * nc + k], 1);
    }
  }
}

// Greedy over nc <= 32 candidates, one per lane of a warp.
__device__ EPLB_RB_COLD void replicate_warp(int nc, int lpn, int ppn, int n, const int64_t *cand_w,
                                            const int32_t *cand_i, int32_t *cand_c, int32_t *p2m,
                                            int32_t *rrank) {
  const int lane = threadIdx.x & 31;
  const int bp = n * ppn;
  const bool valid = lane < nc;
  const int64_t w = valid ? cand_w[n * nc + lane] : 0;
  const int id = valid ? cand_i[n * nc + lane] : 0x7fffffff;
  int c = 1;
  int rounds = 0;
  while ((1 << rounds) < min(nc, 32)) ++rounds;
  for (int r = 0; r < ppn - lpn; ++r) {
    int64_t bw = w;
    int bc = c, bi = id, bl = lane;
    for (int k = rounds - 1; k >= 0; --k) {
      const int64_t ow = static_cast<int64_t>(shfl_xor(static_cast<uint64_t>(bw), 1 << k));
      const int oc = __shfl_xor_sync(0xffffffffu, bc, 1 << k);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, 1 << k);
      const int ol = __shfl_xor_sync(0xffffffffu, bl, 1 << k);
      if (rep_better(ow, oc, oi, bw, bc, bi)) {
        bw = ow;
        bc = oc;
        bi = oi;
        bl = ol;
      }
    }
    if (valid && lane == bl) {
      p2m[bp + lpn + r] = id;
      rrank[bp + lpn + r] = c;
      ++c;
    }
  }
  if (valid) cand_c[n * nc + lane] = c;
  __syncwarp();
}

// Any number of candidates (all experts of the node), counts in shared memory.
__device__ EPLB_RB_COLD void replicate_smem(int lpn, int ppn, int n, const int64_t *wm, int32_t *cnt,
                               int32_t *p2m, int32_t *rrank) {
  const int lane = threadIdx.x & 31;
  const int bm = n * lpn, bp = n * ppn;
  auto local_best = [&](int64_t &bw, int &bc, int &bi) {
    bw = 0;
    bc = 1;
    bi = 0x7fffffff;
#pragma unroll 1
    for (int i = lane; i < lpn; i += 32)
      if (rep_better(wm[bm + i], cnt[bm + i], i, bw, bc, bi)) {
        bw = wm[bm + i];
        bc = cnt[bm + i];
        bi = i;
      }
  };
  int64_t bw;
  int bc, bi;
  local_best(bw, bc, bi);
  for (int r = 0; r < ppn - lpn; ++r) {
    int64_t mw = bw;
    int mc = bc, mi = bi;
    for (int k = 16; k >= 1; k >>= 1) {
      const int64_t ow = static_cast<int64_t>(shfl_xor(static_cast<uint64_t>(mw), k));
      const int oc = __shfl_xor_sync(0xffffffffu, mc, k);
      const int oi = __shfl_xor_sync(0xffffffffu, mi, k);
      if (rep_better(ow, oc, oi, mw, mc, mi)) {
        mw = ow;
        mc = oc;
        mi = oi;
      }
    }
    if (lane == (mi & 31)) {
      cnt[bm + mi] = mc + 1;
      p2m[bp + lpn + r] = mi;
      rrank[bp + lpn + r] = mc;
      local_best(bw, bc, bi);
    }
    __syncwarp();
  }
}

// The plan of a row that cannot be computed: no replicas, log2phy all -1,
// plan quality NaN.
__device__ void write_error_row(const RbArgs &a, int64_t row) {
  const int P = a.s.P, E = a.s.E, X = a.s.X, gpus = a.s.gpus;
#pragma unroll 1
  for (int t = threadIdx.x; t < P; t += nthr()) {
    a.phy2log[row * P + t] = -1;
    a.phyrank[row * P + t] = -1;
  }
#pragma unroll 1
  for (int e = threadIdx.x; e < E; e += nthr()) a.logcnt[row * E + e] = 0;
  int32_t *gl = a.log2phy + row * static_cast<int64_t>(E) * X;
#pragma unroll 1
  for (int i = threadIdx.x; i < E * X; i += nthr()) gl[i] = -1;
  const double nan = __longlong_as_double(0x7ff8000000000000LL);
  if (a.gpu_load) {
#pragma unroll 1
    for (int g = threadIdx.x; g < gpus; g += nthr()) a.gpu_load[row * gpus + g] = nan;
  }
  if (a.stats && threadIdx.x < 4) a.stats[row * 4 + threadIdx.x] = nan;
}

// Plan quality of the row just assembled, by one warp while the others copy
// log2phy out (page "DualPipe и EPLB", Part 2, box "От переводчика: что на
// рисунке": per-GPU loads of the worked example; exercise 2 of "что сделать
// руками": max against mean).  q[p] = w / logcnt of slot p's expert (fp64,
// rounded to nearest); GPU g's load is the sum of its slots' q in slot order
// from 0.0; min and max of the GPU loads (exact in any order: a warp
// butterfly); their mean summed in GPU order from 0.0 divided by gpus; and
// balancedness = mean / max (1 when max is 0).  Every add and divide is an
// explicitly rounded fp64 operation in that fixed order, so the figures are
// bit-identical to the same sums done sequentially on a CPU.  The quotients
// q are divided while step 3 packs (one per expert, by the idle warps: nine
// per lane here took 1.4 us) and placed by the assembly pass; inline: out of
// line, and with a serial min / max loop, it cost 4 us of the 58-row step
// (measured).  q: P slot quotients, gl: gpus doubles of scratch.
// one out-of-line copy of the correctly rounded fp64 divide, off the row's
// straight-line code
__device__ EPLB_RB_COLD double qdiv(double a, double b) { return __ddiv_rn(a, b); }

constexpr int kQualityRegs = 12;  // replicas per GPU summed from registers

__device__ __forceinline__ void plan_quality(double *gpu_load, double *stats, int64_t row,
                                             int gpus, int ppg, const double *q, double *gl) {
  const int lane = threadIdx.x & 31;
  double mn = __longlong_as_double(0x7ff0000000000000LL), mx = 0.0;  // +inf, 0
#pragma unroll 1
  for (int g = lane; g < gpus; g += 32) {
    double acc = 0.0;
    if (ppg <= kQualityRegs) {  // every load issued before the ordered adds
      double v[kQualityRegs];
#pragma unroll
      for (int k = 0; k < kQualityRegs; ++k) v[k] = k < ppg ? q[g * ppg + k] : 0.0;
#pragma unroll
      for (int k = 0; k < kQualityRegs; ++k)
        if (k < ppg) acc = __dadd_rn(acc, v[k]);
    } else {
#pragma unroll 4
      for (int k = 0; k < ppg; ++k) acc = __dadd_rn(acc, q[g * ppg + k]);
    }
    gl[g] = acc;
    if (gpu_load) gpu_load[row * gpus + g] = acc;
    mn = fmin(mn, acc);
    mx = fmax(mx, acc);
  }
  if (stats == nullptr) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  __syncwarp();
  if (lane == 0) {
    double sum = 0.0;
    int g = 0;
    for (; g + 8 <= gpus; g += 8) {  // loads ahead of the ordered adds
      double v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = gl[g + j];
#pragma unroll
      for (int j = 0; j < 8; ++j) sum = __dadd_rn(sum, v[j]);
    }
    for (; g < gpus; ++g) sum = __dadd_rn(sum, gl[g]);
    const double mean = qdiv(sum, static_cast<double>(gpus));
    stats[row * 4 + 0] = mn;
    stats[row * 4 + 1] = mx;
    stats[row * 4 + 2] = mean;
    stats[row * 4 + 3] = mx > 0.0 ? qdiv(mean, mx) : 1.0;
  }
}

// Operands of step 3 as plain values (an out-of-line instance then needs no
// copy of the kernel's parameter block or of the layout on the stack).
struct Step3Ops {
  unsigned char *keys, *sorted, *pw;
  const int64_t *wm;
  const uint64_t *lam;
  const int32_t *cnt, *p2m;
  int32_t *pc, *ipack, *irank;
  int N, npad, lpn, ppn, mpn, ppg;
  int32_t *status;  // the checking build's reports
  uint32_t m_per;   // magic of the keys per node
};

template <typename K, bool kCap2>
__device__ void step3(const Step3Ops &o) {
  K *keys = reinterpret_cast<K *>(o.keys);
  K *sorted = reinterpret_cast<K *>(o.sorted);
  const int64_t *wm = o.wm;
  const uint64_t *lam = o.lam;
  const int32_t *cnt = o.cnt;
  const int32_t *p2m = o.p2m;
  const int N = o.N, npad = o.npad, lpn = o.lpn, ppn = o.ppn;
  const K imask = K(kIdxMask);
  const bool ranked = npad <= kRankSortMax;
  const int per = ranked ? ppn : npad;
#pragma unroll 1
  for (int t = threadIdx.x; t < N * per; t += nthr()) {
    const int n = qdivm(t, per, o.m_per);
    const int j = t - n * per;
    K key = 0;
    if (j < ppn && EPLB_IN(p2m[n * ppn + j] >= 0 && p2m[n * ppn + j] < lpn, o.status)) {
      const int m = n * lpn + p2m[n * ppn + j];
      const uint32_t c = static_cast<uint32_t>(cnt[m]);
      const uint64_t lm = lam[n];
      // Lambda / c exactly; a 32-bit divide when Lambda fits (lcm(1..9) =
      // 2520 on the DeepSeek-V3 shape), the 64-bit routine otherwise
      const uint64_t scale = c == 1 ? lm : (lm >> 32 ? lm / c : static_cast<uint32_t>(lm) / c);
      key = ((K(static_cast<uint64_t>(wm[m])) * K(scale)) << kIdxBits) | (imask - K(j));
    }
    keys[n * npad + j] = key;
  }
  __syncthreads();
  const K *skeys = keys;
  if (ranked) {
    rank_sort<K>(keys, npad, N, ppn, sorted);
    skeys = sorted;
    __syncthreads();
  } else {
    bitonic_desc<K>(keys, npad, N);
  }
  pack_segments<K, kCap2>(skeys, npad, N, ppn, o.mpn, o.ppg, reinterpret_cast<K *>(o.pw), o.pc,
                          o.ipack, o.irank, ppn);
}

// step 3 with 128-bit keys (rows whose weights times Lambda overflow 64 bits);
// left inline: out of line, its call made the kernel spill around it
template <bool kCap2>
__device__ void step3_wide(unsigned char *keys, unsigned char *sorted, unsigned char *pw,
                                        const int64_t *wm, const uint64_t *lam, const int32_t *cnt,
                                        const int32_t *p2m, int32_t *pc, int32_t *ipack,
                                        int32_t *irank, int N, int npad, int lpn, int ppn, int mpn,
                                        int ppg, int32_t *status, uint32_t m_per) {
  step3<u128, kCap2>(Step3Ops{keys, sorted, pw, wm, lam, cnt, p2m, pc, ipack, irank, N, npad, lpn,
                              ppn, mpn, ppg, status, m_per});
}

// One row of rebalance_experts, by the whole CTA, in `smem` (Layout(a.s).total
// bytes).  Called by every thread of the CTA; kCap2 = cap2_shape(a.s) (a
// kernel built without it is correct on every shape, only slower on those).
template <bool kCap2>
__device__ __forceinline__ void rebalance_row(const RbArgs &a, int64_t row, unsigned char *smem) {
  __shared__ int flags[2];  // [0] 128-bit keys needed, [1] exact ratio not representable
  const RebalanceShape &s = a.s;
  const Layout lay(s);
  int64_t *w = reinterpret_cast<int64_t *>(smem + lay.w);
  int64_t *wm = reinterpret_cast<int64_t *>(smem + lay.wm);
  uint64_t *gkey = reinterpret_cast<uint64_t *>(smem + lay.gkey);
  uint64_t *gsorted = reinterpret_cast<uint64_t *>(smem + lay.gsorted);
  uint64_t *lam = reinterpret_cast<uint64_t *>(smem + lay.lam);
  int64_t *cand_w = reinterpret_cast<int64_t *>(smem + lay.cand_w);
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
  int32_t *cand_i = reinterpret_cast<int32_t *>(smem + lay.cand_i);
  int32_t *cand_c = reinterpret_cast<int32_t *>(smem + lay.cand_c);

  const int tid = threadIdx.x;
  if (tid == 0) {
    flags[0] = 0;
    flags[1] = 0;
  }

  // ---- load the row (the window sum over the ring); loads in [0, 2^40) --
  // two threads per expert, each summing half of the ring rows with all its
  // loads in flight
  bool bad = false;
  {
    const int lane = tid & 31;
    const int64_t half = (a.ring_w + 1) >> 1;
#pragma unroll 1
    for (int t = tid; t - lane < 2 * s.E; t += nthr()) {  // warp-uniform for the shuffle
      const bool live = t < 2 * s.E;
      const int e = t >> 1;
      const int64_t at = row * s.E + e;
      const int64_t k0 = (t & 1) * half;
      const int64_t k1 = min(a.ring_w, k0 + half);
      int64_t x = 0;
      if (live) {
#pragma unroll 8
        for (int64_t k = k0; k < k1; ++k) x += __ldcg(a.ring + k * a.ring_stride + at);
      }
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      if (live && !(t & 1)) {
        w[e] = x;
        if (a.loads_out) a.loads_out[at] = x;
        if (a.zero_slot >= 0) a.ring[a.zero_slot * a.ring_stride + at] = 0;
        bad |= (x < 0) | (x >= kLoadLimit);
      }
    }
  }
  if (__syncthreads_or(bad)) {
    write_error_row(a, row);
    if (tid == 0) report(a.status, EPLB_ERR_RANGE);
    return;
  }

  if (table_in_smem(s)) {  // the log2phy table starts all -1 (filled while step 1 runs)
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + lay.table);
#pragma unroll 1
    for (int i = tid; i < s.E * s.X; i += nthr()) tbl[i] = -1;
  }

  // ---- step 1: groups -> nodes ---------------------------------------------
  if (s.gpn == 1) {  // one group per node: the pages' identity short-cut
#pragma unroll 1
    for (int g = tid; g < s.G; g += nthr()) {
      gpack[g] = g;
      grank[g] = 0;
    }
  } else {
#pragma unroll 1
    for (int g = tid >> 5; g < s.G; g += nwarps()) {  // one warp per group
      const int lane = tid & 31;
      uint64_t sum = 0;
#pragma unroll 1
      for (int i = lane; i < s.gs; i += 32) sum += static_cast<uint64_t>(w[g * s.gs + i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) gkey[g] = (sum << kIdxBits) | (kIdxMask - g);
    }
    __syncthreads();
    const uint64_t *gs_keys = gsorted;
    if (s.gpad <= kRankSortMax) {
      rank_sort<uint64_t>(gkey, s.gpad, 1, s.G, gsorted);
    } else {
#pragma unroll 1
      for (int g = s.G + tid; g < s.gpad; g += nthr()) gkey[g] = 0;
      __syncthreads();
      bitonic_desc<uint64_t>(gkey, s.gpad, 1);
      gs_keys = gkey;
    }
    __syncthreads();
    pack_segments<uint64_t, kCap2>(gs_keys, s.gpad, 1, s.G, s.N, s.gpn,
                            reinterpret_cast<uint64_t *>(smem + lay.npw),
                            reinterpret_cast<int32_t *>(smem + lay.npc), gpack, grank, s.G);
  }
  __syncthreads();
  // mlog = logical order after the node permutation; replicate's initial state
#pragma unroll 1
  for (int e = tid; e < s.E; e += nthr()) {
    const int g = qdivm(e, s.gs, a.m_gs);
    const int m = (gpack[g] * s.gpn + grank[g]) * s.gs + (e - g * s.gs);
    if (!EPLB_IN(m >= 0 && m < s.E, a.status)) continue;
    mlog2log[m] = e;
    wm[m] = w[e];
    cnt[m] = 1;
    const int n = qdivm(m, s.lpn, a.m_lpn);
    const int i = m - n * s.lpn;
    p2m[n * s.ppn + i] = i;
    rrank[n * s.ppn + i] = 0;
  }
  __syncthreads();

  // ---- step 2: replicate_experts inside every node -------------------------
  const int nc = num_cand(s);
  if (nc > 0 && nc <= 32) {
    // candidates: the nc heaviest experts of each node (ties by index)
    uint64_t *ckey = reinterpret_cast<uint64_t *>(smem + lay.keys);
#pragma unroll 1
    for (int m = tid; m < s.E; m += nthr()) {
      const int n = qdivm(m, s.lpn, a.m_lpn);
      ckey[m] = (static_cast<uint64_t>(wm[m]) << kIdxBits) | (kIdxMask - (m - n * s.lpn));
    }
    __syncthreads();
    uint64_t *csorted = reinterpret_cast<uint64_t *>(smem + lay.sorted);
    rank_sort<uint64_t>(ckey, s.lpn, s.N, s.lpn, csorted);
    __syncthreads();
#pragma unroll 1
    for (int t = tid; t < s.N * nc; t += nthr()) {  // the nc heaviest of each node
      const int g = qdivm(t, nc, a.m_nc);
      const int j = static_cast<int>(kIdxMask - (csorted[g * s.lpn + (t - g * nc)] & kIdxMask));
      cand_w[t] = wm[g * s.lpn + j];
      cand_i[t] = j;
    }
    __syncthreads();
    if (nc * (s.ppn - s.lpn) <= 256) {
#pragma unroll 1
      for (int t = tid; t < s.N * nc; t += nthr()) cand_c[t] = 1;
      __syncthreads();
      replicate_pairs(s, cand_w, cand_i, cand_c, p2m, rrank, a.m_grid, a.m_r);
    } else {
#pragma unroll 1
      for (int n = tid >> 5; n < s.N; n += nwarps())
        replicate_warp(nc, s.lpn, s.ppn, n, cand_w, cand_i, cand_c, p2m, rrank);
    }
    __syncthreads();
#pragma unroll 1
    for (int t = tid; t < s.N * nc; t += nthr()) {
      const int n = qdivm(t, nc, a.m_nc);
      if (EPLB_IN(cand_i[t] >= 0 && cand_i[t] < s.lpn, a.status)) cnt[n * s.lpn + cand_i[t]] = cand_c[t];
    }
  } else if (nc > 32) {
#pragma unroll 1
    for (int n = tid >> 5; n < s.N; n += nwarps()) replicate_smem(s.lpn, s.ppn, n, wm, cnt, p2m, rrank);
  }
  __syncthreads();

  // ---- Lambda and key width per node (one thread per node) ----------------
  if (s.ppg > 1) {
#pragma unroll 1
    for (int n = tid; n < s.N; n += nthr()) {
      int64_t wmax = 0;
      if (nc > 0 && nc <= 32) {
        wmax = cand_w[n * nc];
      } else {
        for (int i = 0; i < s.lpn; ++i) wmax = max(wmax, wm[n * s.lpn + i]);
      }
      auto width = [&](uint64_t l) -> int {
        const u128 maxsum = static_cast<u128>(static_cast<uint64_t>(wmax)) * l * s.ppg;
        if ((maxsum >> (63 - kIdxBits)) == 0) return 0;
        if ((maxsum >> (127 - kIdxBits)) == 0) return 1;
        return 2;
      };
      uint64_t l = s.lam_fixed;
      int wd = 2;
      if (l != 0) wd = width(l);
      if (wd != 0) {
        // lcm of the counts present in the node
        l = 1;
        bool ok = true;
        if (nc > 0 && nc <= 32 && s.cmax < 64) {
          uint64_t present = 0;  // bit c: some candidate has c replicas
          for (int k = 0; k < nc; ++k) present |= uint64_t(1) << cand_c[n * nc + k];
          present &= ~uint64_t(3);
          while (present && ok) {
            const int c = __ffsll(static_cast<long long>(present)) - 1;
            present &= present - 1;
            ok = lcm_into(l, static_cast<uint32_t>(c));
          }
        } else if (nc > 0 && nc <= 32) {
          for (int k = 0; k < nc && ok; ++k) ok = lcm_into(l, static_cast<uint32_t>(cand_c[n * nc + k]));
        } else {
          for (int i = 0; i < s.lpn && ok; ++i) ok = lcm_into(l, static_cast<uint32_t>(cnt[n * s.lpn + i]));
        }
        wd = ok ? width(l) : 2;
      }
      lam[n] = l;
      if (wd == 2) atomicOr(&flags[1], 1);
      if (wd == 1) atomicOr(&flags[0], 1);
    }
    __syncthreads();
  }
  if (flags[1]) {
    write_error_row(a, row);
    if (tid == 0) report(a.status, EPLB_ERR_RANGE);
    return;
  }

  // ---- step 3: replicas -> GPUs of each node ------------------------------
  if (s.ppg == 1) {  // one replica per GPU: identity short-cut
#pragma unroll 1
    for (int t = tid; t < s.P; t += nthr()) {
      const int n = qdivm(t, s.ppn, a.m_ppn);
      ipack[t] = t - n * s.ppn;
      irank[t] = 0;
    }
  } else if (flags[0] == 0) {
    step3<uint64_t, kCap2>(Step3Ops{smem + lay.keys, smem + lay.sorted, smem + lay.pw, wm, lam, cnt,
                                    p2m, reinterpret_cast<int32_t *>(smem + lay.pc), ipack, irank,
                                    s.N, s.npad, s.lpn, s.ppn, s.mpn, s.ppg, a.status, a.m_per});
  } else {
    step3_wide<kCap2>(smem + lay.keys, smem + lay.sorted, smem + lay.pw, wm, lam, cnt, p2m,
                      reinterpret_cast<int32_t *>(smem + lay.pc), ipack, irank, s.N, s.npad, s.lpn,
                      s.ppn, s.mpn, s.ppg, a.status, a.m_per);
  }
  // plan quality: every logical expert's slot value w / logcnt, by the warps
  // the packing chain leaves idle (the highest thread ids take the first
  // experts), into the raw loads' space (free after step 1)
  const bool quality = a.gpu_load != nullptr || a.stats != nullptr;
  double *qm = reinterpret_cast<double *>(smem + lay.w);
  if (quality) {
#pragma unroll 1
    for (int m = nthr() - 1 - tid; m < s.E; m += nthr())
      qm[m] = qdiv(static_cast<double>(wm[m]), static_cast<double>(cnt[m]));
  }
  __syncthreads();

  // ---- assembly: pphy = node*ppn + gpu*ppg + rank -------------------------
  // phy2log / phyrank / logcnt go straight to global memory; log2phy is
  // scattered into the shared table (filled with -1 before step 1), then
  // copied out row-contiguously
  const int EX = s.E * s.X;
  int32_t *gl = a.log2phy + row * static_cast<int64_t>(EX);
  const bool in_smem = table_in_smem(s);
  int32_t *tbl = reinterpret_cast<int32_t *>(smem + lay.table);
  // plan quality: each slot's quotient, in the sort keys' space (free after
  // step 3)
  double *qslot = reinterpret_cast<double *>(smem + lay.keys);
  bool slots = false;
#pragma unroll 1
  for (int t = tid; t < s.P; t += nthr()) {
    const int n = qdivm(t, s.ppn, a.m_ppn);
    const int pphy = n * s.ppn + ipack[t] * s.ppg + irank[t];
    const int m = n * s.lpn + p2m[t];
    const int e = mlog2log[m];
    const int k = rrank[t];
    if (!EPLB_IN(pphy >= n * s.ppn && pphy < (n + 1) * s.ppn && e >= 0 && e < s.E && k >= 0 &&
                     m >= n * s.lpn && m < (n + 1) * s.lpn,
                 a.status))
      continue;
    if (quality) qslot[pphy] = qm[m];
    a.phy2log[row * s.P + pphy] = e;
    a.phyrank[row * s.P + pphy] = k;
    if (in_smem) {
      if (k < s.X)
        tbl[e * s.X + k] = pphy;
      else
        slots = true;
    } else {
      outp[pphy] = e;
      outr[pphy] = k;
    }
  }
#pragma unroll 1
  for (int m = tid; m < s.E; m += nthr()) {
    const int e = mlog2log[m];
    lc[e] = cnt[m];
    a.logcnt[row * s.E + e] = cnt[m];
  }
  __syncthreads();
  // warp 0 computes the plan quality (scratch in the sort keys' and pack
  // weights' space, free after step 3) while the other warps copy the
  // table out
  if (quality && tid < 32)
    plan_quality(a.gpu_load, a.stats, row, s.gpus, s.ppg, qslot,
                 reinterpret_cast<double *>(smem + lay.pw));
  if (in_smem) {
    const int t0 = quality ? 32 : 0;
    if (tid >= t0) {
      const int nt = nthr() - t0;
      if (a.table_vec4) {
        const int4 *src = reinterpret_cast<const int4 *>(tbl);
        int4 *dst = reinterpret_cast<int4 *>(gl);
#pragma unroll 1
        for (int i = tid - t0; i < (EX >> 2); i += nt) dst[i] = src[i];
      } else {
#pragma unroll 1
        for (int i = tid - t0; i < EX; i += nt) gl[i] = tbl[i];
      }
    }
  } else {
#pragma unroll 1
    for (int t = tid; t < s.P; t += nthr()) {
      const int k = outr[t];
      if (!EPLB_IN(outp[t] >= 0 && outp[t] < s.E && k >= 0, a.status)) continue;
      if (k < s.X)
        gl[outp[t] * s.X + k] = t;
      else
        slots = true;
    }
    const uint32_t X = static_cast<uint32_t>(s.X);
#pragma unroll 1
    for (int i = tid; i < EX; i += nthr()) {
      const uint32_t e = div_magic(static_cast<uint32_t>(i), X, a.x_magic);
      if (static_cast<int>(i - e * X) >= lc[e]) gl[i] = -1;
    }
  }
  if (slots) report(a.status, EPLB_ERR_SLOTS);
}


}  // namespace
}  // namespace eplb
