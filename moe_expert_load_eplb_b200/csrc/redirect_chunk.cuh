// redirect_chunk.cuh -- S5 (and S1 fused): the device code of one redirect
// CTA, shared by redirect.cu's kernel and the serving-step kernel.
//
// A planner maps the router's logical indices to physical ones (page
// "DeepSeek开源LPLB...", usage example).  Replica rule: token t of the call
// (global token t0 + t) uses replica (t0 + t) mod logcnt[l, e] for all K
// slots:  out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]].
//
// HBM-bound gather, streamed like the count kernel: each CTA owns one chunk
// of one layer (a contiguous run of the flattened index array whose interior
// is 16-byte aligned); every thread keeps U = 4 independent 16-byte
// streaming loads in flight, the next U vectors requested into L2 by
// prefetches, and writes 16-byte stores with the default cache policy (the
// evict-first `.cs` stores measured 0.6-0.8% slower on the 1.95 GB stream
// and 1.2 us slower for count+redirect on the 121.6 MB batch; the default
// also leaves the output in L2 for the kernel that reads it next).
// The per-index work decides the speed, so the common case is cut to a
// handful of instructions:
//
// Period table (the fast path).  If every expert's logcnt c divides a fixed
// period M (M = 120 covers c = 1..6, 8, 10, 12, ...; a layer whose counts
// all divide 24 uses M = 24, a fifth of the table to build), then
// (t0 + t) mod c = ((t0 + t) mod M) mod c, so the segment's shared table
//   tab[e][rho] = log2phy[l, e, rho mod c_e],   rho < M  (int16 entries)
// answers every index with one load at tab[e][(t0 + t) mod M]; rho is taken
// once per token.  Indices outside [0, E) are clamped to a sentinel row E of
// -1 (an unsigned min, no branch); an expert with a logcnt outside [1, X]
// gets a row of -1 too.  The CTA votes on the segment's logcnts
// (__syncthreads_and), so the choice of path is uniform.
//
// Descriptors (any plan).  Each expert's replica list becomes one 64-bit
// descriptor:
//   inline:  bits 0..4 = 6 * (c - 1) for c <= 5, bits 5 + 11 j .. = physical
//            index of replica j (all < 2048);
//   other:   bits 0..4 = 31, bits 5..36 = multiply-high magic of c, bits
//            37..52 = c (0: the expert's indices map to -1);
// stored in up to 16 copies (lane l reads copy l mod 16, so a half-warp's
// 64-bit loads hit distinct bank pairs).  Per token a selector word holds,
// in the 6-bit field at 6 * (c - 1), the bit offset of replica
// (t0 + t) mod c for c = 1..5; an "other" descriptor takes (t0 + t) mod c by
// multiply-high and a cached load of the log2phy row.
//
// The same walker with kCount also builds the load histogram of S1 (a
// lane-banked shared histogram, kHistCopies copies per bin, flushed at the
// chunk's end),
// so counting and redirecting one batch read its indices from HBM once:
// 8 bytes per index instead of 4 + 8.
#pragma once

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace eplb {
namespace {


constexpr int kThreads = 512;
constexpr int kU = 4;
constexpr int kInlineMax = 5;       // replicas held in a descriptor
constexpr int kSlotBits = 11;       // inline physical index < 2048
constexpr uint32_t kOther = 31u;    // selector field of a non-inline descriptor
constexpr int kMaxCopies = 16;
// lane copies of each histogram bin (a power of two <= 32): lane l counts
// into copy l mod 16, so a warp-wide atomic meets at most 2-way contention
// whatever the skew of the routing; measured as fast as 32 copies on the
// DeepSeek-V3 prefill batch and 2.6% faster on a 16x larger one, in half the
// shared memory (8 copies, or three CTAs per SM, measured slower)
constexpr int kHistCopies = 16;
constexpr int kStage = 8;           // period table: logcnt <= 8
// shared memory aimed at per CTA: two 512-thread CTAs per SM
constexpr size_t kSmemTarget = 112 * 1024;
constexpr int64_t kChunk = 48 * 1024;  // indices per CTA aimed at
constexpr int64_t kMaxWaves = 8;

struct RedirectArgs {
  const int32_t *idx;
  int64_t *counts;  // kCount only
  int32_t *out;
  int64_t per_layer;  // T * K  (< 2^31)
  int64_t chunks;     // CTAs per layer
  uint32_t K, k_magic;
  uint32_t t0;
  int32_t E, X;
  int32_t copies_log2;  // descriptor copies = 1 << copies_log2
  uint32_t M, m_magic;  // period of the replica table (0: descriptors only)
  uint64_t div_mask;    // bit c set iff c divides M (c < 64)
  const int32_t *log2phy;
  const int32_t *logcnt;
  unsigned long long *bad;
  int32_t *status;
};

__device__ __forceinline__ uint64_t other_desc(uint32_t c) {
  const uint32_t m = c ? 0xffffffffu / c : 0u;
  return kOther | (static_cast<uint64_t>(m) << 5) | (static_cast<uint64_t>(c) << 37);
}

// Descriptor of an expert with c replicas (0: maps to -1) whose first
// entries are p[0..kStage).
__device__ __forceinline__ uint64_t describe(int32_t c, const int32_t *p) {
  if (c <= 0) return other_desc(0);
  if (c > kInlineMax) return other_desc(static_cast<uint32_t>(c));
  uint64_t slots = 0;
  bool fits = true;
#pragma unroll
  for (int j = 0; j < kInlineMax; ++j) {
    if (j < c) {
      fits &= static_cast<uint32_t>(p[j]) < (1u << kSlotBits);
      slots |= static_cast<uint64_t>(static_cast<uint32_t>(p[j]) & ((1u << kSlotBits) - 1u))
               << (5 + kSlotBits * j);
    }
  }
  return fits ? (slots | static_cast<uint64_t>(6 * (c - 1))) : other_desc(static_cast<uint32_t>(c));
}

__host__ __device__ constexpr int gcd_c(int a, int b) { return b == 0 ? a : gcd_c(b, a % b); }

__device__ __forceinline__ uint32_t pack16(int32_t lo, int32_t hi) {
  return (static_cast<uint32_t>(lo) & 0xffffu) | (static_cast<uint32_t>(hi) << 16);
}

// Row of the period table for an expert with C replicas p[0..C): entry rho
// is p[rho mod C].  16-byte block b holds entries 8b .. 8b+7, so the blocks
// repeat with period C / gcd(C, 8); nblocks is a multiple of it (C | M).
template <int C>
__device__ __forceinline__ void fill_row_c(uint4 *row, const int32_t *p, int nblocks) {
  constexpr int PB = C / gcd_c(C, 8);
#pragma unroll
  for (int j = 0; j < PB; ++j) {  // one distinct block at a time: few registers
    uint4 blk;
    blk.x = pack16(p[(8 * j + 0) % C], p[(8 * j + 1) % C]);
    blk.y = pack16(p[(8 * j + 2) % C], p[(8 * j + 3) % C]);
    blk.z = pack16(p[(8 * j + 4) % C], p[(8 * j + 5) % C]);
    blk.w = pack16(p[(8 * j + 6) % C], p[(8 * j + 7) % C]);
#pragma unroll 1
    for (int b = j; b < nblocks; b += PB) row[b] = blk;
  }
}

// c = 0 writes a row of -1.
__device__ __forceinline__ void fill_row(uint4 *row, int c, const int32_t *p, int nblocks) {
  switch (c) {
    case 0: {
      const int32_t neg[1] = {-1};
      fill_row_c<1>(row, neg, nblocks);
      break;
    }
    case 1: fill_row_c<1>(row, p, nblocks); break;
    case 2: fill_row_c<2>(row, p, nblocks); break;
    case 3: fill_row_c<3>(row, p, nblocks); break;
    case 4: fill_row_c<4>(row, p, nblocks); break;
    case 5: fill_row_c<5>(row, p, nblocks); break;
    case 6: fill_row_c<6>(row, p, nblocks); break;
    case 7: fill_row_c<7>(row, p, nblocks); break;
    default: fill_row_c<8>(row, p, nblocks); break;
  }
}

// Selector word of global token u: field 6 (c - 1) = bit offset 5 + 11 r of
// replica r = u mod c, c = 1..5.
__device__ __forceinline__ uint32_t selector(uint32_t u) {
  const uint32_t r3 = mod_magic(u, 3u, 0xffffffffu / 3u);
  const uint32_t r5 = mod_magic(u, 5u, 0xffffffffu / 5u);
  constexpr uint32_t base = 5u * (1u | 1u << 6 | 1u << 12 | 1u << 18 | 1u << 24);
  return base + (u & 1u) * (11u << 6) + r3 * (11u << 12) + (u & 3u) * (11u << 18) +
         r5 * (11u << 24);
}

// Chunk `cta` of the grid (chunk j of layer l = cta / chunks): redirects its
// indices and, with kCount, adds its histogram to a.counts.  Called by every
// thread of a kThreads-thread CTA with the shared memory redirect_plan sized.
template <bool kVecToken, bool kCount>
__device__ __forceinline__ void redirect_chunk(const RedirectArgs &a, unsigned char *smem, int64_t cta) {
  const int E1 = a.E + 1;
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem);  // [E+1][32], kCount only
  unsigned char *region = smem + (kCount ? E1 * kHistCopies * sizeof(uint32_t) : 0);
  int16_t *tab = reinterpret_cast<int16_t *>(region);   // [E+1][M], fast path
  uint64_t *desc = reinterpret_cast<uint64_t *>(region);  // [E+1][copies], otherwise
  const int tid = threadIdx.x;
  const uint32_t lane = tid & 31;
  const int cl2 = a.copies_log2;
  const uint32_t cmask = (1u << cl2) - 1u;
  const uint32_t my_copy = lane & cmask;
  uint32_t *hist_lane = hist + (lane & (kHistCopies - 1));
  const uint32_t E = static_cast<uint32_t>(a.E);
  // the period of the table (the host's choice, or 24 for a layer whose
  // replica counts all divide it: see below)
  uint32_t M = a.M;
  uint32_t m_magic = a.m_magic;
  uint64_t div_mask = a.div_mask;

  // this CTA: part j of layer l.  The layer's 16-byte aligned interior
  // [b0, b1) is cut into slices of kThreads vectors and part j takes slices
  // j, j + chunks, j + 2 * chunks, ... (a thread's kU loads of a batch are
  // kU of them): the layer's CTAs sweep it side by side, so the DRAM pages
  // they read and write are few at a time (the same copy traffic with one
  // contiguous range per CTA measured 2 us slower behind the step's dirty
  // L2; blocks of 2 or 4 batches were slower than single slices).  Part 0
  // also takes the up to 3 elements before b0 and after b1.
  const int64_t layer = cta / a.chunks;
  const int64_t j = cta - layer * a.chunks;
  const int64_t lbase = layer * a.per_layer;
  const int64_t g = lbase, g1 = lbase + a.per_layer;
  const int64_t b0 = min((g + 3) & ~int64_t(3), g1);
  const int64_t b1 = max(g1 & ~int64_t(3), b0);
  const int4 *pin = reinterpret_cast<const int4 *>(a.idx) + (b0 >> 2);
  int4 *pout = reinterpret_cast<int4 *>(a.out) + (b0 >> 2);
  const int nvec = static_cast<int>((b1 - b0) >> 2);
  const uint32_t pos0 = static_cast<uint32_t>(b0 - lbase);
  const int sl = static_cast<int>(a.chunks) * kThreads;  // vectors between a part's slices
  const int step = sl * kU;                                // between its batches

  const int32_t *l2p_layer = a.log2phy + layer * static_cast<int64_t>(a.E) * a.X;
  const int32_t *cnt = a.logcnt + layer * a.E;
  bool range_err = false;
  uint32_t nbad = 0;

  // One round of loads per expert: its logcnt and first kStage entries,
  // issued before the first index vectors so they are not queued behind
  // them.  They give the expert's descriptor (kept in a register for the
  // first expert of this thread) and its row of the period table, written
  // at once.  The period table is used iff every valid logcnt is <= kStage
  // and divides M and all their entries fit int16: the CTA votes.  If the
  // vote fails the descriptors overwrite the rows.
  auto load_expert = [&](int e, int32_t *p) -> int32_t {
    if (e >= a.E) {
#pragma unroll
      for (int q = 0; q < kStage; ++q) p[q] = 0;
      return 0;  // 0: the row maps to -1 (sentinel row E, invalid logcnt)
    }
    const int32_t *row = l2p_layer + static_cast<int64_t>(e) * a.X;
#pragma unroll
    for (int q = 0; q < kStage; ++q) p[q] = q < a.X ? __ldg(row + q) : 0;
    return __ldg(cnt + e);
  };
  bool ok = M != 0;
  uint64_t d_first = 0;
  auto vote_expert = [&](int e, int32_t c, const int32_t *p) {
    if (e < a.E && (c < 1 || c > a.X)) {
      range_err = true;
      c = 0;
    }
    if (e == tid) d_first = describe(c, p);
    bool mine = c <= kStage && (c == 0 || ((div_mask >> c) & 1u));
#pragma unroll
    for (int q = 0; q < kStage; ++q)
      if (q < c && p[q] != static_cast<int16_t>(p[q])) mine = false;
    if (M && mine) fill_row(reinterpret_cast<uint4 *>(tab + e * M), c, p, M / 8);
    ok &= mine;
  };
  int32_t p0[kStage];
  int32_t c0 = tid < E1 ? load_expert(tid, p0) : 0;

  // first vectors in flight while the tables are built, and the batch after
  // them requested into L2 (a prefetch holds no register): twice the bytes
  // in flight while the plan loads are outstanding
  int i = static_cast<int>(j) * kThreads + tid;
  int4 x[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u)
    x[u] = i + u * sl < nvec ? __ldcs(pin + i + u * sl) : make_int4(0, 0, 0, 0);
#pragma unroll
  for (int u = 0; u < kU; ++u)
    if (i + step + u * sl < nvec) prefetch_l2(pin + i + step + u * sl);

  // a layer whose replica counts all divide 24 (1..4, 6, 8, 12, 24) gets the
  // 24-entry period: a fifth of the table to build before streaming
  // (measured: redirect 53.2 -> 51.4 us on the DeepSeek-V3 batch); one vote,
  // taken when every expert has its own thread
  if (M == 120u && E1 <= kThreads) {
    int32_t cc = c0;
    if (tid < a.E && (cc < 1 || cc > a.X)) cc = 0;
    const bool no24 = tid < E1 && cc > 0 && (24 % cc) != 0;
    if (!__syncthreads_or(no24)) {
      M = 24u;
      m_magic = 0xffffffffu / 24u;
      div_mask = (1ull << 1) | (1ull << 2) | (1ull << 3) | (1ull << 4) | (1ull << 6) |
                 (1ull << 8) | (1ull << 12) | (1ull << 24);
    }
  }
  if (tid < E1) vote_expert(tid, c0, p0);
  for (int e = tid + kThreads; e < E1; e += kThreads) {
    int32_t p[kStage];
    const int32_t c = load_expert(e, p);
    vote_expert(e, c, p);
  }
  if (kCount) {
    for (int q = tid; q < E1 * kHistCopies; q += kThreads) hist[q] = 0;
  }
  const bool fast = __syncthreads_and(ok);
  if (!fast) {
    for (int e = tid; e < E1; e += kThreads) {
      uint64_t d = d_first;
      if (e != tid) {  // more experts than threads: load this one again
        int32_t p[kStage];
        const int32_t *row = l2p_layer + static_cast<int64_t>(e) * a.X;
#pragma unroll
        for (int q = 0; q < kStage; ++q) p[q] = e < a.E && q < a.X ? __ldg(row + q) : 0;
        int32_t c = e < a.E ? __ldg(cnt + e) : 0;
        if (c < 1 || c > a.X) c = 0;
        d = describe(c, p);
      }
      // copies in rotated order: the lanes of a warp write distinct bank pairs
      for (int q = 0; q <= static_cast<int>(cmask); ++q)
        desc[(static_cast<uint32_t>(e) << cl2) + ((static_cast<uint32_t>(q + e)) & cmask)] = d;
    }
    __syncthreads();
  }

  // count (or tally as bad) element value e; returns its row, E if invalid
  auto clamp_count = [&](int32_t e) -> uint32_t {
    const uint32_t ee = min(static_cast<uint32_t>(e), E);
    if (kCount)
      atomicAdd(hist_lane + ee * static_cast<uint32_t>(kHistCopies), 1u);
    else
      nbad += ee == E ? 1u : 0u;
    return ee;
  };
  // fast path: ctx = shared address of tab[0][token mod M]
  const uint32_t hist_addr = smem_u32(hist) + 4u * (lane & (kHistCopies - 1));
  const uint32_t tab_addr = smem_u32(tab);
  const uint32_t row_bytes = 2u * M;
  auto map_fast = [&](int32_t e, uint32_t trow) -> int32_t {
    const uint32_t ee = min(static_cast<uint32_t>(e), E);
    if (kCount)
      red_shared_inc(hist_addr + ee * (4u * kHistCopies));
    else
      nbad += ee == E ? 1u : 0u;
    return ld_shared_s16(trow + ee * row_bytes);
  };
  // descriptor path: ctx = {selector(token), token}
  auto map_desc = [&](int32_t e, uint2 ctx) -> int32_t {
    const uint32_t ee = clamp_count(e);
    const uint64_t d = desc[(ee << cl2) + my_copy];
    const uint32_t f = static_cast<uint32_t>(d) & 31u;
    if (f != kOther) {
      const uint32_t sh = (ctx.x >> f) & 63u;
      return static_cast<int32_t>(static_cast<uint32_t>(d >> sh) & ((1u << kSlotBits) - 1u));
    }
    const uint32_t c = static_cast<uint32_t>(d >> 37) & 0xffffu;
    if (c == 0) return -1;
    const uint32_t r = mod_magic(ctx.y, c, static_cast<uint32_t>(d >> 5));
    if (!EPLB_IN(r < c && c <= static_cast<uint32_t>(a.X) && ee < E, a.status)) return -1;
    return __ldg(l2p_layer + ee * static_cast<uint32_t>(a.X) + r);
  };
  auto ctx_fast = [&](uint32_t tok) -> uint32_t {
    const uint32_t r = mod_magic(tok, M, m_magic);
    return tab_addr + 2u * (EPLB_IN(r < M, a.status) ? r : 0u);
  };
  auto ctx_desc = [&](uint32_t tok) -> uint2 { return make_uint2(selector(tok), tok); };

  auto stream = [&](auto ctx_of, auto map1) {
    if (j == 0 && tid < b0 - g) {
      const int64_t p = g + tid;
      const uint32_t tok = a.t0 + div_magic(static_cast<uint32_t>(p - lbase), a.K, a.k_magic);
      a.out[p] = map1(__ldg(a.idx + p), ctx_of(tok));
    }
    if (j == 0 && tid >= 32 && tid - 32 < g1 - b1) {
      const int64_t p = b1 + (tid - 32);
      const uint32_t tok = a.t0 + div_magic(static_cast<uint32_t>(p - lbase), a.K, a.k_magic);
      a.out[p] = map1(__ldg(a.idx + p), ctx_of(tok));
    }
    auto vector = [&](int v, const int4 &xv) {
      const uint32_t pos = pos0 + 4u * static_cast<uint32_t>(v);
      int4 y;
      if (kVecToken) {
        const auto ctx = ctx_of(a.t0 + div_magic(pos, a.K, a.k_magic));
        y.x = map1(xv.x, ctx);
        y.y = map1(xv.y, ctx);
        y.z = map1(xv.z, ctx);
        y.w = map1(xv.w, ctx);
      } else {
        y.x = map1(xv.x, ctx_of(a.t0 + div_magic(pos, a.K, a.k_magic)));
        y.y = map1(xv.y, ctx_of(a.t0 + div_magic(pos + 1, a.K, a.k_magic)));
        y.z = map1(xv.z, ctx_of(a.t0 + div_magic(pos + 2, a.K, a.k_magic)));
        y.w = map1(xv.w, ctx_of(a.t0 + div_magic(pos + 3, a.K, a.k_magic)));
      }
      pout[v] = y;
    };
    // whole batches without per-vector range checks, then the guarded rest
    // (a batch that is not whole is the thread's last: the next one starts
    // past its last slice)
    while (i + (kU - 1) * sl < nvec) {
#pragma unroll
      for (int u = 0; u < kU; ++u) vector(i + u * sl, x[u]);
      i += step;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        x[u] = i + u * sl < nvec ? __ldcs(pin + i + u * sl) : make_int4(0, 0, 0, 0);
      // one batch ahead into L2 (measured: -3 us on the 121.6 MB batch,
      // even on the 1.95 GB stream; two batches ahead was slower)
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (i + step + u * sl < nvec) prefetch_l2(pin + i + step + u * sl);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i + u * sl < nvec) vector(i + u * sl, x[u]);
  };
  if (fast)
    stream(ctx_fast, map_fast);
  else
    stream(ctx_desc, map_desc);

  if (kCount) {
    // two threads per bin, 16 lane copies each (rotated: conflict-free)
    __syncthreads();
    for (int t = tid; t - static_cast<int>(lane) < 2 * E1; t += kThreads) {  // warp-uniform
      const bool live = t < 2 * E1;
      const int b = t >> 1;
      const int h = (t & 1) * (kHistCopies / 2);
      uint32_t sum = 0;
      if (live) {
#pragma unroll 8
        for (int q = 0; q < kHistCopies / 2; ++q)
          sum += hist[b * kHistCopies + ((q + h + b) & (kHistCopies - 1))];
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      if (!live || (t & 1) || sum == 0) continue;
      if (b < a.E)
        atomicAdd(reinterpret_cast<unsigned long long *>(a.counts + layer * a.E + b),
                  static_cast<unsigned long long>(sum));
      else
        nbad += sum;
    }
  }

  if (range_err) report(a.status, EPLB_ERR_RANGE);
  for (int off = 16; off > 0; off >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, off);
  if (lane == 0 && nbad && a.bad) atomicAdd(a.bad, static_cast<unsigned long long>(nbad));
}


// Shared-memory plan of a redirect CTA: the period M of the table (0: none),
// descriptor copies, bytes.  count: with the S1 histogram.
struct RedirectSmem {
  uint32_t M;
  int copies_log2;
  uint64_t div_mask;
  size_t bytes;
};
inline eplb_status redirect_plan(int32_t E, bool count, const DeviceInfo &di, RedirectSmem *out) {
  const size_t E1 = static_cast<size_t>(E) + 1;
  const size_t hist = count ? E1 * kHistCopies * sizeof(uint32_t) : 0;
  // a histogram too large for two CTAs per SM leaves one: then use it all
  const size_t target = hist + E1 * 24 * sizeof(int16_t) > kSmemTarget
                            ? static_cast<size_t>(di.max_smem_optin)
                            : kSmemTarget;
  // the longest period whose table fits; each is a multiple of 8 (16-byte
  // blocks) and of the logcnts it serves: 840 all of 1..8, 120 1..6 and 8,
  // 24 1..4, 6 and 8
  static const uint32_t kPeriods[] = {840, 120, 24};
  uint32_t M = 0;
  for (uint32_t m : kPeriods) {
    if (hist + E1 * m * sizeof(int16_t) <= target) {
      M = m;
      break;
    }
  }
  // rows are written as 16-byte blocks: M must be a multiple of 8
  if (M % 8 != 0) M = 0;
  // as many descriptor copies (up to 16) as fit in the same space
  const size_t room = std::max(target > hist ? target - hist : 0, E1 * M * sizeof(int16_t));
  int cl2 = 4;
  while (cl2 > 0 && (E1 << cl2) * sizeof(uint64_t) > room) --cl2;
  const size_t region = std::max(E1 * M * sizeof(int16_t), (E1 << cl2) * sizeof(uint64_t));
  const size_t smem = (hist + region + 15) & ~size_t(15);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return EPLB_ERR_LIMIT;
  uint64_t div_mask = 0;
  for (uint32_t c = 1; M && c < 64; ++c)
    if (M % c == 0) div_mask |= uint64_t(1) << c;
  static_assert((1 << 4) == kMaxCopies, "copies");
  out->M = M;
  out->copies_log2 = cl2;
  out->div_mask = div_mask;
  out->bytes = smem;
  return EPLB_OK;
}

inline void redirect_fill(RedirectArgs &a, const RedirectSmem &sp, const int32_t *idx, int64_t T,
                          int32_t K, int32_t E, const int32_t *log2phy, int32_t X,
                          const int32_t *logcnt, int64_t t0, int32_t *out, int64_t *counts,
                          unsigned long long *bad, int32_t *status) {
  a.idx = idx;
  a.counts = counts;
  a.out = out;
  a.per_layer = T * K;
  a.K = static_cast<uint32_t>(K);
  a.k_magic = 0xffffffffu / static_cast<uint32_t>(K);
  a.t0 = static_cast<uint32_t>(t0);
  a.E = E;
  a.X = X;
  a.copies_log2 = sp.copies_log2;
  a.M = sp.M;
  a.m_magic = sp.M ? 0xffffffffu / sp.M : 0u;
  a.div_mask = sp.div_mask;
  a.log2phy = log2phy;
  a.logcnt = logcnt;
  a.bad = bad;
  a.status = status;
}

// One CTA per layer chunk: about kChunk indices each, at least one wave and
// at most kMaxWaves of CTAs, and L * chunks just under a whole number of
// waves, so the block scheduler hands the chunks of slow SMs to fast ones
// without leaving a thin last wave.
inline int64_t redirect_chunks(int64_t L, int64_t per_layer, int64_t slots) {
  const int64_t total = per_layer * L;
  const int64_t waves = std::min(std::max<int64_t>(total / (kChunk * slots), 1), kMaxWaves);
  const int64_t chunks = std::max<int64_t>(1, waves * slots / L);
  return std::max<int64_t>(1, std::min(chunks, (per_layer + 4095) / 4096));
}

}  // namespace
}  // namespace eplb
