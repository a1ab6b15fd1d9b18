// Block selection over score rows, one warp per row, and the mask step that
// feeds it through an L2-resident score slab.
//
// SLA post ("Selective Linear Attention", list "the idea"): a fast
// mean-pooling step labels the blocks in advance as critical, marginal or
// negligible.  NABLA post (SberAIScience, points 2-3): the blocks kept are
// the top-ranked ones whose summed softmax mass exceeds 1 - thr.
//
// Selection rules (the same as the row classifier in mask_kernels.cu):
// scores are P = softmax of the row's logits in fp32, ranked by value
// descending and block index ascending; top-k keeps ranks [0, n_c) critical
// and the next n_m marginal; the CDF rule drops, from the lowest rank up,
// every block whose tail sum (it and all lower-ranked blocks, in exact 2^-62
// fixed point) stays below thr, keeps the rest critical (always at least the
// top rank) and marks the next n_m ranks marginal.
//
// Per row, the scores' bit patterns (non-negative floats order like their
// patterns) sit in the warp's shared memory.  One pass builds a 256-bin
// histogram of counts (and, for the CDF rule, fixed-point masses) over equal
// ranges of patterns spanning the row's scores; a scan over the
// bins finds the bin holding each cut; the scores of that bin are compacted
// and the cut value is read off a bitonic warp sort of them (up to 64, two
// per lane), or resolved bit by bit among more; a last pass labels
// the row in index order (equal scores fill the remaining slots by index),
// writes the mask and the ascending block lists and counts near-ties.
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace sla {

namespace {

constexpr int kBins = 256;

struct SelectArgs {
  int nkb, n_c, n_m, from_prob, nrows, per_warp;  // per_warp: shared bytes per warp
  uint64_t thr_fx;
  int8_t* mask;
  sla_block_lists rows;
  float* scores;
  int32_t* tie_count;
};

// Bins: 256 equal ranges of bit patterns from the row's smallest score up,
// 2^shift patterns each, shift the least that covers the row's range.
__device__ __forceinline__ int bin_of(uint32_t v, uint32_t base, int shift) {
  return v >= base ? static_cast<int>(min((v - base) >> shift, 255u)) : 0;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Bin holding the score at rank need - 1 from the top (1 <= need <= row
// length): the bin b with above < need <= above + cnt[b], above = the scores
// in higher bins.  Lane l walks bins 255 - 8l - i.
__device__ __forceinline__ void bin_from_top(const uint32_t* hcnt, int need, int lane, int& bin,
                                             int& above) {
  uint32_t c[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) { c[i] = hcnt[255 - 8 * lane - i]; local += c[i]; }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - local;
  int b = -1, ab = 0;
  if (excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (b < 0 && static_cast<uint32_t>(need) <= acc + c[i]) { b = 255 - 8 * lane - i; ab = acc; }
      acc += c[i];
    }
  }
  const unsigned who = __ballot_sync(0xffffffffu, b >= 0);
  const int src = who ? __ffs(who) - 1 : 0;
  bin = __shfl_sync(0xffffffffu, b, src);
  above = __shfl_sync(0xffffffffu, ab, src);
}

// CDF cut bin: the lowest bin b whose mass together with every lower bin
// reaches thr (thr > 0); below = the mass of the bins under b, above = the
// scores in the bins over b.  found = false when the whole row's mass stays
// under thr.  Lane l walks bins 8l + i.
__device__ __forceinline__ void bin_from_bottom(const uint32_t* hcnt, const uint32_t* hmass,
                                                uint32_t thr, int lane, int& bin,
                                                unsigned long long& below, int& above, bool& found) {
  unsigned long long c[8], local = 0;
  uint32_t n[8], nloc = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hmass[8 * lane + i];
    local += c[i];
    n[i] = hcnt[8 * lane + i];
    nloc += n[i];
  }
  unsigned long long incl = local;
  uint32_t nincl = nloc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    const uint32_t z = __shfl_up_sync(0xffffffffu, nincl, o);
    if (lane >= o) { incl += y; nincl += z; }
  }
  const uint32_t ntot = __shfl_sync(0xffffffffu, nincl, 31);
  const unsigned long long excl = incl - local;
  uint32_t nacc = nincl - nloc;
  int b = -1, ab = 0;
  unsigned long long bl = 0;
  if (excl < thr && thr <= incl) {
    unsigned long long acc = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      nacc += n[i];
      if (b < 0 && thr <= acc + c[i]) {
        b = 8 * lane + i;
        bl = acc;
        ab = static_cast<int>(ntot - nacc);  // scores in bins above b
      }
      acc += c[i];
    }
  }
  const unsigned who = __ballot_sync(0xffffffffu, b >= 0);
  found = who != 0;
  const int src = found ? __ffs(who) - 1 : 0;
  bin = __shfl_sync(0xffffffffu, b, src);
  below = __shfl_sync(0xffffffffu, bl, src);
  above = __shfl_sync(0xffffffffu, ab, src);
}

// Largest pattern t with at least `need` candidates >= t (1 <= need <= n):
// the candidate at rank need - 1 from the top.
__device__ __forceinline__ uint32_t rank_among(const uint32_t* cand, int n, int need, int lane) {
  uint32_t t = 0;
  for (int bit = 30; bit >= 0; --bit) {  // patterns of non-negative floats < 2^31
    const uint32_t c = t | (1u << bit);
    uint32_t k = 0;
    for (int i = lane; i < n; i += 32) k += cand[i] >= c ? 1u : 0u;
    if (__reduce_add_sync(0xffffffffu, k) >= static_cast<uint32_t>(need)) t = c;
  }
  return t;
}

__device__ __forceinline__ int count_greater(const uint32_t* cand, int n, uint32_t v, int lane) {
  uint32_t k = 0;
  for (int i = lane; i < n; i += 32) k += cand[i] > v ? 1u : 0u;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, k));
}
__device__ __forceinline__ int count_equal(const uint32_t* cand, int n, uint32_t v, int lane) {
  uint32_t k = 0;
  for (int i = lane; i < n; i += 32) k += cand[i] == v ? 1u : 0u;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, k));
}

// A cut: every score above v, and the first `fill` scores equal to v in
// index order.  `gap` asks the last pass for the largest score under v
// (the near-tie test at a cut whose group of equal scores is used up).
struct Cut {
  bool on = false;
  uint32_t v = 0;
  int fill = 0;
  int eq = 0;  // scores equal to v in the row
  bool gap = false;
};

constexpr int kCand = 256;  // candidate slots per warp (both cuts)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warp-inclusive prefix sum (Hillis-Steele over shuffles).
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Bitonic sort of one key per lane across the warp, descending (the largest
// at lane 0): 15 compare-exchange steps over shuffles.  Blocks of k lanes
// alternate direction; the last stage (k = 32) runs descending over the
// whole warp.  Only keys move: a candidate's mass is a function of its key,
// recomputed after the sort.
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t x, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
      const bool take_max = ((lane & j) == 0) == ((lane & k) == 0);
      x = take_max ? max(x, y) : min(x, y);
    }
  }
  return x;
}

// The same over 64 keys, two per lane: key r of lane l is element 2l + r,
// so the sorted order runs lane 0 (x0 >= x1), lane 1, ...  An element's
// block direction (element & k) is lane & k/2; at distances of 2 and more
// lane l meets lane l ^ j/2 (each key with its namesake), at distance 1 a
// lane orders its own two keys: 15 exchange steps over shuffles, 6 in
// registers.
__device__ __forceinline__ void warp_sort64_desc(uint32_t& x0, uint32_t& x1, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
    const bool desc = (lane & (k >> 1)) == 0;
#pragma unroll
    for (int j = k >> 1; j >= 2; j >>= 1) {
      const int lj = j >> 1;
      const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, lj);
      const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, lj);
      const bool take_max = ((lane & lj) == 0) == desc;
      x0 = take_max ? max(x0, y0) : min(x0, y0);
      x1 = take_max ? max(x1, y1) : min(x1, y1);
    }
    const uint32_t hi = max(x0, x1), lo = min(x0, x1);
    x0 = desc ? hi : lo;
    x1 = desc ? lo : hi;
  }
}

// The candidate at rank need - 1 from the top among n <= 32 candidates held
// one per lane (`have`; 1 <= need <= n): its value, and how many candidates
// lie above it and equal it.  Lanes without a candidate sort as 0, below or
// level with every real one, which leaves the value at rank need - 1 as it is.
__device__ __forceinline__ void rank_small(uint32_t c, bool have, int need, int lane, uint32_t& v,
                                           int& above, int& eq) {
  const uint32_t key = warp_sort_desc(have ? c : 0u, lane);
  v = __shfl_sync(0xffffffffu, key, need - 1);
  above = __popc(__ballot_sync(0xffffffffu, have && c > v));
  eq = __popc(__ballot_sync(0xffffffffu, have && c == v));
}

// rank_small over 32 < n <= 64 candidates, two per lane (c0 always held, c1
// where h1): rank need - 1 is element need - 1 of the sorted order.
__device__ __forceinline__ void rank_pair(uint32_t c0, uint32_t c1, bool h1, int need, int lane,
                                          uint32_t& v, int& above, int& eq) {
  uint32_t k0 = c0, k1 = h1 ? c1 : 0u;
  warp_sort64_desc(k0, k1, lane);
  const int p = need - 1;
  const uint32_t s0 = __shfl_sync(0xffffffffu, k0, p >> 1);
  const uint32_t s1 = __shfl_sync(0xffffffffu, k1, p >> 1);
  v = (p & 1) ? s1 : s0;
  above = __popc(__ballot_sync(0xffffffffu, c0 > v)) + __popc(__ballot_sync(0xffffffffu, h1 && c1 > v));
  eq = __popc(__ballot_sync(0xffffffffu, c0 == v)) + __popc(__ballot_sync(0xffffffffu, h1 && c1 == v));
}

// CDF cut among n <= 32 candidates held one per lane: the candidate v at
// which lo + (mass of the candidates <= v) first reaches thr, the mass under
// it (`below`, lo included), and the candidates above and equal to it.
// Sorted descending, the suffix sums S_L of the masses (lane L and every
// lane after it) decrease with L; v is the key at the last lane with
// lo + S_L >= thr (a lane of v's group: the group's first lane holds the
// mass of everything <= v, the lane after the group only what is below v).
__device__ __forceinline__ void mass_small(uint32_t c, bool have, unsigned long long lo,
                                           uint64_t thr, int lane, uint32_t& v,
                                           unsigned long long& below, int& above, int& eq) {
  const unsigned long long fx = have ? to_fixed(c) : 0ull;
  const uint32_t key = warp_sort_desc(have ? c : 0u, lane);
  const unsigned long long m = to_fixed(key);  // (0 for the padding)
  unsigned long long suf = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned who = __ballot_sync(0xffffffffu, lo + suf >= thr && m > 0);
  const int src = who ? 31 - __clz(who) : 0;
  v = __shfl_sync(0xffffffffu, key, src);
  unsigned long long under = (have && c < v) ? fx : 0ull;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) under += __shfl_xor_sync(0xffffffffu, under, o);
  below = lo + under;
  above = __popc(__ballot_sync(0xffffffffu, have && c > v));
  eq = __popc(__ballot_sync(0xffffffffu, have && c == v));
}

// mass_small over 32 < n <= 64 candidates, two per lane (c0 always held, c1
// where h1).  In the sorted order lane l holds elements 2l and 2l + 1; with
// U_l the suffix sum of the lanes' pair masses, S(2l) = U_l and
// S(2l + 1) = U_l - m(2l), and v is the key at the last element whose
// lo + S reaches thr.
__device__ __forceinline__ void mass_pair(uint32_t c0, uint32_t c1, bool h1, unsigned long long lo,
                                          uint64_t thr, int lane, uint32_t& v,
                                          unsigned long long& below, int& above, int& eq) {
  uint32_t k0 = c0, k1 = h1 ? c1 : 0u;
  warp_sort64_desc(k0, k1, lane);
  const unsigned long long m0 = to_fixed(k0), m1 = to_fixed(k1);
  unsigned long long suf = m0 + m1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned w0 = __ballot_sync(0xffffffffu, lo + suf >= thr && m0 > 0);
  const unsigned w1 = __ballot_sync(0xffffffffu, lo + (suf - m0) >= thr && m1 > 0);
  const int l0 = w0 ? 31 - __clz(w0) : -1, l1 = w1 ? 31 - __clz(w1) : -1;
  const bool odd = l1 >= 0 && 2 * l1 + 1 > 2 * l0;
  const int src = odd ? l1 : max(l0, 0);
  const uint32_t s0 = __shfl_sync(0xffffffffu, k0, src);
  const uint32_t s1 = __shfl_sync(0xffffffffu, k1, src);
  v = odd ? s1 : s0;
  unsigned long long under = (c0 < v ? to_fixed(c0) : 0ull) + ((h1 && c1 < v) ? to_fixed(c1) : 0ull);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) under += __shfl_xor_sync(0xffffffffu, under, o);
  below = lo + under;
  above = __popc(__ballot_sync(0xffffffffu, c0 > v)) + __popc(__ballot_sync(0xffffffffu, h1 && c1 > v));
  eq = __popc(__ballot_sync(0xffffffffu, c0 == v)) + __popc(__ballot_sync(0xffffffffu, h1 && c1 == v));
}

// Shared memory of one warp (byte offsets; 16-byte aligned pieces).
struct WarpMem {
  size_t mass, pb, bins, hcnt, cand, ctr, total;
};
__host__ __device__ __forceinline__ WarpMem warp_mem(int nkb, bool cdf) {
  const size_t nkb4 = (static_cast<size_t>(nkb) + 3) & ~size_t(3);
  WarpMem w;
  size_t off = 0;
  w.mass = off; off += cdf ? 4 * kBins : 0;
  w.pb = off; off += 4 * nkb4;
  w.bins = off; off += (nkb4 + 15) & ~size_t(15);
  w.hcnt = off; off += 4 * kBins;
  w.cand = off; off += 4 * kCand;
  w.ctr = off; off += 16;
  w.total = off;
  return w;
}

// true if any byte of x equals b (b < 256)
__device__ __forceinline__ bool has_byte(uint32_t x, uint32_t b) {
  const uint32_t y = x ^ (b * 0x01010101u);
  return ((y - 0x01010101u) & ~y & 0x80808080u) != 0;
}

// MARG = false compiles the kernel without the marginal cut (for rules
// that keep no marginal blocks, n_m = 0: the usual NABLA use).
template <bool CDF, bool MARG>
__global__ void __launch_bounds__(256) select_rows_kernel(const float* __restrict__ in,
                                                          SelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * (blockDim.x / 32) + warp;
  if (row >= a.nrows) return;  // whole warps; nothing below syncs beyond the warp
  const unsigned full = 0xffffffffu;
  const int nkb = a.nkb;
  const int nkb4 = (nkb + 3) & ~3, G = nkb4 >> 2;  // groups of four scores
  const WarpMem wm = warp_mem(nkb, CDF);
  unsigned char* wbase = smem + static_cast<size_t>(warp) * wm.total;
  float* pf = reinterpret_cast<float*>(wbase + wm.pb);
  float4* pf4 = reinterpret_cast<float4*>(pf);
  uint4* pb4 = reinterpret_cast<uint4*>(pf);
  const uint32_t* pb = reinterpret_cast<const uint32_t*>(pf);
  uint32_t* bins = reinterpret_cast<uint32_t*>(wbase + wm.bins);  // one byte per score
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(wbase + wm.hcnt);
  uint32_t* hmass = reinterpret_cast<uint32_t*>(wbase + wm.mass);  // approximate masses
  uint32_t* cand = reinterpret_cast<uint32_t*>(wbase + wm.cand);
  uint32_t* ctr = reinterpret_cast<uint32_t*>(wbase + wm.ctr);
  const float* lr = in + i64(row) * nkb;
  const i64 off = i64(row) * nkb;

  // 1. the row into shared memory (16-byte loads when rows are 16-byte
  //    aligned, a batch per lane in flight: the reads come from L2 and
  //    their latency is what a warp waits for), and its max
  float m = -FLT_MAX, mn = FLT_MAX;
  if ((reinterpret_cast<uintptr_t>(lr) & 15u) == 0 && (nkb & 3) == 0) {
    const float4* lv = reinterpret_cast<const float4*>(lr);
    constexpr int kB = 16;
    for (int g0 = 0; g0 < G; g0 += 32 * kB) {
      float4 x[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int g = g0 + lane + 32 * u;
        x[u] = g < G ? __ldcg(lv + g) : make_float4(-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int g = g0 + lane + 32 * u;
        if (g < G) {
          pf4[g] = x[u];
          mn = fminf(mn, fminf(fminf(x[u].x, x[u].y), fminf(x[u].z, x[u].w)));
        }
        m = fmaxf(m, fmaxf(fmaxf(x[u].x, x[u].y), fmaxf(x[u].z, x[u].w)));
      }
    }
  } else {
    constexpr int kB = 16;
    for (int j0 = 0; j0 < nkb4; j0 += 32 * kB) {
      float x[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + lane + 32 * u;
        x[u] = j < nkb ? __ldcg(lr + j) : -FLT_MAX;
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + lane + 32 * u;
        if (j < nkb4) pf[j] = x[u];  // (the padding of the last group: -FLT_MAX)
        if (j < nkb) mn = fminf(mn, x[u]);
        m = fmaxf(m, x[u]);
      }
    }
  }
  for (int b = lane; b < kBins; b += 32) {
    hcnt[b] = 0u;
    if (CDF) hmass[b] = 0u;
  }
  if (lane < 4) ctr[lane] = 0u;
  m = warp_max(m);
  __syncwarp();

  // 2. P = softmax of the row: e = 2^((x - m) log2 e), P = e / sum e;
  //    row-given scores are taken as they are (negative ones as 0).  The
  //    largest P is (largest e) / sum, the same product the scores get.
  float inv = 1.f;
  uint32_t pmax, pmin;
  if (!a.from_prob) {
    constexpr float kLog2e = 1.4426950408889634f;
    const float ml = m * kLog2e;
    float se = 0.f, emax = 0.f, emin = FLT_MAX;
#pragma unroll 2
    for (int g = lane; g < G; g += 32) {
      const float4 x = pf4[g];
      float4 e;
      e.x = ex2(fmaf(x.x, kLog2e, -ml));
      e.y = ex2(fmaf(x.y, kLog2e, -ml));
      e.z = ex2(fmaf(x.z, kLog2e, -ml));
      e.w = ex2(fmaf(x.w, kLog2e, -ml));
      float4 f = e;  // (for the minimum, the padding counts as +inf)
      if (4 * g + 3 >= nkb) {  // the padding of the last group
        if (4 * g + 1 >= nkb) { e.y = 0.f; f.y = FLT_MAX; }
        if (4 * g + 2 >= nkb) { e.z = 0.f; f.z = FLT_MAX; }
        e.w = 0.f;
        f.w = FLT_MAX;
      }
      se += (e.x + e.y) + (e.z + e.w);
      emax = fmaxf(emax, fmaxf(fmaxf(e.x, e.y), fmaxf(e.z, e.w)));
      emin = fminf(emin, fminf(fminf(f.x, f.y), fminf(f.z, f.w)));
      pf4[g] = e;
    }
    se = warp_sum(se);
    inv = 1.0f / se;
    pmax = __float_as_uint(warp_max(emax) * inv);
    pmin = __float_as_uint(-warp_max(-emin) * inv);
  } else {
    pmax = __float_as_uint(fmaxf(m, 0.f));
    pmin = __float_as_uint(fmaxf(-warp_max(-mn), 0.f));
  }
  // (the same products give the scores, so every score lies in [pmin, pmax])
  const uint32_t base = pmin <= pmax ? pmin : pmax;
  const uint32_t range = pmax - base;
  const int shift = range > 255u ? 24 - __clz(range) : 0;  // range >> shift < 256
  __syncwarp();

  // 3. score patterns, their bins, and the histogram of counts (and
  //    fixed-point masses)
#pragma unroll 2
  for (int g = lane; g < G; g += 32) {
    const float4 e = pf4[g];
    const float ev[4] = {e.x, e.y, e.z, e.w};
    uint32_t v[4], bb = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float p = a.from_prob ? fmaxf(ev[k], 0.f) : ev[k] * inv;
      v[k] = __float_as_uint(p);
      const int b = bin_of(v[k], base, shift);
      bb |= static_cast<uint32_t>(b) << (8 * k);
      const int j = 4 * g + k;
      if (j < nkb) {
        atomicAdd(&hcnt[b], 1u);
        if (CDF) atomicAdd(&hmass[b], __float2uint_rz(p * 16777216.f));  // 2^-24 units
        if (a.scores) a.scores[off + j] = p;
      }
    }
    pb4[g] = make_uint4(v[0], v[1], v[2], v[3]);
    bins[g] = bb;
  }
  __syncwarp();

  // candidates of up to two bins: bin c0 from the front of the buffer, bin
  // c1 from the back; returns false if they do not fit
  auto gather = [&](int c0, int c1) -> bool {
    for (int g = lane; g < G; g += 32) {
      const uint32_t bb = bins[g];
      const bool m0 = c0 >= 0 && has_byte(bb, static_cast<uint32_t>(c0));
      const bool m1 = c1 >= 0 && has_byte(bb, static_cast<uint32_t>(c1));
      if (!(m0 || m1)) continue;
      const uint4 v4 = pb4[g];
      const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (4 * g + k >= nkb) continue;
        const int b = static_cast<int>((bb >> (8 * k)) & 255u);
        if (b == c0) {
          const uint32_t s = atomicAdd(&ctr[0], 1u);
          if (s < kCand) cand[s] = v[k];
        } else if (b == c1) {
          const uint32_t s = atomicAdd(&ctr[1], 1u);
          if (s < kCand) cand[kCand - 1 - s] = v[k];
        }
      }
    }
    __syncwarp();
    return ctr[0] + ctr[1] <= static_cast<uint32_t>(kCand);
  };
  // the exact cut value when the candidates do not fit: bit by bit over the
  // whole row, restricted to bin b
  auto rank_in_bin = [&](int b, int need, uint32_t& v, int& above, int& eq) {
    uint32_t t = 0;
    for (int bit = 30; bit >= 0; --bit) {
      const uint32_t c = t | (1u << bit);
      uint32_t k = 0;
      for (int j = lane; j < nkb; j += 32) {
        const uint32_t x = pb[j];
        k += (bin_of(x, base, shift) == b && x >= c) ? 1u : 0u;
      }
      if (__reduce_add_sync(full, k) >= static_cast<uint32_t>(need)) t = c;
    }
    uint32_t gt = 0, sm = 0;
    for (int j = lane; j < nkb; j += 32) {
      const uint32_t x = pb[j];
      if (bin_of(x, base, shift) == b) { gt += x > t ? 1u : 0u; sm += x == t ? 1u : 0u; }
    }
    v = t;
    above = static_cast<int>(__reduce_add_sync(full, gt));
    eq = static_cast<int>(__reduce_add_sync(full, sm));
  };
  // cut at rank need - 1 of the n candidates at cl (or of bin b when they
  // did not fit): value, candidates above, candidates equal
  auto rank_cands = [&](const uint32_t* cl, int n, bool fit, int b, int need, uint32_t& v,
                        int& above, int& eq) {
    if (!fit) {
      rank_in_bin(b, need, v, above, eq);
    } else if (n <= 32) {
      rank_small(lane < n ? cl[lane] : 0u, lane < n, need, lane, v, above, eq);
    } else if (n <= 64) {
      rank_pair(cl[lane], lane + 32 < n ? cl[lane + 32] : 0u, lane + 32 < n, need, lane, v, above, eq);
    } else {
      v = rank_among(cl, n, need, lane);
      above = count_greater(cl, n, v, lane);
      eq = count_equal(cl, n, v, lane);
    }
  };

  // 4. the critical cut (c blocks) and the marginal one (c + nm kept)
  const bool ties_on = a.tie_count != nullptr;
  bool tie = false;
  Cut cc, cm;
  int c = 0;
  if (!CDF) {
    c = a.n_c;
    const int nm = MARG ? min(a.n_m, nkb - c) : 0;
    int bc = -1, ab_c = 0, bm = -1, ab_m = 0;
    if (c > 0) bin_from_top(hcnt, c, lane, bc, ab_c);
    if (nm > 0) bin_from_top(hcnt, c + nm, lane, bm, ab_m);
    const bool shared_bin = c > 0 && nm > 0 && bm == bc;
    const bool fit = gather(bc, shared_bin ? -1 : bm);
    const int n0 = static_cast<int>(min(ctr[0], static_cast<uint32_t>(kCand)));
    const int n1 = static_cast<int>(min(ctr[1], static_cast<uint32_t>(kCand)));
    if (c > 0) {
      uint32_t v;
      int above, eq;
      rank_cands(cand, n0, fit, bc, c - ab_c, v, above, eq);
      above += ab_c;
      cc.on = true;
      cc.v = v;
      cc.fill = c - above;
      cc.eq = eq;
      if (ties_on && c < nkb) {  // gap between ranks c - 1 and c
        if (above + eq > c) tie = true;  // rank c scores v too
        else cc.gap = true;
      }
    }
    if (nm > 0) {
      const uint32_t* cl = shared_bin ? cand : cand + kCand - n1;
      const int nn = shared_bin ? n0 : n1;
      uint32_t v;
      int above, eq;
      rank_cands(cl, nn, fit, bm, c + nm - ab_m, v, above, eq);
      above += ab_m;
      cm.on = true;
      cm.v = v;
      cm.fill = c + nm - above;
      cm.eq = eq;
      if (ties_on && c + nm < nkb) {
        if (above + eq > c + nm) tie = true;
        else cm.gap = true;
      }
    }
  } else {
    if (a.thr_fx == 0) {  // nothing can be dropped
      cc.on = true;
      cc.v = 0u;
      cc.fill = nkb;
      cc.eq = nkb;  // (every score is taken)
      c = nkb;
    } else {
      int b = 0, ab = 0;
      unsigned long long lo = 0;
      bool found = false;
      // the bin on the approximate masses, then confirmed (or moved to a
      // neighbouring non-empty bin) on exact fixed-point sums: the mass under
      // bin b stays below thr and reaching thr takes bin b
      bin_from_bottom(hcnt, hmass, static_cast<uint32_t>(a.thr_fx >> 38), lane, b, lo, ab, found);
      if (!found) b = 255;
      found = false;
      // (the first pass also collects bin b's scores as the cut's candidates,
      // the gather of step 4; the pass is usually the only one)
      int gathered = -1;
      for (int it = 0; it <= kBins; ++it) {
        unsigned long long s_lo = 0, s_b = 0;
        const bool take = it == 0;
        for (int g = lane; g < G; g += 32) {
          const uint32_t bb = bins[g];
          const uint4 v4 = pb4[g];
          const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (4 * g + k >= nkb) continue;
            const int bx = static_cast<int>((bb >> (8 * k)) & 255u);
            if (bx < b) {
              s_lo += to_fixed(v[k]);
            } else if (bx == b) {
              s_b += to_fixed(v[k]);
              if (take) {
                const uint32_t sl = atomicAdd(&ctr[0], 1u);
                if (sl < kCand) cand[sl] = v[k];
              }
            }
          }
        }
        if (take) {
          __syncwarp();
          gathered = b;
        }
        s_lo = warp_sum_u64(s_lo);
        s_b = warp_sum_u64(s_b);
        if (s_lo >= a.thr_fx) {  // thr is reached below b
          int nb = b - 1;
          while (nb > 0 && hcnt[nb] == 0) --nb;
          b = nb;
          continue;
        }
        if (s_lo + s_b < a.thr_fx) {  // thr is not reached within b
          int nb = b + 1;
          while (nb < kBins && hcnt[nb] == 0) ++nb;
          if (nb >= kBins) break;  // the row's whole mass stays under thr
          b = nb;
          continue;
        }
        lo = s_lo;
        found = true;
        break;
      }
      if (found) {
        uint32_t nab = 0;
        for (int i = lane; i < kBins; i += 32) nab += i > b ? hcnt[i] : 0u;
        ab = static_cast<int>(__reduce_add_sync(full, nab));
        bool fit = ctr[0] <= static_cast<uint32_t>(kCand);
        if (gathered != b) {  // the cut moved to another bin: collect that one's
          __syncwarp();
          if (lane < 2) ctr[lane] = 0u;
          __syncwarp();
          fit = gather(b, -1);
        }
        const int n = static_cast<int>(min(ctr[0], static_cast<uint32_t>(kCand)));
        uint32_t v;
        unsigned long long below;
        int above, g;
        if (fit && n <= 32) {
          mass_small(lane < n ? cand[lane] : 0u, lane < n, lo, a.thr_fx, lane, v, below, above, g);
        } else if (fit && n <= 64) {
          mass_pair(cand[lane], lane + 32 < n ? cand[lane + 32] : 0u, lane + 32 < n, lo, a.thr_fx, lane,
                    v, below, above, g);
        } else {
          // bit by bit: the largest t whose mass below it stays under thr
          uint32_t t = 0;
          for (int bit = 30; bit >= 0; --bit) {
            const uint32_t cnd = t | (1u << bit);
            unsigned long long s = 0;
            if (fit) {
              for (int i = lane; i < n; i += 32)
                if (cand[i] < cnd) s += to_fixed(cand[i]);
            } else {
              for (int j = lane; j < nkb; j += 32) {
                const uint32_t x = pb[j];
                if (bin_of(x, base, shift) == b && x < cnd) s += to_fixed(x);
              }
            }
            if (lo + warp_sum_u64(s) < a.thr_fx) t = cnd;
          }
          v = t;
          unsigned long long s = 0;
          uint32_t gt = 0, sm = 0;
          if (fit) {
            for (int i = lane; i < n; i += 32) {
              const uint32_t x = cand[i];
              if (x < v) s += to_fixed(x);
              gt += x > v ? 1u : 0u;
              sm += x == v ? 1u : 0u;
            }
          } else {
            for (int j = lane; j < nkb; j += 32) {
              const uint32_t x = pb[j];
              if (bin_of(x, base, shift) != b) continue;
              if (x < v) s += to_fixed(x);
              gt += x > v ? 1u : 0u;
              sm += x == v ? 1u : 0u;
            }
          }
          below = lo + warp_sum_u64(s);
          above = static_cast<int>(__reduce_add_sync(full, gt));
          g = static_cast<int>(__reduce_add_sync(full, sm));
        }
        above += ab;
        // of the g blocks scoring v, the r lowest-ranked (highest-index)
        // are still below thr when taken alone; the other g - r + 1 are kept
        const uint64_t fx = to_fixed(v);
        const uint64_t r = fx ? (a.thr_fx - below + fx - 1) / fx : 1;
        cc.on = true;
        cc.v = v;
        cc.fill = g - static_cast<int>(r) + 1;
        cc.eq = g;
        c = above + cc.fill;
        if (ties_on) {
          const double thr = static_cast<double>(a.thr_fx) / kFixedOne;
          const uint64_t rk = static_cast<uint64_t>(g - cc.fill + 1);  // kept block's tail count
          const double t_last = static_cast<double>(below + rk * fx) / kFixedOne;
          const double t_next = static_cast<double>(below + (rk - 1) * fx) / kFixedOne;
          if (c > 1) tie |= fabs(t_last - thr) <= kTieEps;
          if (c < nkb) {
            tie |= fabs(thr - t_next) <= kTieEps;
            if (rk >= 2) tie = true;  // the next rank scores v too
            else cc.gap = true;
          }
        }
      } else {
        // the row's whole mass stays under thr: only the top rank is kept
        cc.on = true;
        cc.v = pmax;
        cc.fill = 1;
        uint32_t k = 0;
        unsigned long long s_all = 0;
        for (int j = lane; j < nkb; j += 32) {
          k += pb[j] == pmax ? 1u : 0u;
          s_all += to_fixed(pb[j]);
        }
        cc.eq = static_cast<int>(__reduce_add_sync(full, k));
        s_all = warp_sum_u64(s_all);
        c = 1;
        if (ties_on && nkb > 1) {
          // the decisions at the cut: the tail sum of rank 1 against thr,
          // and rank 1 against the top score (equal, or a relative gap)
          const double thr = static_cast<double>(a.thr_fx) / kFixedOne;
          const double t_next = static_cast<double>(s_all - to_fixed(pmax)) / kFixedOne;
          tie |= fabs(thr - t_next) <= kTieEps;
          if (cc.eq >= 2) tie = true;
          else cc.gap = true;
        }
      }
    }
    const int nm = MARG ? min(a.n_m, nkb - c) : 0;
    if (nm > 0) {
      int bm = 0, ab_m = 0;
      bin_from_top(hcnt, c + nm, lane, bm, ab_m);
      __syncwarp();
      if (lane < 2) ctr[lane] = 0u;
      __syncwarp();
      const bool fit = gather(bm, -1);
      const int n = static_cast<int>(min(ctr[0], static_cast<uint32_t>(kCand)));
      uint32_t v;
      int above, eq;
      rank_cands(cand, n, fit, bm, c + nm - ab_m, v, above, eq);
      above += ab_m;
      cm.on = true;
      cm.v = v;
      cm.fill = c + nm - above;
      cm.eq = eq;
      if (ties_on && c + nm < nkb) {
        if (above + eq > c + nm) tie = true;
        else cm.gap = true;
      }
    }
  }

  // 5. labels in index order (lane l holds scores 4g..4g+3, g = l + 32i):
  //    ranks among equal scores and list positions from packed warp scans;
  //    the mask row, the ascending lists, and the largest scores under the
  //    cut values for the remaining gap tests
  int nc = 0, nmg = 0, eqc = 0, eqm = 0;
  uint32_t mb_c = 0, mb_m = 0;
  const bool mask4 = (reinterpret_cast<uintptr_t>(a.mask + off) & 3u) == 0;
  // Usually every score equal to a cut value is taken (no group of equal
  // scores straddles a cut): labels are then plain comparisons.
  const bool plain = (!cc.on || cc.fill >= cc.eq) && (!cm.on || cm.fill >= cm.eq);
  const bool want_mb = cc.gap || cm.gap;
  // labels of the group g (four scores) as plain comparisons
  auto plain_group = [&](int g, bool is_c[4], bool is_m[4], uint32_t& ncl, uint32_t& nml,
                         uint32_t& lab) {
    uint32_t v[4] = {0u, 0u, 0u, 0u};
    if (g < G) {
      const uint4 v4 = pb4[g];
      v[0] = v4.x; v[1] = v4.y; v[2] = v4.z; v[3] = v4.w;
    }
    ncl = nml = lab = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool valid = g < G && 4 * g + k < nkb;
      is_c[k] = valid && cc.on && v[k] >= cc.v;
      is_m[k] = valid && !is_c[k] && cm.on && v[k] >= cm.v;
      ncl += is_c[k] ? 1u : 0u;
      nml += is_m[k] ? 1u : 0u;
      lab |= static_cast<uint32_t>(is_c[k] ? 2 : (is_m[k] ? 1 : 0)) << (8 * k);
      if (want_mb && valid) {
        if (v[k] < cc.v && v[k] > mb_c) mb_c = v[k];
        if (v[k] < cm.v && v[k] > mb_m) mb_m = v[k];
      }
    }
  };
  auto plain_write = [&](int g, const bool is_c[4], const bool is_m[4], uint32_t lab, int pc,
                         int pm) {
    if (g >= G) return;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (is_c[k]) a.rows.crit_idx[off + pc++] = 4 * g + k;
      if (is_m[k]) a.rows.marg_idx[off + pm++] = 4 * g + k;
    }
    if (mask4 && 4 * g + 3 < nkb) {
      *reinterpret_cast<uint32_t*>(a.mask + off + 4 * g) = lab;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (4 * g + k < nkb) a.mask[off + 4 * g + k] = static_cast<int8_t>((lab >> (8 * k)) & 255u);
    }
  };
  // two groups per lane and step, list positions from one scan of four
  // packed 8-bit counts (at most 4 x 32 = 128 each)
  for (int g0 = 0; plain && g0 < G; g0 += 64) {
    const int ga = g0 + lane, gb = g0 + 32 + lane;
    bool ca[4], ma[4], cb[4], mbk[4];
    uint32_t nca, nma, laba, ncb, nmb, labb;
    plain_group(ga, ca, ma, nca, nma, laba);
    plain_group(gb, cb, mbk, ncb, nmb, labb);
    const uint32_t pk = nca | (nma << 8) | (ncb << 16) | (nmb << 24);
    const uint32_t inc = warp_incl_scan(pk, lane);
    const uint32_t ex = inc - pk;
    const uint32_t tot = __shfl_sync(full, inc, 31);
    const int ta_c = static_cast<int>(tot & 255u), ta_m = static_cast<int>((tot >> 8) & 255u);
    plain_write(ga, ca, ma, laba, nc + static_cast<int>(ex & 255u), nmg + static_cast<int>((ex >> 8) & 255u));
    plain_write(gb, cb, mbk, labb, nc + ta_c + static_cast<int>((ex >> 16) & 255u),
                nmg + ta_m + static_cast<int>(ex >> 24));
    nc += ta_c + static_cast<int>((tot >> 16) & 255u);
    nmg += ta_m + static_cast<int>(tot >> 24);
  }
  for (int g0 = 0; !plain && g0 < G; g0 += 32) {
    const int g = g0 + lane;
    uint32_t v[4] = {0u, 0u, 0u, 0u};
    if (g < G) {
      const uint4 v4 = pb4[g];
      v[0] = v4.x; v[1] = v4.y; v[2] = v4.z; v[3] = v4.w;
    }
    bool valid[4], ec[4], em[4];
    uint32_t nec = 0, nem = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      valid[k] = g < G && 4 * g + k < nkb;
      ec[k] = valid[k] && cc.on && v[k] == cc.v;
      em[k] = valid[k] && cm.on && v[k] == cm.v;
      nec += ec[k] ? 1u : 0u;
      nem += em[k] ? 1u : 0u;
      if (valid[k]) {
        if (v[k] < cc.v && v[k] > mb_c) mb_c = v[k];
        if (v[k] < cm.v && v[k] > mb_m) mb_m = v[k];
      }
    }
    const uint32_t pe = nec | (nem << 16);
    const uint32_t ie = warp_incl_scan(pe, lane);
    const uint32_t te = __shfl_sync(full, ie, 31);
    int rc = eqc + static_cast<int>((ie - pe) & 0xFFFFu);
    int rm = eqm + static_cast<int>((ie - pe) >> 16);
    eqc += static_cast<int>(te & 0xFFFFu);
    eqm += static_cast<int>(te >> 16);
    bool is_c[4], is_m[4];
    uint32_t ncl = 0, nml = 0, lab = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      is_c[k] = valid[k] && cc.on && (v[k] > cc.v || (ec[k] && rc < cc.fill));
      const bool kept = valid[k] && cm.on && (v[k] > cm.v || (em[k] && rm < cm.fill));
      is_m[k] = !is_c[k] && kept;
      rc += ec[k] ? 1 : 0;
      rm += em[k] ? 1 : 0;
      ncl += is_c[k] ? 1u : 0u;
      nml += is_m[k] ? 1u : 0u;
      lab |= static_cast<uint32_t>(is_c[k] ? 2 : (is_m[k] ? 1 : 0)) << (8 * k);
    }
    const uint32_t pl = ncl | (nml << 16);
    const uint32_t il = warp_incl_scan(pl, lane);
    const uint32_t tl = __shfl_sync(full, il, 31);
    int pc = nc + static_cast<int>((il - pl) & 0xFFFFu);
    int pm = nmg + static_cast<int>((il - pl) >> 16);
    nc += static_cast<int>(tl & 0xFFFFu);
    nmg += static_cast<int>(tl >> 16);
    if (g < G) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = 4 * g + k;
        if (is_c[k]) a.rows.crit_idx[off + pc++] = j;
        if (is_m[k]) a.rows.marg_idx[off + pm++] = j;
      }
      if (mask4 && 4 * g + 3 < nkb) {
        *reinterpret_cast<uint32_t*>(a.mask + off + 4 * g) = lab;
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (valid[k]) a.mask[off + 4 * g + k] = static_cast<int8_t>((lab >> (8 * k)) & 255u);
      }
    }
  }
  if (cc.gap) {
    const float hi = __uint_as_float(cc.v), lo = __uint_as_float(__reduce_max_sync(full, mb_c));
    tie |= (hi - lo) <= kTieEps * hi;
  }
  if (cm.gap) {
    const float hi = __uint_as_float(cm.v), lo = __uint_as_float(__reduce_max_sync(full, mb_m));
    tie |= (hi - lo) <= kTieEps * hi;
  }
  if (lane == 0) {
    a.rows.crit_cnt[row] = nc;
    a.rows.marg_cnt[row] = nmg;
    if (ties_on && tie) atomicAdd(a.tie_count, 1);
  }
}

size_t select_per_warp_bytes(int nkb, bool cdf) { return warp_mem(nkb, cdf).total; }

}  // namespace

// Classify `nrows` rows of `in` (logits, or row-softmaxed scores when
// from_prob) with the rules of p; mask, lists and scores are addressed from
// row 0 of this launch.  The near-tie counter is added to, not cleared.
cudaError_t launch_select_rows(const float* in, int nrows, const Geom& g, int8_t* mask,
                               const sla_block_lists& rows, float* scores, int32_t* tie_count,
                               bool from_prob, cudaStream_t s) {
  if (nrows <= 0) return cudaSuccess;
  const bool cdf = g.mode == SLA_MASK_CDF;
  SelectArgs a;
  a.nkb = g.nkb;
  a.n_c = g.n_c;
  a.n_m = g.n_m;
  a.from_prob = from_prob ? 1 : 0;
  a.nrows = nrows;
  a.thr_fx = g.thr_fx;
  a.mask = mask;
  a.rows = rows;
  a.scores = scores;
  a.tie_count = tie_count;
  const size_t per = select_per_warp_bytes(g.nkb, cdf);
  a.per_warp = static_cast<int>(per);
  // Short rows (a warp's share at most 8 KB): CTAs of 2 warps, which the
  // registers, not shared memory, then limit to ~20 resident warps per SM
  // (measured faster than 1, 3, 6 or 8 at rows of 512 blocks).  Longer rows:
  // up to 8 warps (rows) per CTA, at most ~56 KB of shared memory each, so
  // that several CTAs share an SM (measured best at rows of 1182 and 1920).
  const int warps = per <= 8192 ? 2
                                : static_cast<int>(std::max<size_t>(1, std::min<size_t>(8, (56 * 1024) / per)));
  const size_t smem = per * warps;
  const int grid = (nrows + warps - 1) / warps;
  auto launch = [&](auto kern) -> cudaError_t {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, 32 * warps, smem, s>>>(in, a);
    return cudaSuccess;
  };
  cudaError_t e;
  if (cdf) e = g.n_m > 0 ? launch(select_rows_kernel<true, true>) : launch(select_rows_kernel<true, false>);
  else e = launch(select_rows_kernel<false, true>);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sla
