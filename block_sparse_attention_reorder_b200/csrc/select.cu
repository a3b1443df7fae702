// Key-tile selection on a block-score matrix: exact top-k, top-p with a
// top-k floor, and the broadcast of the fixed window lists.
//
// Ordering: tiles run by score descending, equal scores (-0.0 and +0.0 are
// equal) by tile index ascending. A 64-bit composite key (an order-preserving
// integer image of the score << 32 | ~index) is unique per tile and orders
// tiles that way. Both rules come down to one search: walking the row in that
// order with a non-negative weight per tile (1 for a count, the softmax mass
// for top-p), find the first tile at which the running weight reaches a target
// R. Every tile up to and including it is kept; lists are written ascending.
//
// One warp per row; the row is staged in the warp's slice of shared memory
// (lane l's i-th value is tile l + 32 i). The search never sorts the row: the
// scores of the current range are binned into 256 equal-width bins with one
// FMA (monotone in the score, so bins keep the order), a per-warp weight
// histogram locates the bin where the running weight reaches R, and that bin
// becomes the next range. A bin of at most 32 tiles is ranked exactly across
// the warp's lanes; a range of one score value (a run of tied tiles) is
// resolved by index order. A bounded number of levels, then a bit-by-bit
// search over the composite keys, covers whatever is left (infinite scores,
// ranges too narrow to split).
//
// Top-p mass: e_j = exp(s_j - max_j s) in fp64, held as an integer in units of
// 2^-52 (so e_max = 2^52). Integer sums are exact in any order, so the result
// does not depend on atomics or reduction order. With at most 2048 tiles the
// rounding moves a normalised prefix mass by at most 2048 * 2^-53 < 2.3e-13.
#include "internal.h"

namespace {

constexpr int kBins = 256;
constexpr int kCand = 32;   // bin size ranked directly
constexpr int kLevels = 4;  // histogram refinements before the bitwise search

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;  // -0.0 ties with +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ uint64_t comp_key(float x, int j) {
  return ((uint64_t)order_key(x) << 32) | (uint64_t)(0xffffffffu - (uint32_t)j);
}

__device__ __forceinline__ uint64_t shfl_idx_u64(uint64_t v, int src) {
  return ((uint64_t)__shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src) << 32) |
         __shfl_sync(0xffffffffu, (uint32_t)v, src);
}
__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int o) {
  return ((uint64_t)__shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), o) << 32) |
         __shfl_xor_sync(0xffffffffu, (uint32_t)v, o);
}
__device__ __forceinline__ uint64_t shfl_up_u64(uint64_t v, int o) {
  return ((uint64_t)__shfl_up_sync(0xffffffffu, (uint32_t)(v >> 32), o) << 32) |
         __shfl_up_sync(0xffffffffu, (uint32_t)v, o);
}
__device__ __forceinline__ uint64_t shfl_down_u64(uint64_t v, int o) {
  return ((uint64_t)__shfl_down_sync(0xffffffffu, (uint32_t)(v >> 32), o) << 32) |
         __shfl_down_sync(0xffffffffu, (uint32_t)v, o);
}
__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += shfl_xor_u64(v, o);
  return v;
}

// Softmax mass of score x relative to the row max, in units of 2^-52.
__device__ __forceinline__ uint64_t mass_q(float x, double smax) {
  return __double2ull_rn(exp((double)x - smax) * 4503599627370496.0);
}

// Tile weight: 1 for a count, the fixed-point mass otherwise.
template <bool MASS>
__device__ __forceinline__ uint64_t weight_of(float x, double smax) {
  if constexpr (MASS)
    return mass_q(x, smax);
  else
    return 1ull;
}

// Equal-width binning of the range [lo, hi] (lo < hi) without a float-to-int
// conversion: one FMA computes x * sc - lo * sc + 1.5 * 2^23, whose rounding
// to float leaves the bin as an integer in the low mantissa bits once the
// value is clamped to [1.5 * 2^23, 1.5 * 2^23 + 255] (that span has unit
// spacing). Every step is monotone in x, so bins keep the score order; NaN and
// a range that overflows land in bin 0 (the search then moves on to the
// bitwise step).
struct Binning {
  static constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float sc, offm;
  __device__ __forceinline__ Binning(float lo, float hi) {
    sc = (float)kBins / (hi - lo);
    offm = fmaf(-lo, sc, kMagic);
  }
  __device__ __forceinline__ int operator()(float x) const {
    const float t = fminf(fmaxf(fmaf(x, sc, offm), kMagic), kMagic + (float)(kBins - 1));
    return __float_as_int(t) - __float_as_int(kMagic);
  }
};

// The warp's staged row: lane l's i-th value is tile l + 32 i.
struct Row {
  const float* p;  // &slice[lane]
  int N, lane;
  __device__ __forceinline__ float operator[](int i) const { return p[32 * i]; }
  __device__ __forceinline__ bool valid(int i) const { return lane + 32 * i < N; }
};

struct Hist {
  uint32_t* cnt;  // [kBins] tile count per bin
  uint64_t* wt;   // [kBins] weight per bin (mass only)
};

__device__ __forceinline__ bool in_range(float x, float lo, float hi) { return x >= lo && x <= hi; }

template <int VPT, bool MASS>
__device__ __forceinline__ void build_hist(const Row& row, bool whole, float lo, float hi, const Binning& bin,
                                           double smax, Hist h) {
#pragma unroll
  for (int q = 0; q < kBins / 32; ++q) {
    h.cnt[row.lane + 32 * q] = 0;
    if constexpr (MASS) h.wt[row.lane + 32 * q] = 0;
  }
  __syncwarp();
#pragma unroll 8
  for (int i = 0; i < VPT; ++i) {
    const float x = row[i];
    if (row.valid(i) && (whole || in_range(x, lo, hi))) {
      const int b = bin(x);
      atomicAdd(&h.cnt[b], 1u);
      if constexpr (MASS) atomicAdd((unsigned long long*)&h.wt[b], (unsigned long long)mass_q(x, smax));
    }
  }
  __syncwarp();
}

// Bin b (higher bins hold higher scores) in which the running weight, taken
// from the top bin down, reaches R > 0; *above gets the weight of all higher
// bins. Lane l owns bins [8l, 8l+8). Returns -1 if the total is below R.
template <bool MASS>
__device__ __forceinline__ int find_bin(Hist h, uint64_t R, int lane, uint64_t* above) {
  uint64_t c[8], s = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    c[q] = MASS ? h.wt[8 * lane + q] : (uint64_t)h.cnt[8 * lane + q];
    s += c[q];
  }
  uint64_t x = s;  // inclusive suffix sum over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = shfl_down_u64(x, o);
    if (lane + o < 32) x += y;
  }
  uint64_t run = x - s;
  int hit = -1;
  uint64_t hit_above = 0;
#pragma unroll
  for (int q = 7; q >= 0; --q) {
    if (hit < 0 && run < R && R - run <= c[q]) {
      hit = 8 * lane + q;
      hit_above = run;
    }
    run += c[q];
  }
  const uint32_t m = __ballot_sync(0xffffffffu, hit >= 0);
  if (!m) return -1;
  const int src = __ffs(m) - 1;  // at most one bin crosses R
  *above = shfl_idx_u64(hit_above, src);
  return __shfl_sync(0xffffffffu, hit, src);
}

// Largest composite key t whose upper set {keys >= t} weighs at least R: the
// key of the tile at which the running weight reaches R.
template <int VPT, bool MASS>
__device__ uint64_t bisect_key(const Row& row, uint64_t R, double smax) {
  uint64_t t = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const uint64_t c = t | (1ull << bit);
    uint64_t w = 0;
    for (int i = 0; i < VPT; ++i)
      if (row.valid(i) && comp_key(row[i], row.lane + 32 * i) >= c) w += weight_of<MASS>(row[i], smax);
    if (warp_sum_u64(w) >= R) t = c;
  }
  return t;
}

// The search described at the top of the file. On entry `h` holds the
// histogram of the whole row under Binning(lo, hi), [lo, hi] being the row's
// finite-or-not extent. Requires 1 <= R <= the row's total weight.
template <int VPT, bool MASS>
__device__ uint64_t crossing_key(const Row& row, uint64_t R, double smax, float lo, float hi, Hist h,
                                 uint64_t* cand) {
  const int lane = row.lane;
  const uint32_t lt = (1u << lane) - 1u;
  uint64_t A = 0;  // weight of the tiles above the current range
  bool whole = true;
  for (int level = 0; level < kLevels; ++level) {
    if (!(lo < hi)) {
      if (!(lo == hi)) break;  // NaN extent
      // One score value: its tiles run in ascending index order, each with
      // the same weight w; the crossing is the ceil((R - A) / w)-th of them.
      const uint64_t w = weight_of<MASS>(lo, smax);
      if (w == 0 || R <= A) break;
      const uint64_t need = (R - A + w - 1) / w;
      uint64_t base = 0;
      for (int i = 0; i < VPT; ++i) {
        const uint32_t m = __ballot_sync(0xffffffffu, row.valid(i) && row[i] == lo);
        const uint64_t pc = (uint64_t)__popc(m);
        if (base < need && need <= base + pc) {
          uint32_t mm = m;  // drop the lowest (need - base - 1) set lanes
          for (uint64_t s = 1; s < need - base; ++s) mm &= mm - 1;
          return comp_key(lo, 32 * i + __ffs(mm) - 1);
        }
        base += pc;
      }
      break;
    }
    const Binning bin(lo, hi);
    if (!whole) build_hist<VPT, MASS>(row, false, lo, hi, bin, smax, h);
    uint64_t above = 0;
    const int b = find_bin<MASS>(h, R - A, lane, &above);
    if (b < 0) break;
    A += above;
    const uint32_t nb = h.cnt[b];
    if (nb <= (uint32_t)kCand) {
      // Rank the bin's tiles exactly: gather one per lane, sort descending.
      int base = 0;
#pragma unroll 8
      for (int i = 0; i < VPT; ++i) {
        const float x = row[i];
        const bool in = row.valid(i) && (whole || in_range(x, lo, hi)) && bin(x) == b;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        const int pos = base + __popc(m & lt);
        if (in && pos < kCand) cand[pos] = comp_key(x, lane + 32 * i);
        base += __popc(m);
      }
      __syncwarp();
      uint64_t ck = lane < (int)nb ? cand[lane] : 0ull;
      __syncwarp();
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const uint64_t ok = shfl_xor_u64(ck, stride);
          const bool take_max = ((lane & stride) == 0) == ((lane & size) == 0);
          if (take_max ? ok > ck : ok < ck) ck = ok;
        }
      uint64_t c;  // inclusive prefix of the sorted weights
      if constexpr (MASS) {
        c = ck ? mass_q(key_to_float((uint32_t)(ck >> 32)), smax) : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint64_t y = shfl_up_u64(c, o);
          if (lane >= o) c += y;
        }
      } else {
        c = (uint64_t)(lane + 1);
      }
      const uint32_t m = __ballot_sync(0xffffffffu, ck != 0 && A + c >= R);
      if (m) return shfl_idx_u64(ck, __ffs(m) - 1);
      break;
    }
    // Next range: the extent of bin b's scores.
    uint32_t klo = 0xffffffffu, khi = 0u;
#pragma unroll 8
    for (int i = 0; i < VPT; ++i) {
      const float x = row[i];
      if (row.valid(i) && (whole || in_range(x, lo, hi)) && bin(x) == b) {
        const uint32_t k = order_key(x);
        klo = min(klo, k);
        khi = max(khi, k);
      }
    }
    klo = __reduce_min_sync(0xffffffffu, klo);
    khi = __reduce_max_sync(0xffffffffu, khi);
    if (klo > khi) break;
    lo = key_to_float(klo);
    hi = key_to_float(khi);
    whole = false;
  }
  return bisect_key<VPT, MASS>(row, R, smax);
}

// Keep every tile at or above the crossing tile, ascending; returns the count.
template <int VPT>
__device__ __forceinline__ int write_kept(const Row& row, uint64_t kth, int32_t* out, int kmax) {
  const float xth = key_to_float((uint32_t)(kth >> 32));  // NaN for ~0: keeps nothing
  const int jth = (int)(0xffffffffu - (uint32_t)kth);
  const uint32_t lt = (1u << row.lane) - 1u;
  int base = 0;
#pragma unroll 8
  for (int i = 0; i < VPT; ++i) {
    const float x = row[i];
    const int j = row.lane + 32 * i;
    const bool keep = row.valid(i) && (x > xth || (x == xth && j <= jth));
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    const int pos = base + __popc(m & lt);
    if (keep && pos < kmax) out[pos] = j;
    base += __popc(m);
  }
  return min(base, kmax);
}

// NaN-free min and max of the staged row (NaN if it has no other value).
template <int VPT>
__device__ __forceinline__ void row_extent(const Row& row, float* lo, float* hi) {
  float mn = __int_as_float(0x7fc00000), mx = mn;
#pragma unroll 8
  for (int i = 0; i < VPT; ++i)
    if (row.valid(i)) {
      mn = fminf(mn, row[i]);
      mx = fmaxf(mx, row[i]);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  *lo = mn;
  *hi = mx;
}

// One pass over the staged row against bin b: mask[i] gets the 32-tile word
// of chunk i's tiles in bins above b, and the tiles of bin b go to cand (the
// first kCand of them) as composite keys. Returns the number of bin-b tiles.
__device__ __forceinline__ int mask_and_gather(const Row& row, const Binning& bin, int b, uint32_t* mask,
                                               uint64_t* cand) {
  const uint32_t lt = (1u << row.lane) - 1u;
  const int nfull = row.N >> 5, nchunk = (row.N + 31) >> 5;
  int base = 0;
  auto chunk = [&](int i, bool valid) {
    const float x = row[i];
    const int bx = bin(x);
    const uint32_t ma = __ballot_sync(0xffffffffu, valid && bx > b);
    const uint32_t me = __ballot_sync(0xffffffffu, valid && bx == b);
    if (row.lane == 0) mask[i] = ma;
    if (me) {
      const int pos = base + __popc(me & lt);
      if (((me >> row.lane) & 1u) && pos < kCand) cand[pos] = comp_key(x, row.lane + 32 * i);
      base += __popc(me);
    }
  };
#pragma unroll 4
  for (int i = 0; i < nfull; ++i) chunk(i, true);
  if (nchunk > nfull) chunk(nfull, row.valid(nfull));
  __syncwarp();
  return base;
}

// Sorts the warp's candidates (one composite key per lane, 0 for none)
// descending.
__device__ __forceinline__ uint64_t sort_desc32(uint64_t ck, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t ok = shfl_xor_u64(ck, stride);
      const bool take_max = ((lane & stride) == 0) == ((lane & size) == 0);
      if (take_max ? ok > ck : ok < ck) ck = ok;
    }
  return ck;
}

// Writes the tiles whose mask bit is set, ascending, and returns how many
// were written (at most kmax). Lane l owns the words [l*WPL, (l+1)*WPL).
template <int VPT>
__device__ __forceinline__ int compact_mask(const uint32_t* mask, int N, int lane, int32_t* out, int kmax) {
  constexpr int WPL = (VPT + 31) / 32;
  const int nchunk = (N + 31) >> 5;
  uint32_t wv[WPL];
  int c = 0;
#pragma unroll
  for (int t = 0; t < WPL; ++t) {
    const int wi = lane * WPL + t;
    wv[t] = wi < nchunk ? mask[wi] : 0u;
    c += __popc(wv[t]);
  }
  int x = c;  // inclusive prefix over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const int total = __shfl_sync(0xffffffffu, x, 31);
  int pos = x - c;
#pragma unroll
  for (int t = 0; t < WPL; ++t) {
    uint32_t m = wv[t];
    const int jb = 32 * (lane * WPL + t);
    while (m) {
      if (pos < kmax) out[pos] = jb + __ffs(m) - 1;
      ++pos;
      m &= m - 1;
    }
  }
  return min(total, kmax);
}

// Marks the first `keep` sorted candidates in the mask.
__device__ __forceinline__ void mark_kept(uint64_t ck, int lane, int keep, uint32_t* mask) {
  if (lane < keep && ck) {
    const uint32_t j = 0xffffffffu - (uint32_t)ck;
    atomicOr(&mask[j >> 5], 1u << (j & 31));
  }
  __syncwarp();
}

// Rows per CTA: every warp's slice of staged scores, histograms and masks
// must fit the 48 KB of static shared memory.
template <int VPT, bool MASS>
struct Shape {
  static constexpr int per_warp = 32 * VPT * 4 + VPT * 4 + kBins * 4 + (MASS ? kBins * 8 : 0) + kCand * 8;
  static constexpr int warps = (8 * per_warp <= 48 * 1024) ? 8 : 4;
  static_assert(warps * per_warp <= 48 * 1024, "selection shared memory");
};

template <int VPT>
__global__ void __launch_bounds__(32 * Shape<VPT, false>::warps)
topk_kernel(int rows, int N, int k, const float* __restrict__ S, int32_t* __restrict__ idx,
            int32_t* __restrict__ cnt, int kmax, const int32_t* __restrict__ rlist,
            const int* __restrict__ rcount) {
  constexpr int W = Shape<VPT, false>::warps;
  __shared__ float vals_s[W][32 * VPT];
  __shared__ uint32_t hcnt_s[W][kBins];
  __shared__ uint32_t mask_s[W][VPT];
  __shared__ uint64_t cand_s[W][kCand];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // With a row list, warp x takes the list's x-th row (the list's length is
  // read on the device); otherwise row x.
  int r0 = blockIdx.x * W + w;
  if (rlist) {
    if (r0 >= *rcount) return;
    r0 = rlist[r0];
  } else if (r0 >= rows) {
    return;
  }
  const float* s = S + (size_t)r0 * N;
  float* slice = vals_s[w];
  uint32_t* hist = hcnt_s[w];
  const Row row{&slice[lane], N, lane};

  // Pass 1: load the whole row into registers (all loads in flight at once),
  // stage it, histogram it. The bins span the extent of an evenly strided
  // sample of chunks; tiles outside it fall into the edge bins (binning stays
  // monotone).
  constexpr int B0 = VPT < 8 ? VPT : 8;
  constexpr int STEP = VPT / B0;
  float v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int j = lane + 32 * i;
    v[i] = j < N ? __ldg(s + j) : __int_as_float(0x7fc00000);
  }
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int t = 1; t < B0; ++t) {
    mn = fminf(mn, v[t * STEP]);
    mx = fmaxf(mx, v[t * STEP]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const bool spread = mn < mx;
  const Binning bin(spread ? mn : 0.f, spread ? mx : 1.f);
#pragma unroll
  for (int q = 0; q < kBins / 32; ++q) hist[lane + 32 * q] = 0;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int j = lane + 32 * i;
    if (j < N) {
      slice[j] = v[i];
      atomicAdd(&hist[bin(v[i])], 1u);
    }
  }
  __syncwarp();

  const int r = min(k, N);
  int32_t* out = idx + (size_t)r0 * kmax;
  int n = 0;
  uint64_t above = 0;
  const int b = (spread && r >= 1) ? find_bin<false>(Hist{hist, nullptr}, (uint64_t)r, lane, &above) : -1;
  if (b >= 0 && hist[b] <= (uint32_t)kCand) {
    // Pass 2: bins above b are kept whole; rank bin b's tiles exactly.
    const int nb = mask_and_gather(row, bin, b, mask_s[w], cand_s[w]);
    const uint64_t ck = sort_desc32(lane < nb ? cand_s[w][lane] : 0ull, lane);
    mark_kept(ck, lane, r - (int)above, mask_s[w]);
    n = compact_mask<VPT>(mask_s[w], N, lane, out, kmax);
  } else if (r >= 1) {
    // General search over the exact extent.
    float lo, hi;
    row_extent<VPT>(row, &lo, &hi);
    const Hist h{hist, nullptr};
    __syncwarp();
    if (lo < hi) build_hist<VPT, false>(row, true, lo, hi, Binning(lo, hi), 0.0, h);
    const uint64_t kth = crossing_key<VPT, false>(row, (uint64_t)r, 0.0, lo, hi, h, cand_s[w]);
    n = write_kept<VPT>(row, kth, out, kmax);
  }
  if (lane == 0) cnt[r0] = n;
}

// Top-k for rows of a multiple of 4 tiles and at least 128: the row moves as
// float4 (lane l holds tiles 128c + 4l .. 4l+3 of 128-tile chunk c), binning
// uses 128 bins so that four bin indices pack into one 32-bit word, and the
// second pass compares four packed bins with the boundary bin per SWAR
// subtraction instead of binning every score again. The row is not staged in
// shared memory (which keeps eight warps per CTA and the registers low): the
// few boundary-bin candidates and the general search for crowded boundary
// bins (lane-strided view) read it again from global memory, where it is
// still cached.
constexpr int kBins7 = 128;

struct Binning7 {  // Binning with 128 bins (indices fit 7 bits)
  static constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float sc, offm;
  __device__ __forceinline__ Binning7(float lo, float hi) {
    sc = (float)kBins7 / (hi - lo);
    offm = fmaf(-lo, sc, kMagic);
  }
  __device__ __forceinline__ uint32_t operator()(float x) const {
    const float t = fminf(fmaxf(fmaf(x, sc, offm), kMagic), kMagic + (float)(kBins7 - 1));
    return (uint32_t)(__float_as_int(t) - __float_as_int(kMagic));
  }
};

// High bits (7, 15, 23, 31) of a SWAR compare -> 4-bit nibble (bit e = byte e).
__device__ __forceinline__ uint32_t high_bits_nibble(uint32_t m) { return ((m >> 7) * 0x10204080u) >> 28; }

// Bin (of 128) in which the running count, taken from the top bin down,
// reaches r > 0; *above = count of higher bins. Lane l owns bins [4l, 4l+4).
__device__ __forceinline__ int find_bin128(const uint32_t* h, int r, int lane, int* above) {
  uint32_t c[4], s = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    c[q] = h[4 * lane + q];
    s += c[q];
  }
  uint32_t x = s;  // inclusive suffix sum over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  uint32_t run = x - s;
  int hit = -1, hit_above = 0;
#pragma unroll
  for (int q = 3; q >= 0; --q) {
    if (hit < 0 && run < (uint32_t)r && (uint32_t)r - run <= c[q]) {
      hit = 4 * lane + q;
      hit_above = (int)run;
    }
    run += c[q];
  }
  const uint32_t m = __ballot_sync(0xffffffffu, hit >= 0);
  if (!m) return -1;
  const int src = __ffs(m) - 1;
  *above = __shfl_sync(0xffffffffu, hit_above, src);
  return __shfl_sync(0xffffffffu, hit, src);
}

template <int C4>
struct Shape4 {
  static constexpr int per_warp = 128 * C4 + 2 * 4 * C4 * 4 + kBins * 4 + kCand * 8;
  static constexpr int warps = (8 * per_warp <= 48 * 1024) ? 8 : 4;
  static_assert(warps * per_warp <= 48 * 1024, "selection shared memory");
};

template <int C4>
__global__ void __launch_bounds__(32 * Shape4<C4>::warps)
topk4_kernel(int rows, int N, int k, const float* __restrict__ S, int32_t* __restrict__ idx,
             int32_t* __restrict__ cnt, int kmax, const int32_t* __restrict__ rlist,
             const int* __restrict__ rcount) {
  constexpr int W = Shape4<C4>::warps, VPT = 4 * C4;
  __shared__ uint32_t bins_s[W][32 * C4];
  __shared__ uint32_t gt_s[W][4 * C4];
  __shared__ uint32_t eq_s[W][4 * C4];
  __shared__ uint32_t hcnt_s[W][kBins];
  __shared__ uint64_t cand_s[W][kCand];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // With a row list, warp x takes the list's x-th row (the list's length is
  // read on the device); otherwise row x.
  int r0 = blockIdx.x * W + w;
  if (rlist) {
    if (r0 >= *rcount) return;
    r0 = rlist[r0];
  } else if (r0 >= rows) {
    return;
  }
  const float* s = S + (size_t)r0 * N;
  uint32_t* hist = hcnt_s[w];
  const float qnan = __int_as_float(0x7fc00000);
  auto load4 = [&](int c) -> float4 {
    const int j0 = 128 * c + 4 * lane;  // N % 4 == 0: a float4 is all in or all out
    return j0 < N ? __ldg(reinterpret_cast<const float4*>(s + j0)) : make_float4(qnan, qnan, qnan, qnan);
  };

  // Pass 1: bins over the extent of an evenly strided sample of chunks (tiles
  // outside it land in the edge bins), then every chunk binned, loaded in
  // groups of four float4 so that few registers hold the row.
  constexpr int B0 = C4 < 4 ? C4 : 4;
  constexpr int STEP = C4 / B0;
  float mn = qnan, mx = qnan;
  {
    float4 u[B0];
#pragma unroll
    for (int t = 0; t < B0; ++t) u[t] = load4(t * STEP);
#pragma unroll
    for (int t = 0; t < B0; ++t) {
      mn = fminf(fminf(mn, fminf(u[t].x, u[t].y)), fminf(u[t].z, u[t].w));
      mx = fmaxf(fmaxf(mx, fmaxf(u[t].x, u[t].y)), fmaxf(u[t].z, u[t].w));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const bool spread = mn < mx;
  const Binning7 bin(spread ? mn : 0.f, spread ? mx : 1.f);
#pragma unroll
  for (int q = 0; q < kBins7 / 32; ++q) hist[lane + 32 * q] = 0;
  __syncwarp();
  constexpr int G = 4;  // float4 loads in flight per group
#pragma unroll
  for (int c0 = 0; c0 < C4; c0 += G) {
    float4 v[G];
#pragma unroll
    for (int t = 0; t < G; ++t) v[t] = c0 + t < C4 ? load4(c0 + t) : make_float4(qnan, qnan, qnan, qnan);
#pragma unroll
    for (int t = 0; t < G; ++t) {
      const int c = c0 + t;
      if (c >= C4) break;
      uint32_t word = 0;
      if (128 * c + 4 * lane < N) {
        const uint32_t b0 = bin(v[t].x), b1 = bin(v[t].y), b2 = bin(v[t].z), b3 = bin(v[t].w);
        atomicAdd(&hist[b0], 1u);
        atomicAdd(&hist[b1], 1u);
        atomicAdd(&hist[b2], 1u);
        atomicAdd(&hist[b3], 1u);
        word = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
      }
      bins_s[w][32 * c + lane] = word;
    }
  }
  __syncwarp();

  const int r = min(k, N);
  int32_t* out = idx + (size_t)r0 * kmax;
  int n = 0, above = 0;
  const int b = (spread && r >= 1) ? find_bin128(hist, r, lane, &above) : -1;
  if (b >= 0 && hist[b] <= (uint32_t)kCand) {
    // Pass 2: packed bins vs the boundary bin b, four at a time: with every
    // byte x in [0, 127], (x | 0x80) - c keeps its byte and has the high bit
    // set exactly when x >= c (c <= 128).
    const uint32_t cb = (uint32_t)b * 0x01010101u, cb1 = (uint32_t)(b + 1) * 0x01010101u;
    const int nch = (N + 127) >> 7;
    const int sh = 4 * (lane & 7);
    for (int c = 0; c < nch; ++c) {
      const uint32_t x = bins_s[w][32 * c + lane] | 0x80808080u;
      const uint32_t ge1 = (x - cb1) & 0x80808080u, ge0 = (x - cb) & 0x80808080u;
      const uint32_t vm = (128 * c + 4 * lane < N) ? 0xFu : 0u;
      uint32_t gx = (high_bits_nibble(ge1) & vm) << sh;
      uint32_t ex = (high_bits_nibble(ge0 & ~ge1) & vm) << sh;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {  // lanes 8q..8q+7 hold the 32 tiles of word 4c + q
        gx |= __shfl_xor_sync(0xffffffffu, gx, o);
        ex |= __shfl_xor_sync(0xffffffffu, ex, o);
      }
      if ((lane & 7) == 0) {
        gt_s[w][4 * c + (lane >> 3)] = gx;
        eq_s[w][4 * c + (lane >> 3)] = ex;
      }
    }
    __syncwarp();
    // The boundary bin's tiles, one per lane (their order does not matter:
    // they are sorted next).
    const int nw = (N + 31) >> 5;  // <= 64
    const uint32_t e0 = lane < nw ? eq_s[w][lane] : 0u, e1 = lane + 32 < nw ? eq_s[w][lane + 32] : 0u;
    const int pc = __popc(e0) + __popc(e1);
    int x = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int pos = x - pc;
    for (int t = 0; t < 2; ++t) {
      uint32_t m = t ? e1 : e0;
      const int wbase = 32 * (lane + 32 * t);
      while (m) {
        const int j = wbase + __ffs(m) - 1;
        if (pos < kCand) cand_s[w][pos] = comp_key(__ldg(s + j), j);
        ++pos;
        m &= m - 1;
      }
    }
    const int nb = min(__shfl_sync(0xffffffffu, x, 31), kCand);
    __syncwarp();
    // Keep the candidates ranked above r - above (rank by composite key; the
    // keys are unique), no full sort needed.
    const uint64_t mine = lane < nb ? cand_s[w][lane] : 0ull;
    int rank = 0;
    for (int t = 0; t < nb; ++t) rank += shfl_idx_u64(mine, t) > mine ? 1 : 0;
    if (lane < nb && rank < r - above) {
      const uint32_t j = 0xffffffffu - (uint32_t)mine;
      atomicOr(&gt_s[w][j >> 5], 1u << (j & 31));
    }
    __syncwarp();
    n = compact_mask<VPT>(gt_s[w], N, lane, out, kmax);
  } else if (r >= 1) {
    // General search over the exact extent, reading the row from global memory.
    const Row row{s + lane, N, lane};
    float lo, hi;
    row_extent<VPT>(row, &lo, &hi);
    const Hist h{hist, nullptr};
    __syncwarp();
    if (lo < hi) build_hist<VPT, false>(row, true, lo, hi, Binning(lo, hi), 0.0, h);
    const uint64_t kth = crossing_key<VPT, false>(row, (uint64_t)r, 0.0, lo, hi, h, cand_s[w]);
    n = write_kept<VPT>(row, kth, out, kmax);
  }
  if (lane == 0) cnt[r0] = n;
}

// Rows per CTA of the top-p kernel, whose row is not staged in shared memory.
template <int VPT>
struct ShapeP {
  static constexpr int per_warp = VPT * 4 + kBins * 4 + kBins * 8 + kCand * 8;
  static constexpr int warps = (8 * per_warp <= 48 * 1024) ? 8 : 4;
  static_assert(warps * per_warp <= 48 * 1024, "selection shared memory");
};

// Top-p with a top-k floor: in descending order keep the shortest prefix
// whose softmax mass reaches p of the row's total, then at least k and at
// most N tiles. Every pass reads the row from global memory (still cached
// after the first): staging it in shared memory would halve the warps per SM.
template <int VPT>
__global__ void __launch_bounds__(32 * ShapeP<VPT>::warps, 4)
topp_kernel(int rows, int N, int k, double p, const float* __restrict__ S, int32_t* __restrict__ idx,
            int32_t* __restrict__ cnt, int kmax) {
  constexpr int W = ShapeP<VPT>::warps;
  __shared__ uint32_t hcnt_s[W][kBins];
  __shared__ uint64_t hwt_s[W][kBins];
  __shared__ uint32_t mask_s[W][VPT];
  __shared__ uint64_t cand_s[W][kCand];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * W + w;
  if (r0 >= rows) return;
  const float* s = S + (size_t)r0 * N;
  const Row row{s + lane, N, lane};
  // Pass 1: the exact max is needed before any mass.
  float v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int j = lane + 32 * i;
    v[i] = j < N ? __ldg(s + j) : __int_as_float(0x7fc00000);
  }
  float lo = v[0], hi = v[0];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int j = lane + 32 * i;
    lo = fminf(lo, v[i]);
    hi = fmaxf(hi, v[i]);
    (void)j;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const double smax = (double)hi;
  const Hist hm{hcnt_s[w], hwt_s[w]};
  const bool spread = lo < hi;
  const Binning bin0(spread ? lo : 0.f, spread ? hi : 1.f);
  // Pass 2: count and mass histograms and the total mass.
#pragma unroll
  for (int q = 0; q < kBins / 32; ++q) {
    hm.cnt[lane + 32 * q] = 0;
    hm.wt[lane + 32 * q] = 0;
  }
  __syncwarp();
  uint64_t local = 0;
#pragma unroll 4
  for (int i = 0; i < VPT; ++i) {
    if (row.valid(i)) {
      const float x = row[i];
      const uint64_t q = mass_q(x, smax);
      const int b = bin0(x);
      local += q;
      atomicAdd(&hm.cnt[b], 1u);
      atomicAdd((unsigned long long*)&hm.wt[b], (unsigned long long)q);
    }
  }
  __syncwarp();
  const uint64_t total = warp_sum_u64(local);
  // R = ceil(p * total), clamped to [1, total]; a row without finite mass
  // (an infinite score) has total 0 and keeps only the floor.
  const double tgt = ceil(p * (double)total);
  uint64_t R = tgt >= (double)total ? total : (tgt > 1.0 ? (uint64_t)tgt : 1ull);
  if (R > total) R = total;
  int32_t* out = idx + (size_t)r0 * kmax;
  int n = -1;
  uint64_t A = 0;
  const int b = (spread && R >= 1) ? find_bin<true>(hm, R, lane, &A) : -1;
  if (b >= 0 && hm.cnt[b] <= (uint32_t)kCand) {
    // Pass 3: bins above b are kept whole; bin b's tiles in order decide m*.
    int cab = 0;  // tiles in bins above b
#pragma unroll
    for (int q = 0; q < kBins / 32; ++q) {
      const int bb = lane + 32 * q;
      cab += bb > b ? (int)hm.cnt[bb] : 0;
    }
    cab = (int)__reduce_add_sync(0xffffffffu, (uint32_t)cab);
    const int nb = mask_and_gather(row, bin0, b, mask_s[w], cand_s[w]);
    const uint64_t ck = sort_desc32(lane < nb ? cand_s[w][lane] : 0ull, lane);
    uint64_t c = ck ? mass_q(key_to_float((uint32_t)(ck >> 32)), smax) : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = shfl_up_u64(c, o);
      if (lane >= o) c += y;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, ck != 0 && A + c >= R);
    if (hit) {
      const int mstar = cab + __ffs(hit);
      const int r = min(N, max(mstar, k));
      if (r - cab <= nb) {
        mark_kept(ck, lane, r - cab, mask_s[w]);
        n = compact_mask<VPT>(mask_s[w], N, lane, out, kmax);
      } else {
        // The floor reaches past bin b: count search for rank r.
        const uint64_t kth = crossing_key<VPT, false>(row, (uint64_t)r, 0.0, lo, hi, Hist{hm.cnt, nullptr},
                                                      cand_s[w]);
        n = write_kept<VPT>(row, kth, out, kmax);
      }
    }
  }
  if (n < 0) {
    // General search over the exact extent.
    uint64_t kth_m = ~0ull;
    int mstar = 0;
    if (R >= 1) {
      kth_m = crossing_key<VPT, true>(row, R, smax, lo, hi, hm, cand_s[w]);
      const float xth = key_to_float((uint32_t)(kth_m >> 32));
      const int jth = (int)(0xffffffffu - (uint32_t)kth_m);
      uint32_t nm = 0;
#pragma unroll 8
      for (int i = 0; i < VPT; ++i) {
        const float x = row[i];
        nm += (row.valid(i) && (x > xth || (x == xth && lane + 32 * i <= jth))) ? 1u : 0u;
      }
      mstar = (int)__reduce_add_sync(0xffffffffu, nm);
    }
    const int r = min(N, max(mstar, k));
    uint64_t kth = kth_m;
    if (r > mstar) {
      const Hist hc{hcnt_s[w], nullptr};
      if (lo < hi) build_hist<VPT, false>(row, true, lo, hi, bin0, 0.0, hc);
      kth = crossing_key<VPT, false>(row, (uint64_t)r, 0.0, lo, hi, hc, cand_s[w]);
    }
    n = write_kept<VPT>(row, kth, out, kmax);
  }
  if (lane == 0) cnt[r0] = n;
}

__global__ void broadcast_lists_kernel(int N, int kmax, const int32_t* __restrict__ src_idx,
                                       const int32_t* __restrict__ src_cnt, int32_t* __restrict__ idx,
                                       int32_t* __restrict__ cnt) {
  const size_t bh = blockIdx.y;
  const int per = N * kmax;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < per; e += gridDim.x * blockDim.x)
    idx[bh * per + e] = src_idx[e];
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < N; e += gridDim.x * blockDim.x)
    cnt[bh * N + e] = src_cnt[e];
}

template <int VPT>
bsattn_status run_topk(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt, int kmax,
                       const int32_t* rlist, const int* rcount, cudaStream_t st) {
  constexpr int W = Shape<VPT, false>::warps;
  topk_kernel<VPT><<<(rows + W - 1) / W, 32 * W, 0, st>>>(rows, N, k, S, idx, cnt, kmax, rlist, rcount);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

template <int C4>
bsattn_status run_topk4(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt, int kmax,
                        const int32_t* rlist, const int* rcount, cudaStream_t st) {
  constexpr int W = Shape4<C4>::warps;
  topk4_kernel<C4><<<(rows + W - 1) / W, 32 * W, 0, st>>>(rows, N, k, S, idx, cnt, kmax, rlist, rcount);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

template <int VPT>
bsattn_status run_topp(int rows, int N, int k, double p, const float* S, int32_t* idx, int32_t* cnt, int kmax,
                       cudaStream_t st) {
  constexpr int W = ShapeP<VPT>::warps;
  topp_kernel<VPT><<<(rows + W - 1) / W, 32 * W, 0, st>>>(rows, N, k, p, S, idx, cnt, kmax);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

bsattn_status launch_select_topk_rows(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt,
                                      int kmax, const int32_t* rlist, const int* rcount, cudaStream_t st) {
  if (rows <= 0 || N <= 0) return BSATTN_OK;
  if (N % 4 == 0 && N >= 128 && ((uintptr_t)S & 15u) == 0) {
    const int c4 = (N + 127) / 128;
    if (c4 <= 1) return run_topk4<1>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 2) return run_topk4<2>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 3) return run_topk4<3>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 4) return run_topk4<4>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 6) return run_topk4<6>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 8) return run_topk4<8>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 12) return run_topk4<12>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
    if (c4 <= 16) return run_topk4<16>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  }
  const int vpt = (N + 31) / 32;
  if (vpt <= 1) return run_topk<1>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 2) return run_topk<2>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 4) return run_topk<4>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 8) return run_topk<8>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 12) return run_topk<12>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 16) return run_topk<16>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 24) return run_topk<24>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 32) return run_topk<32>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 48) return run_topk<48>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  if (vpt <= 64) return run_topk<64>(rows, N, k, S, idx, cnt, kmax, rlist, rcount, st);
  return BSATTN_ERR_UNSUPPORTED;
}

bsattn_status launch_select_topk(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt, int kmax,
                                 cudaStream_t st) {
  return launch_select_topk_rows(rows, N, k, S, idx, cnt, kmax, nullptr, nullptr, st);
}

bsattn_status launch_select_topp(int rows, int N, int k, double p, const float* S, int32_t* idx, int32_t* cnt,
                                 int kmax, cudaStream_t st) {
  if (rows <= 0 || N <= 0) return BSATTN_OK;
  const int vpt = (N + 31) / 32;
  if (vpt <= 1) return run_topp<1>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 2) return run_topp<2>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 4) return run_topp<4>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 8) return run_topp<8>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 12) return run_topp<12>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 16) return run_topp<16>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 24) return run_topp<24>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 32) return run_topp<32>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 48) return run_topp<48>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (vpt <= 64) return run_topp<64>(rows, N, k, p, S, idx, cnt, kmax, st);
  return BSATTN_ERR_UNSUPPORTED;
}

bsattn_status launch_broadcast_lists(int bh, int N, int kmax, const int32_t* src_idx, const int32_t* src_cnt,
                                     int32_t* idx, int32_t* cnt, cudaStream_t st) {
  const int per = N * kmax;
  dim3 grid((per + 255) / 256 < 64 ? (per + 255) / 256 : 64, bh);
  broadcast_lists_kernel<<<grid, 256, 0, st>>>(N, kmax, src_idx, src_cnt, idx, cnt);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}
