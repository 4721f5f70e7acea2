// tile_rule.cuh -- the index rule as the tensor-core kernel applies it, in 64-key tiles.
//
// Host and device code: the kernel uses it, and a CPU test compiles the same header with g++ to
// check, for many shapes, that the keys visited and unmasked are exactly L(i) and P(i).
//   window  L(i) = [max(0, i - k), i]
//   skips   P(i) = { i - m*pi : m0 <= m <= S, i - m*pi >= 0 },  m0 = floor(k / pi) + 1
// and its bidirectional variant (a sequence of n tokens):
//   window  L(i) = [max(0, i - k), min(n - 1, i + k)]
//   skips   P(i) = { i - m*pi, i + m*pi : m0 <= m <= S, 0 <= key < n }
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define PIA_HD __host__ __device__ __forceinline__
#else
#define PIA_HD inline
#endif

namespace pia {

constexpr int kTileKeys = 64;  // keys per tile (BN)

// floor(a / b) for 0 <= a < 2^52, b >= 1, through a double reciprocal of b (rb = 1.0 / b) and
// an exact +-1 correction -- GPUs have no integer divider, and these run per row and per tile.
PIA_HD long long div_floor(long long a, long long b, double rb) {
  long long q = (long long)((double)a * rb);
  if (q * b > a) --q;
  else if ((q + 1) * b <= a) ++q;
  return q;
}

// Walks, in increasing order, the key tiles that hold at least one key of the union of L(i)
// and P(i) over the query rows [i0, last] of one tile.
struct TileWalk {
  // every field has a value before init() or init_residue()
  long long i0 = 0, last = -1, band_lo = 0, band_hi = -1;  // query rows [i0, last]; window keys [band_lo, band_hi]
  long long n = 0;                       // sequence length (bidirectional: forward keys stop at n - 1)
  int pi = 1, S = 0, m0 = 1;
  bool bidir = false;
  double rpi = 1.0;                      // 1.0 / pi
  PIA_HD void init(long long i0_, long long n_, int rows, int kwin, int pi_, int S_, bool bidir_ = false) {
    i0 = i0_;
    n = n_;
    last = i0_ + rows - 1 < n_ - 1 ? i0_ + rows - 1 : n_ - 1;
    band_lo = i0_ - kwin > 0 ? i0_ - kwin : 0;
    band_hi = bidir_ ? (last + kwin < n_ - 1 ? last + kwin : n_ - 1) : last;
    pi = pi_;
    S = S_;
    m0 = kwin / pi_ + 1;
    bidir = bidir_;
    rpi = 1.0 / (double)pi_;
  }
  // The residue-class view of the split path: rows q0 .. q0 + rows - 1 of a class of T rows,
  // row t reading the band of keys t - S .. t - m0 of the same class (its skips, as a dense band);
  // bidirectional, also the band t + m0 .. t + S (the forward skips).  The walk covers the union.
  PIA_HD void init_residue(long long q0, long long T, int rows, int S_, int m0_, bool bidir_ = false) {
    i0 = q0;
    const long long qlast = q0 + rows - 1 < T - 1 ? q0 + rows - 1 : T - 1;
    last = qlast - m0_;
    band_lo = q0 - S_ > 0 ? q0 - S_ : 0;
    band_hi = S_ < m0_ ? -1 : (bidir_ ? (qlast + S_ < T - 1 ? qlast + S_ : T - 1) : last);  // S < m0: no key
    n = T;
    pi = 1;
    S = 0;
    m0 = 1;
    bidir = false;
    rpi = 1.0;
  }
  // smallest needed key tile index >= t, or -1 when none is left
  PIA_HD int next(int t) const {
    const long long p = (long long)t * kTileKeys;
    long long cand = -1;
    if (p <= band_hi) cand = p > band_lo ? p : band_lo;
    // the skip block of m, [i0 - m pi, last - m pi], reaches row p iff m pi <= last - p;
    // the largest such m has the leftmost block
    const long long room = last - p;
    if (room >= 0 && S >= m0) {
      long long mm = div_floor(room, pi, rpi);
      if (mm > S) mm = S;
      if (mm >= m0) {
        long long st = i0 - mm * pi;
        if (st < p) st = p;
        if (cand < 0 || st < cand) cand = st;
      }
    }
    // bidirectional: the forward block of m, [i0 + m pi, last + m pi], reaches row p iff
    // last + m pi >= p; the smallest such m has the leftmost block
    if (bidir && S >= m0) {
      long long mf = m0;
      if (p - last > (long long)m0 * pi) mf = div_floor(p - last + pi - 1, pi, rpi);  // ceil((p - last) / pi)
      if (mf <= S) {
        long long st = i0 + mf * pi;
        if (st < p) st = p;
        if (st <= n - 1 && (cand < 0 || st < cand)) cand = st;
      }
    }
    return cand < 0 ? -1 : (int)(cand / kTileKeys);
  }
};

// The same walk as an iterator: TileWalk::next's tiles in the same order, with no division per
// step.  The needed keys of the query tile are a union of intervals, taken here in ascending order
// of their starts: the backward skip blocks [i0 - m pi, last - m pi] from the largest m down to m0,
// then the window band, then (bidirectional) the forward blocks [i0 + m pi, last + m pi] from m0
// up.  Each interval covers a contiguous run of tiles; the walk is the union of those runs, each
// tile once, in increasing order.  One division at init (the largest backward m).
struct TileCursor {
  long long i0 = 0, last = -1, band_lo = 0, band_hi = -1, n = 0, pi = 1;
  int S = 0, m0 = 1;
  bool bidir = false;
  int phase = 3;  // 0: backward blocks, 1: band, 2: forward blocks, 3: none left
  int m = 0;      // next block of phase 0 or 2
  int t = -1;     // last tile returned
  int t_end = -1; // last tile of the interval being walked
  PIA_HD void init(const TileWalk& w) {
    i0 = w.i0;
    last = w.last;
    band_lo = w.band_lo;
    band_hi = w.band_hi;
    n = w.n;
    pi = w.pi;
    S = w.S;
    m0 = w.m0;
    bidir = w.bidir;
    t = -1;
    t_end = -1;
    phase = 1;
    m = 0;
    if (S >= m0 && last >= 0) {
      long long mm = div_floor(last, pi, w.rpi);  // blocks with last - m pi >= 0
      if (mm > S) mm = S;
      if (mm >= m0) {
        m = (int)mm;
        phase = 0;
      }
    }
  }
  // the next interval of needed keys [a, b] (0 <= a <= b); false when none is left
  PIA_HD bool interval(long long& a, long long& b) {
    for (;;) {
      if (phase == 0) {
        if (m < m0) {
          phase = 1;
          continue;
        }
        a = i0 - (long long)m * pi;
        if (a < 0) a = 0;
        b = last - (long long)m * pi;
        --m;
        return true;
      }
      if (phase == 1) {
        phase = bidir && S >= m0 ? 2 : 3;
        m = m0;
        if (band_lo <= band_hi) {
          a = band_lo;
          b = band_hi;
          return true;
        }
        continue;
      }
      if (phase == 2) {
        a = i0 + (long long)m * pi;
        if (m > S || a > n - 1) {
          phase = 3;
          continue;
        }
        b = last + (long long)m * pi;
        if (b > n - 1) b = n - 1;
        ++m;
        return true;
      }
      return false;
    }
  }
  // the next tile of the walk, or -1 when none is left
  PIA_HD int next() {
    if (t < t_end) return ++t;
    long long a, b;
    while (interval(a, b)) {
      int ta = (int)(a / kTileKeys);
      const int tb = (int)(b / kTileKeys);
      if (ta <= t) ta = t + 1;
      if (ta <= tb) {
        t = ta;
        t_end = tb;
        return t;
      }
    }
    t_end = t;
    return -1;
  }
};

// One query row's skip keys, in ascending order, taken tile by tile while a walk visits the key
// tiles in increasing order: the backward skips i - m pi (m from its largest value down to m0),
// then (bidirectional) the forward skips i + m pi (m from m0 up, keys below n).  Each key is
// taken by the first tile at or past it, so a walk that visits every tile holding one of the row's
// keys takes each key in its own tile.  One division per row at init, none per tile.
struct RowSkips {
  long long nb = 0, nf = 0, pi = 1;  // next backward / forward skip key
  int lb = 0, lf = 0;                // backward / forward skip keys left
  PIA_HD void init(long long i, int pi_, int S, int m0, double rpi, bool bidir, long long n) {
    pi = pi_;
    lb = lf = 0;
    nb = nf = 0;
    if (S >= m0 && i >= 0) {
      long long mb = div_floor(i, pi_, rpi);
      if (mb > S) mb = S;
      if (mb >= m0) {
        lb = (int)(mb - m0 + 1);
        nb = i - mb * pi_;
      }
    }
    if (bidir && S >= m0 && i + (long long)m0 * pi_ <= n - 1) {
      long long mf = div_floor(n - 1 - i, pi_, rpi);
      if (mf > S) mf = S;
      lf = (int)(mf - m0 + 1);
      nf = i + (long long)m0 * pi_;
    }
  }
  // bit c set for each of the row's skip keys j0 + c in the tile [j0, j0 + kTileKeys)
  PIA_HD uint64_t take(long long j0) {
    uint64_t bits = 0;
    const long long je = j0 + kTileKeys;
    for (; lb > 0 && nb < je; nb += pi, --lb)
      if (nb >= j0) bits |= 1ull << (int)(nb - j0);
    for (; lf > 0 && nf < je; nf += pi, --lf)
      if (nf >= j0) bits |= 1ull << (int)(nf - j0);
    return bits;
  }
};

// The mirror of RowSkips, for a key: the rows that read key j as a skip key, in ascending order,
// taken row tile by row tile while a walk visits the row tiles in increasing order: the
// bidirectional rule's rows j - m pi (m from its largest value down to m0), then the rows j + m pi
// (m from m0 up, rows below n).  One division per key at init, none per tile.
struct KeyReaders {
  long long nb = 0, nf = 0, pi = 1;  // next row before / after the key
  int lb = 0, lf = 0;                // rows left
  PIA_HD void init(long long j, int pi_, int S, int m0, double rpi, bool bidir, long long n) {
    pi = pi_;
    lb = lf = 0;
    nb = nf = 0;
    if (bidir && S >= m0 && j >= 0) {
      long long mb = div_floor(j, pi_, rpi);
      if (mb > S) mb = S;
      if (mb >= m0) {
        lb = (int)(mb - m0 + 1);
        nb = j - mb * pi_;
      }
    }
    if (S >= m0 && j + (long long)m0 * pi_ <= n - 1) {
      long long mf = div_floor(n - 1 - j, pi_, rpi);
      if (mf > S) mf = S;
      lf = (int)(mf - m0 + 1);
      nf = j + (long long)m0 * pi_;
    }
  }
  // bit c set for each row r0 + c in [r0, r0 + kTileKeys) that reads the key as a skip key
  PIA_HD uint64_t take(long long r0) {
    uint64_t bits = 0;
    const long long re = r0 + kTileKeys;
    for (; lb > 0 && nb < re; nb += pi, --lb)
      if (nb >= r0) bits |= 1ull << (int)(nb - r0);
    for (; lf > 0 && nf < re; nf += pi, --lf)
      if (nf >= r0) bits |= 1ull << (int)(nf - r0);
    return bits;
  }
};

// The transposed walk, for the backward: in increasing order, the row tiles (kTileKeys rows each)
// holding at least one row that reads a key of the key block [j0, jl].  Row i reads key j as a
// window key when j in L(i) -- causal: i in [j, j + k]; bidirectional: |i - j| <= k -- and as a
// skip key when i = j + m pi (and, bidirectional, i = j - m pi) for m0 <= m <= S.
struct ReaderWalk {
  long long j0 = 0, jl = -1, w_lo = 0, w_hi = -1, n = 0;  // key block; rows reading it as window keys
  int pi = 1, S = 0, m0 = 1;
  bool bidir = false;
  double rpi = 1.0;
  PIA_HD void init(long long j0_, long long n_, int keys, int kwin, int pi_, int S_, bool bidir_ = false) {
    j0 = j0_;
    n = n_;
    jl = j0_ + keys - 1 < n_ - 1 ? j0_ + keys - 1 : n_ - 1;
    w_lo = bidir_ ? (j0_ - kwin > 0 ? j0_ - kwin : 0) : j0_;
    w_hi = jl + kwin < n_ - 1 ? jl + kwin : n_ - 1;
    pi = pi_;
    S = S_;
    m0 = kwin / pi_ + 1;
    bidir = bidir_;
    rpi = 1.0 / (double)pi_;
  }
  // The residue-class view: keys j0 .. j0 + keys - 1 of a class of T rows, key u read (as a skip
  // key) by the rows u + m0 .. u + S of the same class
  PIA_HD void init_residue(long long j0_, long long T, int keys, int S_, int m0_) {
    j0 = j0_;
    n = T;
    jl = j0_ + keys - 1 < T - 1 ? j0_ + keys - 1 : T - 1;
    w_lo = j0_ + m0_;
    w_hi = jl + S_ < T - 1 ? jl + S_ : T - 1;
    if (w_lo > w_hi || S_ < m0_) w_hi = -1;  // no reader at all
    pi = 1;
    S = 0;
    m0 = 1;
    bidir = false;
    rpi = 1.0;
  }
  // smallest reading row tile index >= t, or -1 when none is left
  PIA_HD int next(int t) const {
    const long long p = (long long)t * kTileKeys;
    long long cand = -1;
    if (p <= w_hi) cand = p > w_lo ? p : w_lo;
    if (S >= m0) {
      // rows after the block, [j0 + m pi, jl + m pi]: the smallest m with jl + m pi >= p
      long long mf = m0;
      if (p - jl > (long long)m0 * pi) mf = div_floor(p - jl + pi - 1, pi, rpi);
      if (mf <= S) {
        long long st = j0 + mf * pi;
        if (st < p) st = p;
        if (st <= n - 1 && (cand < 0 || st < cand)) cand = st;
      }
      // bidirectional: rows before the block, [j0 - m pi, jl - m pi]: the largest m with
      // jl - m pi >= p has the leftmost block
      if (bidir && jl - p >= 0) {
        long long mb = div_floor(jl - p, pi, rpi);
        if (mb > S) mb = S;
        if (mb >= m0) {
          long long st = j0 - mb * pi;
          if (st < p) st = p;
          if (cand < 0 || st < cand) cand = st;
        }
      }
    }
    return cand < 0 ? -1 : (int)(cand / kTileKeys);
  }
};

// For query row i and the key tile starting at j0: window columns [lc_lo, lc_hi] (empty when
// lc_lo > lc_hi) and a bitmask of skip columns (kTileKeys bits).  Skip columns never overlap the window.
// The window of row i is [max(0, i - kwin), i - lo_off]: lo_off = 0 for pi-attention's window;
// the residue-class pass uses it for the skip band of a residue sequence (kwin = S, lo_off = m0,
// no skips).  rpi = 1.0 / pi.
PIA_HD void row_tile_mask(long long i, long long j0, int kwin, int pi, int S, int m0, int& lc_lo, int& lc_hi,
                          uint32_t sk[kTileKeys / 32], int lo_off = 0, double rpi = 0.0, bool bidir = false,
                          long long n = 0) {
  const long long d0 = i - j0;  // i - j at column 0
  const long long lo = (i - kwin > 0 ? i - kwin : 0) - j0;
  const long long hi = bidir ? (i + kwin < n - 1 ? i + kwin : n - 1) - j0 : d0 - lo_off;
  lc_lo = lo < 0 ? 0 : (lo > kTileKeys ? kTileKeys : (int)lo);
  lc_hi = hi > kTileKeys - 1 ? kTileKeys - 1 : (hi < -1 ? -1 : (int)hi);
  static_assert(kTileKeys == 64, "one 64-bit word of skip bits per tile");
  uint64_t bits = 0;  // a register word: an array indexed by c >> 5 would live in local memory
  if (d0 > kwin && S >= m0) {
    // skip columns c = d0 - m pi in 0..kTileKeys-1: from the largest m (smallest c) upwards in c
    long long m = div_floor(d0, pi, rpi > 0.0 ? rpi : 1.0 / (double)pi);
    if (m > S) m = S;
    for (long long c = d0 - m * pi; m >= m0 && c < kTileKeys; --m, c += pi) {
      if (c >= 0) bits |= 1ull << (int)c;
    }
  }
  if (bidir && S >= m0) {
    // forward skip columns c = d0 + m pi (key i + m pi < n) in 0..kTileKeys-1, from the smallest m
    long long m = m0;
    if (-d0 > (long long)m0 * pi) m = div_floor(-d0 + pi - 1, pi, rpi > 0.0 ? rpi : 1.0 / (double)pi);
    for (long long c = d0 + m * pi; m <= S && c < kTileKeys && i + m * pi <= n - 1; ++m, c += pi) {
      if (c >= 0) bits |= 1ull << (int)c;
    }
  }
  sk[0] = (uint32_t)bits;
  sk[1] = (uint32_t)(bits >> 32);
}

// Bits of the window columns [lo, hi] (relative to a 32-column chunk) that fall in 0..31.
PIA_HD uint32_t window_bits(int lo, int hi) {
  if (lo > 31 || hi < 0 || lo > hi) return 0u;
  const int a = lo < 0 ? 0 : lo, b = hi > 31 ? 31 : hi;
  return (b == 31 ? 0xFFFFFFFFu : ((1u << (b + 1)) - 1u)) & ~((1u << a) - 1u);
}

// Cheapest exact treatment of a 32-column chunk cb of a tile for one row:
//   kEmpty  no key of the union: p = 0, no exponential
//   kFull   every column a window key and no skip: one FMA per logit
//   kOne    exactly one skip key and no window key: one exponential for the chunk
//   kMixed  anything else: per-column mask
enum : int { kEmpty = 0, kFull = 1, kOne = 2, kMixed = 3 };
PIA_HD int chunk_class(int cb, int lc_lo, int lc_hi, uint32_t skb) {
  const int c0 = cb * 32;
  const bool any_loc = lc_lo <= c0 + 31 && lc_hi >= c0 && lc_lo <= lc_hi;
  const bool all_loc = lc_lo <= c0 && lc_hi >= c0 + 31;
  if (!any_loc && skb == 0u) return kEmpty;
  if (all_loc && skb == 0u) return kFull;
  if (!any_loc && (skb & (skb - 1u)) == 0u) return kOne;
  return kMixed;
}

}  // namespace pia
