// CPU harness for the tensor-core kernel's index logic (csrc/tile_rule.cuh compiled with g++).
// For query rows 0..n-1 it replays what the kernel does -- walk the key tiles of the row's query
// tile, unmask window columns and skip bits, classify 32-column chunks -- and reports the keys
// that survive, in the oracle's index-table layout, plus consistency counters.
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <vector>

#include "../periodic_sparse_attention_b200/csrc/tile_rule.cuh"

using namespace pia;

extern "C" int tile_rule_sets(int n, int kwin, int pi, int S, int bidir, int width, int32_t* counts, int32_t* idx,
                              int64_t* stats) {
  // stats: [0] tiles visited, [1] keys counted twice, [2] chunk-class violations,
  //        [3] tiles visited out of order, [4] TileCursor steps that differ from TileWalk::next,
  //        [5] tiles where RowSkips and row_tile_mask give different skip bits
  // The keys reported are the tensor-core kernel's: tiles from TileCursor, skip bits from
  // RowSkips, window columns from the row's window bounds.
  for (int s = 0; s < 6; ++s) stats[s] = 0;
  const int BM = 128;
  for (long long i0 = 0; i0 < n; i0 += BM) {
    TileWalk w;
    w.init(i0, n, BM, kwin, pi, S, bidir != 0);
    int prev = -1;
    TileCursor cc;
    cc.init(w);
    for (int t = w.next(0); t >= 0; t = w.next(t + 1)) {
      stats[0]++;
      if (t <= prev) stats[3]++;
      prev = t;
      if (cc.next() != t) stats[4]++;
    }
    if (cc.next() != -1 || cc.next() != -1) stats[4]++;
    for (long long i = i0; i < i0 + BM && i < n; ++i) {
      int32_t* row = idx + i * width;
      int nl = 0, np = 0;
      // window keys ascending, skip keys collected then written by increasing m (descending j)
      int32_t skip_keys[4096];
      TileCursor cur;
      cur.init(w);
      RowSkips rs;
      rs.init(i, pi, S, w.m0, w.rpi, bidir != 0, n);
      const long long w_lo = i - kwin > 0 ? i - kwin : 0;
      const long long w_hi = bidir ? (i + kwin < n - 1 ? i + kwin : n - 1) : i;
      for (int t = cur.next(); t >= 0; t = cur.next()) {
        const long long j0 = (long long)t * kTileKeys;
        int lo, hi;
        uint32_t sk[kTileKeys / 32];
        row_tile_mask(i, j0, kwin, pi, S, w.m0, lo, hi, sk, 0, 0.0, bidir != 0, n);
        const uint64_t bits = rs.take(j0);
        if ((uint32_t)bits != sk[0] || (uint32_t)(bits >> 32) != sk[1]) stats[5]++;
        sk[0] = (uint32_t)bits;
        sk[1] = (uint32_t)(bits >> 32);
        const long long lo64 = w_lo - j0, hi64 = w_hi - j0;
        if ((lo64 < 0 ? 0 : (lo64 > kTileKeys ? kTileKeys : lo64)) != lo ||
            (hi64 > kTileKeys - 1 ? kTileKeys - 1 : (hi64 < -1 ? -1 : hi64)) != hi)
          stats[5]++;
        for (int cb = 0; cb < kTileKeys / 32; ++cb) {
          const int cls = chunk_class(cb, lo, hi, sk[cb]);
          int valid = 0, loc_cnt = 0, skp_cnt = 0;
          for (int e = 0; e < 32; ++e) {
            const int c = cb * 32 + e;
            const bool loc = c >= lo && c <= hi;
            const bool skp = (sk[cb] >> e) & 1u;
            if (loc && skp) stats[1]++;
            if (loc) {
              if (nl < width) row[nl] = (int32_t)(j0 + c);
              ++nl;
              ++loc_cnt;
            }
            if (skp) {
              if (np < 4096) skip_keys[np] = (int32_t)(j0 + c);
              ++np;
              ++skp_cnt;
            }
            valid += loc || skp;
          }
          const bool okc = (cls == kEmpty && valid == 0) || (cls == kFull && loc_cnt == 32 && skp_cnt == 0) ||
                           (cls == kOne && loc_cnt == 0 && skp_cnt == 1) || cls == kMixed;
          if (!okc) stats[2]++;
        }
      }
      // window keys were produced ascending; skips ascending in j -> causal: write by increasing m
      // (descending j); bidirectional: ascending j (the test compares the skip keys as a set)
      int wpos = nl;
      if (bidir)
        for (int s = 0; s < np && wpos < width; ++s) row[wpos++] = skip_keys[s];
      else
        for (int s = np - 1; s >= 0 && wpos < width; --s) row[wpos++] = skip_keys[s];
      while (wpos < width) row[wpos++] = -1;
      counts[2 * i] = nl;
      counts[2 * i + 1] = np;
    }
  }
  return 0;
}

// The transposed walk: for each key block of kTileKeys keys, the row tiles ReaderWalk visits
// (tiles[b * maxper + s], counts[b]); returns 1 if any block visited tiles out of order.
extern "C" int reader_walk_tiles(int n, int kwin, int pi, int S, int bidir, int maxper, int32_t* tiles,
                                 int32_t* counts) {
  int bad = 0;
  const int nb = (n + kTileKeys - 1) / kTileKeys;
  for (int b = 0; b < nb; ++b) {
    ReaderWalk w;
    w.init((long long)b * kTileKeys, n, kTileKeys, kwin, pi, S, bidir != 0);
    int c = 0, prev = -1;
    for (int t = w.next(0); t >= 0; t = w.next(t + 1)) {
      if (t <= prev) bad = 1;
      prev = t;
      if (c < maxper) tiles[b * maxper + c] = t;
      ++c;
    }
    counts[b] = c;
  }
  return bad;
}

// A walk built field by field (as the residue-class pass builds its own): the number of steps at
// which TileCursor and TileWalk::next disagree, over the whole walk.
extern "C" int cursor_vs_walk(long long i0, long long last, long long band_lo, long long band_hi, long long n, int pi,
                              int S, int m0, int bidir) {
  TileWalk w;
  w.i0 = i0;
  w.last = last;
  w.band_lo = band_lo;
  w.band_hi = band_hi;
  w.n = n;
  w.pi = pi;
  w.S = S;
  w.m0 = m0;
  w.bidir = bidir != 0;
  w.rpi = 1.0 / (double)pi;
  TileCursor c;
  c.init(w);
  int bad = 0, steps = 0;
  for (int t = w.next(0); t >= 0 && steps < 100000; t = w.next(t + 1), ++steps)
    if (c.next() != t) ++bad;
  if (c.next() != -1) ++bad;
  return bad;
}

// The backward's key-side view: for key blocks of `keys` keys, walk the reading row tiles with
// ReaderWalk and take each key's reading rows with its window range and KeyReaders; report for
// every (row, key) pair that the rule connects whether the walk produced it as the right kind
// (window or skip), and count pairs produced that the rule does not connect.  reads[i * n + j]:
// 0 none, 1 window, 2 skip, as the oracle's index sets give them (filled by the caller).
extern "C" int key_side_mismatches(int n, int kwin, int pi, int S, int bidir, int keys, const int8_t* reads) {
  int bad = 0;
  const int m0 = kwin / pi + 1;
  for (long long j0 = 0; j0 < n; j0 += keys) {
    ReaderWalk w;
    w.init(j0, n, keys, kwin, pi, S, bidir != 0);
    for (long long j = j0; j < j0 + keys && j < n; ++j) {
      KeyReaders kr;
      kr.init(j, pi, S, m0, w.rpi, bidir != 0, n);
      const long long wlo = bidir ? (j - kwin > 0 ? j - kwin : 0) : j;
      const long long whi = j + kwin < n - 1 ? j + kwin : n - 1;
      std::vector<int8_t> seen(n, 0);
      for (int t = w.next(0); t >= 0; t = w.next(t + 1)) {
        const long long r0 = (long long)t * kTileKeys;
        const uint64_t sk = kr.take(r0);
        for (int c = 0; c < kTileKeys; ++c) {
          const long long i = r0 + c;
          if (i >= n) break;
          const bool win = i >= wlo && i <= whi;
          const bool skp = (sk >> c) & 1ull;
          if (win && skp) ++bad;
          if (win) seen[i] = 1;
          if (skp) seen[i] = 2;
        }
      }
      for (long long i = 0; i < n; ++i)
        if (seen[i] != reads[i * n + j]) ++bad;
    }
  }
  return bad;
}

// The residue-class view's walks, against brute force over one class of T rows: the query walk of
// the rows [q0, q0 + rows) (row t reads keys t - S .. t - m0, clipped at 0) and the reader walk of
// the keys [j0, j0 + rows) (key u read by rows u + m0 .. u + S, clipped below T).  Returns the
// number of tiles produced or missed wrongly, over every block of the class.
extern "C" int residue_walk_mismatches(long long T, int S, int m0, int rows) {
  int bad = 0;
  const long long ntiles = (T + kTileKeys - 1) / kTileKeys;
  std::vector<char> want(ntiles), got(ntiles);
  for (long long b0 = 0; b0 < T; b0 += rows) {
    const long long b1 = b0 + rows < T ? b0 + rows : T;  // block [b0, b1)
    // query side
    std::fill(want.begin(), want.end(), 0);
    std::fill(got.begin(), got.end(), 0);
    for (long long t = b0; t < b1; ++t)
      for (long long key = t - S; key <= t - m0; ++key)
        if (key >= 0) want[key / kTileKeys] = 1;
    TileWalk w;
    w.init_residue(b0, T, rows, S, m0);
    TileCursor c;
    c.init(w);
    int steps = 0;
    for (int t = c.next(); t >= 0 && steps < 100000; t = c.next(), ++steps) {
      if (t >= ntiles || got[t]) ++bad;
      else got[t] = 1;
    }
    for (long long t = 0; t < ntiles; ++t) bad += want[t] != got[t];
    // key side
    std::fill(want.begin(), want.end(), 0);
    std::fill(got.begin(), got.end(), 0);
    for (long long u = b0; u < b1; ++u)
      for (long long r = u + m0; r <= u + S; ++r)
        if (r < T) want[r / kTileKeys] = 1;
    ReaderWalk rw;
    rw.init_residue(b0, T, rows, S, m0);
    steps = 0;
    for (int t = rw.next(0); t >= 0 && steps < 100000; t = rw.next(t + 1), ++steps) {
      if (t >= ntiles || got[t]) ++bad;
      else got[t] = 1;
    }
    for (long long t = 0; t < ntiles; ++t) bad += want[t] != got[t];
  }
  return bad;
}

// The bidirectional residue-class walk (the forward's split of the two-sided rule): rows [q0,
// q0 + rows) of a class of T rows, row t reading keys t - S .. t - m0 and t + m0 .. t + S within
// [0, T).  The walk covers the union of the rows' key ranges as one band; it may also walk the few
// tiles between the two bands of a short block (every row masks them out).  Returns the number of
// needed tiles missed, tiles walked twice, and tiles walked outside [q0 - S, last row + S].
extern "C" int residue_walk_bidir_errors(long long T, int S, int m0, int rows) {
  int bad = 0;
  const long long ntiles = (T + kTileKeys - 1) / kTileKeys;
  std::vector<char> want(ntiles), got(ntiles);
  for (long long b0 = 0; b0 < T; b0 += rows) {
    const long long b1 = b0 + rows < T ? b0 + rows : T;
    std::fill(want.begin(), want.end(), 0);
    std::fill(got.begin(), got.end(), 0);
    for (long long t = b0; t < b1; ++t)
      for (long long m = m0; m <= S; ++m) {
        if (t - m >= 0) want[(t - m) / kTileKeys] = 1;
        if (t + m < T) want[(t + m) / kTileKeys] = 1;
      }
    TileWalk w;
    w.init_residue(b0, T, rows, S, m0, true);
    TileCursor c;
    c.init(w);
    const long long lo = b0 - S < 0 ? 0 : b0 - S, hi = b1 - 1 + S < T - 1 ? b1 - 1 + S : T - 1;
    int steps = 0;
    for (int t = c.next(); t >= 0 && steps < 100000; t = c.next(), ++steps) {
      if (t >= ntiles || got[t]) ++bad;
      else got[t] = 1;
      if ((long long)(t + 1) * kTileKeys - 1 < lo || (long long)t * kTileKeys > hi) ++bad;
    }
    for (long long t = 0; t < ntiles; ++t) bad += want[t] && !got[t];
  }
  return bad;
}
