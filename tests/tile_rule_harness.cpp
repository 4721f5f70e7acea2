// CPU harness for the tensor-core kernel's index logic (csrc/tile_rule.cuh compiled with g++).
// For query rows 0..n-1 it replays what the kernel does -- walk the key tiles of the row's query
// tile, unmask window columns and skip bits, classify 32-column chunks -- and reports the keys
// that survive, in the oracle's index-table layout, plus consistency counters.
#include <cstdint>
#include <cstring>

#include "../periodic_sparse_attention_b200/csrc/tile_rule.cuh"

using namespace pia;

extern "C" int tile_rule_sets(int n, int kwin, int pi, int S, int bidir, int width, int32_t* counts, int32_t* idx,
                              int64_t* stats) {
  // stats: [0] tiles visited, [1] keys counted twice, [2] chunk-class violations,
  //        [3] tiles visited out of order
  for (int s = 0; s < 4; ++s) stats[s] = 0;
  const int BM = 128;
  for (long long i0 = 0; i0 < n; i0 += BM) {
    TileWalk w;
    w.init(i0, n, BM, kwin, pi, S, bidir != 0);
    int prev = -1;
    for (int t = w.next(0); t >= 0; t = w.next(t + 1)) {
      stats[0]++;
      if (t <= prev) stats[3]++;
      prev = t;
    }
    for (long long i = i0; i < i0 + BM && i < n; ++i) {
      int32_t* row = idx + i * width;
      int nl = 0, np = 0;
      // window keys ascending, skip keys collected then written by increasing m (descending j)
      int32_t skip_keys[4096];
      for (int t = w.next(0); t >= 0; t = w.next(t + 1)) {
        const long long j0 = (long long)t * kTileKeys;
        int lo, hi;
        uint32_t sk[kTileKeys / 32];
        row_tile_mask(i, j0, kwin, pi, S, w.m0, lo, hi, sk, 0, 0.0, bidir != 0, n);
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
