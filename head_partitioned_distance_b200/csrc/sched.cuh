// sched.cuh -- band tile scheduler, evaluated identically on host and device.
//
// Head h attends to causal distances in its band [lo, hi) (Balanced Distance
// Partitioning, "Making Every Head Count", Figure 1 caption).  A query tile
// of rows [i0, i0 + Bq) therefore needs only the keys of one diagonal strip:
//   j in [max(0, i0 - hi + 1), i1 - lo],   i1 = min(i0 + Bq, N) - 1,
// and a key tile of keys [j0, j0 + Bk) is reached only by the queries
//   i in [j0 + lo, min(j1 + hi - 1, N - 1)],   j1 = min(j0 + Bk, N) - 1.
// Every tile inside such a range holds at least one permitted element
// (consecutive rows shift the strip by one key and each band is at least one
// wide, so the strips of the rows of a tile overlap into one interval).
//
// A tile is "interior" when all of its Bq x Bk elements are permitted: it lies
// wholly inside [0, N) and its smallest and largest distances
// i0 - (j0 + Bk - 1) and (i0 + Bq - 1) - j0 both fall in [lo, hi).  Interior
// tiles skip the per-element predicate; every other tile in a strip is an
// "edge" tile.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define SPA_HD __host__ __device__ __forceinline__
#else
#define SPA_HD inline
#endif

namespace spa {

enum TileClass : uint8_t { kTileNone = 0, kTileEdge = 1, kTileInterior = 2 };

SPA_HD int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
SPA_HD int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Band of head h under Balanced Distance Partitioning, 64-bit arithmetic.
SPA_HD void band_of_head(int64_t N, int64_t H, int64_t h, int32_t* lo, int32_t* hi) {
  *lo = (int32_t)((h * N) / H);
  *hi = (int32_t)(((h + 1) * N) / H);
}

struct Strip {
  int32_t begin;  // first tile index
  int32_t end;    // last tile index (inclusive); end < begin means no tile
};

// Key tiles that query tile [i0, i0 + Bq) walks.
SPA_HD Strip key_strip(int64_t N, int32_t lo, int32_t hi, int64_t i0, int Bq, int Bk) {
  Strip s{0, -1};
  int64_t i1 = min64(i0 + Bq, N) - 1;
  if (i1 < (int64_t)lo) return s;  // every row precedes the band: empty unit
  int64_t jlo = max64(0, i0 - (int64_t)hi + 1);
  int64_t jhi = i1 - lo;
  s.begin = (int32_t)(jlo / Bk);
  s.end = (int32_t)(jhi / Bk);
  return s;
}

// Query tiles that key tile [j0, j0 + Bk) is reached by.
SPA_HD Strip query_strip(int64_t N, int32_t lo, int32_t hi, int64_t j0, int Bk, int Bq) {
  Strip s{0, -1};
  int64_t ilo = j0 + lo;
  if (ilo > N - 1) return s;  // no query reaches these keys
  int64_t j1 = min64(j0 + Bk, N) - 1;
  int64_t ihi = min64(j1 + (int64_t)hi - 1, N - 1);
  s.begin = (int32_t)(ilo / Bq);
  s.end = (int32_t)(ihi / Bq);
  return s;
}

// Class of a tile known to lie inside a strip.
SPA_HD bool tile_is_interior(int64_t N, int32_t lo, int32_t hi, int64_t i0, int Bq, int64_t j0,
                             int Bk) {
  return (i0 + Bq <= N) && (j0 + Bk <= N) && (i0 - (j0 + Bk - 1) >= (int64_t)lo) &&
         ((i0 + Bq - 1) - j0 < (int64_t)hi);
}

// Class of any tile (t, u).
SPA_HD uint8_t tile_class(int64_t N, int32_t lo, int32_t hi, int t, int Bq, int u, int Bk) {
  Strip s = key_strip(N, lo, hi, (int64_t)t * Bq, Bq, Bk);
  if (u < s.begin || u > s.end) return kTileNone;
  return tile_is_interior(N, lo, hi, (int64_t)t * Bq, Bq, (int64_t)u * Bk, Bk) ? kTileInterior
                                                                                : kTileEdge;
}

}  // namespace spa
