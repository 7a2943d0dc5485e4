// Static tile schedule of the grouped tensor-core product kernels (and one epilogue helper they
// share). A launch is a list of independent problems; problem p owns the tile indices
// [tile_begin, tile_begin + n_tiles), and the persistent grid walks the tile index with a stride
// of the number of CTAs (or pairs).
#pragma once
#include <stdint.h>

namespace muon {

constexpr uint32_t kGroupM = 8;   // row blocks that sweep the column blocks together (L2 reuse)

struct Tile {
  int p;            // problem
  uint32_t bi, bj;  // row block, column block
};

// Problem and block coordinates of global tile t. A symmetric problem enumerates, row block by
// row block, only the tiles that touch the upper triangle: row block bi covers rows
// [TILE_M bi, TILE_M (bi + 1)), and its first such column block is (TILE_M bi) / TILE_N.
template <int TILE_M, int TILE_N, class Prob>
__device__ __forceinline__ Tile decode_tile(const Prob* __restrict__ probs, int nprobs, uint32_t t) {
  int lo = 0, hi = nprobs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (probs[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
  }
  const Prob& P = probs[lo];
  uint32_t l = t - P.tile_begin;
  Tile tl;
  tl.p = lo;
  if (P.sym) {
    uint32_t bi = 0;
    while (true) {
      const uint32_t first = (bi * TILE_M) / TILE_N;
      const uint32_t cnt = P.tiles_n - first;
      if (l < cnt) { tl.bi = bi; tl.bj = first + l; break; }
      l -= cnt;
      ++bi;
    }
  } else {
    const uint32_t per_group = kGroupM * P.tiles_n;
    const uint32_t g = l / per_group;
    const uint32_t first = g * kGroupM;
    const uint32_t gsize = min(kGroupM, P.tiles_m - first);
    const uint32_t r = l - g * per_group;
    tl.bi = first + r % gsize;
    tl.bj = r / gsize;
  }
  return tl;
}

// alpha^e for the small exponents of the epilogue scalars (e = 0, 1, 2)
__device__ __forceinline__ float alpha_pow(float alpha, int e) {
  float s = 1.0f;
  for (int i = 0; i < e; ++i) s *= alpha;
  return s;
}

}  // namespace muon
