// fa_band.cuh -- which key/value tiles a query tile visits, and the reverse, for the
// masks the kernels support (host and device code share these).
//
// Every mask is a key window around the bottom-right diagonal: with off = Nk - Nq,
// query q sees key k iff q + off - wl <= k <= q + off + wr (and 0 <= k < Nk). The
// unmasked case is wl = wr = kUnbounded; the causal mask is wl = kUnbounded, wr = 0;
// a sliding window bounds either side (josueisai.com "flash-attention", section "Que
// ganas y que no", names window attention as the combination for very long
// sequences). Tiles outside the band are never loaded or multiplied; tiles across
// an edge of the band are masked element by element.
#pragma once

namespace fa {

// An edge at least this far from the diagonal bounds nothing (the host clamps every
// window to this, and keeps Nq + Nk below it, so no sum here overflows 32 bits).
constexpr int kUnbounded = 1 << 30;

// Element strides of a 16-bit [B][H][N][d] or [B][N][H][d] tensor: element (b, h, n, t)
// sits at b * sb + h * sh + n * sn + t.
struct Strides {
  long sb, sh, sn;
};

struct TileRange {
  int first;  // first tile index
  int count;  // number of consecutive tiles (0: none)
};

// Key/value tiles (of `tile` keys) that query tile t (rows t*tile .. t*tile+tile-1,
// the last possibly past Nq) has to visit: the union of its rows' windows.
__host__ __device__ inline TileRange kv_tiles_of_query_tile(int t, int tile, int Nq, int Nk,
                                                            int wl, int wr) {
  const int off = Nk - Nq;
  const int q0 = t * tile;
  const int q1 = t * tile + tile - 1 < Nq - 1 ? t * tile + tile - 1 : Nq - 1;  // last real row
  const int lo = q0 + off - wl;  // smallest key any row of the tile sees
  const int hi = q1 + off + wr;  // largest
  const int klo = lo < 0 ? 0 : lo;
  const int khi = hi > Nk - 1 ? Nk - 1 : hi;
  if (klo > khi) return {0, 0};
  return {klo / tile, khi / tile - klo / tile + 1};
}

// Query tiles whose rows see at least one key of key tile j (rows of the last query
// tile past Nq included: they are padding and see what the window gives them).
__host__ __device__ inline TileRange query_tiles_of_kv_tile(int j, int tile, int Nq, int Nk,
                                                            int wl, int wr) {
  const int off = Nk - Nq;
  const int k0 = j * tile;
  const int k1 = j * tile + tile - 1 < Nk - 1 ? j * tile + tile - 1 : Nk - 1;
  const int lo = k0 - off - wr;  // smallest query that sees key k0 .. k1
  const int hi = k1 - off + wl;  // largest
  const int ntq = (Nq + tile - 1) / tile;
  const int qlo = lo < 0 ? 0 : lo;
  const int qhi = hi > ntq * tile - 1 ? ntq * tile - 1 : hi;
  if (qlo > qhi) return {0, 0};
  return {qlo / tile, qhi / tile - qlo / tile + 1};
}

// Order of the work items of a launch with a band (whose items differ in cost): block b
// -> (head bh, rank), rank 0 being each head's heaviest item. Heads go in groups of
// `group`; within a group the items are rank-major, so that every head's heavy items
// start early and the launch ends on light ones (no heavy item left to run alone at
// the end), while the heads in flight at once stay few enough for the tensors they
// stream to share L2. group = 1 is plain head-major order.
__host__ __device__ inline void band_order(int b, int per_head, int BH, int group, int* bh,
                                           int* rank) {
  const int span = group * per_head;
  const int g = b / span;
  const int gg = BH - g * group < group ? BH - g * group : group;  // heads in this group
  const int idx = b - g * span;
  *rank = idx / gg;
  *bh = g * group + (idx - *rank * gg);
}

// Heads per group for band_order: at least `min_groups` groups, and more when a group's
// bytes -- what its heads' work items share through L2: the tensors they stream, and
// in the backward the fp32 dQ accumulator they add into -- would exceed `budget` bytes
// of the 126 MB L2; the groups as even as the head count allows, and never above the
// budget. The forward kernels take at least three groups within 88 MiB: their heaviest
// item (a causal head's last query tiles) runs ~12 % of a launch, and with three groups
// the last group's heaviest items still start early enough to end with it (with more,
// smaller groups they start near the end and run on alone); a group of 88 MiB of K and
// V (22 heads at N = 8192, d = 128) is read from DRAM once, while groups of 96 MiB read
// it about twice. The dK/dV kernel, whose heaviest item runs ~5 % of a launch, takes
// groups within 48 MiB.
inline int band_group(long BH, long bytes_per_head, long min_groups, long budget) {
  if (BH <= 1) return 1;
  long ng = (BH * bytes_per_head + budget - 1) / budget;
  if (ng < min_groups) ng = min_groups;
  if (ng > BH) ng = BH;
  long g = (BH + ng - 1) / ng;
  if (bytes_per_head > 0) {
    const long cap = budget / bytes_per_head > 1 ? budget / bytes_per_head : 1;
    if (g > cap) g = cap;
  }
  return static_cast<int>(g);
}
constexpr long kFwdGroupMin = 3;
constexpr long kFwdGroupBytes = 88L << 20;
constexpr long kBwdGroupMin = 1;
constexpr long kBwdGroupBytes = 48L << 20;

}  // namespace fa
