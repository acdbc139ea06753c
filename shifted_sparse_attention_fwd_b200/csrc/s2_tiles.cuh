// The per-head shift-and-group remap, applied to 128-row tiles.
//
// LongLoRA summary page, §3.4 Algorithm 1: the second chunk of heads is rolled by -G/2
// along N before the attention, cut into independent groups of G consecutive rolled rows,
// attended causally per group, and rolled back after it. Instead of materialising the roll, every kernel
// addresses the original tensors through
//     t = (r + s_h) mod N          (rolled row r -> original token t)
// where s_h is the head's roll (G/2 for the shifted heads, 0 otherwise); group of rolled
// row r is floor(r / G). Tiles are 128 consecutive rolled rows; such a tile maps onto at
// most two contiguous runs of original rows (the run that reaches token N-1 and the run
// that wraps to token 0; three with the Variant 3 reordering), plus zero rows past the end
// of the sequence.
#pragma once

#ifndef __CUDACC__
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace s2 {

constexpr int kTileRows = 128;

// (b, head, group) instances whose tiles the persistent kernels take together: the K/V (or
// Q/dO) tiles of about this many groups stay resident in L2 while their work runs.
constexpr int kL2Chunk = 10;

// No split of the wrap group (see group_begin).
constexpr int kNoWrapSplit = 0x7fffffff;

// The remap of one head. Rolled row r holds original token
//     t = (r + shift) mod N                                   (Algorithm 1's roll)
// and, with `front` (the pages' Variant 3, Table 8: the wrapped tokens swap places with the
// front of the last group), the last rolled group [N - G, N) lists tokens 0..shift-1 first
// and N - G + shift..N - 1 after them:
//     t = r + shift        for r < N - G
//     t = r - (N - G)      for N - G <= r < N - G + shift
//     t = r                for r >= N - G + shift.
// Both are piecewise t = r + const over at most three ranges of r, and so is the inverse.
struct HeadRemap {
  int N, G, shift, front;
  __host__ __device__ __forceinline__ int token(int r) const {
    if (front) return r < N - G ? r + shift : (r < N - G + shift ? r - (N - G) : r);
    const int t = r + shift;
    return t >= N ? t - N : t;
  }
  __host__ __device__ __forceinline__ int rolled(int t) const {
    if (front) return t < shift ? t + (N - G) : (t < N - G + shift ? t - shift : t);
    const int r = t - shift;
    return r < 0 ? r + N : r;
  }
  // Rows where token(r) (rolled(t) when `inverse`) stops being r + const.
  __host__ __device__ __forceinline__ int breaks(bool inverse, int (&br)[2]) const {
    if (shift == 0) return 0;
    if (!front) {
      br[0] = inverse ? shift : N - shift;
      return 1;
    }
    br[0] = inverse ? shift : N - G;
    br[1] = N - G + shift;
    return 2;
  }
};

__host__ __device__ __forceinline__ HeadRemap head_remap(int N, int G, int shift, int front) {
  HeadRemap m;
  m.N = N;
  m.G = G;
  m.shift = shift;
  m.front = shift > 0 ? front : 0;
  return m;
}

// Rows [x0, x0 + len) (clipped to the sequence) of one side of the remap as at most three
// runs, each contiguous on the other side: row x0 + base_k + i maps to src[k] + i for
// i < len[k], base_k = len[0] + ... + len[k-1]. Rows [valid, len) of the range are past the
// end of the sequence.
struct Runs {
  int n, valid;
  int len[3], src[3];
};
// (Loops over the three slots are unrolled with constant indices so the arrays stay in
// registers.)
__host__ __device__ inline Runs remap_runs(const HeadRemap& m, bool inverse, int x0, int len) {
  Runs t;
  t.n = 0;
  t.valid = m.N - x0 < len ? m.N - x0 : len;
  if (!m.front) {
    // the plain roll: the run that reaches the end of the sequence, then the one that wraps
    const int sh = inverse ? (m.shift == 0 ? 0 : m.N - m.shift) : m.shift;
    const int s0 = x0 + sh >= m.N ? x0 + sh - m.N : x0 + sh;
    const int first = t.valid < m.N - s0 ? t.valid : m.N - s0;
    t.n = first < t.valid ? 2 : 1;
    t.len[0] = first;
    t.src[0] = s0;
    t.len[1] = t.valid - first;
    t.src[1] = 0;
    t.len[2] = 0;
    t.src[2] = 0;
    return t;
  }
  int br[2] = {0, 0};
  const int nb = m.breaks(inverse, br);
  const int end = x0 + t.valid;
  int pos = x0;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    t.len[k] = 0;
    t.src[k] = 0;
    if (pos < end) {
      int nxt = end;
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (i < nb && br[i] > pos && br[i] < nxt) nxt = br[i];
      t.len[k] = nxt - pos;
      t.src[k] = inverse ? m.rolled(pos) : m.token(pos);
      t.n = k + 1;
      pos = nxt;
    }
  }
  return t;
}
// The 128-row rolled tile at r0 as runs of original tokens (tile loads, output rows).
__host__ __device__ inline Runs rolled_runs(const HeadRemap& m, int r0) {
  return remap_runs(m, false, r0, kTileRows);
}
// The original tile [t0, t0 + 128) as runs of rolled rows.
__host__ __device__ inline Runs token_runs(const HeadRemap& m, int t0) {
  return remap_runs(m, true, t0, kTileRows);
}
// The original tile [t0, t0 + 128) itself (a single run).
__host__ __device__ inline Runs identity_runs(int t0, int N) {
  Runs t;
  t.n = 1;
  t.valid = N - t0 < kTileRows ? N - t0 : kTileRows;
  t.len[0] = t.valid;
  t.src[0] = t0;
  return t;
}

// TMA moves whole 8-row atoms (one 128-byte swizzle period). An atom that holds rows of two
// different runs (a run boundary that is not a multiple of 8 rows into the tile, which happens
// when G or the roll is not a multiple of 8) cannot be one box: bit a of the result marks such an
// atom a. The kernels load the rows of these atoms with plain loads instead.
__host__ __device__ inline unsigned int straddled_atoms(const Runs& tr) {
  unsigned int m = 0;
  int end = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    end += tr.len[k];
    if (k + 1 < tr.n && (end & 7)) m |= 1u << (end >> 3);
  }
  return m;
}
// The atoms of a 128-row tile that hold a row past the end of the sequence (rows [valid, 128)).
__host__ __device__ inline unsigned int past_end_atoms(const Runs& tr) {
  return tr.valid >= 128 ? 0u : (0xFFFFu & ~((1u << (tr.valid >> 3)) - 1u));
}

// First rolled row of the group containing rolled row r, and one past its last row. With a
// wrap split W < N (the pages' Variant 2, Table 8: in the shifted heads the tokens the roll
// wrapped around, rolled rows [W, N) with W = N - shift, form their own group), the last
// group [N - G, N) is two groups, [N - G, W) and [W, N). When G does not divide N the last
// group is shorter: callers clip group_end at N.
__host__ __device__ __forceinline__ int min_i(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int group_begin(int r, int G, int W = kNoWrapSplit) {
  return r >= W ? W : (r / G) * G;
}
__host__ __device__ inline int group_end(int r, int G, int W = kNoWrapSplit) {
  const int e = (r / G + 1) * G;
  return (r < W && e > W) ? W : e;
}

// Up to three ranges of tile indices [a[i], b[i]], listed in order, no index twice.
struct TileList {
  int n;
  int a[3], b[3];
  __host__ __device__ __forceinline__ int count() const {
    int c = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i < n) c += b[i] - a[i] + 1;
    return c;
  }
  __host__ __device__ __forceinline__ int at(int k) const {
    int r = -1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int c = b[i] - a[i] + 1;
      if (i < n && r < 0) {
        if (k < c) r = a[i] + k;
        else k -= c;
      }
    }
    return r;
  }
  // Position of tile `t` in the list, or -1.
  __host__ __device__ __forceinline__ int index_of(int t) const {
    int k = 0, r = -1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (i < n && r < 0) {
        if (t >= a[i] && t <= b[i]) r = k + (t - a[i]);
        k += b[i] - a[i] + 1;
      }
    }
    return r;
  }
  __host__ __device__ __forceinline__ bool has(int t) const { return index_of(t) >= 0; }
  // Append [lo, hi] minus the tiles already listed. Ranges built from disjoint contiguous
  // runs of rows overlap earlier ranges only in their end tiles, so trimming the ends is
  // enough (a range that would still overlap inside is not added; the index tests check
  // that this never happens).
  __host__ __device__ __forceinline__ void append(int lo, int hi) {
#pragma unroll
    for (int pass = 0; pass < 3; ++pass)
#pragma unroll
      for (int i = 0; i < 3; ++i)
        if (i < n) {
          if (lo >= a[i] && lo <= b[i]) lo = b[i] + 1;
          if (hi >= a[i] && hi <= b[i]) hi = a[i] - 1;
        }
    if (lo > hi) return;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i < n && a[i] <= hi && b[i] >= lo) return;
    bool done = false;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i + 1 == n && b[i] + 1 == lo) {
        b[i] = hi;
        done = true;
      }
    if (done) return;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i == n) {
        a[i] = lo;
        b[i] = hi;
      }
    if (n < 3) ++n;
  }
};

// Query tiles (rolled, 128 rows) of a query head that can see the original kv rows
// [t0, t0 + 128), in increasing order. A kv row at rolled position r is seen by the query rows
// [r, end of r's group), so a run [r0, r1] of rolled kv rows is seen by the query tiles
// r0 / 128 .. (group_end(r1) - 1) / 128.
using QTileRanges = TileList;
__host__ __device__ inline QTileRanges kv_tile_qtiles(const HeadRemap& m, int t0,
                                                      int W = kNoWrapSplit) {
  const Runs tr = token_runs(m, t0);
  if (!m.front) {
    // run A: rolled rows [src0, src0 + len0); run B (after the wrap): rolled rows from 0
    QTileRanges q;
    const int a0 = tr.src[0] / kTileRows;
    const int a1 = (min_i(group_end(tr.src[0] + tr.len[0] - 1, m.G, W), m.N) - 1) / kTileRows;
    q.a[1] = 0; q.b[1] = -1; q.a[2] = 0; q.b[2] = -1;
    if (tr.n == 2) {
      const int b1 = (min_i(group_end(tr.len[1] - 1, m.G, W), m.N) - 1) / kTileRows;
      if (b1 + 1 >= a0) {
        q.n = 1; q.a[0] = 0; q.b[0] = a1 > b1 ? a1 : b1;
      } else {
        q.n = 2; q.a[0] = 0; q.b[0] = b1; q.a[1] = a0; q.b[1] = a1;
      }
    } else {
      q.n = 1; q.a[0] = a0; q.b[0] = a1;
    }
    return q;
  }
  constexpr int kNone = 0x7fffffff;   // sorts after every real range
  int lo[3], hi[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    lo[k] = k < tr.n ? tr.src[k] / kTileRows : kNone;
    hi[k] = k < tr.n ? (min_i(group_end(tr.src[k] + tr.len[k] - 1, m.G, W), m.N) - 1) / kTileRows
                     : kNone;
  }
  // sort the (at most three) ranges by start, then merge overlapping or adjacent ones
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = i + 1; j < 3; ++j)
      if (lo[j] < lo[i]) {
        const int x = lo[i], y = hi[i];
        lo[i] = lo[j]; hi[i] = hi[j];
        lo[j] = x; hi[j] = y;
      }
  QTileRanges q;
  q.n = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    q.a[i] = 0;
    q.b[i] = -1;
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (lo[k] == kNone) continue;
    bool merged = false;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i + 1 == q.n && lo[k] <= q.b[i] + 1) {
        if (hi[k] > q.b[i]) q.b[i] = hi[k];
        merged = true;
      }
    if (merged) continue;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i == q.n) {
        q.a[i] = lo[k];
        q.b[i] = hi[k];
      }
    ++q.n;
  }
  return q;
}

// Original kv tiles that rolled query tile qt reads: its rows see the rolled kv rows
// [start of the group of its first row, its last row]; these map to at most three runs of
// original rows, listed in rolled order, each run's tiles once.
using KvSpan = TileList;
__host__ __device__ inline KvSpan qtile_kv_span(const HeadRemap& m, int qt,
                                               int W = kNoWrapSplit) {
  const int r0 = qt * kTileRows;
  const int last = r0 + kTileRows - 1 < m.N - 1 ? r0 + kTileRows - 1 : m.N - 1;
  const int gb = group_begin(r0, m.G, W);
  KvSpan s;
  if (!m.front) {
    // under the plain roll the rows map to one cyclic range of original rows
    const int T = (m.N + kTileRows - 1) / kTileRows;
    const int len = last - gb + 1;
    const int o0 = gb + m.shift >= m.N ? gb + m.shift - m.N : gb + m.shift;
    int count = o0 + len <= m.N ? (o0 + len - 1) / kTileRows - o0 / kTileRows + 1
                                : (T - o0 / kTileRows) + (o0 + len - m.N - 1) / kTileRows + 1;
    count = count < T ? count : T;
    const int first = o0 / kTileRows;
    s.a[0] = first;
    s.b[0] = first + count - 1 < T - 1 ? first + count - 1 : T - 1;
    s.a[1] = 0;
    s.b[1] = first + count - 1 - T;   // -1 (empty) when the range does not wrap
    s.a[2] = 0;
    s.b[2] = -1;
    s.n = s.b[1] >= 0 ? 2 : 1;
    return s;
  }
  const Runs tr = remap_runs(m, false, gb, last - gb + 1);
  s.n = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    s.a[i] = 0;
    s.b[i] = -1;
  }
#pragma unroll
  for (int k = 0; k < 3; ++k)
    if (k < tr.n) s.append(tr.src[k] / kTileRows, (tr.src[k] + tr.len[k] - 1) / kTileRows);
  return s;
}

// Slots of the bf16 dS tiles that the dK/dV kernel hands to the dQ pass: one 128 x 128 tile
// (32 KB) per (query tile qt, kv tile span.at(i)), i < span.count(), at slot base(qt) + i of
// its (batch, query head). When groups and roll are tile-aligned (and the last group is not
// split or reordered), count = qt mod (G/128) + 1 and the slots are packed (a triangle per
// group); otherwise every query tile gets `stride` slots, the largest count of any query tile.
struct DsSlots {
  int aligned;          // G and every head's roll are multiples of the tile
  int gt;               // G / 128 (aligned case)
  int stride;           // slots per query tile (unaligned case)
  long long per_head;   // slots of one (batch, query head)
  __host__ __device__ __forceinline__ long long base(int qt) const {
    if (aligned) {
      const long long g = qt / gt, i = qt % gt;
      return g * gt * (gt + 1) / 2 + i * (i + 1) / 2;
    }
    return static_cast<long long>(qt) * stride;
  }
};
inline DsSlots ds_slots(int N, int G, int shifted_heads, int shift, int W = kNoWrapSplit,
                        int front = 0) {
  DsSlots d;
  const int T = (N + kTileRows - 1) / kTileRows;
  const int sh = shifted_heads ? shift : 0;
  const int w = shifted_heads ? W : kNoWrapSplit;
  const int fr = shifted_heads ? front : 0;
  d.aligned = (N % G == 0 && G % kTileRows == 0 && sh % kTileRows == 0 && w >= N && !fr) ? 1 : 0;
  d.gt = G / kTileRows;
  d.stride = 0;
  if (d.aligned) {
    d.per_head = static_cast<long long>(N / G) * d.gt * (d.gt + 1) / 2;
  } else {
    const HeadRemap m0 = head_remap(N, G, 0, 0), m1 = head_remap(N, G, sh, fr);
    for (int qt = 0; qt < T; ++qt) {
      const int c0 = qtile_kv_span(m0, qt).count();
      const int c1 = qtile_kv_span(m1, qt, w).count();
      const int c = c0 > c1 ? c0 : c1;
      d.stride = c > d.stride ? c : d.stride;
    }
    d.per_head = static_cast<long long>(T) * d.stride;
  }
  return d;
}

// Block index -> (b, h, rolled query tile) for the forward and dQ kernels. When G is a
// multiple of the tile, tiles late in their group (more key tiles to visit) come first.
__host__ __device__ inline void query_tile_coords(int bid, int B, int Hq, int N, int G, int& b,
                                                  int& h, int& qt) {
  if (N % G == 0 && G % kTileRows == 0) {
    const int tpg = G / kTileRows, ng = N / G;
    const int per = B * Hq * ng;
    const int il = tpg - 1 - bid / per;
    const int rest = bid % per;
    const int g = rest % ng;
    const int bh = rest / ng;
    h = bh % Hq;
    b = bh / Hq;
    qt = g * tpg + il;
  } else {
    const int bh = bid % (B * Hq);
    qt = bid / (B * Hq);
    h = bh % Hq;
    b = bh / Hq;
  }
}

// Block index -> (b, h, rolled query tile), grouped for L2 reuse: the (b, h, group) instances
// are taken `chunk` at a time, and within a chunk the tiles go heaviest first (last tile of
// each group first). Work that runs concurrently then reads the key tiles of only `chunk`
// groups. Falls back to query_tile_coords when G is not a multiple of the tile.
__host__ __device__ inline void query_tile_coords_chunked(int bid, int B, int Hq, int N, int G,
                                                          int chunk, int& b, int& h, int& qt) {
  if (N % G != 0 || G % kTileRows != 0) {
    query_tile_coords(bid, B, Hq, N, G, b, h, qt);
    return;
  }
  const int tpg = G / kTileRows, ng = N / G;
  const int instances = B * Hq * ng;
  const int per_chunk = chunk * tpg;
  const int ck = bid / per_chunk, within = bid % per_chunk;
  const int rest = instances - ck * chunk;
  const int cl = rest < chunk ? rest : chunk;
  const int il = tpg - 1 - within / cl;
  const int inst = ck * chunk + within % cl;
  const int g = inst % ng, bh = inst / ng;
  h = bh % Hq;
  b = bh / Hq;
  qt = g * tpg + il;
}

// Block index -> (b, h, pair) for kernels whose CTA owns the two rolled query tiles 2*pair
// and 2*pair + 1 of one (b, h). When G is a multiple of two tiles, pairs late in their group
// (more key tiles to visit) come first.
__host__ __device__ inline int query_pairs_per_head(int N) {
  return ((N + kTileRows - 1) / kTileRows + 1) / 2;
}
__host__ __device__ inline void query_pair_coords(int bid, int B, int Hq, int N, int G, int& b,
                                                  int& h, int& pair) {
  if (N % G == 0 && G % (2 * kTileRows) == 0) {
    const int ppg = G / (2 * kTileRows), ng = N / G;
    const int per = B * Hq * ng;
    const int pl = ppg - 1 - bid / per;
    const int rest = bid % per;
    const int g = rest % ng;
    const int bh = rest / ng;
    h = bh % Hq;
    b = bh / Hq;
    pair = g * ppg + pl;
  } else {
    const int bh = bid % (B * Hq);
    pair = bid / (B * Hq);
    h = bh % Hq;
    b = bh / Hq;
  }
}

// Block index -> (b, h, pair) with the same L2 grouping as query_tile_coords_chunked: the
// (b, h, group) instances `chunk` at a time, heaviest pairs (last in group) first within a
// chunk. Falls back to query_pair_coords when G is not a multiple of two tiles.
__host__ __device__ inline void query_pair_coords_chunked(int bid, int B, int Hq, int N, int G,
                                                          int chunk, int& b, int& h, int& pair) {
  if (N % G != 0 || G % (2 * kTileRows) != 0) {
    query_pair_coords(bid, B, Hq, N, G, b, h, pair);
    return;
  }
  const int ppg = G / (2 * kTileRows), ng = N / G;
  const int instances = B * Hq * ng;
  const int per_chunk = chunk * ppg;
  const int ck = bid / per_chunk, within = bid % per_chunk;
  const int rest = instances - ck * chunk;
  const int cl = rest < chunk ? rest : chunk;
  const int pl = ppg - 1 - within / cl;
  const int inst = ck * chunk + within % cl;
  const int g = inst % ng, bh = inst / ng;
  h = bh % Hq;
  b = bh / Hq;
  pair = g * ppg + pl;
}

// Block index -> (b, kv head, first original row t0 of the kv tile) for the dK/dV kernel.
// When groups and roll are tile-aligned, kv tiles early in their (rolled) group, which see
// the most query tiles, come first.
__host__ __device__ inline void kv_tile_coords(int bid, int B, int Hq, int Hkv, int N, int G,
                                               int shift_head_begin, int shift, int& b,
                                               int& kvh, int& t0) {
  const int rep = Hq / Hkv;
  if (N % G == 0 && G % kTileRows == 0 && shift % kTileRows == 0) {
    const int ng = N / G;
    const int per = B * Hkv * ng;
    const int jl = bid / per;
    const int rest = bid % per;
    const int g = rest % ng;
    const int bk = rest / ng;
    kvh = bk % Hkv;
    b = bk / Hkv;
    const int sh = (kvh * rep >= shift_head_begin) ? shift : 0;
    const int rs = g * G + jl * kTileRows;
    t0 = rs + sh >= N ? rs + sh - N : rs + sh;
  } else {
    const int bk = bid % (B * Hkv);
    t0 = (bid / (B * Hkv)) * kTileRows;
    kvh = bk % Hkv;
    b = bk / Hkv;
  }
}

// Block index -> (b, kv head, t0) with the L2 grouping of query_tile_coords_chunked: the
// (b, kv head, rolled group) instances `chunk` at a time, kv tiles early in their group (most
// query tiles) first within a chunk. Falls back to kv_tile_coords when groups or roll are not
// tile-aligned.
__host__ __device__ inline void kv_tile_coords_chunked(int bid, int B, int Hq, int Hkv, int N,
                                                       int G, int shift_head_begin, int shift,
                                                       int chunk, int& b, int& kvh, int& t0) {
  if (!(N % G == 0 && G % kTileRows == 0 && shift % kTileRows == 0)) {
    kv_tile_coords(bid, B, Hq, Hkv, N, G, shift_head_begin, shift, b, kvh, t0);
    return;
  }
  const int rep = Hq / Hkv;
  const int tpg = G / kTileRows, ng = N / G;
  const int instances = B * Hkv * ng;
  const int per_chunk = chunk * tpg;
  const int ck = bid / per_chunk, within = bid % per_chunk;
  const int rest = instances - ck * chunk;
  const int cl = rest < chunk ? rest : chunk;
  const int jl = within / cl;
  const int inst = ck * chunk + within % cl;
  const int g = inst % ng, bk = inst / ng;
  kvh = bk % Hkv;
  b = bk / Hkv;
  const int sh = (kvh * rep >= shift_head_begin) ? shift : 0;
  const int rs = g * G + jl * kTileRows;
  t0 = rs + sh >= N ? rs + sh - N : rs + sh;
}

}  // namespace s2
