// The per-head shift-and-group remap, applied to 128-row tiles.
//
// LongLoRA summary page, §3.4 Algorithm 1: the second chunk of heads is rolled by -G/2
// along N (key line 1), viewed as groups of G (".view(B*N/G, G, ...)"), attended causally
// per group, and rolled back (key line 2). Instead of materialising the roll, every kernel
// addresses the original tensors through
//     t = (r + s_h) mod N          (rolled row r -> original token t)
// where s_h is the head's roll (G/2 for the shifted heads, 0 otherwise); group of rolled
// row r is floor(r / G). Tiles are 128 consecutive rolled rows; such a tile maps onto at
// most two contiguous runs of original rows (the run that reaches token N-1 and the run
// that wraps to token 0), plus zero rows past the end of the sequence.
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

struct TileRuns {
  int valid;   // rows of the tile inside the sequence (rows [valid, 128) are padding)
  int first;   // rows [0, first) come from original rows [start, start + first)
  int start;   // original row of tile row 0
  // rows [first, valid) come from original rows [0, valid - first)
};

// Rolled tile starting at rolled row r0, head roll `shift` (0 <= shift < N).
__host__ __device__ inline TileRuns rolled_tile_runs(int r0, int shift, int N) {
  TileRuns t;
  t.valid = N - r0 < kTileRows ? N - r0 : kTileRows;
  long long s = static_cast<long long>(r0) + shift;
  t.start = static_cast<int>(s >= N ? s - N : s);
  const int to_end = N - t.start;
  t.first = t.valid < to_end ? t.valid : to_end;
  return t;
}

// Tile of original rows [t0, t0 + 128): the rolled rows they occupy in a head with roll
// `shift` are (t - shift) mod N, i.e. the tile is the rolled tile starting at
// (t0 - shift) mod N read with the inverse roll. Returns the same run structure in rolled
// coordinates: rows [0, first) are rolled rows [start, start + first), rows [first, valid)
// are rolled rows [0, valid - first).
__host__ __device__ inline TileRuns original_tile_runs(int t0, int shift, int N) {
  const int inv = shift == 0 ? 0 : N - shift;
  return rolled_tile_runs(t0, inv, N);
}

// No split of the wrap group (see group_begin).
constexpr int kNoWrapSplit = 0x7fffffff;

// First rolled row of the group containing rolled row r, and one past its last row. With a
// wrap split W < N (the pages' Variant 2, Table 8: in the shifted heads the tokens the roll
// wrapped around, rolled rows [W, N) with W = N - shift, form their own group), the last
// group [N - G, N) is two groups, [N - G, W) and [W, N).
__host__ __device__ inline int group_begin(int r, int G, int W = kNoWrapSplit) {
  return r >= W ? W : (r / G) * G;
}
__host__ __device__ inline int group_end(int r, int G, int W = kNoWrapSplit) {
  const int e = (r / G + 1) * G;
  return (r < W && e > W) ? W : e;
}

// Query tiles (rolled, 128 rows) of a query head with roll `sh` that can see the original
// kv rows [t0, t0 + 128): up to two disjoint index ranges, [r0a, r0b] then [r1a, r1b].
// A kv row at rolled position r is seen by the query rows [r, end of r's group).
struct QTileRanges {
  int r0a, r0b, r1a, r1b;
  __host__ __device__ __forceinline__ int count() const {
    return (r0b - r0a + 1) + (r1b >= r1a ? r1b - r1a + 1 : 0);
  }
  __host__ __device__ __forceinline__ int at(int i) const {
    const int n0 = r0b - r0a + 1;
    return i < n0 ? r0a + i : r1a + (i - n0);
  }
};

__host__ __device__ inline QTileRanges kv_tile_qtiles(int t0, int sh, int N, int G,
                                                      int W = kNoWrapSplit) {
  const TileRuns tr = original_tile_runs(t0, sh, N);
  // Run A: rolled rows [start, start + first) -> query rows [start, end of group).
  const int a0 = tr.start / kTileRows;
  const int a1 = (group_end(tr.start + tr.first - 1, G, W) - 1) / kTileRows;
  QTileRanges q;
  if (tr.valid > tr.first) {
    // Run B: rolled rows [0, valid - first) -> query rows [0, end of that group).
    const int b1 = (group_end(tr.valid - tr.first - 1, G, W) - 1) / kTileRows;
    if (b1 + 1 >= a0) {
      q.r0a = 0; q.r0b = a1 > b1 ? a1 : b1; q.r1a = 1; q.r1b = 0;
    } else {
      q.r0a = 0; q.r0b = b1; q.r1a = a0; q.r1b = a1;
    }
  } else {
    q.r0a = a0; q.r0b = a1; q.r1a = 1; q.r1b = 0;
  }
  return q;
}

// Original kv tiles that rolled query tile qt (head roll sh) reads. Its rows see the rolled
// kv rows [start of the group of its first row, its last row]; under the roll these are a
// contiguous range of original rows modulo N, covered by `count` consecutive original tiles
// (indices taken modulo the tile count T) starting at `first`.
struct KvSpan {
  int first, count;
};
__host__ __device__ inline KvSpan qtile_kv_span(int qt, int sh, int N, int G,
                                               int W = kNoWrapSplit) {
  const int T = (N + kTileRows - 1) / kTileRows;
  const int r0 = qt * kTileRows;
  const int last = r0 + kTileRows - 1 < N - 1 ? r0 + kTileRows - 1 : N - 1;
  const int gb = group_begin(r0, G, W);
  const int len = last - gb + 1;
  const long long o = static_cast<long long>(gb) + sh;
  const int o0 = static_cast<int>(o >= N ? o - N : o);
  int count;
  if (o0 + len <= N)
    count = (o0 + len - 1) / kTileRows - o0 / kTileRows + 1;
  else
    count = (T - o0 / kTileRows) + (o0 + len - N - 1) / kTileRows + 1;
  KvSpan s;
  s.first = o0 / kTileRows;
  s.count = count < T ? count : T;
  return s;
}

// Slots of the bf16 dS tiles that the dK/dV kernel hands to the dQ pass: one 128 x 128 tile
// (32 KB) per (query tile qt, original kv tile first + i), i < count, at slot base(qt) + i of
// its (batch, query head). When groups and roll are tile-aligned, count = qt mod (G/128) + 1
// and the slots are packed (a triangle per group); otherwise every query tile gets `stride`
// slots, the largest count of any query tile.
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
inline DsSlots ds_slots(int N, int G, int shifted_heads, int shift, int W = kNoWrapSplit) {
  DsSlots d;
  const int T = (N + kTileRows - 1) / kTileRows;
  const int sh = shifted_heads ? shift : 0;
  const int w = shifted_heads ? W : kNoWrapSplit;
  d.aligned = (G % kTileRows == 0 && sh % kTileRows == 0 && w >= N) ? 1 : 0;
  d.gt = G / kTileRows;
  d.stride = 0;
  if (d.aligned) {
    d.per_head = static_cast<long long>(N / G) * d.gt * (d.gt + 1) / 2;
  } else {
    for (int qt = 0; qt < T; ++qt) {
      const int c0 = qtile_kv_span(qt, 0, N, G).count;
      const int c1 = qtile_kv_span(qt, sh, N, G, w).count;
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
  if (G % kTileRows == 0) {
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
  if (G % kTileRows != 0) {
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
  if (G % (2 * kTileRows) == 0) {
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
  if (G % (2 * kTileRows) != 0) {
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
  if (G % kTileRows == 0 && shift % kTileRows == 0) {
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
  if (!(G % kTileRows == 0 && shift % kTileRows == 0)) {
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
