// S²-Attn forward (O and row log-sum-exp) on sm_100a tensor cores.
//
// LongLoRA summary page, §3.4 Algorithm 1: per head, roll (second chunk of heads), view as
// groups of G, causal softmax(scale * q k^T) v inside each group, roll back. A work unit is
// two consecutive 128-row tiles of rolled query rows of one (batch, head); it walks the
// 128-row key/value tiles of the same rolled frame, from the start of the group of its first
// row to its last diagonal tile: work is proportional to N*G rather than N^2. The roll never
// moves data: TMA reads the original rows (s2_tiles.cuh) and the epilogue stores O and LSE at
// the original rows.
//
// The kernel is persistent: one CTA per SM sets up its barriers and TMEM once, decodes its
// first units into a shared-memory table and takes the work units a host-side schedule gives it
// (FwdSchedule: least-loaded-CTA assignment in the L2-grouped unit order, the last units
// heaviest first), so one unit's epilogue and the next unit's loads overlap the tensor-core
// work and the CTAs finish together.
//
// Warp roles (320 threads; 384 with the fused RoPE of the queries):
//   warps 0-3, 4-7  softmax warpgroup of query tile 0 / 1: thread i owns query row i (TMEM
//                   lane i); online softmax in fp32, P written back to TMEM as bf16 over S,
//                   O rescaled in TMEM when the running max grows, epilogue.
//   warp 8          TMA producer: both Q tiles once, then K tiles running one tile ahead of
//                   V tiles (2-slot rings); each ring slot is released by a commit right
//                   after the last MMA that reads it.
//   warp 9          TMEM allocator and MMA issuer (one lane).
//   warps 10, 11    (fused RoPE only) rotate each query tile in shared memory once it has
//                   landed and send the rotated rows out; the MMAs wait for the rotation.
// TMEM columns: S0/P0 [0,128), S1/P1 [128,256), O0 [256,256+D), O1 [256+D, 256+2D).
//
// MMA issue order S0(0) S1(0) PV0(0) S0(1) PV1(0) S1(1) PV0(1) ... lets each warpgroup's
// softmax run while the tensor core works on the other tile. tcgen05 MMAs from one thread
// complete in issue order, so when S_t(j+1) is signalled, PV_t(j) — which read P_t(j) from
// the same columns and accumulated into O_t — is complete: the softmax may rescale O_t at once.
// Tile 1 of a unit has one more key tile than tile 0, so the next unit's first S on tile 0 is
// issued before tile 1's last step when its tiles are already in place.
//
// The epilogue stages each warp's 32 rows of O (64 columns at a time) in shared memory and
// sends them out as 8-row TMA boxes (row stores only where the roll splits an 8-row atom).
#pragma once

#include "s2_common.cuh"
#include "s2_tmem_wide.cuh"

namespace s2 {

struct FwdParams {
  TensorRef q, k, v;      // the inputs again, for rows the TMA boxes cannot move
  __nv_bfloat16* o;
  long long o_sb, o_st;   // element strides of O's batch and token axes
  float* lse;
  int B, Hq, Hkv, N, G, shift_head_begin, shift;
  int wrap;           // wrap split of the shifted heads' last group (kNoWrapSplit: none)
  int front;          // Variant 3: the shifted heads' last group lists the wrapped tokens first
  float scale_log2;   // scale * log2(e)
  unsigned int* err;
  unsigned long long timeout_ns;
  // Fused rotary position embedding of the queries (kernel built with kRope): q holds the
  // un-rotated queries, each query tile is rotated in shared memory before its first MMA and
  // the rotated rows are written to q_rot (contiguous [B, N, Hq, D]).
  __nv_bfloat16* q_rot;
  float rope_log2_base, rope_pi_scale;
};

// Which work units each CTA takes, computed on the host (longest-processing-time-first: the
// units, in their heaviest-first L2-grouped order, each go to the CTA with the least work so
// far, by a cost model of (query tile, key tile) steps plus a per-unit overhead) and passed by
// value with the launch. count = 0: units blockIdx.x, blockIdx.x + gridDim.x, ... instead.
constexpr int kFwdSchedMaxCtas = 160;
constexpr int kFwdSchedMaxUnits = 6144;
struct FwdSchedule {
  int count;                                  // units in the list (0: round robin)
  unsigned short start[kFwdSchedMaxCtas + 1];   // CTA c takes unit[start[c] .. start[c + 1])
  unsigned short unit[kFwdSchedMaxUnits];
};

// The k-th unit of this CTA, or -1 when it has no more.
__device__ __forceinline__ int fwd_unit_index(const FwdSchedule& s, int n_units, int k) {
  if (s.count == 0) {
    const long long u = blockIdx.x + static_cast<long long>(k) * gridDim.x;
    return u < n_units ? static_cast<int>(u) : -1;
  }
  const int i = s.start[blockIdx.x] + k;
  return i < s.start[blockIdx.x + 1] ? s.unit[i] : -1;
}

// Rescale O only when the running max (log2 units) grows by more than this: until then
// exp2(s - stale max) <= 2^8, harmless in fp32 and bf16, and the final 1/l uses the same max.
constexpr float kRescaleThreshold = 8.0f;

// The integer divisions of a unit's decoding: (b, h, pair), the kv head and each tile's first
// key tile. About 2000 cycles on one thread, so a CTA decodes its first kLocalUnits units
// once, at the start, into shared memory (b = -1: no such unit), and every role reads them
// from there at its unit boundaries.
struct FwdUnitRec {
  int b, h, pair, kvh, kb[2];
};
constexpr int kLocalUnits = 64;

template <int D>
struct FwdLayout {
  static constexpr uint32_t kTile = Tile<D>::kBytes;
  static constexpr int kKStages = 2, kVStages = 2;
  static constexpr uint32_t kQ = 0;                         // 2 query tiles
  static constexpr uint32_t kK = kQ + 2 * kTile;            // K ring
  static constexpr uint32_t kV = kK + kKStages * kTile;     // V ring
  static constexpr uint32_t kStageWarp = 32 * 128;          // O staging: 32 rows x 64 columns
  static constexpr uint32_t kStage = kV + kVStages * kTile; // ... for each softmax warp
  static constexpr uint32_t kRecs = kStage + 8 * kStageWarp;   // kLocalUnits FwdUnitRec
  static constexpr uint32_t kBar = kRecs + kLocalUnits * sizeof(FwdUnitRec);
  enum { B_Q = 0, B_QE = 2, B_K = 4, B_KE = B_K + kKStages, B_V = B_KE + kKStages,
         B_VE = B_V + kVStages, B_S = B_VE + kVStages, B_P = B_S + 2, B_ODONE = B_P + 2,
         B_DRAIN = B_ODONE + 2, B_QR = B_DRAIN + 1, B_QW = B_QR + 2, B_RR = B_QW + 2,
         B_COUNT = B_RR + 2 };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  // Dynamic shared memory to request: alignment slack, and at least 116 KB so that only one
  // CTA is resident per SM (each CTA takes all 512 TMEM columns).
  static constexpr uint32_t kLaunchBytes =
      (kBytes + 1024 > 116 * 1024) ? kBytes + 1024 : 116 * 1024;
  static constexpr int kThreads = 320;
  static constexpr int kRopeThreads = 384;   // + the rotation warps (10, 11) of the fused RoPE
  static_assert(kLaunchBytes <= 227 * 1024, "shared memory of one CTA");
};

// Fused RoPE with Position Interpolation of one 128-row query tile in shared memory (the
// 128-byte-swizzled TMA layout), by the kRopeWarps rotation warps together (`part` = this
// warp's index among them): the same rotation as s2_rope_kernel — the pair (x[i], x[i + D/2]) of
// token t turns by (t * pi_scale) * base^(-2i/D) — written back in place, for the MMAs and for
// the TMA stores of the rotated rows. A lane owns one 16-byte chunk of a row's first half (8
// columns) and its partner chunk D/2 columns on: D/16 lanes per row, 16-byte shared-memory
// accesses, packed f32x2 arithmetic on column pairs. The angle of a run's first row is computed
// as there (fp32 product, accurate sincosf); each following row of the run is reached by turning
// by the angle of the rows in between (angle addition in fp32, relative drift about 1e-6 over a
// tile, far below the bf16 rounding of the result).
constexpr int kRopeWarps = 2;
template <int D>
__device__ __forceinline__ uint32_t swz_chunk(uint32_t tile, int row, int col) {
  const int half = col / 64, chunk = (col % 64) / 8;
  return tile + half * Tile<D>::kHalfBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
}
// A lane's frequencies and the turn of one row step, the same for every tile: worked out once.
struct RopeLane {
  float th[8];                  // base^(-2i/D) of the lane's 8 columns
  uint64_t cd[4], sd[4], nsd[4];   // cos, sin and -sin of one step's angle, column pairs packed
};
template <int D>
__device__ __forceinline__ RopeLane rope_lane(float log2_base, float pi_scale) {
  constexpr int kLanesPerRow = D / 16;
  constexpr int kRowsPerStep = (32 / kLanesPerRow) * kRopeWarps;
  const int cl = (threadIdx.x & 31) % kLanesPerRow;
  RopeLane rl;
#pragma unroll
  for (int e = 0; e < 8; ++e) rl.th[e] = exp2f(-(2.0f * (8 * cl + e) / D) * log2_base);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float s0, c0, s1, c1;
    sincosf((kRowsPerStep * pi_scale) * rl.th[2 * k], &s0, &c0);
    sincosf((kRowsPerStep * pi_scale) * rl.th[2 * k + 1], &s1, &c1);
    rl.cd[k] = f2_pack(c0, c1);
    rl.sd[k] = f2_pack(s0, s1);
    rl.nsd[k] = f2_pack(-s0, -s1);
  }
  return rl;
}
template <int D>
__device__ __forceinline__ void rope_query_tile(uint32_t tile, const Runs& tr, const RopeLane& rl,
                                                float pi_scale, int part) {
  constexpr int kLanesPerRow = D / 16;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  constexpr int kRowsPerStep = kRowsPerWarp * kRopeWarps;
  const int lane = threadIdx.x & 31;
  const int cl = lane % kLanesPerRow, r_off = part * kRowsPerWarp + lane / kLanesPerRow;
  const float* th = rl.th;
  const uint64_t* cd = rl.cd;
  const uint64_t* sd = rl.sd;
  const uint64_t* nsd = rl.nsd;
  int base = 0;
  for (int r = 0; r < tr.n; ++r) {
    const int len = tr.len[r], src = tr.src[r];
    uint64_t c[4], sn[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float s0, c0, s1, c1;
      sincosf((static_cast<float>(src + r_off) * pi_scale) * th[2 * k], &s0, &c0);
      sincosf((static_cast<float>(src + r_off) * pi_scale) * th[2 * k + 1], &s1, &c1);
      c[k] = f2_pack(c0, c1);
      sn[k] = f2_pack(s0, s1);
    }
    for (int i = r_off; i < len; i += kRowsPerStep) {
      const int row = base + i;
      const uint32_t a_lo = swz_chunk<D>(tile, row, 8 * cl);
      const uint32_t a_hi = swz_chunk<D>(tile, row, 8 * cl + D / 2);
      uint32_t x[4], y[4];
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]) : "r"(a_lo));
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(y[0]), "=r"(y[1]), "=r"(y[2]), "=r"(y[3]) : "r"(a_hi));
      uint32_t nx[4], ny[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t xf = f2_from_bf16x2(x[k]), yf = f2_from_bf16x2(y[k]);
        // x' = x c - y s, y' = y c + x s
        const uint64_t xr = f2_fma(xf, c[k], f2_mul(yf, sn[k] ^ 0x8000000080000000ull));
        const uint64_t yr = f2_fma(yf, c[k], f2_mul(xf, sn[k]));
        nx[k] = pack_bf16(f2_lo(xr), f2_hi(xr));
        ny[k] = pack_bf16(f2_lo(yr), f2_hi(yr));
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_lo), "r"(nx[0]), "r"(nx[1]),
                   "r"(nx[2]), "r"(nx[3]) : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_hi), "r"(ny[0]), "r"(ny[1]),
                   "r"(ny[2]), "r"(ny[3]) : "memory");
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t cn = f2_fma(c[k], cd[k], f2_mul(sn[k], nsd[k]));
        sn[k] = f2_fma(sn[k], cd[k], f2_mul(c[k], sd[k]));
        c[k] = cn;
      }
    }
    base += len;
  }
  fence_async_smem();   // the MMAs and the TMA stores read the rotated tile (async proxy)
  __syncwarp();
}

// Row maximum of 128 values: eight independent chains of three-input max instructions.
__device__ __forceinline__ float max_tree128(const float (&s)[128]) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = max3f(s[i], s[8 + i], s[16 + i]);
#pragma unroll
  for (int j = 3; j + 1 < 16; j += 2)
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = max3f(m[i], s[8 * j + i], s[8 * (j + 1) + i]);
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], s[120 + i]);
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// One work unit: query tiles 2*pair and 2*pair + 1 of (b, h) and the key tiles they see.
struct FwdUnit {
  int b, h, kvh, wrap_h;
  int shift_h, front_h;   // the head's remap: head_remap(N, G, shift_h, front_h)
  int qt[2], kb[2], ke[2];
  bool tv[2];
  int kv_lo, n_kv;
  __device__ __forceinline__ bool part(int t, int kt) const {
    return tv[t] && kb[t] <= kt && kt <= ke[t];
  }
};

template <bool kFront>
__device__ __forceinline__ FwdUnitRec fwd_unit_rec(const FwdParams& p, int unit) {
  FwdUnitRec r;
  query_pair_coords_chunked(unit, p.B, p.Hq, p.N, p.G, kL2Chunk, r.b, r.h, r.pair);
  r.kvh = r.h / (p.Hq / p.Hkv);
  const int nqt = (p.N + kTileRows - 1) / kTileRows;
  const int wrap_h = r.h >= p.shift_head_begin ? p.wrap : kNoWrapSplit;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * r.pair + t;
    r.kb[t] = qt < nqt ? group_begin(qt * kTileRows, p.G, wrap_h) / kTileRows : 0;
  }
  return r;
}

// kFront: the kernel is built for the Variant 3 reordering (otherwise p.front is ignored and
// the plain-roll index code is all that is compiled in).
template <bool kFront>
__device__ __forceinline__ FwdUnit fwd_unit_from(const FwdParams& p, const FwdUnitRec& r) {
  FwdUnit u;
  u.b = r.b;
  u.h = r.h;
  u.kvh = r.kvh;
  const int nqt = (p.N + kTileRows - 1) / kTileRows;
  const bool shifted = u.h >= p.shift_head_begin;
  u.shift_h = shifted ? p.shift : 0;
  u.front_h = (kFront && shifted) ? p.front : 0;
  u.wrap_h = shifted ? p.wrap : kNoWrapSplit;
  // Tile t = 2*pair + t sees key tiles [kb[t], ke[t]]; tile 0 always exists, tile 1 may not.
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    u.qt[t] = 2 * r.pair + t;
    u.tv[t] = u.qt[t] < nqt;
    u.kb[t] = r.kb[t];
    u.ke[t] = u.qt[t];
  }
  u.kv_lo = u.kb[0];
  u.n_kv = (u.tv[1] ? u.ke[1] : u.ke[0]) - u.kv_lo + 1;
  return u;
}

// The k-th unit of this CTA into u; false when it has no more.
template <bool kFront>
__device__ __forceinline__ bool fwd_unit_k(const FwdParams& p, const FwdSchedule& sched,
                                           int n_units, const FwdUnitRec* recs, int k, FwdUnit& u) {
  FwdUnitRec r;
  if (k < kLocalUnits) {
    r = recs[k];
    if (r.b < 0) return false;
  } else {
    const int unit = fwd_unit_index(sched, n_units, k);
    if (unit < 0) return false;
    r = fwd_unit_rec<kFront>(p, unit);
  }
  u = fwd_unit_from<kFront>(p, r);
  return true;
}

template <int D, bool kFront, bool kRope>
__global__ void __launch_bounds__(kRope ? 384 : 320, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ8,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK8,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmV8,
                  const __grid_constant__ CUtensorMap tmO8,
                  const __grid_constant__ CUtensorMap tmQR, const __grid_constant__ CUtensorMap tmQR8,
                  const FwdParams p, const __grid_constant__ FwdSchedule sched) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return sbase + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_FWD};
  const int n_units = p.B * p.Hq * query_pairs_per_head(p.N);
  FwdUnitRec* recs = reinterpret_cast<FwdUnitRec*>(smem + L::kRecs);

  if (warp == 8 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_Q + s), 1);
      mbar_init(bar(L::B_QE + s), 1);
      mbar_init(bar(L::B_V + s), 1);
      mbar_init(bar(L::B_VE + s), 1);
      mbar_init(bar(L::B_S + s), 1);
      mbar_init(bar(L::B_P + s), 128);
      mbar_init(bar(L::B_ODONE + s), 1);
      mbar_init(bar(L::B_QR + s), 1);
      mbar_init(bar(L::B_QW + s), 1);
      mbar_init(bar(L::B_RR + s), kRopeWarps);
    }
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::B_K + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO8);
  }
  if (warp == 8) {
    for (int i = lane; i < kLocalUnits; i += 32) {
      const int unit = fwd_unit_index(sched, n_units, i);
      FwdUnitRec r{-1, 0, 0, 0, {0, 0}};
      if (unit >= 0) r = fwd_unit_rec<kFront>(p, unit);
      recs[i] = r;
    }
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    // K(i) (i counts every key tile this CTA loads) goes to slot i % 2 once K(i - 2) has been
    // released, V(i) likewise; within a unit K runs one tile ahead of V. Q tile t of a unit is
    // loaded once the previous unit's last S MMA on it is done. Tile rows TMA cannot move are
    // copied by this thread first (produce_tile).
    if (lane == 0) {
      int k_issued = 0, v_issued = 0, q_loads[2] = {0, 0};
      bool ok = true;
      auto issue_k = [&](const FwdUnit& u, int j) -> bool {
        const int i = k_issued, st = i % L::kKStages;
        if (i >= L::kKStages &&
            !wait_bar(bar(L::B_KE + st), ((i / L::kKStages) - 1) & 1, ctx, 1))
          return false;
        produce_tile<D>(sbase + L::kK + st * L::kTile, &tmK, &tmK8, bar(L::B_K + st), p.k, u.b,
                        u.kvh, rolled_runs(head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0),
                                           (u.kv_lo + j) * kTileRows), p.N);
        ++k_issued;
        return true;
      };
      auto issue_v = [&](const FwdUnit& u, int j) -> bool {
        const int i = v_issued, st = i % L::kVStages;
        if (i >= L::kVStages &&
            !wait_bar(bar(L::B_VE + st), ((i / L::kVStages) - 1) & 1, ctx, 9))
          return false;
        produce_tile<D>(sbase + L::kV + st * L::kTile, &tmV, &tmV8, bar(L::B_V + st), p.v, u.b,
                        u.kvh, rolled_runs(head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0),
                                           (u.kv_lo + j) * kTileRows), p.N);
        ++v_issued;
        return true;
      };
      for (int ku = 0; ok; ++ku) {
        FwdUnit u;
        if (!fwd_unit_k<kFront>(p, sched, n_units, recs, ku, u)) break;
        ok = issue_k(u, 0);   // the first key tile can stream while the last unit finishes
        for (int t = 0; ok && t < 2; ++t) {
          if (!u.tv[t]) continue;
          if (q_loads[t] > 0 && !wait_bar(bar(L::B_QE + t), (q_loads[t] - 1) & 1, ctx, 10)) {
            ok = false;
            break;
          }
          // (fused RoPE: and once the TMA unit has read the rotated rows out of the slot)
          if (kRope && q_loads[t] > 0 && !wait_bar(bar(L::B_QW + t), (q_loads[t] - 1) & 1, ctx, 12)) {
            ok = false;
            break;
          }
          produce_tile<D>(sbase + L::kQ + t * L::kTile, &tmQ, &tmQ8, bar(L::B_Q + t), p.q, u.b,
                          u.h, rolled_runs(head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0),
                                           u.qt[t] * kTileRows), p.N);
          ++q_loads[t];
        }
        for (int j = 0; ok && j < u.n_kv; ++j) {
          if (j + 1 < u.n_kv) ok = issue_k(u, j + 1);
          if (ok) ok = issue_v(u, j);
        }
      }
      // Every issued copy lands before the CTA can exit.
      for (int t = 0; t < 2; ++t)
        if (q_loads[t] > 0) drain_wait(bar(L::B_Q + t), (q_loads[t] - 1) & 1, p.timeout_ns);
      for (int i = k_issued - L::kKStages; i < k_issued; ++i)
        if (i >= 0) drain_wait(bar(L::B_K + i % L::kKStages), (i / L::kKStages) & 1, p.timeout_ns);
      for (int i = v_issued - L::kVStages; i < v_issued; ++i)
        if (i >= 0) drain_wait(bar(L::B_V + i % L::kVStages), (i / L::kVStages) & 1, p.timeout_ns);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      int k_used = 0, v_used = 0, q_used[2] = {0, 0}, pcount[2] = {0, 0};
      bool ok = true;
      auto wait_k = [&](int i) {
        return wait_bar(bar(L::B_K + i % L::kKStages), (i / L::kKStages) & 1, ctx, 3);
      };
      bool s0_early = false;   // this unit's first S on tile 0 went out during the last unit
      for (int ku = 0; ok; ++ku) {
        FwdUnit u;
        if (!fwd_unit_k<kFront>(p, sched, n_units, recs, ku, u)) break;
        bool q_ready[2] = {s0_early, false}, first_pv[2] = {true, true};
        // S_t(j) = Q_t K(j)^T into TMEM columns [128 t, 128 t + 128).
        auto issue_s = [&](int t, int kidx) -> bool {
          if (!q_ready[t]) {
            // (with the fused RoPE: once the rotation warp has turned the tile)
            if (!wait_bar(bar((kRope ? L::B_QR : L::B_Q) + t), q_used[t] & 1, ctx, 2)) return false;
            q_ready[t] = true;
            ++q_used[t];
          }
          tc_fence_after();
          gemm_ss_k<D>(tmem + t * 128, sbase + L::kQ + t * L::kTile,
                       sbase + L::kK + (kidx % L::kKStages) * L::kTile, idesc_qk);
          mma_commit(bar(L::B_S + t));
          return true;
        };
        const int k0 = k_used, v0 = v_used;
        if (!wait_k(k0)) { ok = false; break; }
        for (int t = 0; ok && t < 2; ++t) {
          if (!u.part(t, u.kv_lo)) continue;
          if (t != 0 || !s0_early) ok = issue_s(t, k0);
          if (ok && u.kv_lo == u.ke[t]) mma_commit(bar(L::B_QE + t));   // last S on Q_t
        }
        s0_early = false;
        if (!ok) break;
        mma_commit(bar(L::B_KE + k0 % L::kKStages));
        for (int j = 0; ok && j < u.n_kv; ++j) {
          const int kt = u.kv_lo + j, vi = v0 + j, vst = vi % L::kVStages;
          const bool next = j + 1 < u.n_kv;
          bool v_ready = false, k_next_ready = false;
          // Tile 1's last step has no tile-0 work: the next unit's first S on tile 0 goes out
          // before it, so tile 0's softmax finds that S ready when its epilogue ends instead
          // of one softmax pass later — if that unit's query tile (rotated, with the fused
          // RoPE) and first key tile are already in place; this thread does not wait for them
          // here, the unit's start issues the S otherwise.
          if (!next && !u.part(0, kt)) {
            FwdUnit un;
            const int kn = k0 + u.n_kv;
            if (fwd_unit_k<kFront>(p, sched, n_units, recs, ku + 1, un) && un.part(0, un.kv_lo) &&
                mbar_test_wait(bar((kRope ? L::B_QR : L::B_Q) + 0), q_used[0] & 1) &&
                mbar_test_wait(bar(L::B_K + kn % L::kKStages), (kn / L::kKStages) & 1)) {
              ++q_used[0];
              tc_fence_after();
              gemm_ss_k<D>(tmem, sbase + L::kQ, sbase + L::kK + (kn % L::kKStages) * L::kTile,
                           idesc_qk);
              mma_commit(bar(L::B_S + 0));
              s0_early = true;
            }
          }
          for (int t = 0; ok && t < 2; ++t) {
            if (u.part(t, kt)) {
              if (!wait_bar(bar(L::B_P + t), pcount[t] & 1, ctx, 4)) { ok = false; break; }
              if (!v_ready) {
                if (!wait_bar(bar(L::B_V + vst), (vi / L::kVStages) & 1, ctx, 5)) { ok = false; break; }
                v_ready = true;
              }
              tc_fence_after();
              gemm_ts_mn<D>(tmem + 256 + t * D, tmem + t * 128, sbase + L::kV + vst * L::kTile,
                            idesc_pv, !first_pv[t]);
              first_pv[t] = false;
              ++pcount[t];
              if (kt == u.ke[t]) mma_commit(bar(L::B_ODONE + t));
            }
            if (t == 1) mma_commit(bar(L::B_VE + vst));   // V(j) has no reader left
            if (next && u.part(t, kt + 1)) {
              if (!k_next_ready) {
                if (!wait_k(k0 + j + 1)) { ok = false; break; }
                k_next_ready = true;
              }
              if (!issue_s(t, k0 + j + 1)) { ok = false; break; }
              if (kt + 1 == u.ke[t]) mma_commit(bar(L::B_QE + t));   // last S on Q_t
            }
          }
          if (ok && next) mma_commit(bar(L::B_KE + (k0 + j + 1) % L::kKStages));
        }
        k_used = k0 + u.n_kv;
        v_used = v0 + u.n_kv;
      }
    }
  } else if (warp >= 10) {
    // ---------------- rotation warps (fused RoPE of the queries) ----------------
    // Both rotate half of each query tile's rows as soon as it has landed; warp 10 then lets
    // the MMAs at it, sends the rotated rows to q_rot (TMA stores for whole atoms, its own
    // stores for atoms that straddle two runs or reach past the end) and releases the slot
    // for the next load once they have been read out.
    if (kRope) {
      const int part = warp - 10;
      const RopeLane rl = rope_lane<D>(p.rope_log2_base, p.rope_pi_scale);
      int q_loads[2] = {0, 0};
      bool ok = true;
      for (int ku = 0; ok; ++ku) {
        FwdUnit u;
        if (!fwd_unit_k<kFront>(p, sched, n_units, recs, ku, u)) break;
        for (int t = 0; t < 2; ++t) {
          if (!u.tv[t]) continue;
          if (!warp_wait(bar(L::B_Q + t), q_loads[t] & 1, ctx, 11)) { ok = false; break; }
          const int k = q_loads[t]++;
          const Runs tr = rolled_runs(head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0),
                                      u.qt[t] * kTileRows);
          const uint32_t q_s = sbase + L::kQ + t * L::kTile;
          rope_query_tile<D>(q_s, tr, rl, p.rope_pi_scale, part);
          if (lane == 0) mbar_arrive(bar(L::B_RR + t));
          if (part != 0) continue;
          if (!warp_wait(bar(L::B_RR + t), k & 1, ctx, 13)) { ok = false; break; }
          const uint32_t plain = straddled_atoms(tr) | past_end_atoms(tr);
          if (lane == 0) {
            mbar_arrive(bar(L::B_QR + t));
            store_tile<D>(q_s, &tmQR, &tmQR8, u.b, u.h, tr, plain);
          }
          store_atoms_warp<D>(smem + L::kQ + t * L::kTile, plain, tr, p.q_rot, p.N, p.Hq, u.b, u.h);
          __syncwarp();
          if (lane == 0) {
            bulk_wait_read_all();
            mbar_arrive(bar(L::B_QW + t));
          }
        }
      }
      if (lane == 0) bulk_wait_all();   // every rotated row written before the CTA exits
      __syncwarp();
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int wg = warp / 4;
    const int row = threadIdx.x % 128;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const uint32_t s_col = t_lane + wg * 128;
    const uint32_t o_col = t_lane + 256 + wg * D;
    const float c = p.scale_log2;
    int s_cnt = 0, o_cnt = 0;
    bool ok = true;
    for (int ku = 0; ok; ++ku) {
      FwdUnit u;
      if (!fwd_unit_k<kFront>(p, sched, n_units, recs, ku, u)) break;
      if (!u.tv[wg]) continue;
      const int r = u.qt[wg] * kTileRows + row;
      const bool row_valid = r < p.N;
      const int lo = row_valid ? group_begin(r, p.G, u.wrap_h) : u.kb[wg] * kTileRows;
      const int hi = row_valid ? r : u.kb[wg] * kTileRows;
      float m_run = -INFINITY, l_run = 0.f;
      for (int kt = u.kb[wg], cnt = 0; kt <= u.ke[wg]; ++kt, ++cnt, ++s_cnt) {
        if (!warp_wait(bar(L::B_S + wg), s_cnt & 1, ctx, 7)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        {
          uint32_t raw[128];
          tmem_ld128(s_col, raw);
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(raw[i]);
        }
        const int cl = lo - kt * kTileRows, ch = hi - kt * kTileRows;
        if (__any_sync(0xffffffffu, cl > 0 || ch < kTileRows - 1)) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = (i < cl || i > ch) ? -INFINITY : s[i];
        }
        const float m_cand = fmaxf(m_run, max_tree128(s) * c);
        const bool need = m_cand > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          // 0 when m_run = -inf; 1 for a row that has seen no allowed key yet (its O and l
          // are still zero) while others in the warp rescale: -inf - -inf would be NaN
          const float alpha = m_cand == -INFINITY ? 1.f : fast_exp2(m_run - m_cand);
          if (cnt > 0) {
#pragma unroll 1
            for (int j = 0; j < D / 32; ++j) {
              uint32_t ov[32];
              tmem_ld32(o_col + 32 * j, ov);
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st32(o_col + 32 * j, ov);
            }
          }
          l_run *= alpha;
          m_run = m_cand;
        }
        // P = exp2(c s - m), two columns per packed f32x2 multiply-add and sum.
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t a = f2_fma(f2_pack(s[32 * j + 2 * i], s[32 * j + 2 * i + 1]), c2, nm2);
            const float e0 = fast_exp2(f2_lo(a)), e1 = fast_exp2(f2_hi(a));
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(e0, e1));
            pk[i] = pack_bf16(e0, e1);
          }
          tmem_st16(s_col + 16 * j, pk);
        }
        acc[0] = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        l_run += f2_lo(acc[0]) + f2_hi(acc[0]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::B_P + wg));
      }
      if (!ok || !warp_wait(bar(L::B_ODONE + wg), o_cnt & 1, ctx, 8)) { ok = false; break; }
      ++o_cnt;
      tc_fence_after();
      // Epilogue: O / l in bf16 through this warp's staging area (row `lane` of the warp at
      // 128 bytes per 64 columns, 16-byte chunks XOR-swizzled by row: four 8-row atoms in the
      // 128-byte-swizzled layout of an 8-row TMA box). An atom whose 8 rows are all in the
      // sequence and land on 8 consecutive tokens goes out as one TMA box per 64 columns; the
      // rows of other atoms (a run boundary of the roll inside the atom, or the end of the
      // sequence) are stored by the warp, four whole 128-byte rows per instruction. Bulk stores
      // keep the 32 KB of a tile off the SM's load/store path, which the next unit's barrier
      // waits and shared-memory reads share (row stores held them up by ~2700 cycles).
      const float inv_l = 1.f / l_run;
      uint8_t* stage = smem + L::kStage + warp * L::kStageWarp;
      const uint32_t stage_s = sbase + L::kStage + warp * L::kStageWarp;
      const int r_warp = u.qt[wg] * kTileRows + (warp % 4) * 32;
      const HeadRemap hm = head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0);
      const int tok_l = r_warp + lane < p.N ? hm.token(r_warp + lane) : -1;
      const int tok_7 = __shfl_down_sync(0xffffffffu, tok_l, 7);
      const unsigned boxed = __ballot_sync(
          0xffffffffu, (lane & 7) == 0 && r_warp + lane + 7 < p.N && tok_7 - tok_l == 7);
      int tok_atom[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) tok_atom[a] = __shfl_sync(0xffffffffu, tok_l, 8 * a);
#pragma unroll 1
      for (int half = 0; half < D / 64; ++half) {
        // the staging area is free once the TMA unit has read the boxes sent from it
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ov[32];
          tmem_ld32(o_col + 64 * half + 32 * q2, ov);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w4;
            w4.x = pack_bf16(__uint_as_float(ov[8 * v + 0]) * inv_l, __uint_as_float(ov[8 * v + 1]) * inv_l);
            w4.y = pack_bf16(__uint_as_float(ov[8 * v + 2]) * inv_l, __uint_as_float(ov[8 * v + 3]) * inv_l);
            w4.z = pack_bf16(__uint_as_float(ov[8 * v + 4]) * inv_l, __uint_as_float(ov[8 * v + 5]) * inv_l);
            w4.w = pack_bf16(__uint_as_float(ov[8 * v + 6]) * inv_l, __uint_as_float(ov[8 * v + 7]) * inv_l);
            const int chunk = 4 * q2 + v;
            *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) * 16)) = w4;
          }
        }
        fence_async_smem();   // the TMA unit reads the staging area through the async proxy
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int a = 0; a < 4; ++a)
            if ((boxed >> (8 * a)) & 1u)
              tma_store_4d(&tmO8, stage_s + a * 1024, 64 * half, u.h, tok_atom[a], u.b);
          bulk_commit();
        }
        if (boxed != 0x01010101u) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3), chunk = lane & 7;
            const int rq = r_warp + rr;
            if (rq < p.N && !((boxed >> (rr & ~7)) & 1u)) {
              const uint4 w4 = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((chunk ^ (rr & 7)) * 16));
              __nv_bfloat16* dst = p.o + u.b * p.o_sb + hm.token(rq) * p.o_st +
                                   static_cast<long long>(u.h) * D + 64 * half + 8 * chunk;
              *reinterpret_cast<uint4*>(dst) = w4;
            }
          }
        }
        __syncwarp();
      }
      if (row_valid) {
        const int tok = head_remap(p.N, p.G, u.shift_h, kFront ? u.front_h : 0).token(r);
        p.lse[(static_cast<size_t>(u.b) * p.Hq + u.h) * p.N + tok] =
            (m_run + __log2f(l_run)) * 0.6931471805599453f;
      }
      // O_t is read: the next unit's first PV on it waits for this warpgroup's P anyway.
      tc_fence_before();
    }
    // Every box has been written before the CTA's shared memory goes away.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    if (lane == 0) {
      mma_commit(bar(L::B_DRAIN));
      drain_wait(bar(L::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace s2
