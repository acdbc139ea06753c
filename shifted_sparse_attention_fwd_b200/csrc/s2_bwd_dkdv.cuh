// S²-Attn backward, dK and dV, on sm_100a tensor cores.
//
// Gradient of the per-group causal self-attention of LongLoRA's Algorithm 1 (summary page
// §3.4), taken through the roll: a key/value row t of kv head j receives, from every query
// head h that reads it (grouped-query heads h with h / (Hq/Hkv) == j), the contributions of
// the query rows that follow it in h's rolled order inside the same group:
//   P^T  = exp(scale * K Q^T - LSE)             (recomputed, per column = query row)
//   dV  += P^T dO
//   dP^T = V dO^T
//   dS^T = P^T o (dP^T - D)
//   dK  += scale * dS^T Q
// A work tile is 128 ORIGINAL key/value rows of one (batch, kv head), so the tile is shared
// by all its query heads whatever their roll, and dK/dV are written once, without atomics.
// For each query head the rows map to at most two runs of rolled rows (three with the
// Variant 3 reordering); the query tiles
// visited are those covering [rolled row, end of its group) for every row of the tile.
// The kernel is persistent: each CTA claims work tiles from a global counter (heaviest first,
// grouped for L2 reuse), so one tile's epilogue overlaps the next tile's loads and first MMAs
// and the load stays balanced.
//
// Warp roles (608 threads): warps 0-15 elementwise — kv row i (TMEM lane i) is shared by the
// four warps i/32 + 4 g, g = 0..3, warp group g taking query columns [32 g, 32 g + 32), so
// four warps per SM sub-partition hide each other's TMEM and special-function latency;
// warp 16 TMA producer (K, V per tile; Q, dO, LSE2, D per query tile, 2 stages); warp 17
// TMEM allocator + MMA issuer; warp 18 store issuer: the elementwise warps leave each dS
// tile (for the dQ pass) and the finished dV and dK tiles in a shared-memory staging buffer,
// and warp 18 hands them to the TMA unit, so no elementwise warp waits on global stores.
// TMEM: S^T [0,128) and dP^T [128,256); each column group packs its bf16 P^T (dS^T) into the
// first 16 of its own 32 fp32 input columns, so the warps of a row never overwrite each
// other's unread data, and the dV (dK) MMA reads the A operand group by group
// (gemm_ts_mn_grouped); dV [256,256+D), dK [256+D, 256+2D).
#pragma once

#include "s2_common.cuh"
#include "s2_tmem_wide.cuh"

namespace s2 {

struct BwdParams {
  TensorRef q, k, v, dO;   // the inputs again, for rows the TMA boxes cannot move
  const float* lse2;   // [B, Hq, N]  LSE * log2(e)
  const float* dvec;   // [B, Hq, N]  D = rowsum(dO o O)
  __nv_bfloat16* dq;
  long long dq_sb, dq_st;   // element strides of dQ's batch and token axes
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int B, Hq, Hkv, N, G, shift_head_begin, shift;
  int wrap;           // wrap split of the shifted heads' last group (kNoWrapSplit: none)
  int front;          // Variant 3: the shifted heads' last group lists the wrapped tokens first
  float scale_log2;   // scale * log2(e)
  float scale;
  unsigned int* err;
  unsigned long long timeout_ns;
  // kv heads [kvh_begin, kvh_begin + kvh_count) are processed by this pass (with all their
  // query heads); dS tiles, when `ds` is set, are numbered within the pass.
  int kvh_begin, kvh_count;
  __nv_bfloat16* ds;   // bf16 dS tiles for the dQ pass (DsSlots layout), or null
  DsSlots slots;
  unsigned int* sched;   // {next, done} work counter of this launch (claim_unit)
};

constexpr uint32_t kDsTileBytes = kTileRows * kTileRows * 2;   // one bf16 dS tile, 32 KB

// First element of dS slot `slot` of (batch b, query head hq of this pass).
__device__ __forceinline__ __nv_bfloat16* ds_slot_ptr(const BwdParams& p, int b, int hq,
                                                      long long slot) {
  const int rep = p.Hq / p.Hkv;
  const long long hl = static_cast<long long>(b) * (p.kvh_count * rep) + (hq - p.kvh_begin * rep);
  return p.ds + (hl * p.slots.per_head + slot) * (kDsTileBytes / 2);
}

// Elementwise column groups per kv row (warps per TMEM lane quadrant) and their width.
constexpr int kDkdvGroups = 4;
constexpr int kDkdvCols = kTileRows / kDkdvGroups;
constexpr int kDkdvEwWarps = 4 * kDkdvGroups;
constexpr int kDkdvEwThreads = 32 * kDkdvEwWarps;
static_assert(kDkdvCols == 32, "the elementwise code moves 32 columns per TMEM access");

template <int D>
struct DkdvLayout {
  static constexpr uint32_t kTile = Tile<D>::kBytes;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTile;
  static constexpr uint32_t kQ = kV + kTile;          // 2 stages
  static constexpr uint32_t kDO = kQ + 2 * kTile;     // 2 stages
  static constexpr uint32_t kStage = kDO + 2 * kTile; // dS tile, or the dV / dK tile, 32 KB
  static constexpr uint32_t kLse = kStage + kDsTileBytes;   // 2 stages x 128 floats
  static constexpr uint32_t kDv = kLse + 1024;               // 2 stages x 128 floats
  static constexpr uint32_t kRing = kDv + 1024;             // claimed work units
  static constexpr uint32_t kBar = kRing + 4 * kUnitRing;
  enum { B_KV = 0, B_KVE = 1, B_QF = 2, B_QE = 4, B_S = 6, B_DP = 7, B_P = 8, B_DS = 9,
         B_ACC = 10, B_ACCE = 11, B_STF = 12, B_STE = 13, B_DRAIN = 14, B_UF = 15,
         B_UE = B_UF + kUnitRing, B_COUNT = B_UE + kUnitRing };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  // No alignment slack: the kernel checks that the window starts on a 1024-byte boundary.
  static constexpr uint32_t kLaunchBytes = kBytes > 116 * 1024 ? kBytes : 116 * 1024;
  static constexpr int kThreads = 32 * (kDkdvEwWarps + 3);
};

// Work tile u (heaviest first) of this pass -> (b, kv head, first original row).
__device__ __forceinline__ void dkdv_tile(const BwdParams& p, int u, int& b, int& kvh, int& t0) {
  const int rep = p.Hq / p.Hkv;
  int shb = p.shift_head_begin - p.kvh_begin * rep;
  shb = shb < 0 ? 0 : (shb > p.kvh_count * rep ? p.kvh_count * rep : shb);
  kv_tile_coords_chunked(u, p.B, p.kvh_count * rep, p.kvh_count, p.N, p.G, shb, p.shift,
                         kL2Chunk, b, kvh, t0);
  kvh += p.kvh_begin;
}

// The Q and dO tiles and the LSE2 / D values of one query tile when TMA boxes and bulk copies
// cannot move all of it (a remap run starting or ending inside an 8-row atom, or LSE2 / D runs
// that are not 16-byte aligned, which happens when G or the roll is not a multiple of 8): the
// odd parts are copied by this thread first, then `fb` is armed with the bytes the copy engines
// still deliver. Kept out of line so the common path stays as small as it is.
template <int D>
__device__ __noinline__ void dkdv_load_query_tile_slow(
    uint32_t q_dst, uint32_t do_dst, uint32_t sl, uint32_t sd, const CUtensorMap* tmQ,
    const CUtensorMap* tmQ8, const CUtensorMap* tmO, const CUtensorMap* tmO8, uint32_t fb,
    const TensorRef q, const TensorRef dO, const float* lse_row, const float* d_row, int N, int b,
    int hq, const Runs tr, uint32_t skip, bool aligned) {
  if (skip) {
    fill_atoms<D>(q_dst, skip, tr, q, b, hq);
    fill_atoms<D>(do_dst, skip, tr, dO, b, hq);
  }
  if (!aligned) {
    int base = 0;
    for (int r = 0; r < tr.n; ++r) {
      for (int j = 0; j < tr.len[r]; ++j) {
        cp_async4(sl + 4u * (base + j), lse_row + tr.src[r] + j);
        cp_async4(sd + 4u * (base + j), d_row + tr.src[r] + j);
      }
      base += tr.len[r];
    }
    cp_async_wait_all();
  }
  mbar_expect_tx(fb, 2 * tma_tile_bytes<D>(skip) + (aligned ? 8u * tr.valid : 0u));
  load_tile<D>(q_dst, tmQ, tmQ8, fb, b, hq, tr, N, skip);
  load_tile<D>(do_dst, tmO, tmO8, fb, b, hq, tr, N, skip);
  if (aligned) {
    int base = 0;
    for (int r = 0; r < tr.n; ++r) {
      bulk_load(sl + 4u * base, lse_row + tr.src[r], 4u * tr.len[r], fb);
      bulk_load(sd + 4u * base, d_row + tr.src[r], 4u * tr.len[r], fb);
      base += tr.len[r];
    }
  }
}

// kFront: built for the Variant 3 reordering (otherwise p.front is ignored).
template <int D, bool kFront>
__global__ void __launch_bounds__(32 * (kDkdvEwWarps + 3), 1)
    s2_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ8,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK8,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmV8,
                       const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO8,
                       const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                       const BwdParams p) {
  using L = DkdvLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {   // the layout has no slack for realignment: report, do nothing
    if (threadIdx.x == 0) atomicCAS(p.err, 0u, (static_cast<uint32_t>(KID_DKDV) << 8) | 0xFFu);
    return;
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return sbase + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_DKDV};

  const int rep = p.Hq / p.Hkv;
  const int T = (p.N + kTileRows - 1) / kTileRows;
  const int n_tiles = p.B * p.kvh_count * T;
  auto head_map = [&](int hq) {
    const bool shifted = hq >= p.shift_head_begin;
    return head_remap(p.N, p.G, shifted ? p.shift : 0, (kFront && shifted) ? p.front : 0);
  };
  auto head_wrap = [&](int hq) { return hq >= p.shift_head_begin ? p.wrap : kNoWrapSplit; };
  auto pairs_of = [&](int kvh, int t0) {
    int total = 0;
    for (int hq = kvh * rep; hq < (kvh + 1) * rep; ++hq)
      total += kv_tile_qtiles(head_map(hq), t0, head_wrap(hq)).count();
    return total;
  };

  constexpr int kProducer = kDkdvEwWarps, kMma = kDkdvEwWarps + 1, kStore = kDkdvEwWarps + 2;
  if (warp == kProducer && lane == 0) {
    mbar_init(bar(L::B_KV), 1);
    mbar_init(bar(L::B_KVE), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_QF + s), 1);
      mbar_init(bar(L::B_QE + s), 1);
    }
    mbar_init(bar(L::B_S), 1);
    mbar_init(bar(L::B_DP), 1);
    mbar_init(bar(L::B_P), kDkdvEwThreads);
    mbar_init(bar(L::B_DS), kDkdvEwThreads);
    mbar_init(bar(L::B_ACC), 1);
    mbar_init(bar(L::B_ACCE), kDkdvEwThreads);
    mbar_init(bar(L::B_STF), kDkdvEwThreads);
    mbar_init(bar(L::B_STE), 1);
    mbar_init(bar(L::B_DRAIN), 1);
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(bar(L::B_UF + i), 1);
      mbar_init(bar(L::B_UE + i), kDkdvEwWarps + 2);   // MMA, elementwise warps, store
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO);
  }
  if (warp == kMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_s = tmem, tm_dp = tmem + 128, tm_dv = tmem + 256, tm_dk = tmem + 256 + D;
  const uint32_t tm_p = tmem, tm_ds = tmem + 128;   // bf16 P^T and dS^T, grouped A operands
  volatile int* ring = reinterpret_cast<volatile int*>(smem + L::kRing);
  // Every role walks the same sequence of work tiles, claimed by the producer.
  auto next_unit = [&](int k, int& u, bool whole_warp, uint32_t site) {
    return read_unit(k, u, ring, bar(L::B_UF), bar(L::B_UE), ctx, site, whole_warp);
  };

  if (warp == kProducer) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int last_parity[2] = {-1, -1};
      int n = 0, tc = 0, kv_loads = 0;
      bool ok = true;
      // Units are claimed one ahead: unit k + 1 is published as soon as unit k's K and V
      // loads are issued, so the other roles never wait for the producer to finish issuing
      // unit k's query tiles before they can start on the next unit.
      int u_next;
      ok = publish_unit(0, u_next, p.sched, n_tiles, ring, bar(L::B_UF), bar(L::B_UE), ctx, 15);
      for (int k = 0; ok; ++k, ++tc) {
        const int u = u_next;
        if (u < 0) break;
        int b, kvh, t0;
        dkdv_tile(p, u, b, kvh, t0);
        // K and V of the previous tile are free once its last S and dP MMAs are done.
        if (tc > 0 && !wait_bar(bar(L::B_KVE), (tc - 1) & 1, ctx, 11)) { ok = false; break; }
        mbar_expect_tx(bar(L::B_KV), 2 * L::kTile);
        const Runs kv_runs = identity_runs(t0, p.N);
        load_tile<D>(sbase + L::kK, &tmK, &tmK8, bar(L::B_KV), b, kvh, kv_runs, p.N);
        load_tile<D>(sbase + L::kV, &tmV, &tmV8, bar(L::B_KV), b, kvh, kv_runs, p.N);
        ++kv_loads;
        if (!publish_unit(k + 1, u_next, p.sched, n_tiles, ring, bar(L::B_UF), bar(L::B_UE), ctx, 15)) {
          ok = false;
          break;
        }
        for (int hq = kvh * rep; ok && hq < (kvh + 1) * rep; ++hq) {
          const HeadRemap hm = head_map(hq);
          const QTileRanges qr = kv_tile_qtiles(hm, t0, head_wrap(hq));
          const size_t row0 = (static_cast<size_t>(b) * p.Hq + hq) * p.N;
          const float* lse_row = p.lse2 + row0;
          const float* d_row = p.dvec + row0;
          for (int i = 0; i < qr.count(); ++i, ++n) {
            const int st = n & 1;
            if (n >= 2 && !wait_bar(bar(L::B_QE + st), ((n >> 1) - 1) & 1, ctx, 1)) { ok = false; break; }
            const Runs tr = rolled_runs(hm, qr.at(i) * kTileRows);
            const uint32_t fb = bar(L::B_QF + st);
            const uint32_t sl = sbase + L::kLse + st * 512, sd = sbase + L::kDv + st * 512;
            // TMA boxes need runs of whole 8-row atoms, bulk copies 16-byte aligned runs.
            const uint32_t skip = straddled_atoms(tr);
            bool aligned = true;
            {
              int base = 0;
#pragma unroll
              for (int r = 0; r < 3; ++r)
                if (r < tr.n) {
                  aligned = aligned && ((base | tr.len[r]) & 3) == 0 && ((row0 + tr.src[r]) & 3) == 0;
                  base += tr.len[r];
                }
            }
            if (skip != 0 || !aligned) {
              dkdv_load_query_tile_slow<D>(sbase + L::kQ + st * L::kTile,
                                           sbase + L::kDO + st * L::kTile, sl, sd, &tmQ, &tmQ8,
                                           &tmO, &tmO8, fb, p.q, p.dO, lse_row, d_row, p.N, b,
                                           hq, tr, skip, aligned);
            } else {
              mbar_expect_tx(fb, 2 * L::kTile + 8u * tr.valid);
              load_tile<D>(sbase + L::kQ + st * L::kTile, &tmQ, &tmQ8, fb, b, hq, tr, p.N);
              load_tile<D>(sbase + L::kDO + st * L::kTile, &tmO, &tmO8, fb, b, hq, tr, p.N);
              int base = 0;
#pragma unroll
              for (int r = 0; r < 3; ++r) {
                if (r < tr.n) {
                  bulk_load(sl + 4u * base, lse_row + tr.src[r], 4u * tr.len[r], fb);
                  bulk_load(sd + 4u * base, d_row + tr.src[r], 4u * tr.len[r], fb);
                  base += tr.len[r];
                }
              }
            }
            last_parity[st] = (n >> 1) & 1;
          }
        }
      }
      if (kv_loads > 0) drain_wait(bar(L::B_KV), (kv_loads - 1) & 1, p.timeout_ns);
      for (int s = 0; s < 2; ++s)
        if (last_parity[s] >= 0) drain_wait(bar(L::B_QF + s), last_parity[s], p.timeout_ns);
    }
  } else if (warp == kMma) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);  // K Q^T, V dO^T
      constexpr uint32_t idesc_acc = idesc_bf16(128, D, false, true);   // P^T dO, dS^T Q
      int n = 0, tc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++tc) {
        int u;
        if (!next_unit(k, u, false, 16)) break;
        if (u < 0) break;
        int b, kvh, t0;
        dkdv_tile(p, u, b, kvh, t0);
        const int total = pairs_of(kvh, t0);
        ok = wait_bar(bar(L::B_KV), tc & 1, ctx, 2) &&
             wait_bar(bar(L::B_QF + (n & 1)), (n >> 1) & 1, ctx, 3);
        if (!ok) break;
        tc_fence_after();
        gemm_ss_k<D>(tm_s, sbase + L::kK, sbase + L::kQ + (n & 1) * L::kTile, idesc_s);
        mma_commit(bar(L::B_S));
        for (int i = 0; i < total; ++i, ++n) {
          const int st = n & 1;
          const uint32_t q_s = sbase + L::kQ + st * L::kTile, do_s = sbase + L::kDO + st * L::kTile;
          gemm_ss_k<D>(tm_dp, sbase + L::kV, do_s, idesc_s);
          mma_commit(bar(L::B_DP));
          if (i + 1 == total) mma_commit(bar(L::B_KVE));   // last reader of K and V issued
          if (!wait_bar(bar(L::B_P), n & 1, ctx, 4)) { ok = false; break; }
          // The previous tile's dV and dK must have been read out before they restart.
          if (i == 0 && tc > 0 && !wait_bar(bar(L::B_ACCE), (tc - 1) & 1, ctx, 12)) { ok = false; break; }
          tc_fence_after();
          gemm_ts_mn_grouped<D, kDkdvCols>(tm_dv, tm_p, do_s, idesc_acc, i > 0);
          if (i + 1 < total) {
            const int st1 = (n + 1) & 1;
            if (!wait_bar(bar(L::B_QF + st1), ((n + 1) >> 1) & 1, ctx, 5)) { ok = false; break; }
            tc_fence_after();
            gemm_ss_k<D>(tm_s, sbase + L::kK, sbase + L::kQ + st1 * L::kTile, idesc_s);
            mma_commit(bar(L::B_S));
          }
          if (!wait_bar(bar(L::B_DS), n & 1, ctx, 6)) { ok = false; break; }
          tc_fence_after();
          gemm_ts_mn_grouped<D, kDkdvCols>(tm_dk, tm_ds, q_s, idesc_acc, i > 0);
          mma_commit(bar(L::B_QE + st));
        }
        if (ok) mma_commit(bar(L::B_ACC));
      }
    }
  } else if (warp == kStore) {
    // ---------------- store issuer ----------------
    // Mirrors the elementwise warps' use of the staging buffer: per query tile a dS tile
    // (when handing off to the dQ pass), per work tile dV then dK.
    if (lane == 0) {
      int use = 0;
      bool ok = true;
      mbar_arrive(bar(L::B_STE));   // the buffer starts out free
      auto hand_over = [&](auto&& issue) -> bool {
        if (!wait_bar(bar(L::B_STF), use & 1, ctx, 13)) return false;
        issue();
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(bar(L::B_STE));
        ++use;
        return true;
      };
      for (int k = 0; ok; ++k) {
        int u;
        if (!next_unit(k, u, false, 17)) break;
        if (u < 0) break;
        int b, kvh, t0;
        dkdv_tile(p, u, b, kvh, t0);
        if (p.ds) {
          for (int hq = kvh * rep; ok && hq < (kvh + 1) * rep; ++hq) {
            const HeadRemap hm = head_map(hq);
            const QTileRanges qr = kv_tile_qtiles(hm, t0, head_wrap(hq));
            for (int i = 0; ok && i < qr.count(); ++i) {
              const int qt = qr.at(i);
              const int idx = qtile_kv_span(hm, qt, head_wrap(hq)).index_of(t0 / kTileRows);
              ok = hand_over([&] {
                if (idx >= 0)
                  bulk_store(ds_slot_ptr(p, b, hq, p.slots.base(qt) + idx), sbase + L::kStage,
                             kDsTileBytes);
              });
            }
          }
        }
        for (int which = 0; ok && which < 2; ++which)
          ok = hand_over([&] {
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_store_4d(which == 0 ? &tmDV : &tmDK, sbase + L::kStage + h * Tile<D>::kHalfBytes,
                           64 * h, kvh, t0, b);
          });
      }
      bulk_wait_all();
    }
  } else {
    // ---------------- elementwise warps ----------------
    constexpr int W = kDkdvCols;                   // query columns per thread
    constexpr int CPT = D / kDkdvGroups;           // dV / dK columns per thread in the epilogue
    const int grp = warp / 4;                      // query columns [W grp, W grp + W)
    const int row = (warp % 4) * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const float c = p.scale_log2;
    const float* s_lse = reinterpret_cast<const float*>(smem + L::kLse);
    const float* s_dv = reinterpret_cast<const float*>(smem + L::kDv);
    uint8_t* stage = smem + L::kStage;
    int n = 0, tc = 0, use = 0;
    bool ok = true;
    // Wait for the staging buffer, fill it with `fill`, hand it to the store issuer.
    auto stage_out = [&](auto&& fill) -> bool {
      if (!warp_wait(bar(L::B_STE), use & 1, ctx, 14)) return false;
      fill();
      fence_async_smem();
      mbar_arrive(bar(L::B_STF));
      ++use;
      return true;
    };
    for (int k = 0; ok; ++k, ++tc) {
      int u;
      if (!next_unit(k, u, true, 18)) break;
      if (u < 0) break;
      int b, kvh, t0;
      dkdv_tile(p, u, b, kvh, t0);
      const int t = t0 + row;
      const bool kv_valid = t < p.N;
      for (int hq = kvh * rep; ok && hq < (kvh + 1) * rep; ++hq) {
        const HeadRemap hm = head_map(hq);
        const QTileRanges qr = kv_tile_qtiles(hm, t0, head_wrap(hq));
        const int r_k = kv_valid ? hm.rolled(t) : 0;
        const int ge_k = min_i(group_end(r_k, p.G, head_wrap(hq)), p.N);
        for (int i = 0; i < qr.count(); ++i, ++n) {
          const int st = n & 1;
          const int q0 = qr.at(i) * kTileRows + W * grp;
          const int cl = kv_valid ? r_k - q0 : 1;
          const int ch = kv_valid ? ge_k - 1 - q0 : 0;
          const bool mask = __any_sync(0xffffffffu, cl > 0 || ch < W - 1);
          if (!warp_wait(bar(L::B_QF + st), (n >> 1) & 1, ctx, 7)) { ok = false; break; }
          if (!warp_wait(bar(L::B_S), n & 1, ctx, 8)) { ok = false; break; }
          tc_fence_after();
          const float* lse_t = s_lse + st * 128 + W * grp;
          const float* d_t = s_dv + st * 128 + W * grp;
          // P^T phase: W columns of S^T -> P^T (bf16), kept in registers for the dS phase.
          // The columns are read in two halves of 16 to keep fewer values in flight.
          uint32_t pk[W / 2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t raw[16];
            tmem_ld16(t_lane + W * grp + 16 * h, raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int col = 16 * h + 2 * e;
              float x0 = fast_exp2(fmaf(__uint_as_float(raw[2 * e]), c, -lse_t[col]));
              float x1 = fast_exp2(fmaf(__uint_as_float(raw[2 * e + 1]), c, -lse_t[col + 1]));
              if (mask) {
                x0 = (col >= cl && col <= ch) ? x0 : 0.f;
                x1 = (col + 1 >= cl && col + 1 <= ch) ? x1 : 0.f;
              }
              pk[8 * h + e] = pack_bf16(x0, x1);
            }
          }
          tmem_st16(t_lane + W * grp, pk);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(L::B_P));
          // dS^T phase: dS^T = P^T o (dP^T - D).
          if (!warp_wait(bar(L::B_DP), n & 1, ctx, 9)) { ok = false; break; }
          tc_fence_after();
          uint32_t ds[W / 2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t raw[16];
            tmem_ld16(t_lane + 128 + W * grp + 16 * h, raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int col = 16 * h + 2 * e;
              const float2 pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[8 * h + e]));
              float y0 = pf.x * (__uint_as_float(raw[2 * e]) - d_t[col]);
              float y1 = pf.y * (__uint_as_float(raw[2 * e + 1]) - d_t[col + 1]);
              if (mask) {   // exact zeros where P is masked, whatever D holds for padding rows
                y0 = (col >= cl && col <= ch) ? y0 : 0.f;
                y1 = (col + 1 >= cl && col + 1 <= ch) ? y1 : 0.f;
              }
              ds[8 * h + e] = pack_bf16(y0, y1);
            }
          }
          tmem_st16(t_lane + 128 + W * grp, ds);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(L::B_DS));
          if (p.ds) {
            // The dS tile for the dQ pass, in its global layout (DsSlots): 16 blocks of 2 KB,
            // block c holding query columns [8c, 8c + 8) of all 128 kv rows, 16 bytes per row.
            ok = stage_out([&] {
#pragma unroll
              for (int c8 = 0; c8 < W / 8; ++c8)
                *reinterpret_cast<uint4*>(stage + ((W / 8) * grp + c8) * 2048 + row * 16) =
                    make_uint4(ds[4 * c8], ds[4 * c8 + 1], ds[4 * c8 + 2], ds[4 * c8 + 3]);
            });
            if (!ok) break;
          }
        }
      }
      if (!ok || !warp_wait(bar(L::B_ACC), tc & 1, ctx, 10)) { ok = false; break; }
      tc_fence_after();
      // dV, then scale * dK: this thread's CPT columns of its row, in bf16, into the staging
      // buffer in the 128-byte-swizzled layout of the TMA tile (64-column boxes of 128 rows).
#pragma unroll 1
      for (int which = 0; ok && which < 2; ++which) {
        const uint32_t src = (which == 0 ? tm_dv : tm_dk) - tmem + t_lane;
        const float mul = which == 0 ? 1.f : p.scale;
        uint32_t pkd[CPT / 2];
#pragma unroll
        for (int j = 0; j < CPT / 16; ++j) {
          uint32_t rr[16];
          tmem_ld16(src + CPT * grp + 16 * j, rr);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pkd[8 * j + e] = pack_bf16(__uint_as_float(rr[2 * e]) * mul, __uint_as_float(rr[2 * e + 1]) * mul);
        }
        if (which == 1) {   // both accumulators are in registers: the MMA may reuse them
          tc_fence_before();
          mbar_arrive(bar(L::B_ACCE));
        }
        ok = stage_out([&] {
#pragma unroll
          for (int v = 0; v < CPT / 8; ++v) {
            const int col = CPT * grp + 8 * v;   // first of the 8 columns of chunk v
            const int box = col / 64, chunk = (col % 64) / 8;
            *reinterpret_cast<uint4*>(stage + box * Tile<D>::kHalfBytes + row * 128 +
                                      ((chunk ^ (row & 7)) * 16)) =
                make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
          }
        });
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
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
