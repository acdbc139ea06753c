// S²-Attn backward, dQ from the dS tiles that the dK/dV kernel left in the workspace.
//
// The gradient of LongLoRA's per-group causal attention (summary page §3.4, Algorithm 1)
// with respect to a rolled query row is dQ = scale * dS K, where dS = P o (dP - D) is the
// same matrix the dK/dV kernel already forms (transposed) for dK. That kernel stores each
// bf16 dS tile it computes — one per (rolled query tile, original kv tile) — as 16 blocks of
// 8 query columns x 128 kv rows (16 bytes per row), which is the unswizzled core-matrix
// layout of an MN-major A operand (DsSlots in s2_tiles.cuh), so this pass is a plain
// streaming GEMM: no recomputation of S, P or dP, no softmax.
//
// Persistent: one CTA per SM claims rolled query tiles (heaviest first, grouped for L2 reuse)
// from a global counter; for each it accumulates, over the original kv tiles the query
// tile reads (qtile_kv_span), dQ += dS(qt, t) K(t) in TMEM, then scales, rounds to bf16 and
// stores the rows at their original positions. The sum over kv rows is split by ORIGINAL kv
// tile, which is the tiling the dK/dV kernel works in; kv rows a query row cannot see carry
// dS = 0 there.
//
// Warp roles (192 threads): warp 0 loader (dS tile by a plain bulk copy, K tile by TMA, a
// 3-stage ring of 64 KB); warp 1 TMEM allocator and MMA issuer; warps 2-5 epilogue (warp w
// reads TMEM lanes 32 (w mod 4) ..., stages its 32 rows of bf16 dQ in shared memory and sends
// them out as TMA boxes). TMEM: two dQ accumulators of D columns, so one query tile's
// epilogue overlaps the next one's MMAs.
#pragma once

#include "s2_bwd_dkdv.cuh"

namespace s2 {

template <int D>
struct DqDsLayout {
  static constexpr uint32_t kKBytes = Tile<D>::kBytes;
  static constexpr int kStages = 3;
  static constexpr uint32_t kStageBytes = kDsTileBytes + kKBytes;
  // dQ staging of the epilogue warps: 32 rows x D columns of bf16 each, as D/64 column
  // halves of four 8-row atoms in the 128-byte-swizzled layout of an 8-row TMA box.
  static constexpr uint32_t kOut = kStages * kStageBytes;
  static constexpr uint32_t kOutWarp = 32 * D * 2;
  static constexpr uint32_t kRing = kOut + 4 * kOutWarp;   // claimed work units
  static constexpr uint32_t kBar = kRing + 4 * kUnitRing;
  enum { B_FULL = 0, B_EMPTY = kStages, B_ACC = 2 * kStages, B_ACCE = 2 * kStages + 2,
         B_DRAIN = 2 * kStages + 4, B_UF = 2 * kStages + 5, B_UE = B_UF + kUnitRing,
         B_COUNT = B_UE + kUnitRing };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kLaunchBytes = kBytes + 1024;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 2 * D;
  static_assert(kOut % 1024 == 0 && kLaunchBytes <= 227 * 1024, "shared memory of one CTA");
};

// Query tiles of this pass: (b, query head, rolled tile) for work index u, heaviest first.
__device__ __forceinline__ void dq_ds_tile(const BwdParams& p, int u, int& b, int& hq, int& qt) {
  const int rep = p.Hq / p.Hkv;
  int hl;
  query_tile_coords_chunked(u, p.B, p.kvh_count * rep, p.N, p.G, kL2Chunk, b, hl, qt);
  hq = p.kvh_begin * rep + hl;
}

// kFront: built for the Variant 3 reordering (otherwise p.front is ignored).
template <int D, bool kFront>
__global__ void __launch_bounds__(192, 1)
    s2_bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmK8,
                        const __grid_constant__ CUtensorMap tmDQ8, const BwdParams p) {
  using L = DqDsLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return sbase + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_DQDS};

  const int rep = p.Hq / p.Hkv;
  const int T = (p.N + kTileRows - 1) / kTileRows;
  const int units = p.B * p.kvh_count * rep * T;
  auto head_map = [&](int hq) {
    const bool shifted = hq >= p.shift_head_begin;
    return head_remap(p.N, p.G, shifted ? p.shift : 0, (kFront && shifted) ? p.front : 0);
  };
  auto head_wrap = [&](int hq) { return hq >= p.shift_head_begin ? p.wrap : kNoWrapSplit; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::B_FULL + s), 1);
      mbar_init(bar(L::B_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(L::B_ACC + a), 1);
      mbar_init(bar(L::B_ACCE + a), 4);
    }
    mbar_init(bar(L::B_DRAIN), 1);
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(bar(L::B_UF + i), 1);
      mbar_init(bar(L::B_UE + i), 5);   // MMA thread and the 4 epilogue warps
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmDQ8);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* ring = reinterpret_cast<volatile int*>(smem + L::kRing);

  if (warp == 0) {
    // ---------------- loader ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int u;
        if (!publish_unit(k, u, p.sched, units, ring, bar(L::B_UF), bar(L::B_UE), ctx, 5)) break;
        if (u < 0) break;
        int b, hq, qt;
        dq_ds_tile(p, u, b, hq, qt);
        const KvSpan sp = qtile_kv_span(head_map(hq), qt, head_wrap(hq));
        const __nv_bfloat16* ds0 = ds_slot_ptr(p, b, hq, p.slots.base(qt));
        const int kvh = hq / rep;
        const int count = sp.count();
        for (int i = 0; i < count; ++i, ++it) {
          const int s = it % L::kStages;
          if (it >= L::kStages &&
              !wait_bar(bar(L::B_EMPTY + s), ((it / L::kStages) - 1) & 1, ctx, 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(L::B_FULL + s);
          const uint32_t dst = sbase + s * L::kStageBytes;
          mbar_expect_tx(fb, L::kStageBytes);
          bulk_load(dst, ds0 + static_cast<size_t>(i) * (kDsTileBytes / 2), kDsTileBytes, fb);
          load_tile<D>(dst + kDsTileBytes, &tmK, &tmK8, fb, b, kvh,
                       identity_runs(sp.at(i) * kTileRows, p.N), p.N);
        }
      }
      // Wait (bounded) for the copies still in flight before the CTA may exit.
      for (int k = it - L::kStages < 0 ? 0 : it - L::kStages; k < it; ++k)
        drain_wait(bar(L::B_FULL + k % L::kStages), (k / L::kStages) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // dQ[128 x D] += dS[128 q x 128 kv] K[128 kv x D]: A is dS stored kv-row-major
      // (MN-major A), B is the K tile stored kv-row-major (MN-major B).
      constexpr uint32_t idesc = idesc_bf16(128, D, true, true);
      int it = 0, n = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n) {
        int u;
        if (!read_unit(k, u, ring, bar(L::B_UF), bar(L::B_UE), ctx, 6, false)) break;
        if (u < 0) break;
        int b, hq, qt;
        dq_ds_tile(p, u, b, hq, qt);
        const int count = qtile_kv_span(head_map(hq), qt, head_wrap(hq)).count();
        const int a = n & 1;
        if (n >= 2 && !wait_bar(bar(L::B_ACCE + a), ((n >> 1) - 1) & 1, ctx, 2)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + a * D;
        for (int i = 0; i < count; ++i, ++it) {
          const int s = it % L::kStages;
          if (!wait_bar(bar(L::B_FULL + s), (it / L::kStages) & 1, ctx, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + s * L::kStageBytes;
          const uint64_t a0 = sdesc_noswz(st, 128, 2048);
          const uint64_t b0 = sdesc_sw128(st + kDsTileBytes, Tile<D>::kHalfBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < kTileRows / 16; ++kk) {
            // 16 kv rows per step: 256 bytes into every dS block, 2 KB into the K tile
            mma_ss(d_tmem, a0 + static_cast<uint64_t>((kk * 256) >> 4),
                   b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(L::B_EMPTY + s));
        }
        if (!ok) break;
        mma_commit(bar(L::B_ACC + a));
      }
    }
  } else {
    // ---------------- epilogue warps 2-5 ----------------
    const int quad = warp % 4;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    uint8_t* stage = smem + L::kOut + quad * L::kOutWarp;
    const uint32_t stage_s = sbase + L::kOut + quad * L::kOutWarp;
    int n = 0;
    for (int k = 0;; ++k, ++n) {
      int u;
      if (!read_unit(k, u, ring, bar(L::B_UF), bar(L::B_UE), ctx, 7, true)) break;
      if (u < 0) break;
      int b, hq, qt;
      dq_ds_tile(p, u, b, hq, qt);
      const int a = n & 1;
      if (!warp_wait(bar(L::B_ACC + a), (n >> 1) & 1, ctx, 4)) break;
      tc_fence_after();
      // dQ rows in bf16 through this warp's staging area; an 8-row atom whose rows are all in
      // the sequence and land on 8 consecutive tokens goes out as one TMA box per 64 columns,
      // the rows of other atoms (a run boundary of the roll inside the atom, or the end of the
      // sequence) are stored by the warp. Bulk stores keep the 32 KB of a tile off the SM's
      // load/store path, which the loader's barrier waits share.
      const int r_warp = qt * kTileRows + quad * 32;
      const HeadRemap hm = head_map(hq);
      const int tok_l = r_warp + lane < p.N ? hm.token(r_warp + lane) : -1;
      const int tok_7 = __shfl_down_sync(0xffffffffu, tok_l, 7);
      const unsigned boxed = __ballot_sync(
          0xffffffffu, (lane & 7) == 0 && r_warp + lane + 7 < p.N && tok_7 - tok_l == 7);
      int tok_atom[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) tok_atom[i] = __shfl_sync(0xffffffffu, tok_l, 8 * i);
      // the staging area is free once the TMA unit has read the last tile's boxes
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + a * D + 32 * j, rr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(rr[2 * e]) * p.scale,
                            __uint_as_float(rr[2 * e + 1]) * p.scale);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int chunk = (j % 2) * 4 + v;
          *reinterpret_cast<uint4*>(stage + (j / 2) * 4096 + lane * 128 + ((chunk ^ (lane & 7)) * 16)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      fence_async_smem();   // the TMA unit reads the staging area through the async proxy
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(L::B_ACCE + a));   // the accumulator is read: the MMA may reuse it
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if ((boxed >> (8 * i)) & 1u)
              tma_store_4d(&tmDQ8, stage_s + h * 4096 + i * 1024, 64 * h, hq, tok_atom[i], b);
        bulk_commit();
      }
      if (boxed != 0x01010101u) {
#pragma unroll 1
        for (int h = 0; h < D / 64; ++h)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3), chunk = lane & 7;
            const int rq = r_warp + rr;
            if (rq < p.N && !((boxed >> (rr & ~7)) & 1u)) {
              const uint4 w4 =
                  *reinterpret_cast<const uint4*>(stage + h * 4096 + rr * 128 + ((chunk ^ (rr & 7)) * 16));
              __nv_bfloat16* dst = p.dq + b * p.dq_sb + hm.token(rq) * p.dq_st +
                                   static_cast<long long>(hq) * D + 64 * h + 8 * chunk;
              *reinterpret_cast<uint4*>(dst) = w4;
            }
          }
      }
      __syncwarp();
    }
    // Every box has been written before the CTA's shared memory goes away.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      mma_commit(bar(L::B_DRAIN));
      drain_wait(bar(L::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace s2
