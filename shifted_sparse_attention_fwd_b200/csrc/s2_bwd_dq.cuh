// S²-Attn backward, dQ, on sm_100a tensor cores.
//
// Gradient of the per-group causal self-attention of LongLoRA's Algorithm 1 (summary page
// §3.4) with respect to the rolled query rows, stored back at the original rows:
//   P  = exp(scale * Q K^T - LSE)      (recomputed from the forward's LSE)
//   dP = dO V^T
//   dS = P o (dP - D)
//   dQ = scale * dS K
// One CTA owns a 128-row rolled query tile of one (batch, head) and walks the key tiles the
// forward walks (group start to diagonal); dQ is written once, without atomics.
//
// Warp roles (320 threads): warps 0-7 elementwise — query row i (TMEM lane i) is shared by
// warp i/32 (key columns 0-63) and warp i/32 + 4 (columns 64-127), so two warps per SM
// sub-partition work on every tile; warp 8 TMA producer (Q, dO once; K through a 3-slot ring
// one tile ahead of V's 2-slot ring, each slot released right after its last reader); warp 9
// TMEM allocator + MMA issuer.
//
// TMEM: S double buffer [0,128) and [128,256); dP [256,384); dQ [384,384+D). dS (bf16) is
// written into the S buffer it came from, at columns [32,96): each column half packs its
// output inside its own, already consumed, fp32 columns. P stays in registers (bf16) between
// the S and dS phases. Per key tile the MMA issuer runs dP(n), S(n+1), dQ(n): the P phase
// overlaps dP(n) and the dS phase overlaps S(n+1).
#pragma once

#include "s2_bwd_dkdv.cuh"
#include "s2_tmem_wide.cuh"

namespace s2 {

template <int D>
struct DqLayout {
  static constexpr uint32_t kTile = Tile<D>::kBytes;
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kQ + kTile;
  static constexpr uint32_t kK = kDO + kTile;                 // K ring
  static constexpr uint32_t kV = kK + kKStages * kTile;       // V ring
  static constexpr uint32_t kBar = kV + kVStages * kTile;
  enum { B_QDO = 0, B_K = 1, B_KE = 4, B_V = 7, B_VE = 9, B_S = 11, B_DP = 13, B_DS = 14,
         B_ACC = 15, B_DRAIN = 16, B_COUNT = 17 };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kLaunchBytes =
      (kBytes + 1024 > 116 * 1024) ? kBytes + 1024 : 116 * 1024;
  static constexpr int kThreads = 320;
};

// kFront: built for the Variant 3 reordering (otherwise p.front is ignored).
template <int D, bool kFront>
__global__ void __launch_bounds__(320, 1)
    s2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ8,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK8,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmV8,
                     const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO8,
                     const BwdParams p) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return sbase + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_DQ};

  int b, h, qt;
  query_tile_coords(blockIdx.x, p.B, p.Hq, p.N, p.G, b, h, qt);
  const int R0 = qt * kTileRows;
  const bool shifted = h >= p.shift_head_begin;
  const HeadRemap hm = head_remap(p.N, p.G, shifted ? p.shift : 0, (kFront && shifted) ? p.front : 0);
  const int wrap_h = shifted ? p.wrap : kNoWrapSplit;
  const int kvh = h / (p.Hq / p.Hkv);
  const int kt_begin = group_begin(R0, p.G, wrap_h) / kTileRows;
  const int n_kv = qt - kt_begin + 1;

  if (warp == 8 && lane == 0) {
    mbar_init(bar(L::B_QDO), 2);   // the Q tile and the dO tile
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::B_K + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_V + s), 1);
      mbar_init(bar(L::B_VE + s), 1);
      mbar_init(bar(L::B_S + s), 1);
    }
    mbar_init(bar(L::B_DP), 1);
    mbar_init(bar(L::B_DS), 256);
    mbar_init(bar(L::B_ACC), 1);
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO);
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_dp = tmem + 256, tm_dq = tmem + 384;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    // Tile rows TMA cannot move are copied by this thread first (produce_tile).
    if (lane == 0) {
      const Runs q_runs = rolled_runs(hm, R0);
      produce_tile<D>(sbase + L::kQ, &tmQ, &tmQ8, bar(L::B_QDO), p.q, b, h, q_runs, p.N);
      produce_tile<D>(sbase + L::kDO, &tmO, &tmO8, bar(L::B_QDO), p.dO, b, h, q_runs, p.N);
      int k_issued = 0, v_issued = 0;
      auto issue_k = [&]() -> bool {
        const int i = k_issued, st = i % L::kKStages;
        if (i >= L::kKStages &&
            !wait_bar(bar(L::B_KE + st), ((i / L::kKStages) - 1) & 1, ctx, 1))
          return false;
        produce_tile<D>(sbase + L::kK + st * L::kTile, &tmK, &tmK8, bar(L::B_K + st), p.k, b, kvh,
                        rolled_runs(hm, (kt_begin + i) * kTileRows), p.N);
        ++k_issued;
        return true;
      };
      auto issue_v = [&]() -> bool {
        const int i = v_issued, st = i % L::kVStages;
        if (i >= L::kVStages &&
            !wait_bar(bar(L::B_VE + st), ((i / L::kVStages) - 1) & 1, ctx, 10))
          return false;
        produce_tile<D>(sbase + L::kV + st * L::kTile, &tmV, &tmV8, bar(L::B_V + st), p.v, b, kvh,
                        rolled_runs(hm, (kt_begin + i) * kTileRows), p.N);
        ++v_issued;
        return true;
      };
      bool ok = issue_k();
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) ok = issue_k();
        if (ok) ok = issue_v();
      }
      drain_wait(bar(L::B_QDO), 0, p.timeout_ns);
      for (int i = k_issued - L::kKStages; i < k_issued; ++i)
        if (i >= 0) drain_wait(bar(L::B_K + i % L::kKStages), (i / L::kKStages) & 1, p.timeout_ns);
      for (int i = v_issued - L::kVStages; i < v_issued; ++i)
        if (i >= 0) drain_wait(bar(L::B_V + i % L::kVStages), (i / L::kVStages) & 1, p.timeout_ns);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);   // Q K^T, dO V^T
      constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);     // dS K
      auto wait_k = [&](int j) {
        return wait_bar(bar(L::B_K + j % L::kKStages), (j / L::kKStages) & 1, ctx, 3);
      };
      bool ok = wait_bar(bar(L::B_QDO), 0, ctx, 2);
      if (ok) ok = wait_k(0);
      if (ok) {
        tc_fence_after();
        gemm_ss_k<D>(tmem, sbase + L::kQ, sbase + L::kK, idesc_s);
        mma_commit(bar(L::B_S + 0));
      }
      for (int n = 0; ok && n < n_kv; ++n) {
        const int st = n & 1, kst = n % L::kKStages, vst = n % L::kVStages;
        if (!wait_bar(bar(L::B_V + vst), (n / L::kVStages) & 1, ctx, 4)) { ok = false; break; }
        tc_fence_after();
        gemm_ss_k<D>(tm_dp, sbase + L::kDO, sbase + L::kV + vst * L::kTile, idesc_s);
        mma_commit(bar(L::B_DP));
        mma_commit(bar(L::B_VE + vst));   // V(n) has no reader left
        if (n + 1 < n_kv) {
          if (!wait_k(n + 1)) { ok = false; break; }
          tc_fence_after();
          gemm_ss_k<D>(tmem + ((n + 1) & 1) * 128, sbase + L::kQ,
                       sbase + L::kK + ((n + 1) % L::kKStages) * L::kTile, idesc_s);
          mma_commit(bar(L::B_S + ((n + 1) & 1)));
        }
        if (!wait_bar(bar(L::B_DS), n & 1, ctx, 6)) { ok = false; break; }
        tc_fence_after();
        gemm_ts_mn<D>(tm_dq, tmem + st * 128 + 32, sbase + L::kK + kst * L::kTile, idesc_dq, n > 0);
        mma_commit(bar(L::B_KE + kst));   // K(n): read by S(n) and dQ(n)
      }
      if (ok) mma_commit(bar(L::B_ACC));
    }
  } else {
    // ---------------- elementwise warps 0-7 ----------------
    const int half = warp / 4;                     // key columns [64 half, 64 half + 64)
    const int row = (warp % 4) * 32 + lane;
    const int r = R0 + row;
    const bool row_valid = r < p.N;
    const int lo = row_valid ? group_begin(r, p.G, wrap_h) : kt_begin * kTileRows;
    const int hi = row_valid ? r : kt_begin * kTileRows;
    const int t = row_valid ? hm.token(r) : 0;
    const size_t lrow = (static_cast<size_t>(b) * p.Hq + h) * p.N + t;
    const float lse2 = row_valid ? p.lse2[lrow] : 0.f;
    const float dd = row_valid ? p.dvec[lrow] : 0.f;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const float c = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < n_kv; ++n) {
      const int st = n & 1;
      // P phase: 64 columns of S -> P (bf16, registers).
      if (!warp_wait(bar(L::B_S + st), (n >> 1) & 1, ctx, 7)) { ok = false; break; }
      tc_fence_after();
      const int c0 = (kt_begin + n) * kTileRows + 64 * half;
      const int cl = lo - c0, ch = hi - c0;
      uint32_t pk[32];
      {
        uint32_t raw[64];
        tmem_ld64(t_lane + st * 128 + 64 * half, raw);
        const bool mask = __any_sync(0xffffffffu, cl > 0 || ch < 63);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = 2 * e;
          float x0 = fast_exp2(fmaf(__uint_as_float(raw[col]), c, -lse2));
          float x1 = fast_exp2(fmaf(__uint_as_float(raw[col + 1]), c, -lse2));
          if (mask) {
            x0 = (col < cl || col > ch) ? 0.f : x0;
            x1 = (col + 1 < cl || col + 1 > ch) ? 0.f : x1;
          }
          pk[e] = pack_bf16(x0, x1);
        }
      }
      // dS phase: dS = P o (dP - D), packed into this half's own consumed S columns.
      if (!warp_wait(bar(L::B_DP), n & 1, ctx, 8)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t raw[64];
        tmem_ld64(tm_dp - tmem + t_lane + 64 * half, raw);
        uint32_t ds[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[e]));
          ds[e] = pack_bf16(pf.x * (__uint_as_float(raw[2 * e]) - dd),
                            pf.y * (__uint_as_float(raw[2 * e + 1]) - dd));
        }
        tmem_st32(t_lane + st * 128 + 32 + 32 * half, ds);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_DS));
    }
    if (ok && warp_wait(bar(L::B_ACC), 0, ctx, 9)) {
      tc_fence_after();
      __nv_bfloat16* qrow = p.dq + b * p.dq_sb + t * p.dq_st + static_cast<long long>(h) * D;
#pragma unroll
      for (int j = half * (D / 64); j < (half + 1) * (D / 64); ++j) {
        uint32_t rr[32];
        tmem_ld32(tm_dq - tmem + t_lane + 32 * j, rr);
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w4;
            w4.x = pack_bf16(__uint_as_float(rr[8 * v + 0]) * p.scale, __uint_as_float(rr[8 * v + 1]) * p.scale);
            w4.y = pack_bf16(__uint_as_float(rr[8 * v + 2]) * p.scale, __uint_as_float(rr[8 * v + 3]) * p.scale);
            w4.z = pack_bf16(__uint_as_float(rr[8 * v + 4]) * p.scale, __uint_as_float(rr[8 * v + 5]) * p.scale);
            w4.w = pack_bf16(__uint_as_float(rr[8 * v + 6]) * p.scale, __uint_as_float(rr[8 * v + 7]) * p.scale);
            reinterpret_cast<uint4*>(qrow + 32 * j)[v] = w4;
          }
        }
      }
    }
  }

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
