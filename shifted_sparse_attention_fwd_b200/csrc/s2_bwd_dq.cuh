// S²-Attn backward, dQ, on sm_100a tensor cores.
//
// Gradient of the per-group causal self-attention of LongLoRA's Algorithm 1 (summary page
// §3.4) with respect to the rolled query rows, stored back at the original rows:
//   P  = exp(scale * Q K^T - LSE)      (recomputed from the forward's LSE)
//   dP = dO V^T
//   dS = P o (dP - D)
//   dQ = scale * dS K
// One CTA owns a 128-row rolled query tile of one (batch, head) and walks the same key
// tiles as the forward (group start to diagonal); dQ is written once, without atomics.
//
// Warp roles (192 threads): warps 0-3 elementwise (thread i owns query row i), warp 4 TMA
// producer (Q, dO once; K through a 3-stage ring one tile ahead of V's 2-stage ring, each slot
// released by a commit right after its last reader: dP for V, dQ for K), warp 5 TMEM
// allocator + MMA issuer.
// TMEM: S/dS double buffer [0,128) and [128,256); dP [256,384); dQ [384, 384+D).
#pragma once

#include "s2_bwd_dkdv.cuh"

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
         B_ACC = 16, B_DRAIN = 17, B_COUNT = 18 };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kLaunchBytes =
      (kBytes + 1024 > 116 * 1024) ? kBytes + 1024 : 116 * 1024;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
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

  // Same tile order as the forward.
  int b, h, qt;
  query_tile_coords(blockIdx.x, p.B, p.Hq, p.N, p.G, b, h, qt);
  const int R0 = qt * kTileRows;
  const int shift_h = h >= p.shift_head_begin ? p.shift : 0;
  const int kvh = h / (p.Hq / p.Hkv);
  const int kt_begin = group_begin(R0, p.G) / kTileRows;
  const int n_kv = qt - kt_begin + 1;

  if (warp == 4 && lane == 0) {
    mbar_init(bar(L::B_QDO), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_V + s), 1);
      mbar_init(bar(L::B_VE + s), 1);
      mbar_init(bar(L::B_S + s), 1);
      mbar_init(bar(L::B_DS + s), 128);
    }
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::B_K + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    mbar_init(bar(L::B_DP), 1);
    mbar_init(bar(L::B_ACC), 1);
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_dp = tmem + 256, tm_dq = tmem + 384;

  if (warp == 4) {
    if (lane == 0) {
      const TileRuns q_runs = rolled_tile_runs(R0, shift_h, p.N);
      mbar_expect_tx(bar(L::B_QDO), 2 * L::kTile);
      load_tile<D>(sbase + L::kQ, &tmQ, &tmQ8, bar(L::B_QDO), b, h, q_runs, p.N);
      load_tile<D>(sbase + L::kDO, &tmO, &tmO8, bar(L::B_QDO), b, h, q_runs, p.N);
      int k_issued = 0, v_issued = 0;
      auto issue_k = [&]() -> bool {
        const int i = k_issued, st = i % L::kKStages;
        if (i >= L::kKStages &&
            !wait_bar(bar(L::B_KE + st), ((i / L::kKStages) - 1) & 1, ctx, 1))
          return false;
        mbar_expect_tx(bar(L::B_K + st), L::kTile);
        load_tile<D>(sbase + L::kK + st * L::kTile, &tmK, &tmK8, bar(L::B_K + st), b, kvh,
                     rolled_tile_runs((kt_begin + i) * kTileRows, shift_h, p.N), p.N);
        ++k_issued;
        return true;
      };
      auto issue_v = [&]() -> bool {
        const int i = v_issued, st = i % L::kVStages;
        if (i >= L::kVStages &&
            !wait_bar(bar(L::B_VE + st), ((i / L::kVStages) - 1) & 1, ctx, 10))
          return false;
        mbar_expect_tx(bar(L::B_V + st), L::kTile);
        load_tile<D>(sbase + L::kV + st * L::kTile, &tmV, &tmV8, bar(L::B_V + st), b, kvh,
                     rolled_tile_runs((kt_begin + i) * kTileRows, shift_h, p.N), p.N);
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
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);   // Q K^T, dO V^T
      constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);     // dS K
      auto issue_nt = [&](uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * Tile<D>::kHalfBytes + (kk % 4) * 32;
          mma_ss(d_tmem, sdesc_sw128(a_base + off, 16, 1024), sdesc_sw128(b_base + off, 16, 1024),
                 idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto wait_k = [&](int j) {
        return wait_bar(bar(L::B_K + j % L::kKStages), (j / L::kKStages) & 1, ctx, 3);
      };
      bool ok = wait_bar(bar(L::B_QDO), 0, ctx, 2);
      if (ok) ok = wait_k(0);
      if (ok) {
        tc_fence_after();
        issue_nt(tmem, sbase + L::kQ, sbase + L::kK);
        mma_commit(bar(L::B_S + 0));
      }
      for (int n = 0; ok && n < n_kv; ++n) {
        const int st = n & 1, kst = n % L::kKStages, vst = n % L::kVStages;
        if (!wait_bar(bar(L::B_V + vst), (n / L::kVStages) & 1, ctx, 4)) { ok = false; break; }
        tc_fence_after();
        issue_nt(tm_dp, sbase + L::kDO, sbase + L::kV + vst * L::kTile);
        mma_commit(bar(L::B_DP));
        mma_commit(bar(L::B_VE + vst));   // V(n) has no reader left
        if (n + 1 < n_kv) {
          if (!wait_k(n + 1)) { ok = false; break; }
          tc_fence_after();
          issue_nt(tmem + ((n + 1) & 1) * 128, sbase + L::kQ,
                   sbase + L::kK + ((n + 1) % L::kKStages) * L::kTile);
          mma_commit(bar(L::B_S + ((n + 1) & 1)));
        }
        if (!wait_bar(bar(L::B_DS + st), (n >> 1) & 1, ctx, 6)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = sbase + L::kK + kst * L::kTile;
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)
          mma_ts(tm_dq, tmem + st * 128 + kk * 8,
                 sdesc_sw128(k_base + kk * 2048, Tile<D>::kHalfBytes, 1024), idesc_dq,
                 (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(L::B_KE + kst));   // K(n): read by S(n) and dQ(n)
      }
      if (ok) mma_commit(bar(L::B_ACC));
    }
  } else {
    const int row = threadIdx.x;
    const int r = R0 + row;
    const bool row_valid = r < p.N;
    const int lo = row_valid ? group_begin(r, p.G) : kt_begin * kTileRows;
    const int hi = row_valid ? r : kt_begin * kTileRows;
    long long tt = static_cast<long long>(r) + shift_h;
    const int t = row_valid ? static_cast<int>(tt >= p.N ? tt - p.N : tt) : 0;
    const size_t lrow = (static_cast<size_t>(b) * p.Hq + h) * p.N + t;
    const float lse2 = row_valid ? p.lse2[lrow] : 0.f;
    const float dd = row_valid ? p.dvec[lrow] : 0.f;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < n_kv; ++n) {
      const int st = n & 1;
      if (!warp_wait(bar(L::B_S + st), (n >> 1) & 1, ctx, 7)) { ok = false; break; }
      tc_fence_after();
      const int c0 = (kt_begin + n) * kTileRows;
      const int cl = lo - c0, ch = hi - c0;
      float pv[128];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + st * 128 + 32 * j, rr);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = 32 * j + e;
          const float x = fast_exp2(fmaf(__uint_as_float(rr[e]), c, -lse2));
          pv[col] = (col >= cl && col <= ch) ? x : 0.f;
        }
      }
      if (!warp_wait(bar(L::B_DP), n & 1, ctx, 8)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + 256 + 32 * j, rr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int col = 32 * j + 2 * e;
          pk[e] = pack_bf16(pv[col] * (__uint_as_float(rr[2 * e]) - dd),
                            pv[col + 1] * (__uint_as_float(rr[2 * e + 1]) - dd));
        }
        tmem_st16(t_lane + st * 128 + 16 * j, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_DS + st));
    }
    if (ok && warp_wait(bar(L::B_ACC), 0, ctx, 9)) {
      tc_fence_after();
      __nv_bfloat16* qrow = p.dq + ((static_cast<size_t>(b) * p.N + t) * p.Hq + h) * D;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + 384 + 32 * j, rr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(rr[2 * e]) * p.scale, __uint_as_float(rr[2 * e + 1]) * p.scale);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(qrow + 32 * j);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    if (lane == 0) {
      mma_commit(bar(L::B_DRAIN));
      drain_wait(bar(L::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  (void)tm_dq;
}

}  // namespace s2
