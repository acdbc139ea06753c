// S²-Attn backward, dQ, on sm_100a tensor cores.
//
// Gradient of the per-group causal self-attention of LongLoRA's Algorithm 1 (summary page
// §3.4) with respect to the rolled query rows, stored back at the original rows:
//   P  = exp(scale * Q K^T - LSE)      (recomputed from the forward's LSE)
//   dP = dO V^T
//   dS = P o (dP - D)
//   dQ = scale * dS K
// One CTA owns two consecutive 128-row rolled query tiles of one (batch, head) and walks the
// key tiles the forward walks (group start to diagonal); dQ is written once, without atomics.
//
// Warp roles (320 threads): warps 0-3 and 4-7 elementwise for query tile 0 and 1 (thread i
// owns query row i), warp 8 TMA producer (Q and dO of both tiles once; K through a 2-slot
// ring, V through a 1-slot ring, each slot released right after its last reader), warp 9
// TMEM allocator + MMA issuer.
//
// TMEM: tile t uses columns R_t = [128 t, 128 t + 128) in turn for S, then dP, then dS (bf16),
// and dQ_t = [256 + 128 t, 384 + 128 t). P is kept in registers (bf16) between the S and dP
// phases, which is what frees R_t for dP. The MMA issuer interleaves the tiles
// (dP0 dP1 dQ0 S0' dQ1 S1' ...) so one tile's elementwise phase overlaps the other's MMAs.
#pragma once

#include "s2_bwd_dkdv.cuh"
#include "s2_tmem_wide.cuh"

namespace s2 {

template <int D>
struct DqLayout {
  static constexpr uint32_t kTile = Tile<D>::kBytes;
  static constexpr int kKStages = 2, kVStages = 1;
  static constexpr uint32_t kQ = 0;                          // Q0, Q1
  static constexpr uint32_t kDO = kQ + 2 * kTile;            // dO0, dO1
  static constexpr uint32_t kK = kDO + 2 * kTile;            // K ring
  static constexpr uint32_t kV = kK + kKStages * kTile;      // V ring
  static constexpr uint32_t kBar = kV + kVStages * kTile;
  enum { B_QD = 0, B_K = 2, B_KE = 4, B_V = 6, B_VE = 7, B_S = 8, B_PF = 10, B_DP = 12,
         B_DS = 14, B_ACC = 16, B_DRAIN = 18, B_COUNT = 19 };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kLaunchBytes =
      (kBytes + 1024 > 116 * 1024) ? kBytes + 1024 : 116 * 1024;
  static constexpr int kThreads = 320;
};

template <int D>
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

  // Same work decomposition as the forward: tiles 2*pair and 2*pair + 1 of (b, h).
  int b, h, pair;
  query_pair_coords(blockIdx.x, p.B, p.Hq, p.N, p.G, b, h, pair);
  const int nqt = (p.N + kTileRows - 1) / kTileRows;
  const int shift_h = h >= p.shift_head_begin ? p.shift : 0;
  const int kvh = h / (p.Hq / p.Hkv);
  int qt[2], kb[2], ke[2];
  bool tv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    qt[t] = 2 * pair + t;
    tv[t] = qt[t] < nqt;
    kb[t] = tv[t] ? group_begin(qt[t] * kTileRows, p.G) / kTileRows : 0;
    ke[t] = qt[t];
  }
  const int kv_lo = kb[0];
  const int n_kv = (tv[1] ? ke[1] : ke[0]) - kv_lo + 1;
  auto part = [&](int t, int kt) { return tv[t] && kb[t] <= kt && kt <= ke[t]; };

  if (warp == 8 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_QD + s), 1);
      mbar_init(bar(L::B_K + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
      mbar_init(bar(L::B_S + s), 1);
      mbar_init(bar(L::B_PF + s), 128);
      mbar_init(bar(L::B_DP + s), 1);
      mbar_init(bar(L::B_DS + s), 128);
      mbar_init(bar(L::B_ACC + s), 1);
    }
    mbar_init(bar(L::B_V), 1);
    mbar_init(bar(L::B_VE), 1);
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

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      for (int t = 0; t < 2; ++t) {
        if (!tv[t]) continue;
        const TileRuns q_runs = rolled_tile_runs(qt[t] * kTileRows, shift_h, p.N);
        mbar_expect_tx(bar(L::B_QD + t), 2 * L::kTile);
        load_tile<D>(sbase + L::kQ + t * L::kTile, &tmQ, &tmQ8, bar(L::B_QD + t), b, h, q_runs, p.N);
        load_tile<D>(sbase + L::kDO + t * L::kTile, &tmO, &tmO8, bar(L::B_QD + t), b, h, q_runs, p.N);
      }
      int k_issued = 0, v_issued = 0;
      auto issue_k = [&]() -> bool {
        const int i = k_issued, st = i % L::kKStages;
        if (i >= L::kKStages &&
            !wait_bar(bar(L::B_KE + st), ((i / L::kKStages) - 1) & 1, ctx, 1))
          return false;
        mbar_expect_tx(bar(L::B_K + st), L::kTile);
        load_tile<D>(sbase + L::kK + st * L::kTile, &tmK, &tmK8, bar(L::B_K + st), b, kvh,
                     rolled_tile_runs((kv_lo + i) * kTileRows, shift_h, p.N), p.N);
        ++k_issued;
        return true;
      };
      auto issue_v = [&]() -> bool {
        const int i = v_issued;
        if (i >= L::kVStages && !wait_bar(bar(L::B_VE), (i - 1) & 1, ctx, 11)) return false;
        mbar_expect_tx(bar(L::B_V), L::kTile);
        load_tile<D>(sbase + L::kV, &tmV, &tmV8, bar(L::B_V), b, kvh,
                     rolled_tile_runs((kv_lo + i) * kTileRows, shift_h, p.N), p.N);
        ++v_issued;
        return true;
      };
      bool ok = issue_k();
      for (int j = 0; ok && j < n_kv; ++j) {
        if (ok) ok = issue_v();
        if (ok && j + 1 < n_kv) ok = issue_k();
      }
      for (int t = 0; t < 2; ++t)
        if (tv[t]) drain_wait(bar(L::B_QD + t), 0, p.timeout_ns);
      for (int i = k_issued - L::kKStages; i < k_issued; ++i)
        if (i >= 0) drain_wait(bar(L::B_K + i % L::kKStages), (i / L::kKStages) & 1, p.timeout_ns);
      if (v_issued > 0) drain_wait(bar(L::B_V), (v_issued - 1) & 1, p.timeout_ns);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);   // Q K^T, dO V^T
      constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);     // dS K
      bool qd_ready[2] = {false, false}, first_dq[2] = {true, true};
      int pf_cnt[2] = {0, 0}, ds_cnt[2] = {0, 0};
      bool ok = true;
      auto issue_nt = [&](uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * Tile<D>::kHalfBytes + (kk % 4) * 32;
          mma_ss(d_tmem, sdesc_sw128(a_base + off, 16, 1024), sdesc_sw128(b_base + off, 16, 1024),
                 idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto ensure_qd = [&](int t) -> bool {
        if (qd_ready[t]) return true;
        if (!wait_bar(bar(L::B_QD + t), 0, ctx, 2)) return false;
        qd_ready[t] = true;
        return true;
      };
      auto wait_k = [&](int i) {
        return wait_bar(bar(L::B_K + i % L::kKStages), (i / L::kKStages) & 1, ctx, 3);
      };
      auto issue_s = [&](int t, int kidx) -> bool {
        if (!ensure_qd(t)) return false;
        tc_fence_after();
        issue_nt(tmem + t * 128, sbase + L::kQ + t * L::kTile,
                 sbase + L::kK + (kidx % L::kKStages) * L::kTile);
        mma_commit(bar(L::B_S + t));
        return true;
      };
      if (!wait_k(0)) ok = false;
      for (int t = 0; ok && t < 2; ++t)
        if (part(t, kv_lo)) ok = issue_s(t, 0);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int kt = kv_lo + j, kst = j % L::kKStages;
        const bool next = j + 1 < n_kv;
        // dP_t(j) = dO_t V(j)^T into R_t once the elementwise warps hold P_t(j) in registers.
        bool v_ready = false;
        for (int t = 0; ok && t < 2; ++t) {
          if (!part(t, kt)) continue;
          if (!wait_bar(bar(L::B_PF + t), pf_cnt[t] & 1, ctx, 4)) { ok = false; break; }
          ++pf_cnt[t];
          if (!v_ready) {
            if (!wait_bar(bar(L::B_V), j & 1, ctx, 5)) { ok = false; break; }
            v_ready = true;
          }
          tc_fence_after();
          issue_nt(tmem + t * 128, sbase + L::kDO + t * L::kTile, sbase + L::kV);
          mma_commit(bar(L::B_DP + t));
        }
        if (!ok) break;
        mma_commit(bar(L::B_VE));   // V(j) has no reader left
        // dQ_t += dS_t(j) K(j), then S_t(j+1) into R_t.
        bool k_next_ready = false;
        for (int t = 0; ok && t < 2; ++t) {
          if (part(t, kt)) {
            if (!wait_bar(bar(L::B_DS + t), ds_cnt[t] & 1, ctx, 6)) { ok = false; break; }
            ++ds_cnt[t];
            tc_fence_after();
            const uint32_t k_base = sbase + L::kK + kst * L::kTile;
#pragma unroll
            for (int kk = 0; kk < kTileRows / 16; ++kk)
              mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                     sdesc_sw128(k_base + kk * 2048, Tile<D>::kHalfBytes, 1024), idesc_dq,
                     (!first_dq[t] || kk > 0) ? 1u : 0u);
            first_dq[t] = false;
            if (kt == ke[t]) mma_commit(bar(L::B_ACC + t));
          }
          if (next && part(t, kt + 1)) {
            if (!k_next_ready) {
              if (!wait_k(j + 1)) { ok = false; break; }
              k_next_ready = true;
            }
            if (!issue_s(t, j + 1)) { ok = false; break; }
          }
        }
        if (ok) mma_commit(bar(L::B_KE + kst));   // K(j): read by S(j) and dQ(j)
      }
    }
  } else {
    // ---------------- elementwise warpgroups ----------------
    const int wg = warp / 4;
    if (tv[wg]) {
      const int row = threadIdx.x % 128;
      const int r = qt[wg] * kTileRows + row;
      const bool row_valid = r < p.N;
      const int lo = row_valid ? group_begin(r, p.G) : kb[wg] * kTileRows;
      const int hi = row_valid ? r : kb[wg] * kTileRows;
      const long long tt = static_cast<long long>(r) + shift_h;
      const int t = row_valid ? static_cast<int>(tt >= p.N ? tt - p.N : tt) : 0;
      const size_t lrow = (static_cast<size_t>(b) * p.Hq + h) * p.N + t;
      const float lse2 = row_valid ? p.lse2[lrow] : 0.f;
      const float dd = row_valid ? p.dvec[lrow] : 0.f;
      const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
      const uint32_t r_col = t_lane + wg * 128;
      const uint32_t dq_col = t_lane + 256 + wg * 128;
      const float c = p.scale_log2;
      bool ok = true;
      int cnt = 0;
      for (int kt = kb[wg]; kt <= ke[wg]; ++kt, ++cnt) {
        // P phase: S_t(j) -> P (bf16, registers); R_t is then free for dP.
        if (!warp_wait(bar(L::B_S + wg), cnt & 1, ctx, 7)) { ok = false; break; }
        tc_fence_after();
        uint32_t pk[64];
        {
          const int cl = lo - kt * kTileRows, ch = hi - kt * kTileRows;
          const bool mask = __any_sync(0xffffffffu, cl > 0 || ch < kTileRows - 1);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t raw[64];
            tmem_ld64(r_col + 64 * half, raw);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = 64 * half + 2 * i;
              float e0 = fast_exp2(fmaf(__uint_as_float(raw[2 * i]), c, -lse2));
              float e1 = fast_exp2(fmaf(__uint_as_float(raw[2 * i + 1]), c, -lse2));
              if (mask) {
                e0 = (col < cl || col > ch) ? 0.f : e0;
                e1 = (col + 1 < cl || col + 1 > ch) ? 0.f : e1;
              }
              pk[32 * half + i] = pack_bf16(e0, e1);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(L::B_PF + wg));
        // dS phase: dS = P o (dP - D) into R_t (bf16).
        if (!warp_wait(bar(L::B_DP + wg), cnt & 1, ctx, 8)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t dp[16];
          tmem_ld16(r_col + 16 * j, dp);
          uint32_t ds[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[8 * j + e]));
            ds[e] = pack_bf16(pf.x * (__uint_as_float(dp[2 * e]) - dd),
                              pf.y * (__uint_as_float(dp[2 * e + 1]) - dd));
          }
          tmem_st8(r_col + 8 * j, ds);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::B_DS + wg));
      }
      if (ok && warp_wait(bar(L::B_ACC + wg), 0, ctx, 9)) {
        tc_fence_after();
        __nv_bfloat16* qrow = p.dq + ((static_cast<size_t>(b) * p.N + t) * p.Hq + h) * D;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          uint32_t rr[32];
          tmem_ld32(dq_col + 32 * j, rr);
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
