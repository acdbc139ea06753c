// S²-Attn forward (O and row log-sum-exp) on sm_100a tensor cores.
//
// LongLoRA summary page, §3.4 Algorithm 1: per head, roll (second chunk of heads), view as
// groups of G, causal softmax(scale * q k^T) v inside each group, roll back. One CTA owns a
// 128-row tile of rolled query rows of one (batch, head); it walks the 128-row key/value
// tiles of the same rolled frame from the start of the group of its first row up to its
// own diagonal tile, so work is proportional to N*G rather than N^2. The roll never moves
// data: TMA reads the original rows (see s2_tiles.cuh) and the epilogue stores O and LSE at
// the original rows.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i); online softmax in fp32,
//              P written back to TMEM as bf16, O rescaled in TMEM, epilogue.
//   warp 4     TMA producer: Q once, then K/V tiles through a 2-stage ring.
//   warp 5     TMEM allocator and MMA issuer (one lane): S = Q K^T (SS), O += P V (TS).
// TMEM columns: S/P double buffer at [0,128) and [128,256); O at [256, 256+D).
#pragma once

#include "s2_common.cuh"

namespace s2 {

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, N, G, shift_head_begin, shift;
  float scale_log2;   // scale * log2(e)
  unsigned int* err;
  unsigned long long timeout_ns;
};

template <int D>
struct FwdLayout {
  static constexpr uint32_t kTile = Tile<D>::kBytes;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;        // 2 stages
  static constexpr uint32_t kV = kK + 2 * kTile;    // 2 stages
  static constexpr uint32_t kBar = kV + 2 * kTile;
  enum { B_Q = 0, B_K = 1, B_V = 3, B_EMPTY = 5, B_S = 7, B_P = 9, B_O = 11, B_DRAIN = 12,
         B_COUNT = 13 };
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  // Dynamic shared memory to request: alignment slack, and at least 116 KB so that only one
  // CTA is resident per SM (each CTA takes all 512 TMEM columns).
  static constexpr uint32_t kLaunchBytes =
      (kBytes + 1024 > 116 * 1024) ? kBytes + 1024 : 116 * 1024;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ8,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK8,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmV8,
                  const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return sbase + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_FWD};

  int b, h, qt;
  query_tile_coords(blockIdx.x, p.B, p.Hq, p.N, p.G, b, h, qt);
  const int R0 = qt * kTileRows;
  const int shift_h = h >= p.shift_head_begin ? p.shift : 0;
  const int kvh = h / (p.Hq / p.Hkv);
  const int kt_begin = group_begin(R0, p.G) / kTileRows;
  const int n_kv = qt - kt_begin + 1;

  if (warp == 4 && lane == 0) {
    mbar_init(bar(L::B_Q), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_K + s), 1);
      mbar_init(bar(L::B_V + s), 1);
      mbar_init(bar(L::B_EMPTY + s), 1);
      mbar_init(bar(L::B_S + s), 1);
      mbar_init(bar(L::B_P + s), 128);
    }
    mbar_init(bar(L::B_O), 1);
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int last_parity[2] = {-1, -1};
      mbar_expect_tx(bar(L::B_Q), L::kTile);
      load_tile<D>(sbase + L::kQ, &tmQ, &tmQ8, bar(L::B_Q), b, h,
                   rolled_tile_runs(R0, shift_h, p.N), p.N);
      for (int it = 0; it < n_kv; ++it) {
        const int st = it & 1;
        if (it >= 2 && !wait_bar(bar(L::B_EMPTY + st), ((it >> 1) - 1) & 1, ctx, 1)) break;
        const TileRuns tr = rolled_tile_runs((kt_begin + it) * kTileRows, shift_h, p.N);
        mbar_expect_tx(bar(L::B_K + st), L::kTile);
        load_tile<D>(sbase + L::kK + st * L::kTile, &tmK, &tmK8, bar(L::B_K + st), b, kvh, tr, p.N);
        mbar_expect_tx(bar(L::B_V + st), L::kTile);
        load_tile<D>(sbase + L::kV + st * L::kTile, &tmV, &tmV8, bar(L::B_V + st), b, kvh, tr, p.N);
        last_parity[st] = (it >> 1) & 1;
      }
      // Every issued copy lands before the CTA can exit.
      drain_wait(bar(L::B_Q), 0, p.timeout_ns);
      for (int s = 0; s < 2; ++s) {
        if (last_parity[s] >= 0) {
          drain_wait(bar(L::B_K + s), last_parity[s], p.timeout_ns);
          drain_wait(bar(L::B_V + s), last_parity[s], p.timeout_ns);
        }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      const uint32_t tm_o = tmem + 256;
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!wait_bar(bar(L::B_P + st), ph, ctx, 2)) return false;
        if (!wait_bar(bar(L::B_V + st), ph, ctx, 3)) return false;
        tc_fence_after();
        const uint32_t v_base = sbase + L::kV + st * L::kTile;
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(v_base + kk * 2048, Tile<D>::kHalfBytes, 1024);
          mma_ts(tm_o, tmem + st * 128 + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(L::B_EMPTY + st));
        mma_commit(bar(L::B_O));
        return true;
      };
      bool ok = wait_bar(bar(L::B_Q), 0, ctx, 4);
      for (int it = 0; ok && it < n_kv; ++it) {
        const int st = it & 1;
        if (!wait_bar(bar(L::B_K + st), (it >> 1) & 1, ctx, 5)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_base = sbase + L::kQ;
        const uint32_t k_base = sbase + L::kK + st * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * Tile<D>::kHalfBytes + (kk % 4) * 32;
          mma_ss(tmem + st * 128, sdesc_sw128(q_base + off, 16, 1024),
                 sdesc_sw128(k_base + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::B_S + st));
        if (it > 0) ok = issue_pv(it - 1);
      }
      if (ok) issue_pv(n_kv - 1);
    }
  } else {
    // ---------------- softmax warps 0-3 ----------------
    const int row = threadIdx.x;
    const int r = R0 + row;
    const bool row_valid = r < p.N;
    const int lo = row_valid ? group_begin(r, p.G) : kt_begin * kTileRows;
    const int hi = row_valid ? r : kt_begin * kTileRows;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      const int st = it & 1;
      if (!warp_wait(bar(L::B_S + st), (it >> 1) & 1, ctx, 6)) { ok = false; break; }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + st * 128 + 32 * j, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * j + i] = __uint_as_float(rr[i]);
      }
      const int c0 = (kt_begin + it) * kTileRows;
      const int cl = lo - c0, ch = hi - c0;
      if (cl > 0 || ch < kTileRows - 1) {
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = (i < cl || i > ch) ? -INFINITY : s[i];
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m_run, mx * c);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        s[i] = fast_exp2(fmaf(s[i], c, -m_use));
        sum += s[i];
      }
      const float alpha = fast_exp2(m_run - m_use);
      if (it > 0) {
        if (!warp_wait(bar(L::B_O), (it - 1) & 1, ctx, 7)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            uint32_t rr[32];
            tmem_ld32(t_lane + 256 + 32 * j, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(t_lane + 256 + 32 * j, rr);
          }
        }
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(s[32 * j + 2 * i], s[32 * j + 2 * i + 1]);
        tmem_st16(t_lane + st * 128 + 16 * j, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_P + st));
    }
    if (ok && warp_wait(bar(L::B_O), (n_kv - 1) & 1, ctx, 8)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      long long tt = static_cast<long long>(r) + shift_h;
      const int t = static_cast<int>(tt >= p.N ? tt - p.N : tt);
      __nv_bfloat16* orow =
          p.o + ((static_cast<size_t>(b) * p.N + (row_valid ? t : 0)) * p.Hq + h) * D;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t rr[32];
        tmem_ld32(t_lane + 256 + 32 * j, rr);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16(__uint_as_float(rr[2 * i]) * inv_l, __uint_as_float(rr[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * j);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row_valid)
        p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.N + t] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
    }
  }

  // ---------------- teardown ----------------
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
}

}  // namespace s2
