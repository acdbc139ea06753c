// Pieces shared by the tensor-core kernels: tile loads through the remap, shared-memory
// carving, and the end-of-kernel drain that makes an aborted CTA exit cleanly.
#pragma once

#include "s2_device.cuh"
#include "s2_tiles.cuh"

namespace s2 {

// Bytes of one 128-row tile of head dimension D (bf16): D/64 column halves of 16 KB, each
// a TMA box of 64 columns written with the 128-byte swizzle.
template <int D>
struct Tile {
  static constexpr uint32_t kHalfBytes = kTileRows * 128;
  static constexpr uint32_t kBytes = kTileRows * D * 2;
  static constexpr int kHalves = D / 64;
};

// A [B, N, H, D] bf16 tensor by address and element strides (batch, token), for the rows that
// are loaded with plain loads instead of TMA.
struct TensorRef {
  const __nv_bfloat16* p;
  long long sb, st;
};

// Bytes the TMA unit delivers for a tile whose atoms in `skip` are filled by plain loads.
template <int D>
__device__ __forceinline__ uint32_t tma_tile_bytes(uint32_t skip) {
  return Tile<D>::kBytes - static_cast<uint32_t>(__popc(skip)) * (8u * 128u) * Tile<D>::kHalves;
}

// 16-byte (or 4-byte) asynchronous copy global -> shared by one thread; with src_bytes = 0 the
// destination is filled with zeros. Completed by cp_async_wait_all.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src))
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// One thread: the rows of the atoms in `skip` (see straddled_atoms), copied with 16-byte
// asynchronous copies from the tensor into the 128-byte-swizzled tile layout the TMA boxes
// produce (16-byte chunk c of a row's 64-column half at chunk c XOR (row mod 8)); rows past the
// end of the sequence become zeros. Returns when the copies have landed and are visible to the
// tensor core (proxy fence), so the caller may signal the tile's barrier.
template <int D>
__device__ __forceinline__ void fill_atoms(uint32_t dst, uint32_t skip, const Runs& tr,
                                           const TensorRef& t, int b, int h) {
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
  for (uint32_t m = skip; m != 0; m &= m - 1) {
    const int a = __ffs(m) - 1;
    for (int row = 8 * a; row < 8 * a + 8; ++row) {
      int src = -1, base = 0;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        if (k < tr.n && row >= base && row < base + tr.len[k]) src = tr.src[k] + (row - base);
        base += k < tr.n ? tr.len[k] : 0;
      }
      const __nv_bfloat16* g = t.p + b * t.sb + (src < 0 ? 0 : src) * t.st + static_cast<long long>(h) * D;
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        cp_async16(dst + (c / 8) * Tile<D>::kHalfBytes + row * 128 + (((c % 8) ^ (row & 7)) * 16),
                   g + 8 * c, src < 0 ? 0u : 16u);
    }
  }
  cp_async_wait_all();
  fence_async_smem();
}

// Issue the TMA loads of one 128-row tile of a [B, N, H, D] tensor whose rows are given by
// `tr`, except the atoms in `skip`. A single run of 128 rows uses the 128-row box; anything
// else is moved in 8-row boxes (one swizzle atom each), with rows past the sequence read out
// of bounds so TMA writes zeros. Delivers tma_tile_bytes<D>(skip) on `bar`.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* m128,
                                          const CUtensorMap* m8, uint32_t bar, int b, int h,
                                          const Runs& tr, int N, uint32_t skip = 0) {
  if (tr.n == 1 && tr.len[0] == kTileRows) {
#pragma unroll
    for (int half = 0; half < Tile<D>::kHalves; ++half)
      tma_load_4d(dst + half * Tile<D>::kHalfBytes, m128, bar, half * 64, h, tr.src[0], b);
  } else {
    for (int row = 0; row < kTileRows; row += 8) {
      if ((skip >> (row >> 3)) & 1u) continue;
      int src = N, base = 0;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        if (k < tr.n && row >= base && row < base + tr.len[k]) src = tr.src[k] + (row - base);
        base += k < tr.n ? tr.len[k] : 0;
      }
#pragma unroll
      for (int half = 0; half < Tile<D>::kHalves; ++half)
        tma_load_4d(dst + half * Tile<D>::kHalfBytes + row * 128, m8, bar, half * 64, h, src, b);
    }
  }
}

// A tile with atoms TMA cannot move: those are copied by this thread first, then `bar` is
// armed with the bytes TMA still delivers (one arrival) and the other boxes are issued. Kept out
// of line so the common path stays as small as it is.
template <int D>
__device__ __noinline__ void load_tile_slow(uint32_t dst, const CUtensorMap* m128,
                                            const CUtensorMap* m8, uint32_t bar, const TensorRef t,
                                            int b, int h, const Runs tr, int N, uint32_t skip) {
  fill_atoms<D>(dst, skip, tr, t, b, h);
  mbar_expect_tx(bar, tma_tile_bytes<D>(skip));
  load_tile<D>(dst, m128, m8, bar, b, h, tr, N, skip);
}

// Producer thread: one tile through the remap, one arrival on `bar` with its bytes.
template <int D>
__device__ __forceinline__ void produce_tile(uint32_t dst, const CUtensorMap* m128,
                                             const CUtensorMap* m8, uint32_t bar,
                                             const TensorRef& t, int b, int h, const Runs& tr,
                                             int N) {
  const uint32_t skip = straddled_atoms(tr);
  if (skip) {
    load_tile_slow<D>(dst, m128, m8, bar, t, b, h, tr, N, skip);
    return;
  }
  mbar_expect_tx(bar, Tile<D>::kBytes);
  load_tile<D>(dst, m128, m8, bar, b, h, tr, N);
}

// The reverse of load_tile for one thread: TMA stores of a 128-row tile in shared memory (the
// layout load_tile produces) to the rows `tr` gives, except the atoms in `skip`, which must
// include every atom that straddles two runs or reaches past the end of the sequence
// (straddled_atoms | past_end_atoms); committed as one bulk group.
template <int D>
__device__ __forceinline__ void store_tile(uint32_t src, const CUtensorMap* m128,
                                           const CUtensorMap* m8, int b, int h, const Runs& tr,
                                           uint32_t skip) {
  if (tr.n == 1 && tr.len[0] == kTileRows && skip == 0) {
#pragma unroll
    for (int half = 0; half < Tile<D>::kHalves; ++half)
      tma_store_4d(m128, src + half * Tile<D>::kHalfBytes, half * 64, h, tr.src[0], b);
  } else {
    for (int row = 0; row < kTileRows; row += 8) {
      if ((skip >> (row >> 3)) & 1u) continue;
      int dst = -1, base = 0;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        if (k < tr.n && row >= base && row < base + tr.len[k]) dst = tr.src[k] + (row - base);
        base += k < tr.n ? tr.len[k] : 0;
      }
      if (dst < 0) continue;
#pragma unroll
      for (int half = 0; half < Tile<D>::kHalves; ++half)
        tma_store_4d(m8, src + half * Tile<D>::kHalfBytes + row * 128, half * 64, h, dst, b);
    }
  }
  bulk_commit();
}

// The rows of the atoms in `skip` that are in the sequence, stored by a whole warp from a
// 128-row tile in shared memory (load_tile's layout) to a contiguous [B, N, H, D] tensor.
template <int D>
__device__ __forceinline__ void store_atoms_warp(const uint8_t* tile, uint32_t skip,
                                                 const Runs& tr, __nv_bfloat16* out, int N,
                                                 int H, int b, int h) {
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
  const int lane = threadIdx.x & 31;
  for (uint32_t m = skip; m != 0; m &= m - 1) {
    const int a = __ffs(m) - 1;
    for (int i = lane; i < 8 * kChunks; i += 32) {
      const int row = 8 * a + i / kChunks, c = i % kChunks;
      int dst = -1, base = 0;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        if (k < tr.n && row >= base && row < base + tr.len[k]) dst = tr.src[k] + (row - base);
        base += k < tr.n ? tr.len[k] : 0;
      }
      if (dst < 0) continue;
      const uint4 v = *reinterpret_cast<const uint4*>(
          tile + (c / 8) * Tile<D>::kHalfBytes + row * 128 + (((c % 8) ^ (row & 7)) * 16));
      *reinterpret_cast<uint4*>(out + ((static_cast<long long>(b) * N + dst) * H + h) * D + 8 * c) = v;
    }
  }
}

// Whole-tile GEMMs issued by the MMA thread. Operand descriptors are built once per call and
// advanced by constant offsets: the tensor core's issue queue is only a few instructions
// deep, so per-instruction scalar work in the issuing thread shows up as tensor-core idle time.
//
// D[128 x 128] (+)= A[128 x D] * B[128 x D]^T, both operands 128-row K-major tiles (SW128).
template <int D>
__device__ __forceinline__ void gemm_ss_k(uint32_t d_tmem, uint32_t a_base, uint32_t b_base,
                                          uint32_t idesc) {
  const uint64_t a0 = sdesc_sw128(a_base, 16, 1024), b0 = sdesc_sw128(b_base, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = static_cast<uint64_t>(((kk / 4) * Tile<D>::kHalfBytes + (kk % 4) * 32) >> 4);
    mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
  }
}
// D[128 x D] (+)= A[128 x 128 bf16, in TMEM] * B[128 (K) x D], B an MN-major tile (SW128).
template <int D>
__device__ __forceinline__ void gemm_ts_mn(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base,
                                           uint32_t idesc, bool accumulate) {
  const uint64_t b0 = sdesc_sw128(b_base, Tile<D>::kHalfBytes, 1024);
#pragma unroll
  for (int kk = 0; kk < kTileRows / 16; ++kk)
    mma_ts(d_tmem, a_tmem + kk * 8, b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// Dynamic work distribution for the persistent kernels. One thread of the CTA claims units
// from a global counter {next, done} (heaviest units have the lowest indices, so claiming in
// counter order is longest-first and balances the load) and publishes each claimed unit, or
// -1 when none is left, to the CTA's other roles through a 4-slot ring in shared memory:
// ring slot k % 4 is filled after the slot's previous unit was acknowledged by every consumer.
// The last CTA to run out of units resets the counter, so the next launch starts from zero.
constexpr int kUnitRing = 4;
__device__ __forceinline__ int claim_unit(unsigned int* sched, int n_units) {
  const unsigned int u = atomicAdd(sched, 1u);
  if (u < static_cast<unsigned int>(n_units)) return static_cast<int>(u);
  __threadfence();
  if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
    atomicExch(sched, 0u);
    atomicExch(sched + 1, 0u);
  }
  return -1;
}
// Producer side: claim the k-th unit of this CTA and publish it (slot k % 4).
__device__ __forceinline__ bool publish_unit(int k, int& u, unsigned int* sched, int n_units,
                                             volatile int* ring, uint32_t full0, uint32_t empty0,
                                             const WaitCtx& ctx, uint32_t site) {
  const int slot = k % kUnitRing;
  if (k >= kUnitRing &&
      !wait_bar(empty0 + 8u * slot, ((k / kUnitRing) - 1) & 1, ctx, site)) return false;
  u = claim_unit(sched, n_units);
  ring[slot] = u;
  mbar_arrive(full0 + 8u * slot);
  return true;
}
// Consumer side (a whole warp, or one thread with lanes == 1): read the k-th unit.
__device__ __forceinline__ bool read_unit(int k, int& u, volatile const int* ring, uint32_t full0,
                                          uint32_t empty0, const WaitCtx& ctx, uint32_t site,
                                          bool whole_warp) {
  const int slot = k % kUnitRing;
  bool ok = wait_bar(full0 + 8u * slot, (k / kUnitRing) & 1, ctx, site);
  if (whole_warp) ok = __all_sync(0xffffffffu, ok);
  if (!ok) return false;
  u = ring[slot];
  if (whole_warp) __syncwarp();
  if (!whole_warp || (threadIdx.x % 32) == 0) mbar_arrive(empty0 + 8u * slot);
  return true;
}

// As gemm_ts_mn, with the bf16 A operand written by kGroups column groups of W = 128 / kGroups
// columns, each packed into the first W/2 TMEM columns of its own range: the 16 K-values of
// step kk sit at a_tmem + W * (16 kk / W) + (16 kk % W) / 2.
template <int D, int W>
__device__ __forceinline__ void gemm_ts_mn_grouped(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base,
                                                   uint32_t idesc, bool accumulate) {
  const uint64_t b0 = sdesc_sw128(b_base, Tile<D>::kHalfBytes, 1024);
#pragma unroll
  for (int kk = 0; kk < kTileRows / 16; ++kk)
    mma_ts(d_tmem, a_tmem + W * ((16 * kk) / W) + ((16 * kk) % W) / 2,
           b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// Wait used only while tearing down: ignores the abort flag, bounded by the timeout.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity,
                                           unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) return;
  }
}

// Warp-uniform wait: every lane waits (each needs the acquire), and the warp proceeds only
// if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& ctx,
                                          uint32_t site) {
  const bool ok = wait_bar(bar, parity, ctx, site);
  return __all_sync(0xffffffffu, ok);
}

// 1024-byte aligned base of the dynamic shared memory window (swizzle atoms need it).
__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return raw + (((a + 1023u) & ~1023u) - a);
}

}  // namespace s2
