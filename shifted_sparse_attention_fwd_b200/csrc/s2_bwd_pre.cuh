// Backward preprocess: D[b,h,t] = sum_c dO[b,t,h,c] * O[b,t,h,c] in fp32, and the row
// log-sum-exp rescaled to base 2, LSE2 = LSE * log2(e), both laid out [B, Hq, N].
//
// D is the row term of the softmax derivative, dS = P o (dP - D) with
// D_i = sum_j P_ij dP_ij = dO_i . O_i (the backward of the causal self-attention that
// LongLoRA's Algorithm 1 applies per group, §3.4). Memory bound: every byte of O and dO is
// read once. Block 0 also clears the work counters the persistent gradient kernels claim their
// units from.
//
// s2_bwd_pre_stream_kernel (the common case): one CTA per SM streams a contiguous range of
// tokens. A producer warp moves each token's (Hq x D) block of O and of dO into a 3-stage
// shared-memory ring with bulk copies (one 8-32 KB copy per token and tensor, completion counted
// on an mbarrier); eight warps reduce the rows from shared memory (D/8 lanes per row, 16-byte
// reads of consecutive chunks) and write D and LSE2 for the stage's tokens, consecutive threads
// taking consecutive tokens of one head. s2_bwd_pre_kernel, the plain-load version, covers
// heads too wide for the ring.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "s2_common.cuh"

namespace s2 {

// A block covers kPreTokens consecutive tokens of one batch and every head: for contiguous O
// and dO the rows it reads (token-major, head-minor) are one contiguous range of memory.
// O and dO are addressed through their batch and token strides (elements).
constexpr int kPreTokens = 8;

template <int D>
__global__ void __launch_bounds__(256) s2_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ dvec,
                                                         float* __restrict__ lse2,
                                                         unsigned int* __restrict__ sched,
                                                         int sched_words, int Hq, int N,
                                                         long long o_sb, long long o_st,
                                                         long long do_sb, long long do_st) {
  constexpr int kLanesPerRow = D / 8;            // 16-byte chunks per (token, head) row
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  // The work counters of the gradient kernels that follow start from zero.
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < sched_words; i += blockDim.x) sched[i] = 0u;

  const int tblocks = (N + kPreTokens - 1) / kPreTokens;
  const int b = blockIdx.x / tblocks;
  const int t0 = (blockIdx.x % tblocks) * kPreTokens;
  const int nt = N - t0 < kPreTokens ? N - t0 : kPreTokens;
  const int rows = nt * Hq;                      // rows r = (t - t0) * Hq + h
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int sub = lane / kLanesPerRow, li = lane % kLanesPerRow;

  constexpr int kUnroll = 4;                     // row pairs in flight per thread
  for (int r0 = warp * kRowsPerWarp; r0 < rows; r0 += kUnroll * 8 * kRowsPerWarp) {
    uint4 ov[kUnroll], gv[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int rr = r0 + k * 8 * kRowsPerWarp + sub;
      if (rr < rows) {
        const long long t = t0 + rr / Hq, hd = static_cast<long long>(rr % Hq) * D + li * 8;
        ov[k] = __ldg(reinterpret_cast<const uint4*>(o + b * o_sb + t * o_st + hd));
        gv[k] = __ldg(reinterpret_cast<const uint4*>(dO + b * do_sb + t * do_st + hd));
      } else {
        ov[k] = make_uint4(0, 0, 0, 0);
        gv[k] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int rr = r0 + k * 8 * kRowsPerWarp + sub;
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ov[k]);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv[k]);
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fg = __bfloat1622float2(g2[e]);
        acc = fmaf(fa.x, fg.x, acc);
        acc = fmaf(fa.y, fg.y, acc);
      }
#pragma unroll
      for (int sh = kLanesPerRow / 2; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
      if (li == 0 && rr < rows) {
        const int h = rr % Hq, t = t0 + rr / Hq;
        const size_t idx = (static_cast<size_t>(b) * Hq + h) * N + t;
        dvec[idx] = acc;
        lse2[idx] = lse[idx] * 1.4426950408889634f;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Streaming version.
// ---------------------------------------------------------------------------------------
struct PreParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  long long o_sb, o_st, do_sb, do_st;   // element strides of the batch and token axes
  const float* lse;
  float* dvec;
  float* lse2;
  unsigned int* sched;
  int sched_words;
  int B, Hq, N;
  int tps;          // tokens per stage (tps * Hq * D * 2 bytes of each tensor)
  unsigned int* err;
  unsigned long long timeout_ns;
};

constexpr int kPreStages = 3;
constexpr int kPreComputeWarps = 8;
constexpr int kPreThreads = 32 * (kPreComputeWarps + 1);
constexpr uint32_t kPreStageMax = 32768;   // bytes of each tensor per stage (at least one token)

// Shared-memory layout: kPreStages x {O block, dO block}, the D values of one stage
// (token-major), the full / empty barriers, the abort flag.
__host__ __device__ inline uint32_t pre_stage_bytes(int tps, int Hq, int D) {
  return static_cast<uint32_t>(tps) * Hq * D * 2;
}
__host__ __device__ inline uint32_t pre_bar_offset(int tps, int Hq, int D) {
  return (kPreStages * 2 * pre_stage_bytes(tps, Hq, D) + 4u * tps * Hq + 7u) & ~7u;
}
__host__ __device__ inline uint32_t pre_smem_bytes(int tps, int Hq, int D) {
  return pre_bar_offset(tps, Hq, D) + 8u * (2 * kPreStages) + 8u;
}

__device__ __forceinline__ void pre_compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(32 * kPreComputeWarps) : "memory");
}
// Barrier of the compute warps that also ORs a predicate over them: every warp gets the same
// answer, so they leave the loop together.
__device__ __forceinline__ bool pre_compute_any(bool q) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(q ? 1u : 0u), "r"(32 * kPreComputeWarps)
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kPreThreads, 1) s2_bwd_pre_stream_kernel(const PreParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t stage_bytes = pre_stage_bytes(p.tps, p.Hq, D);
  float* s_d = reinterpret_cast<float*>(smem + kPreStages * 2 * stage_bytes);
  const uint32_t bar_off = pre_bar_offset(p.tps, p.Hq, D);
  const uint32_t bars = smem_u32(smem + bar_off);
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kPreStages + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + bar_off + 8u * (2 * kPreStages));
  const WaitCtx ctx{abort_flag, p.err, p.timeout_ns, KID_PRE};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.sched_words; i += blockDim.x) p.sched[i] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPreStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kPreComputeWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // This CTA's stages: a contiguous range, so its tokens are consecutive.
  const long long tokens = static_cast<long long>(p.B) * p.N;
  const long long n_stages = (tokens + p.tps - 1) / p.tps;
  const long long s_begin = n_stages * blockIdx.x / gridDim.x;
  const long long s_end = n_stages * (blockIdx.x + 1) / gridDim.x;
  const int row_bytes = p.Hq * D * 2;

  if (warp == kPreComputeWarps) {
    // ---------------- producer: one bulk copy per token and tensor ----------------
    if (lane == 0) {
      int k = 0;
      for (long long s = s_begin; s < s_end; ++s, ++k) {
        const int slot = k % kPreStages;
        if (k >= kPreStages && !wait_bar(empty(slot), ((k / kPreStages) - 1) & 1, ctx, 1)) break;
        const long long g0 = s * p.tps;
        const int nt = static_cast<int>(tokens - g0 < p.tps ? tokens - g0 : p.tps);
        mbar_expect_tx(full(slot), 2u * nt * row_bytes);
        const uint32_t dst = smem_u32(smem + slot * 2 * stage_bytes);
        for (int i = 0; i < nt; ++i) {
          const long long g = g0 + i, b = g / p.N, t = g % p.N;
          bulk_load(dst + i * row_bytes, p.o + b * p.o_sb + t * p.o_st, row_bytes, full(slot));
          bulk_load(dst + stage_bytes + i * row_bytes, p.dO + b * p.do_sb + t * p.do_st, row_bytes,
                    full(slot));
        }
      }
      // Every issued copy lands before the CTA can exit.
      for (int j = (k > kPreStages ? k - kPreStages : 0); j < k; ++j)
        drain_wait(full(j % kPreStages), (j / kPreStages) & 1, p.timeout_ns);
    }
  } else {
    // ---------------- reduction: D/8 lanes per (token, head) row ----------------
    constexpr int kLanesPerRow = D / 8;
    constexpr int kRowsPerStep = 32 / kLanesPerRow;
    const int sub = lane / kLanesPerRow, li = lane % kLanesPerRow;
    int k = 0;
    for (long long s = s_begin; s < s_end; ++s, ++k) {
      const int slot = k % kPreStages;
      const bool ok = warp_wait(full(slot), (k / kPreStages) & 1, ctx, 2);
      // Every compute warp passes this barrier each stage and gets the same verdict, so a wait
      // that gave up (here or in the producer) ends the loop of all of them together; the
      // barrier also frees s_d of the previous stage.
      if (pre_compute_any(!ok || *abort_flag != 0)) break;
      const long long g0 = s * p.tps;
      const int nt = static_cast<int>(tokens - g0 < p.tps ? tokens - g0 : p.tps);
      const int nrows = nt * p.Hq;
      const uint8_t* so = smem + slot * 2 * stage_bytes;
      const uint8_t* sg = so + stage_bytes;
      for (int r0 = warp * kRowsPerStep; r0 < nrows; r0 += kPreComputeWarps * kRowsPerStep) {
        const int r = r0 + sub;                 // warp-uniform loop, per-lane row
        float acc = 0.f;
        if (r < nrows) {
          const uint4 a = *reinterpret_cast<const uint4*>(so + r * (D * 2) + li * 16);
          const uint4 c = *reinterpret_cast<const uint4*>(sg + r * (D * 2) + li * 16);
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
          const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fa = __bfloat1622float2(a2[e]);
            const float2 fc = __bfloat1622float2(c2[e]);
            acc = fmaf(fa.x, fc.x, acc);
            acc = fmaf(fa.y, fc.y, acc);
          }
        }
#pragma unroll
        for (int sh = kLanesPerRow / 2; sh > 0; sh >>= 1)
          acc += __shfl_xor_sync(0xffffffffu, acc, sh);
        if (li == 0 && r < nrows) s_d[r] = acc;   // row r = token r / Hq, head r % Hq
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(slot));   // this warp is done reading the slot
      pre_compute_sync();
      // D and LSE2 of the stage's tokens, consecutive threads on consecutive tokens of one
      // head (the [B, Hq, N] layout).
      for (int i = threadIdx.x; i < nrows; i += 32 * kPreComputeWarps) {
        const int h = i / nt, tt = i % nt;
        const long long g = g0 + tt, b = g / p.N, t = g % p.N;
        const size_t idx = (static_cast<size_t>(b) * p.Hq + h) * p.N + t;
        p.dvec[idx] = s_d[tt * p.Hq + h];
        p.lse2[idx] = p.lse[idx] * 1.4426950408889634f;
      }
    }
  }
}

}  // namespace s2
