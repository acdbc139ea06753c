// Backward preprocess: D[b,h,t] = sum_c dO[b,t,h,c] * O[b,t,h,c] in fp32, and the row
// log-sum-exp rescaled to base 2, LSE2 = LSE * log2(e), both laid out [B, Hq, N].
//
// D is the row term of the softmax derivative, dS = P o (dP - D) with
// D_i = sum_j P_ij dP_ij = dO_i . O_i (the backward of the causal self-attention that
// LongLoRA's Algorithm 1 applies per group, §3.4). Memory bound: every byte of O and dO is
// read once with 16-byte loads, each block streaming one contiguous range of memory (a few
// tokens, all heads); the small [B, Hq, N] outputs are written as 32-byte pieces. Block 0
// also clears the work counters the persistent gradient kernels claim their units from.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

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
  constexpr int kStride = 8 * kRowsPerWarp;      // rows between a thread's unrolled loads
  // Row rr of the block is (token t0 + rr / Hq, head rr % Hq). Each thread's rows advance by
  // fixed steps, so their (token, head) pairs are stepped instead of divided per load: the
  // integer divisions had made this memory-bound kernel issue-bound.
  int tk[kUnroll], hk[kUnroll];
#pragma unroll
  for (int k = 0; k < kUnroll; ++k) {
    const int rr = warp * kRowsPerWarp + k * kStride + sub;
    tk[k] = rr / Hq;
    hk[k] = rr % Hq;
  }
  const int step_rows = kUnroll * kStride;       // rows from one iteration to the next
  const int dt = step_rows / Hq, dh = step_rows % Hq;
  const long long o_base = b * o_sb + t0 * o_st + li * 8, do_base = b * do_sb + t0 * do_st + li * 8;
  for (int r0 = warp * kRowsPerWarp; r0 < rows; r0 += step_rows) {
    uint4 ov[kUnroll], gv[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int rr = r0 + k * kStride + sub;
      if (rr < rows) {
        const long long hd = static_cast<long long>(hk[k]) * D;
        ov[k] = __ldg(reinterpret_cast<const uint4*>(o + o_base + tk[k] * o_st + hd));
        gv[k] = __ldg(reinterpret_cast<const uint4*>(dO + do_base + tk[k] * do_st + hd));
      } else {
        ov[k] = make_uint4(0, 0, 0, 0);
        gv[k] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int rr = r0 + k * kStride + sub;
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
        const size_t idx = (static_cast<size_t>(b) * Hq + hk[k]) * N + t0 + tk[k];
        dvec[idx] = acc;
        lse2[idx] = lse[idx] * 1.4426950408889634f;
      }
      // this thread's next row of slot k
      tk[k] += dt;
      hk[k] += dh;
      if (hk[k] >= Hq) {
        hk[k] -= Hq;
        ++tk[k];
      }
    }
  }
}

}  // namespace s2
