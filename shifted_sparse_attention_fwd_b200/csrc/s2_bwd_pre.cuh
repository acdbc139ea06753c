// Backward preprocess: D[b,h,t] = sum_c dO[b,t,h,c] * O[b,t,h,c] in fp32, and the row
// log-sum-exp rescaled to base 2, LSE2 = LSE * log2(e), both laid out [B, Hq, N].
//
// D is the row term of the softmax derivative, dS = P o (dP - D) with
// D_i = sum_j P_ij dP_ij = dO_i . O_i (the backward of the causal self-attention that
// LongLoRA's Algorithm 1 applies per group, §3.4). Memory bound: every byte of O and dO is
// read once with 16-byte loads; each block covers 128 consecutive tokens of one (b, h) so
// that the [B, Hq, N] outputs are written as coalesced 512-byte rows. Block 0 also clears the
// work counters the persistent gradient kernels claim their units from.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace s2 {

template <int D>
__global__ void __launch_bounds__(256) s2_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ dvec,
                                                         float* __restrict__ lse2,
                                                         unsigned int* __restrict__ sched,
                                                         int sched_words, int Hq, int N) {
  constexpr int kLanesPerRow = D / 8;            // 16-byte chunks per row
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  constexpr int kPasses = 16 / kRowsPerPass;     // 16 rows per warp, 8 warps per block
  __shared__ float s_d[128];
  // The work counters of the gradient kernels that follow start from zero.
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < sched_words; i += blockDim.x) sched[i] = 0u;

  const int tiles = (N + 127) / 128;
  const int tile = blockIdx.x % tiles;
  const int bh = blockIdx.x / tiles;
  const int h = bh % Hq, b = bh / Hq;
  const int t0 = tile * 128;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int sub = lane / kLanesPerRow, li = lane % kLanesPerRow;

  uint4 ov[kPasses], gv[kPasses];
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int t = t0 + warp * 16 + i * kRowsPerPass + sub;
    if (t < N) {
      const size_t off = ((static_cast<size_t>(b) * N + t) * Hq + h) * D + li * 8;
      ov[i] = __ldg(reinterpret_cast<const uint4*>(o + off));
      gv[i] = __ldg(reinterpret_cast<const uint4*>(dO + off));
    } else {
      ov[i] = make_uint4(0, 0, 0, 0);
      gv[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&ov[i]);
    const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(&gv[i]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(a[e]);
      const float2 fg = __bfloat1622float2(g[e]);
      acc = fmaf(fa.x, fg.x, acc);
      acc = fmaf(fa.y, fg.y, acc);
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (li == 0) s_d[warp * 16 + i * kRowsPerPass + sub] = acc;
  }
  __syncthreads();
  if (threadIdx.x < 128) {
    const int t = t0 + threadIdx.x;
    if (t < N) {
      const size_t idx = (static_cast<size_t>(b) * Hq + h) * N + t;
      dvec[idx] = s_d[threadIdx.x];
      lse2[idx] = lse[idx] * 1.4426950408889634f;
    }
  }
}

}  // namespace s2
