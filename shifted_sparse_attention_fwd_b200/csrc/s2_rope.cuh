// Rotary position embedding with Position Interpolation, applied to a [B, N, H, D] bf16
// tensor: the step just before the attention (LongLoRA summary page, §3 "Phase 1" step 2
// "Position Embedding Modification", and §4 "Model setup": RoPE with positions rescaled by
// Position Interpolation). For token t (original order) and i < D/2 the pair
// (x[i], x[i + D/2]) turns by the angle (t * pi_scale) * base^(-2i/D) (the Llama half-split
// pairing); `inverse` turns by the opposite angle, which is the transpose of the rotation and
// so maps gradients with respect to the rotated tensor back to the input.
//
// Memory bound: each block takes kRopeTokens consecutive tokens of one batch element, first
// computes the cos/sin of their D/2 angles once (shared by every head), then streams all heads
// of those tokens with 16-byte loads and stores. In place (y == x) is allowed: every element is
// read and written by the same thread.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace s2 {

constexpr int kRopeTokens = 8;
constexpr int kRopeThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRopeThreads) s2_rope_kernel(
    const __nv_bfloat16* x, __nv_bfloat16* y, int N, int H,
    long long x_sb, long long x_st, long long y_sb, long long y_st, float log2_base,
    float pi_scale, float sin_sign) {
  constexpr int kHalf = D / 2;
  constexpr int kChunks = kHalf / 8;             // 8 pairs per 16-byte chunk of each half
  __shared__ float s_cos[kRopeTokens][kHalf], s_sin[kRopeTokens][kHalf];
  const int tblocks = (N + kRopeTokens - 1) / kRopeTokens;
  const int b = blockIdx.x / tblocks;
  const int t0 = (blockIdx.x % tblocks) * kRopeTokens;
  const int nt = N - t0 < kRopeTokens ? N - t0 : kRopeTokens;
  for (int k = threadIdx.x; k < kRopeTokens * kHalf; k += blockDim.x) {
    const int tt = k / kHalf, i = k % kHalf;
    // theta_i = base^(-2i/D); the angle in fp32 (exact position product, one rounding of
    // theta), cos and sin with the library's accurate sincosf
    const float theta = exp2f(-(2.0f * i / D) * log2_base);
    const float ang = (static_cast<float>(t0 + tt) * pi_scale) * theta;
    float sv, cv;
    sincosf(ang, &sv, &cv);
    s_cos[tt][i] = cv;
    s_sin[tt][i] = sin_sign * sv;
  }
  __syncthreads();
  // work item = (token, head, chunk): chunk c covers pairs 8c .. 8c + 7, i.e. the 16 bytes at
  // column 8c of the first half and those at column D/2 + 8c. Each thread loads kRopeUnroll
  // items before computing, to keep more bytes in flight.
  constexpr int kRopeUnroll = 4;
  const int items = nt * H * kChunks;
  for (int w0 = threadIdx.x; w0 < items; w0 += kRopeUnroll * blockDim.x) {
    uint4 lo[kRopeUnroll], hi[kRopeUnroll];
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int w = w0 + u * blockDim.x;
      if (w < items) {
        const int c = w % kChunks, th = w / kChunks;
        const int h = th % H, tt = th / H;
        const __nv_bfloat16* src =
            x + b * x_sb + (t0 + tt) * x_st + static_cast<long long>(h) * D + 8 * c;
        lo[u] = *reinterpret_cast<const uint4*>(src);
        hi[u] = *reinterpret_cast<const uint4*>(src + kHalf);
      }
    }
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int w = w0 + u * blockDim.x;
      if (w >= items) break;
      const int c = w % kChunks, th = w / kChunks;
      const int h = th % H, tt = th / H;
      __nv_bfloat16* dst = y + b * y_sb + (t0 + tt) * y_st + static_cast<long long>(h) * D + 8 * c;
      const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo[u]);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi[u]);
      uint4 olo, ohi;
      __nv_bfloat162* ol = reinterpret_cast<__nv_bfloat162*>(&olo);
      __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = __bfloat1622float2(l2[j]), bb = __bfloat1622float2(h2[j]);
        const int i = 8 * c + 2 * j;
        const float c0 = s_cos[tt][i], c1 = s_cos[tt][i + 1];
        const float s0 = s_sin[tt][i], s1 = s_sin[tt][i + 1];
        ol[j] = __floats2bfloat162_rn(a.x * c0 - bb.x * s0, a.y * c1 - bb.y * s1);
        oh[j] = __floats2bfloat162_rn(bb.x * c0 + a.x * s0, bb.y * c1 + a.y * s1);
      }
      *reinterpret_cast<uint4*>(dst) = olo;
      *reinterpret_cast<uint4*>(dst + kHalf) = ohi;
    }
  }
}

}  // namespace s2
