// K1: LayerNorm statistics prologue.
//
// One CTA of 256 threads per row. Each thread loads 16-byte vectors (8 bf16)
// of x, residual (and bias_in) with coalesced row loads, forms h = x + r (+b)
// in fp32, writes residual_out = bf16_rne(h), and keeps h in registers for the
// two-pass statistics: mean = sum(h)/K, then var = sum((h-mean)^2)/K, both
// reduced with warp shuffles and one shared-memory exchange; rstd =
// 1/sqrt(var + eps). The order is the fused_layernorm_qkv order of TensorRT-LLM
// 深度工程实践, §2.3 (mean, variance, rsqrt(var + epsilon)).
//
// The kernel triggers its dependents at entry (programmatic dependent launch):
// the GEMM kernel that follows starts its prologue and weight stream at once and
// waits (griddepcontrol.wait) only before it reads the statistics.
#pragma once

#include "common.cuh"

namespace fnl {

constexpr int kK1Threads = 256;

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();   // red[] reuse guard
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kK1Threads / 32; ++w) s += red[w];
  return s;
}

template <int MAXV>
__global__ void __launch_bounds__(kK1Threads) k1_layernorm_stats(const bf16* __restrict__ x,
                                                                 const bf16* __restrict__ residual,
                                                                 const bf16* __restrict__ bias_in,
                                                                 bf16* __restrict__ residual_out,
                                                                 float2* __restrict__ stats,
                                                                 float* __restrict__ mean_out,
                                                                 float* __restrict__ rstd_out, int M, int K,
                                                                 float eps) {
  pdl_launch_dependents();
  __shared__ float red[kK1Threads / 32];
  const int row = blockIdx.x;
  if (row >= M) return;
  const int nvec = K >> 3;
  const size_t rbase = static_cast<size_t>(row) * K;
  float h[MAXV][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * kK1Threads;
    if (v < nvec) {
      float xr[8], rr[8], bb[8];
      unpack8(ldg16(x + rbase + v * 8), xr);
      unpack8(ldg16(residual + rbase + v * 8), rr);
      load8_or_zero(bias_in, v * 8, true, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[i][e] = (xr[e] + rr[e]) + bb[e];
        s += h[i][e];
      }
      *reinterpret_cast<uint4*>(residual_out + rbase + v * 8) = pack8(h[i]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) h[i][e] = 0.f;
    }
  }
  const float mean = block_sum_256(s, red) / static_cast<float>(K);
  float s2 = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * kK1Threads;
    if (v < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = h[i][e] - mean;
        s2 = fmaf(d, d, s2);
      }
    }
  }
  const float var = block_sum_256(s2, red) / static_cast<float>(K);
  const float rstd = 1.f / sqrtf(var + eps);
  if (threadIdx.x == 0) {
    stats[row] = make_float2(mean, rstd);
    if (mean_out) mean_out[row] = mean;
    if (rstd_out) rstd_out[row] = rstd;
  }
}

}  // namespace fnl
