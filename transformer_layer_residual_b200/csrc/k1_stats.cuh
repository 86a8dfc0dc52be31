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

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = 0.f;
#pragma unroll
  for (int w = 0; w < kK1Threads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// Sum and max over the block's 256 threads with one shared-memory exchange.
__device__ __forceinline__ void block_sum_max_256(float& s, float& m, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) {
    red[warp] = s;
    red[kK1Threads / 32 + warp] = m;
  }
  __syncthreads();
  s = 0.f;
  m = 0.f;
#pragma unroll
  for (int w = 0; w < kK1Threads / 32; ++w) {
    s += red[w];
    m = fmaxf(m, red[kK1Threads / 32 + w]);
  }
}

// FP8 pre-pass of the fused ops (per-token dynamic quantisation, TensorRT-LLM
// 深度工程实践, §3.3 FP4/FP8 动态量化加速: activation ranges from runtime
// statistics). One CTA per row: h = x + r (+ bias_in) in fp32, residual_out =
// bf16(h), the row's statistics (LayerNorm: two-pass mean and variance;
// RMSNorm: mean of h^2), then the value the FP8 converters quantise, computed
// exactly as they compute it, and its amax: LayerNorm a = (h - mean) rstd
// gamma + beta; RMSNorm a = h gamma (1/rms is a positive per-token factor, so
// it joins the token's dequantisation scale instead). Writes stats8[row] =
// (mean, rstd, dequantisation scale, 448 / amax) with the scale amax / 448
// (times rstd for RMSNorm); 1 and 1 for a zero row; and the row's activation
// codes q8[row][k] = e4m3(a * 448 / amax) (round to nearest even, saturating),
// which the GEMM loads as its operand: the row is quantised once, not once per
// weight tile.
template <int MAXV, bool RMS>
__global__ void __launch_bounds__(kK1Threads) k1_fp8_prepass(const bf16* __restrict__ x,
                                                             const bf16* __restrict__ residual,
                                                             const bf16* __restrict__ bias_in,
                                                             const bf16* __restrict__ gamma,
                                                             const bf16* __restrict__ beta,
                                                             bf16* __restrict__ residual_out,
                                                             float4* __restrict__ stats8,
                                                             uint8_t* __restrict__ q8,
                                                             float* __restrict__ mean_out,
                                                             float* __restrict__ rstd_out, int M, int K,
                                                             float eps) {
  pdl_launch_dependents();
  __shared__ float red[2 * kK1Threads / 32];
  const int row = blockIdx.x;
  if (row >= M) return;
  const int nvec = K >> 3;
  const size_t rbase = static_cast<size_t>(row) * K;
  f32x2 h[MAXV][4];
  float s = 0.f;
  float amax = 0.f;   // RMSNorm: max |h gamma|, taken in the first pass
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * kK1Threads;
    if (v < nvec) {
      const uint4 xv = ldg16(x + rbase + v * 8), rv = ldg16(residual + rbase + v * 8);
      const uint4 bv = bias_in != nullptr ? ldg16(bias_in + v * 8) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, rw[4] = {rv.x, rv.y, rv.z, rv.w};
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t ho[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        h[i][e] = add2(bf2_to_f2(xw[e]), bf2_to_f2(rw[e]));
        if (bias_in != nullptr) h[i][e] = add2(h[i][e], bf2_to_f2(bw[e]));
        float lo, hi;
        unpk2(h[i][e], lo, hi);
        s += RMS ? fmaf(lo, lo, hi * hi) : lo + hi;
        ho[e] = f2_to_bf2(h[i][e]);
      }
      if (RMS) {   // the value the converters quantise: h * gamma
        const uint4 gv = ldg16(gamma + v * 8);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float lo, hi;
          unpk2(mul2(h[i][e], bf2_to_f2(gw[e])), lo, hi);
          amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        }
      }
      *reinterpret_cast<uint4*>(residual_out + rbase + v * 8) = make_uint4(ho[0], ho[1], ho[2], ho[3]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) h[i][e] = 0ull;
    }
  }
  float mean = 0.f, rstd;
  if (RMS) {
    block_sum_max_256(s, amax, red);
    rstd = 1.f / sqrtf(s / static_cast<float>(K) + eps);
  } else {
    mean = block_sum_256(s, red) / static_cast<float>(K);
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = threadIdx.x + i * kK1Threads;
      if (v < nvec) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float lo, hi;
          unpk2(h[i][e], lo, hi);
          const float d0 = lo - mean, d1 = hi - mean;
          s2 = fmaf(d0, d0, s2);
          s2 = fmaf(d1, d1, s2);
        }
      }
    }
    rstd = 1.f / sqrtf(block_sum_256(s2, red) / static_cast<float>(K) + eps);
  }
  const f32x2 mu2 = pk2(mean, mean), rs2 = pk2(rstd, rstd);
#pragma unroll
  for (int i = 0; i < MAXV && !RMS; ++i) {   // LayerNorm: amax of the normalised value
    const int v = threadIdx.x + i * kK1Threads;
    if (v < nvec) {
      const uint4 gv = ldg16(gamma + v * 8);
      const uint4 bv = beta != nullptr ? ldg16(beta + v * 8) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const f32x2 a = fma2(mul2(sub2(h[i][e], mu2), rs2), bf2_to_f2(gw[e]), bf2_to_f2(bw[e]));
        float lo, hi;
        unpk2(a, lo, hi);
        amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
      }
    }
  }
  if (!RMS) amax = block_max_256(amax, red);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (threadIdx.x == 0) {
    const float sa = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    stats8[row] = make_float4(mean, rstd, RMS ? rstd * sa : sa, inv);
    if (mean_out) mean_out[row] = mean;
    if (rstd_out) rstd_out[row] = rstd;
  }
  // the codes: the same fp32 operations, in the same order, as the amax above
  const f32x2 inv2 = pk2(inv, inv);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * kK1Threads;
    if (v < nvec) {
      const uint4 gv = ldg16(gamma + v * 8);
      const uint4 bv = (!RMS && beta != nullptr) ? ldg16(beta + v * 8) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
      f32x2 a[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const f32x2 y = RMS ? mul2(h[i][e], bf2_to_f2(gw[e]))
                            : fma2(mul2(sub2(h[i][e], mu2), rs2), bf2_to_f2(gw[e]), bf2_to_f2(bw[e]));
        a[e] = mul2(y, inv2);
      }
      *reinterpret_cast<uint2*>(q8 + rbase + v * 8) = make_uint2(e4m3x4(a[0], a[1]), e4m3x4(a[2], a[3]));
    }
  }
}

// Static per-output-channel FP8 weights: one CTA per W row, s_w = amax / 448
// (1 for a zero row) and codes e4m3(w / s_w), both divisions IEEE in fp32.
__global__ void __launch_bounds__(kK1Threads) k0_quantize_weight_fp8(const bf16* __restrict__ W,
                                                                    uint8_t* __restrict__ Wq,
                                                                    float* __restrict__ w_scale, int N, int K) {
  __shared__ float red[kK1Threads / 32];
  const int row = blockIdx.x;
  if (row >= N) return;
  const size_t base = static_cast<size_t>(row) * K;
  const int nvec = K >> 3;
  float amax = 0.f;
  for (int v = threadIdx.x; v < nvec; v += kK1Threads) {
    float f[8];
    unpack8(ldg16(W + base + v * 8), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
  amax = block_max_256(amax, red);
  const float sw = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  for (int v = threadIdx.x; v < nvec; v += kK1Threads) {
    float f[8];
    unpack8(ldg16(W + base + v * 8), f);
    uint32_t c[2];
#pragma unroll
    for (int e = 0; e < 2; ++e)
      c[e] = e4m3x4(pk2(__fdiv_rn(f[4 * e], sw), __fdiv_rn(f[4 * e + 1], sw)),
                    pk2(__fdiv_rn(f[4 * e + 2], sw), __fdiv_rn(f[4 * e + 3], sw)));
    *reinterpret_cast<uint2*>(Wq + base + v * 8) = make_uint2(c[0], c[1]);
  }
  if (threadIdx.x == 0) w_scale[row] = sw;
}

}  // namespace fnl
