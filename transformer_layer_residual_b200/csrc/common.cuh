// Parameters and epilogue arithmetic shared by the fused-op kernels.
#pragma once

#include "ptx.cuh"

namespace fnl {

typedef __nv_bfloat16 bf16;

enum Epi : int { kEpiQKV = 0, kEpiSwiGLU = 1, kEpiGELU = 2 };
enum Norm : int { kLayerNorm = 0, kRMSNorm = 1 };

struct OpParams {
  int M, K, N;       // tokens, hidden, rows of W
  int I;             // SwiGLU intermediate size (N = 2I)
  int Hq, Hkv, D;    // QKV heads
  float eps;
  const bf16* gamma;
  const bf16* beta;      // LayerNorm shift, may be null
  const bf16* bias_in;   // [K], may be null
  const bf16* bias;      // [N] output bias, may be null
  bf16* residual_out;    // written in the GEMM kernels for RMSNorm, by the stats kernel for LayerNorm
  float* rstd_out;       // RMSNorm statistics output (GEMM kernels), may be null
  const float2* stats;   // LayerNorm (mean, rstd) per row, written by the stats kernel
  bf16* q;
  bf16* k;
  bf16* v;
  bf16* out;
  // small-M split-K workspace
  float* part;           // [T][max_seg][mpad][128] fp32 partial accumulators
  float* part_ss;        // [T][max_seg][mpad] partial sums of h^2 (RMSNorm)
  unsigned* counters;    // [T] arrival counters, zero between launches
  int max_seg;
  int mpad;
  int stages;
  int split;             // 1: operand = bf16 hi + bf16 lo (two UMMAs), 0: single bf16 rounding
  int* status;           // device status word (bounded-wait failures)
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Round a[8] to bf16 (hi) and, if `split`, also the remainder a - hi to bf16 (lo).
__device__ __forceinline__ void round_split8(const float (&a)[8], bool split, uint4& hi, uint4& lo) {
  hi = pack8(a);
  if (split) {
    float h[8], r[8];
    unpack8(hi, h);
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = a[e] - h[e];
    lo = pack8(r);
  }
}

// Per-stage copies of the k-block's slices of gamma, beta and bias_in
// (64 bf16 each), brought in by the producer with the stage's tiles.
constexpr int kVecElems = 64;
constexpr int kVecStageBytes = 3 * kVecElems * 2;   // 384

// Bytes of the k-block's vector slices; the producer adds them to the stage's
// expected transaction count.
__device__ __forceinline__ uint32_t issue_vec_loads(const OpParams& p, bool has_beta, bool has_bias_in, int kb,
                                                    bf16* vec, uint64_t* bar) {
  const int k0 = kb * kVecElems;
  const int kvalid = min(kVecElems, p.K - k0);
  const uint32_t vb = static_cast<uint32_t>(kvalid) * 2;
  bulk_load(vec, p.gamma + k0, vb, bar);
  uint32_t n = vb;
  if (has_beta) {
    bulk_load(vec + kVecElems, p.beta + k0, vb, bar);
    n += vb;
  }
  if (has_bias_in) {
    bulk_load(vec + 2 * kVecElems, p.bias_in + k0, vb, bar);
    n += vb;
  }
  return n;
}

__device__ __forceinline__ uint32_t vec_bytes(const OpParams& p, bool has_beta, bool has_bias_in, int kb) {
  const int kvalid = min(kVecElems, p.K - kb * kVecElems);
  return static_cast<uint32_t>(kvalid) * 2 * (1 + (has_beta ? 1 : 0) + (has_bias_in ? 1 : 0));
}

// The converter's 8 gamma / beta / bias_in values of chunk c from the stage copy.
__device__ __forceinline__ void stage_vec8(const bf16* vec, int which, bool present, int c, bool kin,
                                           float (&f)[8]) {
  if (present && kin) {
    unpack8(ld_shared_v4(smem_u32(vec + which * kVecElems + c * 8)), f);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = 0.f;
  }
}

// 8 consecutive elements of one token row: h = x + r (+ bias_in) in fp32,
// a = normalise(h) rounded to bf16 (hi) and, if split, the bf16 remainder (lo).
// LayerNorm: a = (h - mean) * rstd * gamma + beta. RMSNorm (deferred scale):
// a = h * gamma and sq += h^2 (even and odd elements in the two lanes).
// g, be, bi: the chunk's gamma / beta / bias_in as four fp32 pairs.
template <int NORM>
__device__ __forceinline__ void convert8(const uint4& xv, const uint4& rv, const f32x2 (&g)[4], const f32x2 (&be)[4],
                                         const f32x2 (&bi)[4], bool has_beta, bool has_bias_in, float mean,
                                         float rstd, bool split, bool want_h, f32x2& sq, uint4& hi, uint4& lo,
                                         uint4& hres) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
  uint32_t ho[4], lw[4], hw[4];
  const f32x2 mu2 = pk2(mean, mean), rs2 = pk2(rstd, rstd);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f32x2 h = add2(bf2_to_f2(xw[i]), bf2_to_f2(rw[i]));
    if (has_bias_in) h = add2(h, bi[i]);
    f32x2 a;
    if (NORM == kLayerNorm) {
      a = mul2(sub2(h, mu2), rs2);
      a = has_beta ? fma2(a, g[i], be[i]) : mul2(a, g[i]);
    } else {
      a = mul2(h, g[i]);
      sq = fma2(h, h, sq);
    }
    ho[i] = f2_to_bf2(a);
    if (split) lw[i] = f2_to_bf2(sub2(a, bf2_to_f2(ho[i])));
    if (want_h) hw[i] = f2_to_bf2(h);
  }
  hi = make_uint4(ho[0], ho[1], ho[2], ho[3]);
  if (split) lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  if (want_h) hres = make_uint4(hw[0], hw[1], hw[2], hw[3]);
}

// A 16-byte vector of 8 bf16 as four fp32 pairs (zeros when absent).
__device__ __forceinline__ void vec_pairs(const bf16* vec, int which, bool present, int c, bool kin,
                                          f32x2 (&f)[4]) {
  if (present && kin) {
    const uint4 v = ld_shared_v4(smem_u32(vec + which * kVecElems + c * 8));
    f[0] = bf2_to_f2(v.x);
    f[1] = bf2_to_f2(v.y);
    f[2] = bf2_to_f2(v.z);
    f[3] = bf2_to_f2(v.w);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = 0ull;
  }
}

__device__ __forceinline__ void load8_or_zero(const bf16* base, int k0, bool ok, float (&f)[8]) {
  if (base != nullptr && ok) {
    unpack8(ldg16(base + k0), f);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = 0.f;
  }
}

// SiLU(g) = g / (1 + e^-g).
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.f + __expf(-g)); }

// GELU, tanh form: 0.5 z (1 + tanh(u)) with u = sqrt(2/pi)(z + 0.044715 z^3),
// evaluated as z / (1 + e^(-2u)) (the same function: 0.5(1 + tanh u) is the
// logistic function of 2u), which avoids the cancellation of 1 + tanh(u) for
// negative z.
__device__ __forceinline__ float gelu_tanh_f(float z) {
  const float u2 = -1.5957691216057308f * z * fmaf(0.044715f * z, z, 1.f);   // -2u
  return __fdividef(z, 1.f + __expf(u2));
}

// Store 8 consecutive output columns [n, n+8) of row m (QKV or GELU epilogue).
// acc is the raw fp32 accumulator, scale the deferred RMSNorm 1/rms (1 for LN).
template <int EPI>
__device__ __forceinline__ void store_out8(const OpParams& p, int m, int n, const float (&acc)[8], float scale) {
  float y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = acc[e] * scale;
  if (p.bias != nullptr) {
    float b[8];
    unpack8(ldg16(p.bias + n), b);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] += b[e];
  }
  bf16* dst;
  if (EPI == kEpiGELU) {
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = gelu_tanh_f(y[e]);
    dst = p.out + static_cast<size_t>(m) * p.N + n;
  } else {
    const int D = p.D;
    const int nq = p.Hq * D;
    const int nk = nq + p.Hkv * D;
    if (n < nq) {
      const int h = n / D;
      dst = p.q + (static_cast<size_t>(h) * p.M + m) * D + (n - h * D);
    } else if (n < nk) {
      const int n2 = n - nq, h = n2 / D;
      dst = p.k + (static_cast<size_t>(h) * p.M + m) * D + (n2 - h * D);
    } else {
      const int n2 = n - nk, h = n2 / D;
      dst = p.v + (static_cast<size_t>(h) * p.M + m) * D + (n2 - h * D);
    }
  }
  *reinterpret_cast<uint4*>(dst) = pack8(y);
}

// SwiGLU epilogue for output columns [j, j+8) of row m.
__device__ __forceinline__ void store_swiglu8(const OpParams& p, int m, int j, const float (&gate)[8],
                                              const float (&up)[8], float scale) {
  float g[8], u[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    g[e] = gate[e] * scale;
    u[e] = up[e] * scale;
  }
  if (p.bias != nullptr) {
    float bg[8], bu[8];
    unpack8(ldg16(p.bias + j), bg);
    unpack8(ldg16(p.bias + p.I + j), bu);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      g[e] += bg[e];
      u[e] += bu[e];
    }
  }
  float y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = silu_f(g[e]) * u[e];
  *reinterpret_cast<uint4*>(p.out + static_cast<size_t>(m) * p.I + j) = pack8(y);
}

}  // namespace fnl
