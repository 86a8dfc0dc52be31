// Parameters and epilogue arithmetic shared by the fused-op kernels.
#pragma once

#include "ptx.cuh"

namespace fnl {

typedef __nv_bfloat16 bf16;

// kEpiResidual with kNoNorm is the residual-stream projection (o_proj /
// down_proj): the activation operand is used as loaded (no add, no norm, no
// converters) and the epilogue adds the residual stream: out = residual + y.
enum Epi : int { kEpiQKV = 0, kEpiSwiGLU = 1, kEpiGELU = 2, kEpiResidual = 3 };
enum Norm : int { kLayerNorm = 0, kRMSNorm = 1, kNoNorm = 2 };

struct OpParams {
  int M, K, N;       // tokens, hidden, rows of W
  int I;             // SwiGLU intermediate size (N = 2I)
  int Hq, Hkv, D;    // QKV heads
  float eps;
  const bf16* x_in;      // x and residual [M][K] (read directly by the small-M kernel's
  const bf16* r_in;      // residual_out writers; the GEMM operands come through tensor maps)
  const bf16* gamma;
  const bf16* beta;      // LayerNorm shift, may be null
  const bf16* bias_in;   // [K], may be null
  const bf16* bias;      // [N] output bias, may be null
  bf16* residual_out;    // written in the GEMM kernels for RMSNorm, by the statistics kernel for LayerNorm
  float* rstd_out;       // RMSNorm statistics output (GEMM kernels), may be null
  const float2* stats;   // LayerNorm (mean, rstd) per row, written by the stats kernel
  bf16* q;
  bf16* k;
  bf16* v;
  bf16* out;
  const float4* stats8;  // FP8 ops: per token (mean, rstd, dequantisation scale, 448 / amax), from the pre-pass
  int fp8_rms;           // FP8 ops: 1 = RMSNorm (codes of h * gamma, rstd in the scale), 0 = LayerNorm
  const float* w_scale;  // FP8 ops: per W row dequantisation scale s_w [N] (null for the bf16 ops)
  const bf16* res_in;    // residual-stream projection: the residual [M][N] added in the epilogue
                         // (may be the same buffer as out: each element is read, then written,
                         // by one thread)
  // small-M split-K workspace
  float* part;           // [T][max_seg][mpad][128] fp32 partial accumulators
  float* part_ss;        // [T][max_seg][mpad] partial sums of h^2 (RMSNorm)
  unsigned* counters;    // [T] arrival counters, zero between launches
  int max_seg;
  int mpad;
  int stages;
  int cls;               // small-M kernel: CTAs per cluster (one W tile per cluster), 0 = stream-K form
  int sk;                // 128x256 tile and pair kernels: 1 = stream-K over (tile, k-block) units, 0 = whole tiles
  int sk_full;           // pair kernel, stream-K: tiles [0, sk_full) whole, round robin; the rest split
  int split;             // 1: operand = bf16 hi + bf16 lo (two UMMAs), 0: single bf16 rounding
  int* status;           // device status word (bounded-wait failures)
  unsigned long long wait_ns;   // limit of the main-loop waits (the drain waits keep FNL_WAIT_NS)
  int stall;             // fault injection for the status-path tests: 1 = CTA 0's producer never
                         // issues its first weight copy, so the wait for it runs out (0 = off)
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
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

// Split-K work units (W tile, k-block) dealt evenly over G CTAs: CTA g takes
// units [g U / G, (g + 1) U / G).
// Index of the CTA whose unit range contains unit u (units split as g*U/G).
__host__ __device__ inline int unit_owner(long long u, int G, long long U) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}
// The same in double precision (exact: every operand is an integer below 2^53
// and a quotient that is not an integer is at least 1/U away from one).
__device__ __forceinline__ int unit_owner_fast(long long u, int G, long long U) {
  return static_cast<int>((static_cast<double>(u + 1) * G - 1.0) / static_cast<double>(U));
}

// Compile-time flag for code specialised on a condition that is uniform over a
// stage (a generic lambda takes it as its argument type).
template <bool B>
struct BoolC {
  static constexpr bool value = B;
};

// Set elements [from, n) of the three per-stage vector slices (gamma, beta,
// bias_in; n elements apart) to zero. Called by a converter warp on the last
// k-block when K is not a multiple of the k-block: the slices' loads covered only
// the first K - k0 elements, and with zeros there the columns past K (whose x,
// residual and W entries the tensor copies fill with zeros) give exactly a = 0
// and h = 0, so the chunk loops need no bounds test.
__device__ __forceinline__ void zero_vec_tails(bf16* vec, int n, int from) {
  uint16_t* v = reinterpret_cast<uint16_t*>(vec);
  for (int i = from + static_cast<int>(threadIdx.x & 31); i < n; i += 32) {
    v[i] = 0;
    v[n + i] = 0;
    v[2 * n + i] = 0;
  }
  __syncwarp();
}

// Zero all per-stage vector slices once, before the first copy into them, so a
// slice whose vector the call does not have (beta, bias_in) reads as zeros.
// All threads of the block; the proxy fence orders these stores before the
// tensor-copy engine's later writes to the same words.
__device__ __forceinline__ void zero_vec_slices(bf16* vecs, int elems) {
  uint16_t* v = reinterpret_cast<uint16_t*>(vecs);
  for (int i = threadIdx.x; i < elems; i += blockDim.x) v[i] = 0;
  fence_proxy_async_smem();
}

// 8 consecutive elements of one token row: h = x + r (+ bias_in) in fp32,
// a = normalise(h) rounded to bf16 (hi) and, with SPLIT, the bf16 remainder a - hi
// (lo); with WANT_H also bf16(h) for residual_out.
// LayerNorm: a = (h - mean) * rstd * gamma + beta (beta = 0 when absent).
// RMSNorm (deferred scale): a = h * gamma and sq += h^2 (even and odd elements
// in the two lanes of the pair).
// g, be, bi: the chunk's gamma / beta / bias_in as four fp32 pairs.
// Every choice is a template parameter, so the converter loops carry no
// per-element branches.
template <int NORM, bool BIAS_IN, bool SPLIT, bool WANT_H>
__device__ __forceinline__ void convert8(const uint4& xv, const uint4& rv, const f32x2 (&g)[4], const f32x2 (&be)[4],
                                         const f32x2 (&bi)[4], float mean, float rstd, f32x2& sq, uint4& hi,
                                         uint4& lo, uint4& hres) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
  uint32_t ho[4], lw[4], hw[4];
  const f32x2 mu2 = pk2(mean, mean), rs2 = pk2(rstd, rstd);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f32x2 h = add2(bf2_to_f2(xw[i]), bf2_to_f2(rw[i]));
    if (BIAS_IN) h = add2(h, bi[i]);
    f32x2 a;
    if (NORM == kLayerNorm) {
      a = fma2(mul2(sub2(h, mu2), rs2), g[i], be[i]);
    } else {
      a = mul2(h, g[i]);
      sq = fma2(h, h, sq);
    }
    ho[i] = f2_to_bf2(a);
    if (SPLIT) lw[i] = f2_to_bf2(sub2(a, bf2_to_f2(ho[i])));
    if (WANT_H) hw[i] = f2_to_bf2(h);
  }
  hi = make_uint4(ho[0], ho[1], ho[2], ho[3]);
  if (SPLIT) lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  if (WANT_H) hres = make_uint4(hw[0], hw[1], hw[2], hw[3]);
}

// The 8 bf16 at a 16-byte aligned shared-memory address as four fp32 pairs.
__device__ __forceinline__ void vec_pairs(uint32_t addr, f32x2 (&f)[4]) {
  const uint4 v = ld_shared_v4(addr);
  f[0] = bf2_to_f2(v.x);
  f[1] = bf2_to_f2(v.y);
  f[2] = bf2_to_f2(v.z);
  f[3] = bf2_to_f2(v.w);
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

// 16 bytes from global memory through L2 only (no L1 allocation: read once).
__device__ __forceinline__ uint4 ldcg16(const void* p) {
  return __ldcg(reinterpret_cast<const uint4*>(p));
}

// Store 8 consecutive output columns [n, n+8) of row m (QKV, GELU or residual
// epilogue). acc is the raw fp32 accumulator, scale the deferred RMSNorm 1/rms
// (1 for LN and for the residual-stream projection).
// FP8 ops: the accumulator holds sum of code products; y = acc s_a[m] s_w[n]
// (s_a includes rstd for RMSNorm).
__device__ __forceinline__ void fp8_dequant8(const OpParams& p, int m, int n, float (&y)[8]) {
  const float sa = p.stats8[m].z;
  const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.w_scale + n));
  const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.w_scale + n + 4));
  const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] *= sa * ws[e];
}

// Debug builds (FNL_DEBUG_CHECKS: libfnl_debug.so, built beside libfnl.so) check
// every output store against its buffer: an out-of-range store is skipped and
// the status word records kStatusBounds, which fnl_check reports. It stands in
// for compute-sanitizer on the outputs, where a wrong index would otherwise
// corrupt memory silently. Release builds compile the check away.
__device__ __forceinline__ bool store_in_bounds(const OpParams& p, const bf16* dst, const bf16* base,
                                                size_t elems) {
#ifdef FNL_DEBUG_CHECKS
  if (base == nullptr || dst < base || dst + 8 > base + elems) {
    if (p.status != nullptr) atomicCAS(p.status, 0, kStatusBounds);
    return false;
  }
#endif
  return true;
}

template <int EPI>
__device__ __forceinline__ void store_out8(const OpParams& p, int m, int n, const float (&acc)[8], float scale) {
  float y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = acc[e] * scale;
  if (p.w_scale != nullptr) fp8_dequant8(p, m, n, y);
  if (p.bias != nullptr) {
    float b[8];
    unpack8(ldg16(p.bias + n), b);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] += b[e];
  }
  bf16* dst;
  const bf16* base = p.out;
  size_t elems = static_cast<size_t>(p.M) * p.N;
  if (EPI == kEpiResidual) {
    const size_t off = static_cast<size_t>(m) * p.N + n;
    float r[8];
    unpack8(ldcg16(p.res_in + off), r);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] += r[e];
    dst = p.out + off;
  } else if (EPI == kEpiGELU) {
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
      base = p.q;
      elems = static_cast<size_t>(p.Hq) * p.M * D;
    } else if (n < nk) {
      const int n2 = n - nq, h = n2 / D;
      dst = p.k + (static_cast<size_t>(h) * p.M + m) * D + (n2 - h * D);
      base = p.k;
      elems = static_cast<size_t>(p.Hkv) * p.M * D;
    } else {
      const int n2 = n - nk, h = n2 / D;
      dst = p.v + (static_cast<size_t>(h) * p.M + m) * D + (n2 - h * D);
      base = p.v;
      elems = static_cast<size_t>(p.Hkv) * p.M * D;
    }
  }
  if (!store_in_bounds(p, dst, base, elems)) return;
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
  if (p.w_scale != nullptr) {
    fp8_dequant8(p, m, j, g);
    fp8_dequant8(p, m, p.I + j, u);
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
  bf16* dst = p.out + static_cast<size_t>(m) * p.I + j;
  if (!store_in_bounds(p, dst, p.out, static_cast<size_t>(p.M) * p.I)) return;
  *reinterpret_cast<uint4*>(dst) = pack8(y);
}

}  // namespace fnl
