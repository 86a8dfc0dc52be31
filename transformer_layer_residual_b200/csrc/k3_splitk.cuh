// K3: small-M (decode) fused norm + GEMM + epilogue, split-K over all SMs.
//
// With M <= 128 tokens the op is bound by streaming W from HBM once. The
// product is computed transposed ("swap AB"): the W tile is the UMMA M=128
// operand and the (padded) tokens are the N operand, so a tcgen05.mma
// M=128 x N=mpad x K=16 does useful work even for one token. Work units are
// (128-row W tile, 64-wide k-block) pairs, in one of two forms:
// - stream-K: the units are split evenly over the grid, CTA g taking
//   [g*U/G, (g+1)*U/G), cut at tile boundaries into segments. Each segment's
//   fp32 partial goes to a workspace slot; an arrival counter per tile (one
//   acquire-release atomic per segment) elects the last-arriving CTA, which
//   sums the slots in slot order (deterministic), applies the deferred RMSNorm
//   scale and the epilogue, and resets the counter. A CTA's last segment is
//   summed by all its warps from shared memory, after bulk copies of the slots.
// - cluster: one W tile per cluster of cls CTAs, CTA r taking k-blocks
//   [r nkb / cls, (r+1) nkb / cls); partials stay in shared memory and each CTA
//   sums its share of the tile over distributed shared memory, in rank order,
//   between two cluster barriers. Used when the clusters fill the GPU.
// Nothing spins on another CTA except the cluster barriers, which every thread
// of every CTA reaches after its role loop.
//
// Warp roles (10 warps): 0 TMA producer (W tile + x/residual tiles), 1 TMEM
// owner and UMMA issuer, 2-5 epilogue / split-K reduction (and, for RMSNorm,
// residual_out while the main loop runs), 6-9 converters (normalised bf16
// operand built in place in shared memory, as in K2).
//
// Each stage has two barriers: full_w (the W tile, from HBM) and full_x (the
// x / residual tiles and the gamma / beta / bias_in slices, from L2), so the
// converters start on a stage as soon as its activations land instead of
// waiting for its weights. The kernel is launched as a programmatic dependent
// of the previous kernel on the stream, so its CTAs are resident and set up
// (barriers, TMEM, tensor maps) when that kernel completes; every global access
// except the tensor-map prefetch comes after griddepcontrol.wait.
#pragma once

#include "common.cuh"

namespace fnl {
namespace k3 {

constexpr int BW = 128;   // W rows per tile (UMMA M)
constexpr int BK = 64;
constexpr int MAX_STAGES = 8;        // bf16 forms
constexpr int MAX_STAGES_FP8 = 16;   // FP8 form: 8 KB weight stages, so twice as many for the same bytes in flight
constexpr int RING = MAX_STAGES_FP8;
constexpr int W_BYTES = BW * BK * 2;   // 16 KB
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_EPI0 = 2, NUM_EPI_WARPS = 4;
constexpr int WARP_CONV0 = 6, NUM_CONV_WARPS = 4;
constexpr int NUM_THREADS = (WARP_CONV0 + NUM_CONV_WARPS) * 32;   // 320
constexpr int MAX_MPAD = 128;
// Weight stages fetched before griddepcontrol.wait. Zero: back to back, the
// previous call's tail (partial-sum stores, arrival atomics, the last CTA's
// reduction) is a chain of dependent L2 round trips, and weight traffic issued
// during it lengthens the chain by more than it saves (decode 32 x 6144 x 4096:
// 18.7 us per call with 8 stages, 18.2 with 2, 17.7 with none).
constexpr int PREWAIT_STAGES = 0;
// The FP8 form's predecessor is always its own light pre-pass (one CTA per
// token), so its whole first ring of weight stages streams before the wait.
constexpr int PREWAIT_STAGES_FP8 = MAX_STAGES_FP8;

struct Ctrl {
  uint64_t full_w[RING], full_x[RING], conv[RING], empty[RING];
  uint64_t tfull[2], tempty[2], sfull[2], drain, esync, rbar;
  long long u0, u1;   // this CTA's unit range
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int fin_go, fin_t, fin_nseg;   // the CTA's last segment completes its tile: reduced by all warps
  float ssw[2][NUM_CONV_WARPS][MAX_MPAD];   // per converter warp partial sums of h^2 (RMSNorm)
  float css[MAX_MPAD];                      // cluster form: this CTA's sum of h^2 per token
};

__host__ __device__ inline int stage_bytes(int mpad) { return W_BYTES + 2 * mpad * BK * 2; }
// FP8 form: the W tile is 128 rows x 64 e4m3 (8 KB, 64-byte swizzle) and the
// activation operand [mpad][64] e4m3 codes (64-byte swizzle), both as loaded:
// the pre-pass has quantised each token's row once, so no W tile re-does it.
constexpr int W8_BYTES = BW * BK;   // 8 KB
__host__ __device__ inline int stage_bytes8(int mpad) { return W8_BYTES + mpad * BK; }
constexpr int VEC_BYTES = MAX_STAGES * kVecStageBytes;   // 3 KB (the bf16 forms' gamma / beta / bias_in slices)
__host__ __device__ inline int smem_bytes(int mpad, int stages, bool fp8 = false) {
  return stages * (fp8 ? stage_bytes8(mpad) : stage_bytes(mpad)) + VEC_BYTES + static_cast<int>(sizeof(Ctrl)) + 1024;
}
__host__ __device__ inline uint32_t tmem_cols(int mpad) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(2 * mpad)) c <<= 1;
  return c;
}
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > FNL_WAIT_NS) return false;
  }
  return true;
}

// Iterates this CTA's segments: (tile, first k-block, k-block count, slot, #segments of the tile).
struct SegIter {
  long long u, u1, U;
  int G, g, nkb;
  __device__ SegIter(long long u0_, long long u1_, long long U_, int nkb_, int G_, int g_)
      : u(u0_), u1(u1_), U(U_), G(G_), g(g_), nkb(nkb_) {}
  __device__ bool next(int& t, int& kb0, int& nk, int& slot, int& nseg) {
    if (u >= u1) return false;
    t = static_cast<int>(u / nkb);
    kb0 = static_cast<int>(u - static_cast<long long>(t) * nkb);
    const long long tile_end = static_cast<long long>(t + 1) * nkb;
    const long long e = tile_end < u1 ? tile_end : u1;
    nk = static_cast<int>(e - u);
    const int first = unit_owner_fast(static_cast<long long>(t) * nkb, G, U);
    const int last = unit_owner_fast(tile_end - 1, G, U);
    slot = g - first;
    nseg = last - first + 1;
    u = e;
    return true;
  }
};

}  // namespace k3

// Last-arriving CTA of tile t: out = epilogue(sum over slots 0..nseg-1 of the
// fp32 partials), summed in slot order so the result does not depend on which
// CTA arrives last. Run by NT threads (et = 0..NT-1): the epilogue warps for a
// tile that is not the CTA's last, the whole CTA for its last one (nothing else
// is left to do then). Each thread takes ITEMS (row, 8-column) items at a time and
// issues the loads of up to 4 slots of all of them before adding, so the
// reduction costs about one L2 round trip per 4 slots instead of one per slot.
template <int EPI, int NORM, int NT>
__device__ __forceinline__ void k3_reduce_tile(const OpParams& p, int t, int nseg, int et) {
  using namespace k3;
  constexpr int ITEMS = (EPI == kEpiSwiGLU) ? 1 : 2;
  const int mpad = p.mpad;
  const size_t slot_stride = static_cast<size_t>(mpad) * BW;
  const float* tp = p.part + static_cast<size_t>(t) * p.max_seg * slot_stride;
  const float* tss = p.part_ss + static_cast<size_t>(t) * p.max_seg * mpad;
  const int G8 = (EPI == kEpiSwiGLU) ? 8 : 16;
  const int n_items = p.M * G8;
  for (int it0 = et; it0 < n_items; it0 += ITEMS * NT) {
    float acc[ITEMS][8], up[ITEMS][8], ssum[ITEMS];
    int mi[ITEMS], gi[ITEMS];
    bool ok[ITEMS];
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int item = it0 + q * NT;
      ok[q] = item < n_items;
      mi[q] = ok[q] ? item / G8 : 0;
      gi[q] = ok[q] ? item - mi[q] * G8 : 0;
      ssum[q] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[q][e] = up[q][e] = 0.f;
    }
    for (int base = 0; base < nseg; base += 4) {
      float4 va[ITEMS][4][2], vu[ITEMS][4][2];
      float vs[ITEMS][4];
#pragma unroll
      for (int q = 0; q < ITEMS; ++q) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int sl = base + j;
          if (ok[q] && sl < nseg) {
            const float* row = tp + sl * slot_stride + static_cast<size_t>(mi[q]) * BW + gi[q] * 8;
            va[q][j][0] = __ldcg(reinterpret_cast<const float4*>(row));
            va[q][j][1] = __ldcg(reinterpret_cast<const float4*>(row + 4));
            if (EPI == kEpiSwiGLU) {
              vu[q][j][0] = __ldcg(reinterpret_cast<const float4*>(row + 64));
              vu[q][j][1] = __ldcg(reinterpret_cast<const float4*>(row + 68));
            }
            if (NORM == kRMSNorm) vs[q][j] = __ldcg(tss + static_cast<size_t>(sl) * mpad + mi[q]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < ITEMS; ++q) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (ok[q] && base + j < nseg) {
            acc[q][0] += va[q][j][0].x; acc[q][1] += va[q][j][0].y; acc[q][2] += va[q][j][0].z; acc[q][3] += va[q][j][0].w;
            acc[q][4] += va[q][j][1].x; acc[q][5] += va[q][j][1].y; acc[q][6] += va[q][j][1].z; acc[q][7] += va[q][j][1].w;
            if (EPI == kEpiSwiGLU) {
              up[q][0] += vu[q][j][0].x; up[q][1] += vu[q][j][0].y; up[q][2] += vu[q][j][0].z; up[q][3] += vu[q][j][0].w;
              up[q][4] += vu[q][j][1].x; up[q][5] += vu[q][j][1].y; up[q][6] += vu[q][j][1].z; up[q][7] += vu[q][j][1].w;
            }
            if (NORM == kRMSNorm) ssum[q] += vs[q][j];
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      if (!ok[q]) continue;
      const int m = mi[q], g = gi[q];
      float scale = 1.f;
      if (NORM == kRMSNorm) {
        scale = 1.f / sqrtf(ssum[q] / static_cast<float>(p.K) + p.eps);
        if (t == 0 && g == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
      }
      if (EPI == kEpiSwiGLU) {
        const int j = t * 64 + g * 8;
        if (j < p.I) store_swiglu8(p, m, j, acc[q], up[q], scale);
      } else {
        const int n = t * BW + g * 8;
        if (n < p.N) store_out8<EPI>(p, m, n, acc[q], scale);
      }
    }
  }
}

// The last segment's tile reduced from shared memory: slot sl's rows [0, M) of
// partial sums at part + sl M 128 (fp32 [M][128]), its sum(h^2) per token at
// ss + sl mpad; summed in slot order like k3_reduce_tile. All the CTA's threads.
template <int EPI, int NORM>
__device__ __forceinline__ void k3_reduce_tile_smem(const OpParams& p, int t, int nseg, const float* part,
                                                    const float* ss) {
  using namespace k3;
  const int G8 = (EPI == kEpiSwiGLU) ? 8 : 16;
  const int n_items = p.M * G8;
  const int slot = p.M * BW;
  for (int item = threadIdx.x; item < n_items; item += NUM_THREADS) {
    const int m = item / G8, g = item - m * G8;
    const uint32_t base = smem_u32(part + m * BW + g * 8);
    float acc[8], up[8], ssum = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = up[e] = 0.f;
    for (int sl = 0; sl < nseg; ++sl) {
      const uint32_t a = base + static_cast<uint32_t>(sl * slot) * 4;
      const uint4 v0 = ld_shared_v4(a), v1 = ld_shared_v4(a + 16);
      acc[0] += __uint_as_float(v0.x); acc[1] += __uint_as_float(v0.y);
      acc[2] += __uint_as_float(v0.z); acc[3] += __uint_as_float(v0.w);
      acc[4] += __uint_as_float(v1.x); acc[5] += __uint_as_float(v1.y);
      acc[6] += __uint_as_float(v1.z); acc[7] += __uint_as_float(v1.w);
      if (EPI == kEpiSwiGLU) {   // the up rows are rows 64..127 of the tile
        const uint4 u0 = ld_shared_v4(a + 256), u1 = ld_shared_v4(a + 272);
        up[0] += __uint_as_float(u0.x); up[1] += __uint_as_float(u0.y);
        up[2] += __uint_as_float(u0.z); up[3] += __uint_as_float(u0.w);
        up[4] += __uint_as_float(u1.x); up[5] += __uint_as_float(u1.y);
        up[6] += __uint_as_float(u1.z); up[7] += __uint_as_float(u1.w);
      }
      if (NORM == kRMSNorm) ssum += ss[sl * p.mpad + m];
    }
    float scale = 1.f;
    if (NORM == kRMSNorm) {
      scale = 1.f / sqrtf(ssum / static_cast<float>(p.K) + p.eps);
      if (t == 0 && g == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
    }
    if (EPI == kEpiSwiGLU) {
      const int j = t * 64 + g * 8;
      if (j < p.I) store_swiglu8(p, m, j, acc, up, scale);
    } else {
      const int n = t * BW + g * 8;
      if (n < p.N) store_out8<EPI>(p, m, n, acc, scale);
    }
  }
}

// Cluster form of the small-M kernel: CTA r of the cluster (rank order 0..cls-1)
// sums items [r n / cls, (r + 1) n / cls) of the tile's n (row, 8-column) items
// over the partial sums that the cluster's CTAs hold in shared memory, in rank
// order (the same sum on every run), and runs the epilogue on them.
template <int EPI, int NORM>
__device__ __forceinline__ void k3_cluster_reduce(const OpParams& p, uint32_t part_local, uint32_t css_local, int t,
                                                  int r, int cls) {
  using namespace k3;
  const int G8 = (EPI == kEpiSwiGLU) ? 8 : 16;
  const int n_items = p.M * G8;
  const int i1 = (r + 1) * n_items / cls;
  for (int item = r * n_items / cls + static_cast<int>(threadIdx.x); item < i1; item += NUM_THREADS) {
    const int m = item / G8, g = item - m * G8;
    const uint32_t off = static_cast<uint32_t>(m * BW + g * 8) * 4;
    float acc[8], up[8], ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = up[e] = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < cls) {
        const uint32_t a = dsmem_addr(part_local + off, q);
        const float4 v0 = ld_dsmem_f4(a), v1 = ld_dsmem_f4(a + 16);
        acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
        acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
        if (EPI == kEpiSwiGLU) {   // the up rows are rows 64..127 of the tile
          const float4 u0 = ld_dsmem_f4(a + 256), u1 = ld_dsmem_f4(a + 272);
          up[0] += u0.x; up[1] += u0.y; up[2] += u0.z; up[3] += u0.w;
          up[4] += u1.x; up[5] += u1.y; up[6] += u1.z; up[7] += u1.w;
        }
        if (NORM == kRMSNorm) ss += ld_dsmem_f32(dsmem_addr(css_local + m * 4, q));
      }
    }
    float scale = 1.f;
    if (NORM == kRMSNorm) {
      scale = 1.f / sqrtf(ss / static_cast<float>(p.K) + p.eps);
      if (t == 0 && g == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
    }
    if (EPI == kEpiSwiGLU) {
      const int j = t * 64 + g * 8;
      if (j < p.I) store_swiglu8(p, m, j, acc, up, scale);
    } else {
      const int n = t * BW + g * 8;
      if (n < p.N) store_out8<EPI>(p, m, n, acc, scale);
    }
  }
}

// FP8 (e4m3 weights and activations, kind::f8f6f4 UMMA): the pre-pass has
// normalised and quantised each token's row once (e4m3 codes [M][K] in the
// workspace, tm_x maps them), so the codes tile is the UMMA's B operand as
// loaded and the converter warps have nothing to do; the epilogue multiplies by
// s_a[m] s_w[n] (p.stats8, p.w_scale). Instantiated with NORM = kLayerNorm.
template <int EPI, int NORM, bool SPLIT, bool FP8 = false>
__global__ void __launch_bounds__(k3::NUM_THREADS, 1)
    k3_splitk_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                     const __grid_constant__ CUtensorMap tm_w, const OpParams p) {
  using namespace k3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int mpad = p.mpad, S = p.stages;
  const int SB = FP8 ? stage_bytes8(mpad) : stage_bytes(mpad);
  const int WB = FP8 ? W8_BYTES : W_BYTES;   // x tile offset within a stage
  // the activation tile is the UMMA operand as loaded: no norm (residual-stream
  // projection), or the FP8 form's pre-quantised codes
  constexpr bool DIRECT = NORM == kNoNorm || FP8;
  const int XB = mpad * BK * 2;
  bf16* vecs = reinterpret_cast<bf16*>(smem + S * SB);   // [S][3][64]
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + S * SB + VEC_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_beta = NORM == kLayerNorm && p.beta != nullptr;
  const bool has_bias_in = EPI == kEpiGELU && p.bias_in != nullptr;   // only the GELU entry point has one

  const int M = p.M, K = p.K;
  const int T = (EPI == kEpiSwiGLU) ? (p.I + 63) / 64 : (p.N + BW - 1) / BW;
  const int nkb = (K + BK - 1) / BK;
  const uint32_t ncols = tmem_cols(mpad);
  const bool cl = p.cls > 0;
  constexpr bool BIAS_IN = EPI == kEpiGELU;   // only the GELU entry point has a bias_in

  const long long U = static_cast<long long>(T) * nkb;
  if (threadIdx.x == 0) {
    pdl_launch_dependents();   // the next call's CTAs may take SMs as ours retire
    if (p.cls > 0) {   // cluster form: CTA r of cluster t takes k-blocks [r nkb / cls, (r + 1) nkb / cls) of tile t
      const long long t0 = blockIdx.x / p.cls, r = blockIdx.x % p.cls;
      ctrl->u0 = t0 * nkb + r * nkb / p.cls;
      ctrl->u1 = t0 * nkb + (r + 1) * nkb / p.cls;
    } else {
      ctrl->u0 = static_cast<long long>(blockIdx.x) * U / gridDim.x;
      ctrl->u1 = static_cast<long long>(blockIdx.x + 1) * U / gridDim.x;
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&ctrl->full_w[s], 1);
      mbar_init(&ctrl->full_x[s], 1);
      mbar_init(&ctrl->conv[s], 1);   // one converter warp per stage
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], NUM_EPI_WARPS);
      mbar_init(&ctrl->sfull[b], NUM_CONV_WARPS);
    }
    mbar_init(&ctrl->drain, 1);
    mbar_init(&ctrl->esync, NUM_EPI_WARPS);
    mbar_init(&ctrl->rbar, 1);
    ctrl->abort_flag = 0;
    ctrl->last_flag = 0;
    ctrl->fin_go = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_r);
    prefetch_tmap(&tm_w);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&ctrl->tmem_base, ncols);
    tmem_relinquish();
  }
  if (!DIRECT) zero_vec_slices(vecs, S * 3 * kVecElems);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int* abortf = &ctrl->abort_flag;
  const long long u0 = ctrl->u0, u1 = ctrl->u1;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int P = static_cast<int>(u1 - u0);   // positions (units) of this CTA
      const int npre = P < S ? P : S;
      uint32_t armed_w = 0, armed_x = 0, par_w = 0, par_x = 0;
      bool ok = true;
      // fault injection (status-path tests only): CTA 0 withholds its first weight copy
      bool withhold = p.stall != 0 && blockIdx.x == 0;
      const uint64_t pol_w = policy_evict_first();   // W is streamed exactly once
      // two cursors over the unit sequence (tile t, k-block kb, stage s, parity)
      struct Cur {
        int t, kb, s;
        uint32_t ph;
      };
      const int t0 = static_cast<int>(u0 / nkb);
      Cur cw{t0, static_cast<int>(u0 - static_cast<long long>(t0) * nkb), 0, 0u};
      Cur cx = cw;
      auto step = [&](Cur& c) {
        if (++c.kb == nkb) {
          c.kb = 0;
          ++c.t;
        }
        if (++c.s == S) {
          c.s = 0;
          c.ph ^= 1u;
        }
      };
      auto issue_w = [&](const Cur& c) {
        if (withhold) {
          withhold = false;
          return;
        }
        uint8_t* st = smem + c.s * SB;
        mbar_arrive_expect_tx(&ctrl->full_w[c.s], WB);
        if (EPI == kEpiSwiGLU) {
          tma_load_2d_hint(st, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.t * 64, pol_w);
          tma_load_2d_hint(st + WB / 2, &tm_w, &ctrl->full_w[c.s], c.kb * BK, p.I + c.t * 64, pol_w);
        } else {
          tma_load_2d_hint(st, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.t * BW, pol_w);
        }
        armed_w |= 1u << c.s;
        par_w = (par_w & ~(1u << c.s)) | (c.ph << c.s);
      };
      auto issue_x = [&](const Cur& c) {
        uint8_t* st = smem + c.s * SB;
        if (DIRECT) {   // the activation tile is the operand as loaded
          mbar_arrive_expect_tx(&ctrl->full_x[c.s], FP8 ? mpad * BK : XB);
          tma_load_2d(st + WB, &tm_x, &ctrl->full_x[c.s], c.kb * BK, 0);
          armed_x |= 1u << c.s;
          par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
          return;
        }
        mbar_arrive_expect_tx(&ctrl->full_x[c.s], 2 * XB + vec_bytes(p, has_beta, has_bias_in, c.kb));
        issue_vec_loads(p, has_beta, has_bias_in, c.kb, vecs + c.s * 3 * kVecElems, &ctrl->full_x[c.s]);
        tma_load_2d(st + WB, &tm_x, &ctrl->full_x[c.s], c.kb * BK, 0);
        tma_load_2d(st + WB + XB, &tm_r, &ctrl->full_x[c.s], c.kb * BK, 0);
        armed_x |= 1u << c.s;
        par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
      };
      // Weight stages that may stream before griddepcontrol.wait (weights are
      // never written by the previous kernel; activations are read only after it).
      constexpr int kPre = FP8 ? PREWAIT_STAGES_FP8 : PREWAIT_STAGES;
      const int npre0 = npre < kPre ? npre : kPre;
      for (int q = 0; q < npre0; ++q) {
        issue_w(cw);
        step(cw);
      }
      pdl_wait();
      for (int q = 0; q < P; ++q) {
        if (q >= npre0 && q < npre) {   // the rest of the first ring
          issue_w(cw);
          step(cw);
        } else if (q >= npre) {
          if (!mbar_wait(&ctrl->empty[cw.s], cw.ph ^ 1, abortf, p.status, kStatusWaitEmpty, p.wait_ns)) {
            ok = false;
            break;
          }
          issue_w(cw);
          step(cw);
        }
        issue_x(cx);
        step(cx);
      }
      if (!ok) {   // let every issued copy land before the CTA can exit
        for (int i = 0; i < S; ++i) {
          if (armed_w & (1u << i)) drain_wait(&ctrl->full_w[i], (par_w >> i) & 1);
          if (armed_x & (1u << i)) drain_wait(&ctrl->full_x[i], (par_x >> i) & 1);
        }
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      SegIter it(u0, u1, U, nkb, gridDim.x, blockIdx.x);
      int t, kb0, nk, slot, nseg;
      uint32_t s = 0, ph = 0;
      bool ok = true;
      const uint32_t idesc = FP8 ? idesc_e4m3(BW, mpad) : idesc_bf16(BW, mpad);
      int i = 0;
      while (ok && it.next(t, kb0, nk, slot, nseg)) {
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!mbar_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * mpad;
        for (int kb = 0; kb < nk; ++kb) {
          // the converted operand (or, without a norm, the activation tile as loaded)
          uint64_t* ready = DIRECT ? &ctrl->full_x[s] : &ctrl->conv[s];
          if (!mbar_wait(ready, ph, abortf, p.status, kStatusWaitConv, p.wait_ns) ||
              !mbar_wait(&ctrl->full_w[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(smem + s * SB);
          if (FP8) {   // 64 e4m3 per row: two K = 32 steps of 32 bytes
            const uint64_t ad = sw64_desc(wa);
            const uint64_t bd = sw64_desc(wa + WB);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              umma_f8(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          } else {
            const uint64_t ad = sw128_desc(wa);
            const uint64_t bd = sw128_desc(wa + WB);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
            if (SPLIT) {
              const uint64_t ld = sw128_desc(wa + WB + XB);
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) umma_bf16(d, ad + 2 * kk, ld + 2 * kk, idesc, 1u);
            }
          }
          umma_commit(&ctrl->empty[s]);
          if (++s == static_cast<uint32_t>(S)) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&ctrl->tfull[b]);
        ++i;
      }
      umma_commit(&ctrl->drain);
      drain_wait(&ctrl->drain, 0);
    }
  } else if (warp < WARP_CONV0) {
    // ------------------------------------------------------------ epilogue + split-K reduction
    const int q = warp & 3;
    const int et = threadIdx.x - WARP_EPI0 * 32;   // 0..127
    const int nl = q * 32 + lane;                  // W row within the tile = TMEM lane
    pdl_wait();   // workspace and outputs may still be in use by the previous kernel
    if (NORM == kRMSNorm) {
      // residual_out = bf16(x + r (+ bias_in)), fp32 sum as in the converters:
      // this CTA's share of the M x K/8 16-byte chunks, written while the
      // mainloop runs (LayerNorm's comes from the statistics kernel).
      const int kc = K / 8;
      const long long nch = static_cast<long long>(M) * kc;
      const long long ch1 = nch * (blockIdx.x + 1) / gridDim.x;
      for (long long ch = nch * blockIdx.x / gridDim.x + et; ch < ch1; ch += NUM_EPI_WARPS * 32) {
        const int m = static_cast<int>(ch / kc);
        const int k0 = static_cast<int>(ch - static_cast<long long>(m) * kc) * 8;
        const size_t off = static_cast<size_t>(m) * K + k0;
        const uint4 xv = ldg16(p.x_in + off), rv = ldg16(p.r_in + off);
        const uint4 bv = (BIAS_IN && p.bias_in != nullptr) ? ldg16(p.bias_in + k0) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, rw[4] = {rv.x, rv.y, rv.z, rv.w};
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
        uint32_t hw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f32x2 h = add2(bf2_to_f2(xw[e]), bf2_to_f2(rw[e]));
          if (BIAS_IN) h = add2(h, bf2_to_f2(bw[e]));
          hw[e] = f2_to_bf2(h);
        }
        if (store_in_bounds(p, p.residual_out + off, p.residual_out, static_cast<size_t>(p.M) * p.K))
          *reinterpret_cast<uint4*>(p.residual_out + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
    }
    SegIter it(u0, u1, U, nkb, gridDim.x, blockIdx.x);
    int t, kb0, nk, slot, nseg;
    int i = 0;
    uint32_t eph = 0;
    while (it.next(t, kb0, nk, slot, nseg)) {
      const int b = i & 1;
      const uint32_t use = static_cast<uint32_t>(i >> 1);
      if (!warp_wait(&ctrl->tfull[b], use & 1, abortf, p.status, kStatusWaitTmemFull, p.wait_ns)) break;
      if (NORM == kRMSNorm) {
        if (!warp_wait(&ctrl->sfull[b], use & 1, abortf, p.status, kStatusWaitStats, p.wait_ns)) break;
      }
      tc_fence_after();
      // stream-K form: the partial goes to the tile's workspace slot; cluster
      // form: to this CTA's own shared memory (the stage buffers, all consumed
      // once the last UMMA has completed), [mpad][128] fp32
      const size_t base = static_cast<size_t>(t) * p.max_seg + slot;
      float* part = cl ? reinterpret_cast<float*>(smem) : p.part + base * mpad * BW;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * mpad;
      for (int mc = 0; mc < mpad; mc += 16) {
        uint32_t v[16];
        tmem_ld16(tbase + mc, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (mc + e < M) part[static_cast<size_t>(mc + e) * BW + nl] = __uint_as_float(v[e]);
      }
      if (NORM == kRMSNorm && et < M) {
        float ssum = 0.f;
#pragma unroll
        for (int w = 0; w < NUM_CONV_WARPS; ++w) ssum += ctrl->ssw[b][w][et];   // fixed order
        if (cl) ctrl->css[et] = ssum;
        else p.part_ss[base * mpad + et] = ssum;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->tempty[b]);
      ++i;
      if (cl) continue;   // the cluster sums its tile after the role loops

      // arrival: the last CTA of this tile reduces all slots in slot order.
      // The epilogue warps meet on an mbarrier (bounded wait), not bar.sync,
      // so a warp that gave up a wait can never leave the others blocked.
      // Ordering needs no fence of its own: the mbarrier orders this CTA's
      // slot stores before thread et 0's arrival, whose acquire-release atomic
      // publishes them at GPU scope (release is cumulative over what the
      // barrier ordered before it) and, for the last arrival, makes the other
      // CTAs' slots visible (acquire); the next barrier passes that on to the
      // threads that read the slots (L2 loads).
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->esync);
      if (!warp_wait(&ctrl->esync, eph, abortf, p.status, kStatusWaitDrain, p.wait_ns)) break;
      eph ^= 1;
      if (et == 0) {
        const unsigned old = atom_add_acq_rel_gpu(&p.counters[t], 1u);
        ctrl->last_flag = (old == static_cast<unsigned>(nseg - 1)) ? 1 : 0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->esync);
      if (!warp_wait(&ctrl->esync, eph, abortf, p.status, kStatusWaitDrain, p.wait_ns)) break;
      eph ^= 1;
      if (ctrl->last_flag) {
        if (it.u >= it.u1) {   // the CTA's last segment: handed to all warps below
          if (et == 0) {
            ctrl->fin_t = t;
            ctrl->fin_nseg = nseg;
            ctrl->fin_go = 1;
          }
        } else {
          k3_reduce_tile<EPI, NORM, NUM_EPI_WARPS * 32>(p, t, nseg, et);
          if (et == 0) p.counters[t] = 0u;
        }
      }
    }
  } else if (!DIRECT) {
    // ------------------------------------------------------------ converters
    // Converter warp cw owns pipeline positions cw, cw + 4, cw + 8, ... of this
    // CTA's unit sequence, so up to four stages are converted at once. Lanes
    // are split into groups of L lanes per token row (L = 8 for M <= 4 down to
    // 1 for M > 16): lane = (row slot, first chunk); a lane walks chunks
    // cf, cf + L, ... of rows rb, rb + 32/L, ... (< M; padding rows keep the
    // zeros TMA filled in, a valid operand whose columns are never read).
    // sum(h^2) stays in registers and is reduced over the L lanes once per segment.
    const int cw = warp - WARP_CONV0;
    const int L = M <= 4 ? 8 : (M <= 8 ? 4 : (M <= 16 ? 2 : 1));
    const int rpp = 32 / L;              // rows per pass of the warp
    const int rb = lane / L, cf = lane - rb * L;
    const int npass = (M + rpp - 1) / rpp;   // 1..4
    const int cpl = 8 / L;                   // chunks per lane per row
    float mu[4], rs[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) mu[j] = rs[j] = 0.f;
    if (NORM == kLayerNorm) {
      pdl_wait();   // statistics come from the previous kernel
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = rb + rpp * j;
        if (j < npass && row < M) {
          const float2 st = p.stats[row];
          mu[j] = st.x;
          rs[j] = st.y;
        }
      }
    }
    SegIter it(u0, u1, U, nkb, gridDim.x, blockIdx.x);
    int t, kb0, nk, slot, nseg;
    int pos = 0;   // first position of the current segment
    int i = 0;     // segment index
    int cq = cw, cs = cw;   // this warp's next position and its stage (S >= NUM_CONV_WARPS)
    uint32_t cph = 0;
    bool ok = true;
    while (ok && it.next(t, kb0, nk, slot, nseg)) {
      const int b = i & 1;
      f32x2 sq[4] = {0ull, 0ull, 0ull, 0ull};   // this warp's share of the segment's sum(h^2) per row
      for (; cq < pos + nk; cq += NUM_CONV_WARPS) {
        const int q = cq;
        const int s = cs;
        const uint32_t ph = cph;
        cs += NUM_CONV_WARPS;
        if (cs >= S) {
          cs -= S;
          cph ^= 1u;
        }
        const int kb = kb0 + (q - pos);
        if (!warp_wait(&ctrl->full_x[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint32_t xs = smem_u32(smem + s * SB) + W_BYTES;
        const uint32_t rsm = xs + XB;
        bf16* vec = vecs + s * 3 * kVecElems;
        if (K - kb * BK < BK) zero_vec_tails(vec, kVecElems, K - kb * BK);
        const uint32_t vaddr = smem_u32(vec);
        // For each row slot j of this lane, the lane's chunks of that row in
        // batches of 4: all shared-memory loads of a batch are issued before its
        // arithmetic and stores, so chunks overlap instead of running in series.
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = rb + rpp * j;
          if (j < npass && row < M) {
            for (int c0 = 0; c0 < cpl; c0 += 4) {
              uint4 xv[4], rv[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                if (c0 + u < cpl) {
                  const int c = cf + L * (c0 + u);
                  const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
                  xv[u] = ld_shared_v4(xs + off);
                  rv[u] = ld_shared_v4(rsm + off);
                }
              }
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                if (c0 + u < cpl) {
                  const int c = cf + L * (c0 + u);
                  const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
                  f32x2 g2[4], be2[4] = {}, bi2[4] = {};
                  vec_pairs(vaddr + c * 16, g2);
                  if (NORM == kLayerNorm) vec_pairs(vaddr + 2 * kVecElems + c * 16, be2);
                  if (BIAS_IN) vec_pairs(vaddr + 4 * kVecElems + c * 16, bi2);
                  uint4 hi, lo, hres;
                  convert8<NORM, BIAS_IN, SPLIT, false>(xv[u], rv[u], g2, be2, bi2, mu[j], rs[j], sq[j], hi, lo, hres);
                  st_shared_v4(xs + off, hi);
                  if (SPLIT) st_shared_v4(rsm + off, lo);
                }
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->conv[s]);
      }
      if (!ok) break;
      if (NORM == kRMSNorm) {
        // publish this warp's share once the epilogue has read the segment
        // that used this buffer two segments ago
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!warp_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty, p.wait_ns)) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float lo_, hi_;
          unpk2(sq[j], lo_, hi_);
          float t = lo_ + hi_;
          for (int o = 1; o < L; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
          const int row = rb + rpp * j;
          if (cf == 0 && j < npass && row < M) ctrl->ssw[b][cw][row] = t;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull[b]);
      }
      pos += nk;
      ++i;
    }
  }

  // Every role's loop is over (each bounded wait returns), so all warps meet
  // here; the tile completed by this CTA's last segment is summed by all of them.
  __syncthreads();
  if (cl) {
    // Cluster form: every CTA of the cluster holds its partial sums of the
    // cluster's tile in its shared memory; each sums its share of the tile's
    // items over the cluster (distributed shared memory, rank order).
    cluster_sync();
    if (*abortf == 0)
      k3_cluster_reduce<EPI, NORM>(p, smem_u32(smem), smem_u32(ctrl->css), blockIdx.x / p.cls, blockIdx.x % p.cls,
                                   p.cls);
    cluster_sync();   // no CTA leaves while the others still read its shared memory
  } else if (ctrl->fin_go && *abortf == 0) {
    // The tile's slots are bulk-copied into the (idle) stage buffers and summed
    // there: one deep stream of copies instead of every thread's scattered L2
    // loads. Falls back to direct loads when they do not fit.
    const int t = ctrl->fin_t, nseg = ctrl->fin_nseg;
    const uint32_t slot_bytes = static_cast<uint32_t>(M) * BW * 4;
    const uint32_t ss_bytes = NORM == kRMSNorm ? static_cast<uint32_t>(mpad) * 4 : 0u;
    if (static_cast<long long>(nseg) * (slot_bytes + ss_bytes) <= static_cast<long long>(S) * SB) {
      if (threadIdx.x == 0) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&ctrl->rbar, static_cast<uint32_t>(nseg) * (slot_bytes + ss_bytes));
        const size_t slot_stride = static_cast<size_t>(mpad) * BW;
        const float* tp = p.part + static_cast<size_t>(t) * p.max_seg * slot_stride;
        const float* tss = p.part_ss + static_cast<size_t>(t) * p.max_seg * mpad;
        for (int sl = 0; sl < nseg; ++sl) {
          bulk_load(smem + sl * slot_bytes, tp + sl * slot_stride, slot_bytes, &ctrl->rbar);
          if (NORM == kRMSNorm)
            bulk_load(smem + nseg * slot_bytes + sl * ss_bytes, tss + static_cast<size_t>(sl) * mpad, ss_bytes,
                      &ctrl->rbar);
        }
      }
      if (warp_wait(&ctrl->rbar, 0, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
        k3_reduce_tile_smem<EPI, NORM>(p, t, nseg, reinterpret_cast<const float*>(smem),
                                       reinterpret_cast<const float*>(smem + nseg * slot_bytes));
      } else if (threadIdx.x == 0) {
        drain_wait(&ctrl->rbar, 0);   // the copies land before the CTA can exit
      }
    } else {
      k3_reduce_tile<EPI, NORM, NUM_THREADS>(p, t, nseg, threadIdx.x);
    }
    if (threadIdx.x == 0) p.counters[t] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace fnl
