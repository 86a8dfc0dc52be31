// K3: small-M (decode) fused norm + GEMM + epilogue, stream-K over all SMs.
//
// With M <= 128 tokens the op is bound by streaming W from HBM once. The
// product is computed transposed ("swap AB"): the W tile is the UMMA M=128
// operand and the (padded) tokens are the N operand, so a tcgen05.mma
// M=128 x N=mpad x K=16 does useful work even for one token. The work units
// (128-row W tile, 64-wide k-block) are split evenly over the grid (stream-K):
// CTA g takes units [g*U/G, (g+1)*U/G), cutting at tile boundaries into
// segments. Each segment's fp32 partial goes to a workspace slot; an arrival
// counter per tile elects the last-arriving CTA, which sums the slots in a
// fixed order (deterministic), applies the deferred RMSNorm scale and the
// epilogue, and resets the counter. Nothing spins on another CTA.
//
// Warp roles (10 warps): 0 TMA producer (W tile + x/residual tiles), 1 TMEM
// owner and UMMA issuer, 2-5 epilogue / split-K reduction, 6-9 converters
// (normalised bf16 operand built in place in shared memory, as in K2).
#pragma once

#include "common.cuh"

namespace fnl {
namespace k3 {

constexpr int BW = 128;   // W rows per tile (UMMA M)
constexpr int BK = 64;
constexpr int MAX_STAGES = 8;
constexpr int W_BYTES = BW * BK * 2;   // 16 KB
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_EPI0 = 2, NUM_EPI_WARPS = 4;
constexpr int WARP_CONV0 = 6, NUM_CONV_WARPS = 4;
constexpr int NUM_THREADS = (WARP_CONV0 + NUM_CONV_WARPS) * 32;   // 320
constexpr int MAX_MPAD = 128;

struct Ctrl {
  uint64_t full[MAX_STAGES], conv[MAX_STAGES], empty[MAX_STAGES];
  uint64_t tfull[2], tempty[2], sfull[2], drain, esync;
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  float ss[2][MAX_MPAD];
};

__host__ __device__ inline int stage_bytes(int mpad) { return W_BYTES + 2 * mpad * BK * 2; }
__host__ __device__ inline int smem_bytes(int mpad, int stages) {
  return stages * stage_bytes(mpad) + static_cast<int>(sizeof(Ctrl)) + 1024;
}
__host__ __device__ inline uint32_t tmem_cols(int mpad) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(2 * mpad)) c <<= 1;
  return c;
}
// Index of the CTA whose unit range contains unit u (units split as g*U/G).
__host__ __device__ inline int unit_owner(long long u, int G, long long U) {
  return static_cast<int>(((u + 1) * G - 1) / U);
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
  __device__ SegIter(int T, int nkb_, int G_, int g_) : nkb(nkb_), G(G_), g(g_) {
    U = static_cast<long long>(T) * nkb_;
    u = static_cast<long long>(g_) * U / G_;
    u1 = static_cast<long long>(g_ + 1) * U / G_;
  }
  __device__ bool next(int& t, int& kb0, int& nk, int& slot, int& nseg) {
    if (u >= u1) return false;
    t = static_cast<int>(u / nkb);
    kb0 = static_cast<int>(u - static_cast<long long>(t) * nkb);
    const long long tile_end = static_cast<long long>(t + 1) * nkb;
    const long long e = tile_end < u1 ? tile_end : u1;
    nk = static_cast<int>(e - u);
    const int first = unit_owner(static_cast<long long>(t) * nkb, G, U);
    const int last = unit_owner(tile_end - 1, G, U);
    slot = g - first;
    nseg = last - first + 1;
    u = e;
    return true;
  }
};

}  // namespace k3

template <int EPI, int NORM>
__global__ void __launch_bounds__(k3::NUM_THREADS, 1)
    k3_splitk_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                     const __grid_constant__ CUtensorMap tm_w, const OpParams p) {
  using namespace k3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int mpad = p.mpad, S = p.stages;
  const int SB = stage_bytes(mpad);
  const int XB = mpad * BK * 2;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + S * SB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int M = p.M, K = p.K;
  const int T = (EPI == kEpiSwiGLU) ? (p.I + 63) / 64 : (p.N + BW - 1) / BW;
  const int nkb = (K + BK - 1) / BK;
  const uint32_t ncols = tmem_cols(mpad);
  const bool split = p.split != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->conv[s], NUM_CONV_WARPS);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], NUM_EPI_WARPS);
      mbar_init(&ctrl->sfull[b], NUM_CONV_WARPS);
    }
    mbar_init(&ctrl->drain, 1);
    mbar_init(&ctrl->esync, NUM_EPI_WARPS);
    ctrl->abort_flag = 0;
    ctrl->last_flag = 0;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int* abortf = &ctrl->abort_flag;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      SegIter it(T, nkb, gridDim.x, blockIdx.x);
      int t, kb0, nk, slot, nseg;
      uint32_t s = 0, ph = 0, armed = 0, last_par = 0;
      bool ok = true;
      const uint64_t pol_w = policy_evict_first();   // W is streamed exactly once
      while (ok && it.next(t, kb0, nk, slot, nseg)) {
        for (int kb = kb0; kb < kb0 + nk; ++kb) {
          if (!mbar_wait(&ctrl->empty[s], ph ^ 1, abortf, p.status, kStatusWaitEmpty)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * SB;
          mbar_arrive_expect_tx(&ctrl->full[s], SB);
          if (EPI == kEpiSwiGLU) {
            tma_load_2d_hint(st, &tm_w, &ctrl->full[s], kb * BK, t * 64, pol_w);
            tma_load_2d_hint(st + W_BYTES / 2, &tm_w, &ctrl->full[s], kb * BK, p.I + t * 64, pol_w);
          } else {
            tma_load_2d_hint(st, &tm_w, &ctrl->full[s], kb * BK, t * BW, pol_w);
          }
          tma_load_2d(st + W_BYTES, &tm_x, &ctrl->full[s], kb * BK, 0);
          tma_load_2d(st + W_BYTES + XB, &tm_r, &ctrl->full[s], kb * BK, 0);
          armed |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
          if (++s == static_cast<uint32_t>(S)) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < S; ++i)
          if (armed & (1u << i)) drain_wait(&ctrl->full[i], (last_par >> i) & 1);
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      SegIter it(T, nkb, gridDim.x, blockIdx.x);
      int t, kb0, nk, slot, nseg;
      uint32_t s = 0, ph = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16(BW, mpad);
      int i = 0;
      while (ok && it.next(t, kb0, nk, slot, nseg)) {
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!mbar_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * mpad;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&ctrl->conv[s], ph, abortf, p.status, kStatusWaitConv) ||
              !mbar_wait(&ctrl->full[s], ph, abortf, p.status, kStatusWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(smem + s * SB);
          const uint64_t ad = sw128_desc(wa);
          const uint64_t bd = sw128_desc(wa + W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          if (split) {
            const uint64_t ld = sw128_desc(wa + W_BYTES + XB);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) umma_bf16(d, ad + 2 * kk, ld + 2 * kk, idesc, 1u);
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
    SegIter it(T, nkb, gridDim.x, blockIdx.x);
    int t, kb0, nk, slot, nseg;
    int i = 0;
    uint32_t eph = 0;
    while (it.next(t, kb0, nk, slot, nseg)) {
      const int b = i & 1;
      const uint32_t use = static_cast<uint32_t>(i >> 1);
      if (!warp_wait(&ctrl->tfull[b], use & 1, abortf, p.status, kStatusWaitTmemFull)) break;
      if (NORM == kRMSNorm) {
        if (!warp_wait(&ctrl->sfull[b], use & 1, abortf, p.status, kStatusWaitStats)) break;
      }
      tc_fence_after();
      const size_t base = static_cast<size_t>(t) * p.max_seg + slot;
      float* part = p.part + base * mpad * BW;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * mpad;
      for (int mc = 0; mc < mpad; mc += 16) {
        uint32_t v[16];
        tmem_ld16(tbase + mc, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (mc + e < M) part[static_cast<size_t>(mc + e) * BW + nl] = __uint_as_float(v[e]);
      }
      if (NORM == kRMSNorm && et < M) p.part_ss[base * mpad + et] = ctrl->ss[b][et];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->tempty[b]);
      ++i;

      // arrival: the last CTA of this tile reduces all slots in slot order.
      // The epilogue warps meet on an mbarrier (bounded wait), not bar.sync,
      // so a warp that gave up a wait can never leave the others blocked.
      __threadfence();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->esync);
      if (!warp_wait(&ctrl->esync, eph, abortf, p.status, kStatusWaitDrain)) break;
      eph ^= 1;
      if (et == 0) {
        __threadfence();
        const unsigned old = atomicAdd(&p.counters[t], 1u);
        ctrl->last_flag = (old == static_cast<unsigned>(nseg - 1)) ? 1 : 0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->esync);
      if (!warp_wait(&ctrl->esync, eph, abortf, p.status, kStatusWaitDrain)) break;
      eph ^= 1;
      if (ctrl->last_flag) {
        __threadfence();
        const float* tp = p.part + static_cast<size_t>(t) * p.max_seg * mpad * BW;
        const float* tss = p.part_ss + static_cast<size_t>(t) * p.max_seg * mpad;
        const int G8 = (EPI == kEpiSwiGLU) ? 8 : 16;
        for (int item = et; item < M * G8; item += NUM_EPI_WARPS * 32) {
          const int m = item / G8, g = item - (item / G8) * G8;
          float scale = 1.f;
          if (NORM == kRMSNorm) {
            float ssum = 0.f;
            for (int sl = 0; sl < nseg; ++sl) ssum += __ldcg(tss + static_cast<size_t>(sl) * mpad + m);
            scale = 1.f / sqrtf(ssum / static_cast<float>(K) + p.eps);
            if (t == 0 && g == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
          }
          if (EPI == kEpiSwiGLU) {
            const int j = t * 64 + g * 8;
            if (j >= p.I) continue;
            float ga[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ua[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int sl = 0; sl < nseg; ++sl) {
              const float* row = tp + (static_cast<size_t>(sl) * mpad + m) * BW;
              const float4 a0 = __ldcg(reinterpret_cast<const float4*>(row + g * 8));
              const float4 a1 = __ldcg(reinterpret_cast<const float4*>(row + g * 8 + 4));
              const float4 b0 = __ldcg(reinterpret_cast<const float4*>(row + 64 + g * 8));
              const float4 b1 = __ldcg(reinterpret_cast<const float4*>(row + 64 + g * 8 + 4));
              ga[0] += a0.x; ga[1] += a0.y; ga[2] += a0.z; ga[3] += a0.w;
              ga[4] += a1.x; ga[5] += a1.y; ga[6] += a1.z; ga[7] += a1.w;
              ua[0] += b0.x; ua[1] += b0.y; ua[2] += b0.z; ua[3] += b0.w;
              ua[4] += b1.x; ua[5] += b1.y; ua[6] += b1.z; ua[7] += b1.w;
            }
            store_swiglu8(p, m, j, ga, ua, scale);
          } else {
            const int n = t * BW + g * 8;
            if (n >= p.N) continue;
            float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int sl = 0; sl < nseg; ++sl) {
              const float* row = tp + (static_cast<size_t>(sl) * mpad + m) * BW;
              const float4 a0 = __ldcg(reinterpret_cast<const float4*>(row + g * 8));
              const float4 a1 = __ldcg(reinterpret_cast<const float4*>(row + g * 8 + 4));
              acc[0] += a0.x; acc[1] += a0.y; acc[2] += a0.z; acc[3] += a0.w;
              acc[4] += a1.x; acc[5] += a1.y; acc[6] += a1.z; acc[7] += a1.w;
            }
            store_out8<EPI>(p, m, n, acc, scale);
          }
        }
        if (et == 0) p.counters[t] = 0u;
      }
    }
  } else {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - WARP_CONV0 * 32;   // 0..127
    const int c = ct & 7;
    const int rg = ct >> 3;                          // rows rg + 16 j
    const int nj = mpad / 16;
    float mu[8], rs[8], ss[8];
    if (NORM == kLayerNorm) pdl_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = rg + 16 * j;
      mu[j] = 0.f;
      rs[j] = 0.f;
      if (NORM == kLayerNorm && j < nj && row < M) {
        const float2 st = p.stats[row];
        mu[j] = st.x;
        rs[j] = st.y;
      }
    }
    SegIter it(T, nkb, gridDim.x, blockIdx.x);
    int t, kb0, nk, slot, nseg;
    uint32_t s = 0, ph = 0;
    int i = 0;
    bool ok = true;
    while (ok && it.next(t, kb0, nk, slot, nseg)) {
#pragma unroll
      for (int j = 0; j < 8; ++j) ss[j] = 0.f;
      const bool write_res = (NORM == kRMSNorm) && t == 0;
      for (int kb = kb0; kb < kb0 + nk; ++kb) {
        if (!warp_wait(&ctrl->full[s], ph, abortf, p.status, kStatusWaitFull)) {
          ok = false;
          break;
        }
        const int k0 = kb * BK + c * 8;
        const bool kin = k0 < K;
        float g[8], be[8], bi[8];
        load8_or_zero(p.gamma, k0, kin, g);
        load8_or_zero(NORM == kLayerNorm ? p.beta : nullptr, k0, kin, be);
        load8_or_zero(p.bias_in, k0, kin, bi);
        const uint32_t xs = smem_u32(smem + s * SB) + W_BYTES;
        const uint32_t rsm = xs + XB;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < nj) {
            const int row = rg + 16 * j;
            const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
            float h[8], rr[8], a[8];
            unpack8(ld_shared_v4(xs + off), h);
            unpack8(ld_shared_v4(rsm + off), rr);
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = (h[e] + rr[e]) + bi[e];
            if (NORM == kLayerNorm) {
#pragma unroll
              for (int e = 0; e < 8; ++e) a[e] = fmaf((h[e] - mu[j]) * rs[j], g[e], be[e]);
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                a[e] = h[e] * g[e];
                ss[j] = fmaf(h[e], h[e], ss[j]);
              }
            }
            uint4 hi, lo;
            round_split8(a, split, hi, lo);
            st_shared_v4(xs + off, hi);
            if (split) st_shared_v4(rsm + off, lo);
            if (write_res && row < M && kin)
              *reinterpret_cast<uint4*>(p.residual_out + static_cast<size_t>(row) * K + k0) = pack8(h);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->conv[s]);
        if (++s == static_cast<uint32_t>(S)) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      if (NORM == kRMSNorm) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], 1);
          ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], 2);
          ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], 4);
        }
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!warp_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty)) break;
        if (c == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < nj) ctrl->ss[b][rg + 16 * j] = ss[j];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull[b]);
      }
      ++i;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace fnl
