// K2: large-M fused norm + GEMM + epilogue, persistent, one CTA per SM.
//
// Tile: 128 tokens x 256 W rows (SwiGLU: 128 gate rows + the matching 128 up
// rows), K in blocks of 64. Warp roles (18 warps):
//   warp 0      TMA producer: per k-block, x and residual tiles [128 x 64] and
//               the W tile [256 x 64], 128-byte swizzled, into one of 3 stages;
//   warp 1      TMEM owner and UMMA issuer (one thread): 4 x
//               tcgen05.mma M=128 N=256 K=16 per k-block into one of two
//               256-column fp32 accumulators;
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (lane = token row),
//               deferred RMSNorm scale, bias, QKV head-major split / SwiGLU /
//               GELU, bf16 stores straight to the outputs;
//   warps 6-17  converters: in place in shared memory, turn the x tile into the
//               normalised bf16 A operand a = norm(x + r (+ bias_in)) using the
//               residual tile, so the normalised activations never touch global
//               memory (the "shared memory caching of normalised values /
//               eliminating the intermediate write-back" of TensorRT-LLM
//               深度工程实践, §2.3).
// LayerNorm: (mean, rstd) per row come from the statistics kernel (K1).
// RMSNorm: deferred scaling. The converters write a' = bf16(gamma * h) and sum
// h^2 per row over the K loop; 1/rms is applied per accumulator row in the
// epilogue (y = rstd * sum_k a'_k W_nk is the same product). Tiles in the first
// N column also write residual_out and rstd_out, so RMSNorm needs no extra pass.
// Each stage has a weight barrier (full_w) and an activation barrier (full_x);
// the kernel is a programmatic dependent of the previous kernel on the stream
// (first weight tiles before griddepcontrol.wait, everything else after it).
#pragma once

#include "common.cuh"

namespace fnl {
namespace k2 {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 3;
constexpr int X_BYTES = BM * BK * 2;                 // 16 KB
constexpr int W_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = 2 * X_BYTES + W_BYTES;   // 64 KB
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_EPI0 = 2, NUM_EPI_WARPS = 4;
constexpr int WARP_CONV0 = 6, NUM_CONV_WARPS = 12;
constexpr int ROW_STRIDE = NUM_CONV_WARPS * 32 / 8;              // rows between a thread's rows
constexpr int ROWS_PER_THREAD = (BM + ROW_STRIDE - 1) / ROW_STRIDE;   // 3
constexpr int NUM_THREADS = (WARP_CONV0 + NUM_CONV_WARPS) * 32;   // 576
constexpr int TMEM_COLS = 2 * BN;                                  // 512
constexpr int GROUP_M = 16;  // tile raster: 16 M-blocks share each W tile while it is hot in L2

struct Ctrl {
  uint64_t full_w[STAGES], full_x[STAGES], conv[STAGES], empty[STAGES];
  uint64_t tfull[2], tempty[2], sfull[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  float rs[2][BM];
};
constexpr int VEC_BYTES = (STAGES * kVecStageBytes + 127) / 128 * 128;   // [STAGES][3][64] bf16
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + VEC_BYTES + static_cast<int>(sizeof(Ctrl)) + 1024;

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = GROUP_M * num_n;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(GROUP_M, num_m - first_m);
  const int r = t - group * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > FNL_WAIT_NS) return false;
  }
  return true;
}

}  // namespace k2

template <int EPI, int NORM, bool SPLIT>
__global__ void __launch_bounds__(k2::NUM_THREADS, 1)
    k2_tile_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                   const __grid_constant__ CUtensorMap tm_w, const OpParams p) {
  using namespace k2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  bf16* vecs = reinterpret_cast<bf16*>(smem + STAGES * STAGE_BYTES);   // [STAGES][3][64]
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + STAGES * STAGE_BYTES + VEC_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_beta = NORM == kLayerNorm && p.beta != nullptr;
  const bool has_bias_in = EPI == kEpiGELU && p.bias_in != nullptr;   // only the GELU entry point has one

  const int M = p.M, K = p.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (EPI == kEpiSwiGLU) ? (p.I + 127) / 128 : (p.N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int nkb = (K + BK - 1) / BK;
  constexpr bool BIAS_IN = EPI == kEpiGELU;   // only the GELU entry point has a bias_in

  if (threadIdx.x == 0) {
    pdl_launch_dependents();   // the next call's CTAs may take SMs as ours retire
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full_w[s], 1);
      mbar_init(&ctrl->full_x[s], 1);
      mbar_init(&ctrl->conv[s], NUM_CONV_WARPS);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], NUM_EPI_WARPS);
      mbar_init(&ctrl->sfull[b], NUM_CONV_WARPS);
    }
    mbar_init(&ctrl->drain, 1);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_r);
    prefetch_tmap(&tm_w);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  zero_vec_slices(vecs, STAGES * 3 * kVecElems);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int* abortf = &ctrl->abort_flag;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // positions q = (local tile index) * nkb + k-block, stage q % STAGES
      const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const int P = my_tiles * nkb;
      const int npre = P < STAGES ? P : STAGES;
      uint32_t armed_w = 0, armed_x = 0, par_w = 0, par_x = 0;
      bool ok = true;
      struct Cur {
        int t, mb, nb, kb, s;
        uint32_t ph;
      };
      Cur cw{static_cast<int>(blockIdx.x), 0, 0, 0, 0, 0u};
      if (P > 0) tile_coords(cw.t, num_m, num_n, cw.mb, cw.nb);
      Cur cx = cw;
      auto step = [&](Cur& c) {
        if (++c.kb == nkb) {
          c.kb = 0;
          c.t += gridDim.x;
          if (c.t < tiles) tile_coords(c.t, num_m, num_n, c.mb, c.nb);
        }
        if (++c.s == STAGES) {
          c.s = 0;
          c.ph ^= 1u;
        }
      };
      auto issue_w = [&](const Cur& c) {
        uint8_t* st = smem + c.s * STAGE_BYTES;
        mbar_arrive_expect_tx(&ctrl->full_w[c.s], W_BYTES);
        if (EPI == kEpiSwiGLU) {
          tma_load_2d(st + 2 * X_BYTES, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.nb * 128);
          tma_load_2d(st + 2 * X_BYTES + W_BYTES / 2, &tm_w, &ctrl->full_w[c.s], c.kb * BK, p.I + c.nb * 128);
        } else {
          tma_load_2d(st + 2 * X_BYTES, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.nb * BN);
        }
        armed_w |= 1u << c.s;
        par_w = (par_w & ~(1u << c.s)) | (c.ph << c.s);
      };
      auto issue_x = [&](const Cur& c) {
        uint8_t* st = smem + c.s * STAGE_BYTES;
        mbar_arrive_expect_tx(&ctrl->full_x[c.s], 2 * X_BYTES + vec_bytes(p, has_beta, has_bias_in, c.kb));
        issue_vec_loads(p, has_beta, has_bias_in, c.kb, vecs + c.s * 3 * kVecElems, &ctrl->full_x[c.s]);
        tma_load_2d(st, &tm_x, &ctrl->full_x[c.s], c.kb * BK, c.mb * BM);
        tma_load_2d(st + X_BYTES, &tm_r, &ctrl->full_x[c.s], c.kb * BK, c.mb * BM);
        armed_x |= 1u << c.s;
        par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
      };
      // Weights of the first stages stream while the previous kernel finishes
      // (they are never written by it); activations only after it is done.
      for (int q = 0; q < npre; ++q) {
        issue_w(cw);
        step(cw);
      }
      pdl_wait();
      for (int q = 0; q < P; ++q) {
        if (q >= npre) {
          if (!mbar_wait(&ctrl->empty[cw.s], cw.ph ^ 1, abortf, p.status, kStatusWaitEmpty)) {
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
        for (int i = 0; i < STAGES; ++i) {
          if (armed_w & (1u << i)) drain_wait(&ctrl->full_w[i], (par_w >> i) & 1);
          if (armed_x & (1u << i)) drain_wait(&ctrl->full_x[i], (par_x >> i) & 1);
        }
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16(BM, BN);
      int i = 0;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!mbar_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctrl->conv[s], ph, abortf, p.status, kStatusWaitConv) ||
              !mbar_wait(&ctrl->full_w[s], ph, abortf, p.status, kStatusWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t ad = sw128_desc(xa);
          const uint64_t bd = sw128_desc(xa + 2 * X_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          if (SPLIT) {   // + lo(a) W^T into the same accumulator
            const uint64_t ld = sw128_desc(xa + X_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) umma_bf16(d, ld + 2 * kk, bd + 2 * kk, idesc, 1u);
          }
          umma_commit(&ctrl->empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&ctrl->tfull[b]);
      }
      umma_commit(&ctrl->drain);   // every issued UMMA done before TMEM is freed
      drain_wait(&ctrl->drain, 0);
    }
  } else if (warp < WARP_CONV0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;   // TMEM lane quadrant this warp may read
    const int row_local = q * 32 + lane;
    pdl_wait();   // outputs may still be in use by the previous kernel
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const uint32_t use = static_cast<uint32_t>(i >> 1);
      if (!warp_wait(&ctrl->tfull[b], use & 1, abortf, p.status, kStatusWaitTmemFull)) break;
      float scale = 1.f;
      if (NORM == kRMSNorm) {
        if (!warp_wait(&ctrl->sfull[b], use & 1, abortf, p.status, kStatusWaitStats)) break;
        scale = ctrl->rs[b][row_local];
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      const int m = mb * BM + row_local;
      const bool row_ok = m < M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
      if (EPI == kEpiSwiGLU) {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t g0[16], g1[16], u0[16], u1[16];
          tmem_ld16(tbase + cc * 32, g0);
          tmem_ld16(tbase + cc * 32 + 16, g1);
          tmem_ld16(tbase + 128 + cc * 32, u0);
          tmem_ld16(tbase + 128 + cc * 32 + 16, u1);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const int j = nb * 128 + cc * 32 + g8 * 8;
              if (j < p.I) {
                float gv[8], uv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int c = g8 * 8 + e;
                  gv[e] = __uint_as_float(c < 16 ? g0[c] : g1[c - 16]);
                  uv[e] = __uint_as_float(c < 16 ? u0[c] : u1[c - 16]);
                }
                store_swiglu8(p, m, j, gv, uv, scale);
              }
            }
          }
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t a0[16], a1[16];
          tmem_ld16(tbase + cc * 32, a0);
          tmem_ld16(tbase + cc * 32 + 16, a1);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const int n = nb * BN + cc * 32 + g8 * 8;
              if (n < p.N) {
                float av[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int c = g8 * 8 + e;
                  av[e] = __uint_as_float(c < 16 ? a0[c] : a1[c - 16]);
                }
                store_out8<EPI>(p, m, n, av, scale);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->tempty[b]);
    }
  } else {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - WARP_CONV0 * 32;   // 0 .. NUM_CONV_WARPS*32-1
    const int c = ct & 7;                            // 16-byte chunk of the 128-byte row
    const int rbase = ct >> 3;                       // rows rbase + ROW_STRIDE j (< BM)
    constexpr int RPT = ROWS_PER_THREAD;
    if (NORM == kLayerNorm) pdl_wait();              // statistics come from the previous kernel
    uint32_t s = 0, ph = 0;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      float mu[RPT], rs[RPT];
      f32x2 ss[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int gm = mb * BM + rbase + ROW_STRIDE * j;
        ss[j] = 0ull;
        mu[j] = 0.f;
        rs[j] = 0.f;
        if (NORM == kLayerNorm && gm < M) {
          const float2 st = p.stats[gm];
          mu[j] = st.x;
          rs[j] = st.y;
        }
      }
      const bool write_res = (NORM == kRMSNorm) && nb == 0;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!warp_wait(&ctrl->full_x[s], ph, abortf, p.status, kStatusWaitFull)) {
          ok = false;
          break;
        }
        bf16* vec = vecs + s * 3 * kVecElems;
        if (K - kb * BK < BK) zero_vec_tails(vec, kVecElems, K - kb * BK);
        const uint32_t vaddr = smem_u32(vec) + c * 16;
        f32x2 g2[4], be2[4] = {}, bi2[4] = {};
        vec_pairs(vaddr, g2);
        if (NORM == kLayerNorm) vec_pairs(vaddr + 2 * kVecElems, be2);
        if (BIAS_IN) vec_pairs(vaddr + 4 * kVecElems, bi2);
        const uint32_t xs = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t rsm = xs + X_BYTES;
        // loads of all of this thread's rows first, then arithmetic and stores,
        // so the chunks overlap instead of running in series
        uint4 xv[RPT], rv[RPT];
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          const int row = rbase + ROW_STRIDE * j;
          if (row < BM) {
            const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
            xv[j] = ld_shared_v4(xs + off);
            rv[j] = ld_shared_v4(rsm + off);
          }
        }
        // instantiated with and without the residual_out store (first N column)
        auto convert_stage = [&](auto wres_tag) {
          constexpr bool WRES = decltype(wres_tag)::value;
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            const int row = rbase + ROW_STRIDE * j;
            if (row >= BM) continue;
            const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
            uint4 hi, lo, hres;
            convert8<NORM, BIAS_IN, SPLIT, WRES>(xv[j], rv[j], g2, be2, bi2, mu[j], rs[j], ss[j], hi, lo, hres);
            st_shared_v4(xs + off, hi);
            if (SPLIT) st_shared_v4(rsm + off, lo);   // residual chunk already consumed by this thread
            if (WRES) {
              const int gm = mb * BM + row;
              const int k0 = kb * BK + c * 8;
              if (gm < M && k0 < K)
                *reinterpret_cast<uint4*>(p.residual_out + static_cast<size_t>(gm) * K + k0) = hres;
            }
          }
        };
        if (write_res) convert_stage(BoolC<true>{});
        else convert_stage(BoolC<false>{});
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->conv[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      if (NORM == kRMSNorm) {
        float sst[RPT];
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          float lo_, hi_;
          unpk2(ss[j], lo_, hi_);
          sst[j] = lo_ + hi_;
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 1);
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 2);
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 4);
        }
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!warp_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty)) break;
        if (c == 0) {
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            const int row = rbase + ROW_STRIDE * j;
            if (row >= BM) continue;
            const float r = 1.f / sqrtf(sst[j] / static_cast<float>(K) + p.eps);
            ctrl->rs[b][row] = r;
            const int gm = mb * BM + row;
            if (write_res && p.rstd_out != nullptr && gm < M) p.rstd_out[gm] = r;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull[b]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fnl
