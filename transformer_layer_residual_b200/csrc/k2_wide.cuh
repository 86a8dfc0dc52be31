// K2W: large-M fused norm + GEMM + epilogue with 128 x 512 tiles (persistent).
//
// Same dataflow as K2 (TMA x / residual / W tiles -> converters build the
// normalised bf16 operand in place in shared memory -> tcgen05.mma into TMEM ->
// epilogue), with the tile shaped to cut the bytes per FLOP that the fused
// operand costs: the tile is 128 tokens x 512 W rows (SwiGLU: 256 gate rows +
// the matching 256 up rows), the k-block is 32 wide (64-byte rows, 64-byte
// swizzle). A stage is then x 8 KB + residual 8 KB + W 32 KB for 512 UMMA
// cycles: half the conversion work and three quarters of the L2->SM traffic of
// the 128 x 256 x 64 tile per FLOP, and four stages fit in shared memory. The
// accumulator takes all 512 TMEM columns, so the epilogue of a tile is not
// overlapped with the next tile's MMAs (the producer and converters keep
// running ahead meanwhile).
//
// Warp roles (14 warps): 0 TMA producer, 1 TMEM owner + UMMA issuer,
// 2-5 epilogue, 6-13 converters. RMSNorm uses the deferred scale as in K2;
// LayerNorm statistics come from the statistics kernel.
#pragma once

#include "common.cuh"

namespace fnl {
namespace k2w {

constexpr int BM = 128, BN = 512, BK = 32, STAGES = 4;
constexpr int X_BYTES = BM * BK * 2;                 // 8 KB
constexpr int W_BYTES = BN * BK * 2;                 // 32 KB
constexpr int W_HALF = W_BYTES / 2;                  // 256 rows
constexpr int STAGE_BYTES = 2 * X_BYTES + W_BYTES;   // 48 KB
constexpr int VEC = BK;                              // gamma / beta / bias_in elements per stage
constexpr int VEC_STAGE_BYTES = 3 * VEC * 2;         // 192
constexpr int VEC_BYTES = STAGES * VEC_STAGE_BYTES;
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_EPI0 = 2, NUM_EPI_WARPS = 4;
constexpr int WARP_CONV0 = 6, NUM_CONV_WARPS = 8;
constexpr int NUM_THREADS = (WARP_CONV0 + NUM_CONV_WARPS) * 32;   // 448
constexpr int TMEM_COLS = 512;
constexpr int GROUP_M = 16;

struct Ctrl {
  uint64_t full_w[STAGES], full_x[STAGES], conv[STAGES], empty[STAGES];
  uint64_t tfull, tempty, sfull, drain;
  uint32_t tmem_base;
  int abort_flag;
  float rs[BM];
};
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

}  // namespace k2w

template <int EPI, int NORM, bool SPLIT>
__global__ void __launch_bounds__(k2w::NUM_THREADS, 1)
    k2w_tile_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                    const __grid_constant__ CUtensorMap tm_w, const OpParams p) {
  using namespace k2w;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  bf16* vecs = reinterpret_cast<bf16*>(smem + STAGES * STAGE_BYTES);   // [STAGES][3][32]
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + STAGES * STAGE_BYTES + VEC_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_beta = NORM == kLayerNorm && p.beta != nullptr;
  const bool has_bias_in = EPI == kEpiGELU && p.bias_in != nullptr;

  const int M = p.M, K = p.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (EPI == kEpiSwiGLU) ? (p.I + 255) / 256 : (p.N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int nkb = (K + BK - 1) / BK;
  constexpr bool BIAS_IN = EPI == kEpiGELU;   // only the GELU entry point has a bias_in

  if (threadIdx.x == 0) {
    pdl_launch_dependents();
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full_w[s], 1);
      mbar_init(&ctrl->full_x[s], 1);
      mbar_init(&ctrl->conv[s], NUM_CONV_WARPS);
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->tfull, 1);
    mbar_init(&ctrl->tempty, NUM_EPI_WARPS);
    mbar_init(&ctrl->sfull, NUM_CONV_WARPS);
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
  zero_vec_slices(vecs, STAGES * 3 * VEC);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int* abortf = &ctrl->abort_flag;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const int P = my_tiles * nkb;
      const int npre = P < STAGES ? P : STAGES;
      uint32_t armed_w = 0, armed_x = 0, par_w = 0, par_x = 0;
      bool ok = true;
      // fault injection (status-path tests only): CTA 0 withholds its first weight copy
      bool withhold = p.stall != 0 && blockIdx.x == 0;
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
        if (withhold) {
          withhold = false;
          return;
        }
        uint8_t* st = smem + c.s * STAGE_BYTES + 2 * X_BYTES;
        mbar_arrive_expect_tx(&ctrl->full_w[c.s], W_BYTES);
        if (EPI == kEpiSwiGLU) {
          tma_load_2d(st, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.nb * 256);
          tma_load_2d(st + W_HALF, &tm_w, &ctrl->full_w[c.s], c.kb * BK, p.I + c.nb * 256);
        } else {
          tma_load_2d(st, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.nb * BN);
          tma_load_2d(st + W_HALF, &tm_w, &ctrl->full_w[c.s], c.kb * BK, c.nb * BN + 256);
        }
        armed_w |= 1u << c.s;
        par_w = (par_w & ~(1u << c.s)) | (c.ph << c.s);
      };
      auto issue_x = [&](const Cur& c) {
        uint8_t* st = smem + c.s * STAGE_BYTES;
        if (NORM == kNoNorm) {   // the activation tile is the operand as loaded
          mbar_arrive_expect_tx(&ctrl->full_x[c.s], X_BYTES);
          tma_load_2d(st, &tm_x, &ctrl->full_x[c.s], c.kb * BK, c.mb * BM);
          armed_x |= 1u << c.s;
          par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
          return;
        }
        bf16* vec = vecs + c.s * 3 * VEC;
        const int k0 = c.kb * BK;
        const uint32_t vb = static_cast<uint32_t>(min(VEC, K - k0)) * 2;
        const uint32_t nvec = 1 + (has_beta ? 1 : 0) + (has_bias_in ? 1 : 0);
        mbar_arrive_expect_tx(&ctrl->full_x[c.s], 2 * X_BYTES + vb * nvec);
        bulk_load(vec, p.gamma + k0, vb, &ctrl->full_x[c.s]);
        if (has_beta) bulk_load(vec + VEC, p.beta + k0, vb, &ctrl->full_x[c.s]);
        if (has_bias_in) bulk_load(vec + 2 * VEC, p.bias_in + k0, vb, &ctrl->full_x[c.s]);
        tma_load_2d(st, &tm_x, &ctrl->full_x[c.s], k0, c.mb * BM);
        tma_load_2d(st + X_BYTES, &tm_r, &ctrl->full_x[c.s], k0, c.mb * BM);
        armed_x |= 1u << c.s;
        par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
      };
      for (int q = 0; q < npre; ++q) {
        issue_w(cw);
        step(cw);
      }
      pdl_wait();
      for (int q = 0; q < P; ++q) {
        if (q >= npre) {
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
      if (!ok) {
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
      const uint32_t idesc = idesc_bf16(BM, 256);
      int i = 0;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
        if (!mbar_wait(&ctrl->tempty, (static_cast<uint32_t>(i) & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty, p.wait_ns))
          break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          // the converted operand (or, without a norm, the activation tile as loaded)
          uint64_t* ready = NORM == kNoNorm ? &ctrl->full_x[s] : &ctrl->conv[s];
          if (!mbar_wait(&ctrl->full_w[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns) ||
              !mbar_wait(ready, ph, abortf, p.status, kStatusWaitConv, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t ad = sw64_desc(xa);
          const uint64_t ld = sw64_desc(xa + X_BYTES);
          const uint64_t bd0 = sw64_desc(xa + 2 * X_BYTES);
          const uint64_t bd1 = sw64_desc(xa + 2 * X_BYTES + W_HALF);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(tmem, ad + 2 * kk, bd0 + 2 * kk, idesc, acc);
            umma_bf16(tmem + 256, ad + 2 * kk, bd1 + 2 * kk, idesc, acc);
            if (SPLIT) {   // + lo(a) W^T into the same accumulators
              umma_bf16(tmem, ld + 2 * kk, bd0 + 2 * kk, idesc, 1u);
              umma_bf16(tmem + 256, ld + 2 * kk, bd1 + 2 * kk, idesc, 1u);
            }
          }
          umma_commit(&ctrl->empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&ctrl->tfull);
      }
      umma_commit(&ctrl->drain);
      drain_wait(&ctrl->drain, 0);
    }
  } else if (warp < WARP_CONV0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    pdl_wait();
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const uint32_t par = static_cast<uint32_t>(i) & 1;
      if (!warp_wait(&ctrl->tfull, par, abortf, p.status, kStatusWaitTmemFull, p.wait_ns)) break;
      float scale = 1.f;
      if (NORM == kRMSNorm) {
        if (!warp_wait(&ctrl->sfull, par, abortf, p.status, kStatusWaitStats, p.wait_ns)) break;
        scale = ctrl->rs[row_local];
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      const int m = mb * BM + row_local;
      const bool row_ok = m < M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
      if (EPI == kEpiSwiGLU) {
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t g0[16], g1[16], u0[16], u1[16];
          tmem_ld16(tbase + cc * 32, g0);
          tmem_ld16(tbase + cc * 32 + 16, g1);
          tmem_ld16(tbase + 256 + cc * 32, u0);
          tmem_ld16(tbase + 256 + cc * 32 + 16, u1);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const int j = nb * 256 + cc * 32 + g8 * 8;
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
      if (lane == 0) mbar_arrive(&ctrl->tempty);
    }
  } else if (NORM != kNoNorm) {
    // ------------------------------------------------------------ converters
    // Thread ct: 16-byte chunk c (0..3) of the 64-byte row, rows rbase and
    // rbase + 64. 64-byte swizzle: chunk c of row r sits at c ^ ((r >> 1) & 3).
    const int ct = threadIdx.x - WARP_CONV0 * 32;   // 0..255
    const int c = ct & 3;
    const int rbase = ct >> 2;                       // 0..63
    if (NORM == kLayerNorm) pdl_wait();
    uint32_t s = 0, ph = 0;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      float mu[2], rs[2];
      f32x2 ss[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int gm = mb * BM + rbase + 64 * j;
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
        if (!warp_wait(&ctrl->full_x[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
          ok = false;
          break;
        }
        bf16* vec = vecs + s * 3 * VEC;
        if (K - kb * BK < BK) zero_vec_tails(vec, VEC, K - kb * BK);
        const uint32_t vaddr = smem_u32(vec) + c * 16;
        f32x2 g2[4], be2[4] = {}, bi2[4] = {};
        vec_pairs(vaddr, g2);
        if (NORM == kLayerNorm) vec_pairs(vaddr + 2 * VEC, be2);
        if (BIAS_IN) vec_pairs(vaddr + 4 * VEC, bi2);
        const uint32_t xs = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t rsm = xs + X_BYTES;
        uint4 xv[2], rv[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = rbase + 64 * j;
          const uint32_t off = row * 64 + ((c ^ ((row >> 1) & 3)) << 4);
          xv[j] = ld_shared_v4(xs + off);
          rv[j] = ld_shared_v4(rsm + off);
        }
        // instantiated with and without the residual_out store (first N column)
        auto convert_stage = [&](auto wres_tag) {
          constexpr bool WRES = decltype(wres_tag)::value;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int row = rbase + 64 * j;
            const uint32_t off = row * 64 + ((c ^ ((row >> 1) & 3)) << 4);
            uint4 hi, lo, hres;
            convert8<NORM, BIAS_IN, SPLIT, WRES>(xv[j], rv[j], g2, be2, bi2, mu[j], rs[j], ss[j], hi, lo, hres);
            st_shared_v4(xs + off, hi);
            if (SPLIT) st_shared_v4(rsm + off, lo);
            if (WRES) {
              const int gm = mb * BM + row;
              const int k0 = kb * BK + c * 8;
              if (gm < M && k0 < K) {
                bf16* dst = p.residual_out + static_cast<size_t>(gm) * K + k0;
                if (store_in_bounds(p, dst, p.residual_out, static_cast<size_t>(M) * K))
                  *reinterpret_cast<uint4*>(dst) = hres;
              }
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
        float sst[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float lo_, hi_;
          unpk2(ss[j], lo_, hi_);
          sst[j] = lo_ + hi_;
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 1);
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 2);
        }
        // the epilogue of the previous tile has read rs once tempty completes
        if (!warp_wait(&ctrl->tempty, (static_cast<uint32_t>(i) & 1) ^ 1, abortf, p.status,
                       kStatusWaitTmemEmpty, p.wait_ns))
          break;
        if (c == 0) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int row = rbase + 64 * j;
            const float r = 1.f / sqrtf(sst[j] / static_cast<float>(K) + p.eps);
            ctrl->rs[row] = r;
            const int gm = mb * BM + row;
            if (write_res && p.rstd_out != nullptr && gm < M) p.rstd_out[gm] = r;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull);
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
