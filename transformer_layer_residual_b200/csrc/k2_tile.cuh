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
//               residual tile, so the normalised activations stay on chip and
//               are never written back (the LayerNorm + projection fusion of
//               TensorRT-LLM 深度工程实践, §2.3).
// LayerNorm: (mean, rstd) per row come from the statistics kernel (K1).
// RMSNorm: deferred scaling. The converters write a' = bf16(gamma * h) and sum
// h^2 per row over their k-blocks; the epilogue turns the sum into 1/rms and
// applies it per accumulator row (y = rstd * sum_k a'_k W_nk is the same
// product), writing rstd_out for the first N column. Tiles in the first N
// column also write residual_out, so RMSNorm needs no extra pass.
// Work: whole tiles g, g + G, ... per CTA; when the tiles are fewer than the
// CTAs by a fifth or more, stream-K instead: even shares of the (tile, k-block)
// units, partial tiles summed from fp32 slots by their last CTA.
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
  uint64_t tfull[2], tempty[2], sfull[2], drain, esync;
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int fin_go, fin_t, fin_nseg;   // stream-K: the CTA's last segment completes its tile (summed by all warps)
  float rs[2][BM];               // RMSNorm: sum(h^2) per row of the segment, from the converters
};
// Stream-K partial of one segment: fp32 [BN / 8][BM][8] (8-column chunks, rows
// contiguous, so a warp's 32 rows read and write 1 KB runs) and sum(h^2) [BM].
constexpr int SLOT_FLOATS = BM * BN + BM;

// The CTA's segments. Tile mode (p.sk == 0): whole tiles g, g + G, ...
// Stream-K (p.sk != 0, used when there are fewer tiles than CTAs): the
// (tile, k-block) units [g U / G, (g + 1) U / G), cut at tile ends; slot /
// nseg locate the segment among the tile's CTAs.
struct Segs {
  long long u, u1, U;
  int t_next, tiles, nkb, G, g;
  bool sk;
  __device__ bool next(int& t, int& kb0, int& nk, int& slot, int& nseg) {
    if (!sk) {
      if (t_next >= tiles) return false;
      t = t_next;
      t_next += G;
      kb0 = 0;
      nk = nkb;
      slot = 0;
      nseg = 1;
      return true;
    }
    if (u >= u1) return false;
    t = static_cast<int>(u / nkb);
    kb0 = static_cast<int>(u - static_cast<long long>(t) * nkb);
    const long long te = static_cast<long long>(t + 1) * nkb;
    const long long e = te < u1 ? te : u1;
    nk = static_cast<int>(e - u);
    const int first = unit_owner_fast(static_cast<long long>(t) * nkb, G, U);
    const int last = unit_owner_fast(te - 1, G, U);
    slot = g - first;
    nseg = last - first + 1;
    u = e;
    return true;
  }
  __device__ bool done() const { return sk ? u >= u1 : t_next >= tiles; }
};
__device__ __forceinline__ Segs make_segs(bool sk, int tiles, int nkb) {
  Segs it;
  it.sk = sk;
  it.tiles = tiles;
  it.nkb = nkb;
  it.G = gridDim.x;
  it.g = blockIdx.x;
  it.t_next = blockIdx.x;
  it.U = static_cast<long long>(tiles) * nkb;
  it.u = it.U * blockIdx.x / gridDim.x;
  it.u1 = it.U * (blockIdx.x + 1) / gridDim.x;
  return it;
}
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

// Stream-K fix-up of tile t by the CTA that arrived last: sum the nseg slots in
// slot order (the same sum on every run) and run the epilogue, NT threads
// (et = 0..NT-1). Item = (row, 8-column chunk), rows fastest so that a warp
// reads 1 KB runs; each thread loads ITEMS items' slots before adding.
template <int EPI, int NORM, int NT>
__device__ __forceinline__ void k2_reduce_tile(const OpParams& p, int t, int nseg, int et, int num_m, int num_n) {
  using namespace k2;
  int mb, nb;
  tile_coords(t, num_m, num_n, mb, nb);
  const float* tp = p.part + static_cast<size_t>(t) * p.max_seg * SLOT_FLOATS;
  constexpr int CH = (EPI == kEpiSwiGLU) ? BN / 16 : BN / 8;   // SwiGLU: gate chunks (up = chunk + BN / 16)
  constexpr int ITEMS = (EPI == kEpiSwiGLU) ? 1 : 2;   // SwiGLU carries gate and up sums
  const int n_items = BM * CH;
  for (int it0 = et; it0 < n_items; it0 += ITEMS * NT) {
    float acc[ITEMS][8], up[ITEMS][8], ssum[ITEMS];
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      ssum[q] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[q][e] = up[q][e] = 0.f;
    }
    for (int sl = 0; sl < nseg; ++sl) {
      const float* sp = tp + static_cast<size_t>(sl) * SLOT_FLOATS;
      float4 va[ITEMS][2], vu[ITEMS][2];
      float vs[ITEMS];
#pragma unroll
      for (int q = 0; q < ITEMS; ++q) {
        const int item = it0 + q * NT;
        if (item < n_items) {
          const int row = item % BM, c8 = item / BM;
          const float* a = sp + (static_cast<size_t>(c8) * BM + row) * 8;
          va[q][0] = __ldcg(reinterpret_cast<const float4*>(a));
          va[q][1] = __ldcg(reinterpret_cast<const float4*>(a + 4));
          if (EPI == kEpiSwiGLU) {
            const float* u = a + static_cast<size_t>(CH) * BM * 8;
            vu[q][0] = __ldcg(reinterpret_cast<const float4*>(u));
            vu[q][1] = __ldcg(reinterpret_cast<const float4*>(u + 4));
          }
          if (NORM == kRMSNorm) vs[q] = __ldcg(sp + BM * BN + row);
        }
      }
#pragma unroll
      for (int q = 0; q < ITEMS; ++q) {
        if (it0 + q * NT < n_items) {
          acc[q][0] += va[q][0].x; acc[q][1] += va[q][0].y; acc[q][2] += va[q][0].z; acc[q][3] += va[q][0].w;
          acc[q][4] += va[q][1].x; acc[q][5] += va[q][1].y; acc[q][6] += va[q][1].z; acc[q][7] += va[q][1].w;
          if (EPI == kEpiSwiGLU) {
            up[q][0] += vu[q][0].x; up[q][1] += vu[q][0].y; up[q][2] += vu[q][0].z; up[q][3] += vu[q][0].w;
            up[q][4] += vu[q][1].x; up[q][5] += vu[q][1].y; up[q][6] += vu[q][1].z; up[q][7] += vu[q][1].w;
          }
          if (NORM == kRMSNorm) ssum[q] += vs[q];
        }
      }
    }
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int item = it0 + q * NT;
      if (item >= n_items) continue;
      const int row = item % BM, c8 = item / BM;
      const int m = mb * BM + row;
      if (m >= p.M) continue;
      float scale = 1.f;
      if (NORM == kRMSNorm) {
        scale = 1.f / sqrtf(ssum[q] / static_cast<float>(p.K) + p.eps);
        if (nb == 0 && c8 == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
      }
      if (EPI == kEpiSwiGLU) {
        const int j = nb * (BN / 2) + c8 * 8;
        if (j < p.I) store_swiglu8(p, m, j, acc[q], up[q], scale);
      } else {
        const int n = nb * BN + c8 * 8;
        if (n < p.N) store_out8<EPI>(p, m, n, acc[q], scale);
      }
    }
  }
}

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
  const bool sk = p.sk != 0;

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
    mbar_init(&ctrl->esync, NUM_EPI_WARPS);
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
      const Segs segs = make_segs(sk, tiles, nkb);
      const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const int P = sk ? static_cast<int>(segs.u1 - segs.u) : my_tiles * nkb;
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
      if (sk) {
        cw.t = static_cast<int>(segs.u / nkb);
        cw.kb = static_cast<int>(segs.u - static_cast<long long>(cw.t) * nkb);
      }
      if (P > 0) tile_coords(cw.t, num_m, num_n, cw.mb, cw.nb);
      Cur cx = cw;
      auto step = [&](Cur& c) {
        if (++c.kb == nkb) {
          c.kb = 0;
          c.t += sk ? 1 : static_cast<int>(gridDim.x);
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
        if (NORM == kNoNorm) {   // the activation tile is the operand as loaded
          mbar_arrive_expect_tx(&ctrl->full_x[c.s], X_BYTES);
          tma_load_2d(st, &tm_x, &ctrl->full_x[c.s], c.kb * BK, c.mb * BM);
          armed_x |= 1u << c.s;
          par_x = (par_x & ~(1u << c.s)) | (c.ph << c.s);
          return;
        }
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
      Segs segs = make_segs(sk, tiles, nkb);
      int t, kb0, nk, slot, nseg;
      while (ok && segs.next(t, kb0, nk, slot, nseg)) {
        const int b = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        ++i;
        if (!mbar_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb) {   // kb counts the segment's k-blocks
          // the converted operand (or, without a norm, the activation tile as loaded)
          uint64_t* ready = NORM == kNoNorm ? &ctrl->full_x[s] : &ctrl->conv[s];
          if (!mbar_wait(ready, ph, abortf, p.status, kStatusWaitConv, p.wait_ns) ||
              !mbar_wait(&ctrl->full_w[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
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
    pdl_wait();   // outputs and workspace may still be in use by the previous kernel
    const int et = threadIdx.x - WARP_EPI0 * 32;   // 0..127
    int i = 0;
    uint32_t eph = 0;
    Segs segs = make_segs(sk, tiles, nkb);
    int t, kb0, nk, slot, nseg;
    while (segs.next(t, kb0, nk, slot, nseg)) {
      const int b = i & 1;
      const uint32_t use = static_cast<uint32_t>(i >> 1);
      ++i;
      if (!warp_wait(&ctrl->tfull[b], use & 1, abortf, p.status, kStatusWaitTmemFull, p.wait_ns)) break;
      float ssq = 0.f;
      if (NORM == kRMSNorm) {
        if (!warp_wait(&ctrl->sfull[b], use & 1, abortf, p.status, kStatusWaitStats, p.wait_ns)) break;
        ssq = ctrl->rs[b][row_local];
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      const int m = mb * BM + row_local;
      const bool row_ok = m < M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
      if (nk < nkb) {
        // stream-K: a part of the tile's K. The fp32 partial and sum(h^2) go to
        // the tile's slot; the last CTA to arrive sums the slots.
        float* sp = p.part + (static_cast<size_t>(t) * p.max_seg + slot) * SLOT_FLOATS;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t a0[16], a1[16];
          tmem_ld16(tbase + cc * 32, a0);
          tmem_ld16(tbase + cc * 32 + 16, a1);
          tmem_ld_wait();
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            float* dst = sp + (static_cast<size_t>(cc * 4 + g8) * BM + row_local) * 8;
            float4 lo4, hi4;
            const uint32_t* src = g8 < 2 ? a0 + g8 * 8 : a1 + (g8 - 2) * 8;
            lo4.x = __uint_as_float(src[0]); lo4.y = __uint_as_float(src[1]);
            lo4.z = __uint_as_float(src[2]); lo4.w = __uint_as_float(src[3]);
            hi4.x = __uint_as_float(src[4]); hi4.y = __uint_as_float(src[5]);
            hi4.z = __uint_as_float(src[6]); hi4.w = __uint_as_float(src[7]);
            reinterpret_cast<float4*>(dst)[0] = lo4;
            reinterpret_cast<float4*>(dst)[1] = hi4;
          }
        }
        if (NORM == kRMSNorm) sp[BM * BN + row_local] = ssq;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->tempty[b]);
        // arrival (as in the small-M kernel: the epilogue mbarrier orders the
        // slot stores before thread et 0's acquire-release atomic)
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
          if (segs.done()) {   // the CTA's last segment: summed by all warps below
            if (et == 0) {
              ctrl->fin_t = t;
              ctrl->fin_nseg = nseg;
              ctrl->fin_go = 1;
            }
          } else {
            k2_reduce_tile<EPI, NORM, NUM_EPI_WARPS * 32>(p, t, nseg, et, num_m, num_n);
            if (et == 0) p.counters[t] = 0u;
          }
        }
        continue;
      }
      float scale = 1.f;
      if (NORM == kRMSNorm) {
        scale = 1.f / sqrtf(ssq / static_cast<float>(K) + p.eps);
        if (nb == 0 && row_ok && p.rstd_out != nullptr) p.rstd_out[m] = scale;
      }
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
  } else if (NORM != kNoNorm) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - WARP_CONV0 * 32;   // 0 .. NUM_CONV_WARPS*32-1
    const int c = ct & 7;                            // 16-byte chunk of the 128-byte row
    const int rbase = ct >> 3;                       // rows rbase + ROW_STRIDE j (< BM)
    constexpr int RPT = ROWS_PER_THREAD;
    if (NORM == kLayerNorm) pdl_wait();              // statistics come from the previous kernel
    uint32_t s = 0, ph = 0;
    int i = 0;
    bool ok = true;
    Segs segs = make_segs(sk, tiles, nkb);
    int t, kb0, nk, slot, nseg;
    while (ok && segs.next(t, kb0, nk, slot, nseg)) {
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
      for (int kb = kb0; kb < kb0 + nk; ++kb) {
        if (!warp_wait(&ctrl->full_x[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
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
        if (!warp_wait(&ctrl->tempty[b], (use & 1) ^ 1, abortf, p.status, kStatusWaitTmemEmpty, p.wait_ns)) break;
        if (c == 0) {   // the segment's sum(h^2) per row; the epilogue turns it into 1/rms
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            const int row = rbase + ROW_STRIDE * j;
            if (row < BM) ctrl->rs[b][row] = sst[j];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull[b]);
      }
      ++i;
    }
  }

  // Every role's loop is over (each bounded wait returns), so all warps meet
  // here; a tile completed by this CTA's last stream-K segment is summed by all.
  __syncthreads();
  if (ctrl->fin_go && *abortf == 0) {
    k2_reduce_tile<EPI, NORM, NUM_THREADS>(p, ctrl->fin_t, ctrl->fin_nseg, threadIdx.x, num_m, num_n);
    if (threadIdx.x == 0) p.counters[ctrl->fin_t] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fnl
