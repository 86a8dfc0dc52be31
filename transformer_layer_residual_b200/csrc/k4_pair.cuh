// K4: large-M fused norm + GEMM + epilogue on CTA pairs (tcgen05 cta_group::2).
//
// Same dataflow as the 128 x 512 kernel (TMA x / residual / W tiles ->
// converter warps build the normalised bf16 operand in shared memory ->
// tcgen05.mma into TMEM -> fused epilogue), with the pair tile spread over two
// CTAs of a cluster: 256 tokens x 512 W rows (SwiGLU: 256 gate rows + the
// matching 256 up rows). Each CTA holds its 128 tokens' x, residual and
// normalised operand, and half of each weight operand; the pair's even CTA
// issues tcgen05.mma.cta_group::2 M=256 N=256 K=16, which reads A from both
// CTAs' shared memory (128 rows each) and B from both (128 of the 256 W rows
// each) and writes each CTA's 128 accumulator rows into its own TMEM. Per CTA
// and 32-wide k-block that is x 8 KB + residual 8 KB + W 16 KB of tensor copies
// and 32 KB of UMMA operand reads for 512 tensor cycles, against 48 KB and
// 48 KB in the single-CTA 128 x 512 kernel: shared-memory bytes per FLOP, the
// bound of the fused operand's pipeline, drop by about a quarter.
//
// Two rings per CTA. The operand ring (OST slots: normalised A [+ its lo part
// for the split form], W half 0, W half 1) holds what the UMMA reads; a slot is
// refilled once the UMMA that read it has completed. The raw ring (RST slots:
// x, residual and the gamma / beta / bias_in slices) only feeds the
// converters, and a raw slot is refilled as soon as its converters have read
// it. So the activation copies run ahead of the UMMA, and an operand slot's
// turnaround (UMMA done -> W copy and conversion -> next UMMA) no longer
// includes the activation copy's latency: on B200 that turnaround was about
// 1.1 us against 6 x 0.31 us of tensor work buffered, and the tensor pipe
// waited on the ring for about 40% of the time when both copies sat in one slot.
//
// Warp roles (15 warps per CTA): 0 raw-ring producer (x, residual, vectors),
// 1 TMEM (allocated for the pair) and, in the even CTA, UMMA issuer; 2-5
// epilogue (own 128 rows); 6-13 converters, in two groups of four that take
// alternate positions (the conversion latency of one position overlaps the
// next); 14 operand-ring producer (W halves; without a norm also the
// activation tile, which is the operand as loaded). An operand slot is ready
// for the UMMA when both CTAs' converters have built their operand and seen
// their own weight halves land: every converter warp of the position's group in
// both CTAs arrives on the even CTA's conv[s] after waiting for its CTA's
// full_w[s], so no tensor copy ever signals the other CTA and each CTA drains
// only its own copies. The UMMA commits arrive on both CTAs' empty[s] / tfull
// (multicast commit); the epilogue warps of both CTAs arrive on the even
// CTA's tempty. RMSNorm uses the deferred scale of the other kernels (each
// CTA's converters sum h^2 of its rows for its own epilogue); LayerNorm
// statistics come from the statistics kernel. A wait that gives up raises the
// abort flag of both CTAs; both CTAs meet at a cluster barrier after their role
// loops (and after the last UMMA completed), so neither leaves while the other
// may still touch its shared memory.
//
// Work split: each pair takes whole tiles in turn, or, when the tiles fill the
// pairs' waves poorly (70B QKV at M = 256: 20 tiles for 74 pairs; M = 2048: 2.2
// waves), stream-K: the (tile, k-block) units are dealt evenly over the pairs.
// A pair that holds only part of a tile's k-blocks stores its fp32 partial sums
// in a slot and moves on; the fix-up kernel k6_pair_fixup, launched right after,
// adds each split tile's slots in slot order and runs the epilogue, spread over
// the whole GPU. (Summed inside this kernel by the last pair to arrive, the
// gather of up to 5 x 256 KB of partial sums per CTA through L2 ran on 128
// threads of one pair and held that pair's next segment: 70B QKV at M = 256
// took 187 us, against 85 us for the 128 x 256 stream-K kernel.)
#pragma once

#include "common.cuh"

namespace fnl {
namespace k4 {

constexpr int BM = 128;            // tokens per CTA (256 per pair)
constexpr int BN = 512;            // W rows per pair tile (all in each CTA's TMEM)
constexpr int BK = 32;             // k-block: 64-byte rows, 64-byte swizzle
constexpr int X_BYTES = BM * BK * 2;              // 8 KB: x, residual, A or lo(A) of one k-block
constexpr int WH_BYTES = 128 * BK * 2;            // 8 KB: one 128-row half of an N=256 operand
constexpr int RAW_BYTES = 2 * X_BYTES;            // raw slot: x, residual
// operand ring: A [lo(A)] W0 W1; the split form's larger slots leave room for fewer
__host__ __device__ constexpr int op_stages(bool split) { return split ? 5 : 6; }
__host__ __device__ constexpr int raw_stages(bool split) { return split ? 3 : 4; }
__host__ __device__ constexpr int op_a_bytes(bool split) { return (split ? 2 : 1) * X_BYTES; }
__host__ __device__ constexpr int op_bytes(bool split) { return op_a_bytes(split) + 2 * WH_BYTES; }
constexpr int MAX_OST = 6, MAX_RST = 4;
constexpr int RINGS_BYTES = 6 * (X_BYTES + 2 * WH_BYTES) + 4 * RAW_BYTES;   // 208 KB (the split form: the same)
static_assert(op_stages(true) * op_bytes(true) + raw_stages(true) * RAW_BYTES == RINGS_BYTES, "ring sizes");
static_assert(op_stages(false) * op_bytes(false) + raw_stages(false) * RAW_BYTES == RINGS_BYTES, "ring sizes");
constexpr int VEC = BK;
constexpr int VEC_STAGE_BYTES = 3 * VEC * 2;
constexpr int VEC_BYTES = MAX_RST * VEC_STAGE_BYTES;
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_EPI0 = 2, NUM_EPI_WARPS = 4;
constexpr int WARP_CONV0 = 6, NUM_CONV_WARPS = 8;
constexpr int WARP_WTMA = WARP_CONV0 + NUM_CONV_WARPS;                  // 14
constexpr int CONV_GROUPS = 2;                                          // positions converted at once
constexpr int CONV_GROUP_WARPS = NUM_CONV_WARPS / CONV_GROUPS;          // 4
constexpr int CONV_GROUP_THREADS = CONV_GROUP_WARPS * 32;               // 128
constexpr int CONV_ROWS_PER_PASS = CONV_GROUP_THREADS / 4;              // 32 rows x 4 chunks
constexpr int NUM_THREADS = (WARP_WTMA + 1) * 32;   // 480
// The epilogue is shared by the epilogue warps and each converter group for
// LayerNorm and for the no-norm projection (on B200: LayerNorm + GELU 0.60 ->
// 0.64 of the sustained tensor peak, the down projection 0.96 -> 0.99). Not with
// RMSNorm: there the converters also carry the h^2 sums, the shared form needs
// more registers than the 128 a thread of this 480-thread CTA can have, and in
// the long power-capped runs the busier SM clocked lower and lost 2-3%. Nor in
// the split form, which is bound by the tensor pipe (two UMMAs per operand).
__host__ __device__ constexpr int epi_shares(bool split, int norm) {
  return (split || norm == kRMSNorm) ? 1 : 1 + CONV_GROUPS;
}
constexpr int TMEM_COLS = 512;
constexpr int GROUP_M = 8;         // pair rows (of 256 tokens) sharing a W tile while it is hot in L2

struct Ctrl {
  uint64_t full_w[MAX_OST], conv[MAX_OST], empty[MAX_OST];   // operand ring
  uint64_t raw_full[MAX_RST], raw_empty[MAX_RST];            // raw ring
  uint64_t tfull, tempty, sfull[2], efree[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  float rs[2][CONV_GROUPS][BM];   // RMSNorm: per segment buffer, per converter group, sum of h^2 per row
};
constexpr int SMEM_BYTES = RINGS_BYTES + VEC_BYTES + static_cast<int>(sizeof(Ctrl)) + 1024;

__device__ __forceinline__ void tile_coords(int t, int num_m2, int num_n, int& mb2, int& nb) {
  const int per_group = GROUP_M * num_n;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(GROUP_M, num_m2 - first_m);
  const int r = t - group * per_group;
  mb2 = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > FNL_WAIT_NS) return false;
  }
  return true;
}

// The pair's work as segments (tile t, k-blocks [kb0, kb0 + nk), slot, nseg):
// whole tiles t = pair, pair + npairs, ... below `full` (nseg = 1), then, with
// stream-K, the contiguous units [pair U / G, (pair + 1) U / G) of the U =
// (tiles - full) x nkb (tile, k-block) units of the remaining tiles, cut at tile
// boundaries, where slot is this pair's index among the nseg pairs that share
// tile t. The whole waves keep the pairs on neighbouring tiles (their W and
// activation tiles stay in L2); only the last, partial wave is split.
struct PairSegs {
  long long u, u1, U;
  int nkb, G, g, t, full;
  bool sk;
  __device__ PairSegs(bool sk_, int full_, int tiles, int nkb_, int G_, int g_)
      : u(0), u1(0), U(static_cast<long long>(tiles - full_) * nkb_), nkb(nkb_), G(G_), g(g_), t(g_),
        full(full_), sk(sk_) {
    if (sk) {
      u = static_cast<long long>(g) * U / G;
      u1 = static_cast<long long>(g + 1) * U / G;
    }
  }
  __device__ int positions() const {
    const int whole = g < full ? ((full - 1 - g) / G + 1) * nkb : 0;
    return whole + static_cast<int>(u1 - u);
  }
  // slot storage index of tile t (stream-K tiles only)
  __device__ int sk_tile(int tt) const { return tt - full; }
  __device__ bool next(int& tt, int& kb0, int& nk, int& slot, int& nseg) {
    if (t < full) {
      tt = t;
      kb0 = 0;
      nk = nkb;
      slot = 0;
      nseg = 1;
      t += G;
      return true;
    }
    if (u >= u1) return false;
    const int ts = static_cast<int>(u / nkb);   // index among the split tiles
    tt = full + ts;
    kb0 = static_cast<int>(u - static_cast<long long>(ts) * nkb);
    const long long tile_end = static_cast<long long>(ts + 1) * nkb;
    const long long e = tile_end < u1 ? tile_end : u1;
    nk = static_cast<int>(e - u);
    const int first = unit_owner_fast(static_cast<long long>(ts) * nkb, G, U);
    const int last = unit_owner_fast(tile_end - 1, G, U);
    slot = g - first;
    nseg = last - first + 1;
    u = e;
    return true;
  }
};

// The producers' walk over the pair's positions: tile coordinates and k-block
// of each (tile, k-block) unit in order.
struct PosCur {
  PairSegs segs;
  int num_m2, num_n, t, kb, kb_end, mb2, nb;
  __device__ PosCur(const PairSegs& s_, int num_m2_, int num_n_) : segs(s_), num_m2(num_m2_), num_n(num_n_) {
    kb = kb_end = 0;
    step();
  }
  __device__ void step() {
    if (++kb < kb_end) return;
    int kb0, nk, slot, nseg;
    if (segs.next(t, kb0, nk, slot, nseg)) {
      kb = kb0;
      kb_end = kb0 + nk;
      tile_coords(t, num_m2, num_n, mb2, nb);
    }
  }
};

}  // namespace k4

template <int EPI, int NORM, bool SPLIT>
__global__ void __launch_bounds__(k4::NUM_THREADS, 1)
    k4_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                   const __grid_constant__ CUtensorMap tm_w, const OpParams p) {
  using namespace k4;
  constexpr int OST = op_stages(SPLIT), RST = raw_stages(SPLIT);
  constexpr int OPB = op_bytes(SPLIT), OPA = op_a_bytes(SPLIT);
  constexpr int EPI_SHARES = epi_shares(SPLIT, NORM);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* raw = smem + OST * OPB;                                        // [RST][x | residual]
  bf16* vecs = reinterpret_cast<bf16*>(smem + RINGS_BYTES);               // [RST][3][32]
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + RINGS_BYTES + VEC_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();       // 0: the pair's UMMA issuer
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;
  const bool has_beta = NORM == kLayerNorm && p.beta != nullptr;
  const bool has_bias_in = EPI == kEpiGELU && p.bias_in != nullptr;
  constexpr bool BIAS_IN = EPI == kEpiGELU;

  const int M = p.M, K = p.K;
  const int num_m2 = (M + 2 * BM - 1) / (2 * BM);
  const int num_n = (EPI == kEpiSwiGLU) ? (p.I + 255) / 256 : (p.N + BN - 1) / BN;
  const int tiles = num_m2 * num_n;
  const int nkb = (K + BK - 1) / BK;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const PairSegs segs0(p.sk != 0, p.sk != 0 ? p.sk_full : tiles, tiles, nkb, npairs, pair);
  const int P = segs0.positions();   // positions (tile, k-block) of this CTA

  if (threadIdx.x == 0) {
    pdl_launch_dependents();
    for (int s = 0; s < OST; ++s) {
      mbar_init(&ctrl->full_w[s], 1);
      mbar_init(&ctrl->conv[s], 2 * CONV_GROUP_WARPS);   // (even CTA) one group's warps of both CTAs
      mbar_init(&ctrl->empty[s], 1);                     // multicast UMMA commit
    }
    for (int r = 0; r < RST; ++r) {
      mbar_init(&ctrl->raw_full[r], 1);
      mbar_init(&ctrl->raw_empty[r], CONV_GROUP_WARPS);  // the warps of the group that converted it
    }
    mbar_init(&ctrl->tfull, 1);
    mbar_init(&ctrl->tempty, 2 * NUM_EPI_WARPS * EPI_SHARES);   // (even CTA) every epilogue share of both CTAs
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->sfull[b], NUM_CONV_WARPS);
      mbar_init(&ctrl->efree[b], NUM_EPI_WARPS);
    }
    mbar_init(&ctrl->drain, 1);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_r);
  }
  if (warp == WARP_WTMA && lane == 0) prefetch_tmap(&tm_w);
  if (warp == WARP_MMA) {
    tmem_alloc_pair(&ctrl->tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  zero_vec_slices(vecs, RST * 3 * VEC);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int* abortf = &ctrl->abort_flag;
  // a wait that gave up (or saw the flag) also stops the other CTA of the pair
  auto abort_pair = [&]() { st_remote_u32(&ctrl->abort_flag, peer, 1u); };

  // The epilogue of the pair's i-th segment (tile t, slot of nseg) for this
  // warp's TMEM lane quarter (rows q32 .. q32 + 31 of the CTA's 128): share j of
  // EPI_SHARES, 16-column chunks cc = j, j + EPI_SHARES, ... The epilogue warps
  // take share 0; with EPI_SHARES > 1 the converter warps, idle while the UMMA
  // waits for the accumulator, take shares 1 and 2 (group 0 and 1) before they
  // start on the next segment. Every taking warp of both CTAs arrives on the
  // even CTA's tempty.
  // A segment that is only part of its tile's k-blocks (stream-K, nseg > 1)
  // stores this CTA's 128 rows of partial sums (fp32 [128][512], and the rows'
  // partial sums of h^2) in its slot instead; k6_pair_fixup finishes the tile.
  auto epilogue_share = [&](int i, int t, int slot, int nseg, int j) -> bool {
    const int q32 = (warp & 3) * 32;
    const int row_local = q32 + lane;
    if (!warp_wait(&ctrl->tfull, static_cast<uint32_t>(i) & 1, abortf, p.status, kStatusWaitTmemFull,
                   p.wait_ns)) {
      if (lane == 0) abort_pair();
      return false;
    }
    float ssum = 0.f;   // RMSNorm: this segment's sum of h^2 of the row
    if (NORM == kRMSNorm) {
      const int b = i & 1;
      if (!warp_wait(&ctrl->sfull[b], static_cast<uint32_t>(i >> 1) & 1, abortf, p.status, kStatusWaitStats,
                     p.wait_ns)) {
        if (lane == 0) abort_pair();
        return false;
      }
#pragma unroll
      for (int g = 0; g < CONV_GROUPS; ++g) ssum += ctrl->rs[b][g][row_local];   // fixed order
      __syncwarp();
      if (j == 0 && lane == 0) mbar_arrive(&ctrl->efree[b]);   // the converters may refill rs[b] (see below)
    }
    tc_fence_after();
    int mb2, nb;
    tile_coords(t, num_m2, num_n, mb2, nb);
    const int m = mb2 * 2 * BM + static_cast<int>(rank) * BM + row_local;
    const bool row_ok = m < M;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(q32) << 16);
    // TMEM column of 16-column chunk cc: the gate and up halves for SwiGLU
    constexpr int NCH = EPI == kEpiSwiGLU ? 16 : BN / 16;
    const bool partial = nseg > 1;
    if (partial) {
      // slot `slot` of this tile half: 128 rows x 512 fp32 partial sums, 128 partial sums of h^2
      const size_t half =
          (static_cast<size_t>(segs0.sk_tile(t)) * p.max_seg + static_cast<size_t>(slot)) * 2 + rank;
      float* own = p.part + (half * BM + row_local) * 512;
#pragma unroll 1
      for (int cc = j; cc < NCH; cc += EPI_SHARES) {
        uint32_t a0[16];
        tmem_ld16(tbase + cc * 16, a0);
        if (EPI == kEpiSwiGLU) {
          uint32_t u0[16];
          tmem_ld16(tbase + 256 + cc * 16, u0);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            *reinterpret_cast<uint4*>(own + cc * 16 + e) = make_uint4(a0[e], a0[e + 1], a0[e + 2], a0[e + 3]);
            *reinterpret_cast<uint4*>(own + 256 + cc * 16 + e) = make_uint4(u0[e], u0[e + 1], u0[e + 2], u0[e + 3]);
          }
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<uint4*>(own + cc * 16 + e) = make_uint4(a0[e], a0[e + 1], a0[e + 2], a0[e + 3]);
        }
      }
      if (NORM == kRMSNorm && j == 0) p.part_ss[half * BM + row_local] = ssum;
    } else {
      float scale = 1.f;
      if (NORM == kRMSNorm) scale = 1.f / sqrtf(ssum / static_cast<float>(K) + p.eps);
      if (NORM == kRMSNorm && j == 0 && nb == 0 && row_ok && p.rstd_out != nullptr) p.rstd_out[m] = scale;
      auto gather16 = [&](int col, float (&v)[16]) {
        uint32_t a0[16];
        tmem_ld16(tbase + col, a0);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(a0[e]);
      };
      // 16-column chunks: few registers held, so the converter warps can take shares without spilling
      if (EPI == kEpiSwiGLU) {
#pragma unroll 1
        for (int cc = j; cc < NCH; cc += EPI_SHARES) {
          float g0[16], u0[16];
          gather16(cc * 16, g0);
          gather16(256 + cc * 16, u0);
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
              const int jj = nb * 256 + cc * 16 + g8 * 8;
              if (jj < p.I) {
                float gv[8], uv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  gv[e] = g0[g8 * 8 + e];
                  uv[e] = u0[g8 * 8 + e];
                }
                store_swiglu8(p, m, jj, gv, uv, scale);
              }
            }
          }
        }
      } else {
#pragma unroll 1
        for (int cc = j; cc < NCH; cc += EPI_SHARES) {
          float a0[16];
          gather16(cc * 16, a0);
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
              const int n = nb * BN + cc * 16 + g8 * 8;
              if (n < p.N) {
                float av[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) av[e] = a0[g8 * 8 + e];
                store_out8<EPI>(p, m, n, av, scale);
              }
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {   // the pair's accumulator may be overwritten once every share of both CTAs is done
      if (leader) mbar_arrive(&ctrl->tempty);
      else mbar_arrive_remote(&ctrl->tempty, 0);
    }
    return true;
  };

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ raw-ring producer (own rows)
    if (lane == 0 && NORM != kNoNorm) {
      uint32_t armed = 0, par = 0;
      bool ok = true;
      PosCur c(segs0, num_m2, num_n);
      pdl_wait();   // activations may be written by the previous kernel
      for (int q = 0; q < P; ++q, c.step()) {
        const int r = q % RST;
        const uint32_t ph = static_cast<uint32_t>(q / RST) & 1u;
        if (q >= RST &&
            !mbar_wait(&ctrl->raw_empty[r], ph ^ 1u, abortf, p.status, kStatusWaitEmpty, p.wait_ns)) {
          ok = false;
          break;
        }
        uint8_t* st = raw + r * RAW_BYTES;
        const int k0 = c.kb * BK;
        const int row0 = c.mb2 * 2 * BM + static_cast<int>(rank) * BM;
        bf16* vec = vecs + r * 3 * VEC;
        const uint32_t vb = static_cast<uint32_t>(min(VEC, K - k0)) * 2;
        const uint32_t nvec = 1 + (has_beta ? 1 : 0) + (has_bias_in ? 1 : 0);
        mbar_arrive_expect_tx(&ctrl->raw_full[r], 2 * X_BYTES + vb * nvec);
        bulk_load(vec, p.gamma + k0, vb, &ctrl->raw_full[r]);
        if (has_beta) bulk_load(vec + VEC, p.beta + k0, vb, &ctrl->raw_full[r]);
        if (has_bias_in) bulk_load(vec + 2 * VEC, p.bias_in + k0, vb, &ctrl->raw_full[r]);
        tma_load_2d(st, &tm_x, &ctrl->raw_full[r], k0, row0);
        tma_load_2d(st + X_BYTES, &tm_r, &ctrl->raw_full[r], k0, row0);
        armed |= 1u << r;
        par = (par & ~(1u << r)) | (ph << r);
      }
      if (!ok) {
        abort_pair();
        for (int i = 0; i < RST; ++i)   // let every issued copy land before the CTA can exit
          if (armed & (1u << i)) drain_wait(&ctrl->raw_full[i], (par >> i) & 1);
      }
    }
  } else if (warp == WARP_WTMA) {
    // ------------------------------------------------------------ operand-ring producer (own halves)
    if (lane == 0) {
      const int npre = P < OST ? P : OST;
      uint32_t armed = 0, par = 0;
      bool ok = true;
      // fault injection (status-path tests only): CTA 0 withholds position 0's copies
      const int skip = (p.stall != 0 && blockIdx.x == 0) ? 0 : -1;
      PosCur cw(segs0, num_m2, num_n), cx = cw;
      auto step = [&](PosCur& c) { c.step(); };
      // one arrive_expect_tx per slot use: the W halves (+ the activation tile without a norm)
      auto arm = [&](int q) {
        if (q == skip) return;
        const int s = q % OST;
        const uint32_t ph = static_cast<uint32_t>(q / OST) & 1u;
        mbar_arrive_expect_tx(&ctrl->full_w[s], 2 * WH_BYTES + (NORM == kNoNorm ? X_BYTES : 0));
        armed |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      };
      auto issue_w = [&](int q, const PosCur& c) {
        if (q == skip) return;
        const int s = q % OST;
        uint8_t* st = smem + s * OPB + OPA;
        // this CTA's 128-row halves of the two N=256 operands
        int r0, r1;
        if (EPI == kEpiSwiGLU) {
          r0 = c.nb * 256 + static_cast<int>(rank) * 128;          // gate rows
          r1 = p.I + c.nb * 256 + static_cast<int>(rank) * 128;    // the matching up rows
        } else {
          r0 = c.nb * BN + static_cast<int>(rank) * 128;
          r1 = c.nb * BN + 256 + static_cast<int>(rank) * 128;
        }
        tma_load_2d(st, &tm_w, &ctrl->full_w[s], c.kb * BK, r0);
        tma_load_2d(st + WH_BYTES, &tm_w, &ctrl->full_w[s], c.kb * BK, r1);
      };
      auto issue_x = [&](int q, const PosCur& c) {   // no norm: the activation tile is the operand
        if (q == skip) return;
        const int s = q % OST;
        tma_load_2d(smem + s * OPB, &tm_x, &ctrl->full_w[s], c.kb * BK,
                    c.mb2 * 2 * BM + static_cast<int>(rank) * BM);
      };
      for (int q = 0; q < npre; ++q) {   // weights stream before the dependency wait
        arm(q);
        issue_w(q, cw);
        step(cw);
      }
      if (NORM == kNoNorm) {
        pdl_wait();
        for (int q = 0; q < npre; ++q) {
          issue_x(q, cx);
          step(cx);
        }
      }
      for (int q = npre; q < P; ++q) {
        const int s = q % OST;
        const uint32_t ph = static_cast<uint32_t>(q / OST) & 1u;
        if (!mbar_wait(&ctrl->empty[s], ph ^ 1u, abortf, p.status, kStatusWaitEmpty, p.wait_ns)) {
          ok = false;
          break;
        }
        arm(q);
        issue_w(q, cw);
        step(cw);
        if (NORM == kNoNorm) {
          issue_x(q, cx);
          step(cx);
        }
      }
      if (!ok) {
        abort_pair();
        for (int i = 0; i < OST; ++i)   // let every issued copy land before the CTA can exit
          if (armed & (1u << i)) drain_wait(&ctrl->full_w[i], (par >> i) & 1);
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issuer (even CTA)
    if (leader && lane == 0) {
      uint32_t s = 0, ph = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16(2 * BM, 256);
      PairSegs segs = segs0;
      int t, kb0, nk, slot, nseg;
      for (int i = 0; ok && segs.next(t, kb0, nk, slot, nseg); ++i) {
        if (!mbar_wait_cluster(&ctrl->tempty, (static_cast<uint32_t>(i) & 1) ^ 1, abortf, p.status,
                               kStatusWaitTmemEmpty, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {   // accumulate from the segment's first k-block
          if (!mbar_wait_cluster(&ctrl->conv[s], ph, abortf, p.status, kStatusWaitConv, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(smem + s * OPB);
          const uint64_t ad = sw64_desc(xa);
          const uint64_t ld = sw64_desc(xa + X_BYTES);
          const uint64_t bd0 = sw64_desc(xa + OPA);
          const uint64_t bd1 = sw64_desc(xa + OPA + WH_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16_pair(tmem, ad + 2 * kk, bd0 + 2 * kk, idesc, acc);
            umma_bf16_pair(tmem + 256, ad + 2 * kk, bd1 + 2 * kk, idesc, acc);
            if (SPLIT) {   // + lo(a) W^T into the same accumulators
              umma_bf16_pair(tmem, ld + 2 * kk, bd0 + 2 * kk, idesc, 1u);
              umma_bf16_pair(tmem + 256, ld + 2 * kk, bd1 + 2 * kk, idesc, 1u);
            }
          }
          umma_commit_pair(&ctrl->empty[s], 0x3);   // the slot is free in both CTAs
          if (++s == static_cast<uint32_t>(OST)) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(&ctrl->tfull, 0x3);
      }
      if (!ok) abort_pair();
      umma_commit_pair(&ctrl->drain, 0x1);   // every issued UMMA done before the pair's exit
      drain_wait(&ctrl->drain, 0);
    }
  } else if (warp < WARP_CONV0) {
    // ------------------------------------------------------------ epilogue (own 128 rows, share 0)
    pdl_wait();
    PairSegs segs = segs0;
    int t, kb0, nk, slot, nseg;
    for (int i = 0; segs.next(t, kb0, nk, slot, nseg); ++i)
      if (!epilogue_share(i, t, slot, nseg, 0)) break;
  } else {
    // ------------------------------------------------------------ converters (own 128 rows)
    // Two groups of four warps: group g converts positions q = g, g + 2, ...
    // of this CTA's (tile, k-block) sequence, reading raw slot q % RST and
    // writing operand slot q % OST, so two positions are converted at once and
    // the conversion latency of one overlaps the next. Thread gt of a group
    // (0..127): 16-byte chunk c = gt & 3 of the 64-byte row, rows rb + 32 j
    // (rb = gt >> 2, j = 0..3). 64-byte swizzle: chunk c of row r sits at
    // c ^ ((r >> 1) & 3). RMSNorm: each group sums h^2 over its k-blocks; the
    // epilogue adds the two groups' sums in group order. Without a norm
    // (residual-stream projection) the warps only relay the slot's readiness
    // to the even CTA. Before segment i + 1 each group takes its share of
    // segment i's epilogue: the UMMA cannot start segment i + 1 before the
    // accumulator is read, so the shares shorten the gap between segments.
    constexpr int RPT = BM / CONV_ROWS_PER_PASS;   // rows per thread (4)
    const int ct = threadIdx.x - WARP_CONV0 * 32;   // 0..255
    const int grp = ct / CONV_GROUP_THREADS;          // 0..CONV_GROUPS-1
    const int gt = ct - grp * CONV_GROUP_THREADS;     // 0..127
    const int c = gt & 3;
    const int rb = gt >> 2;                           // 0..31
    if (NORM == kLayerNorm) pdl_wait();
    int i = 0;
    bool ok = true;
    long long q0 = 0;   // first position of the current segment
    PairSegs segs = segs0;
    int t, kb0, nk, slot, nseg;
    int pt = 0, pslot = 0, pnseg = 1;   // the previous segment, for its epilogue share
    for (; ok && segs.next(t, kb0, nk, slot, nseg); ++i, q0 += nk) {
      // this group's share of the previous segment's epilogue, before any of this segment's state is live
      if (EPI_SHARES > 1 && i > 0 && !epilogue_share(i - 1, pt, pslot, pnseg, 1 + grp)) {
        ok = false;
        break;
      }
      pt = t;
      pslot = slot;
      pnseg = nseg;
      int mb2, nb;
      tile_coords(t, num_m2, num_n, mb2, nb);
      const int mrow0 = mb2 * 2 * BM + static_cast<int>(rank) * BM;
      float mu[RPT], rs[RPT];
      f32x2 ss[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int gm = mrow0 + rb + CONV_ROWS_PER_PASS * j;
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
      // this group's positions of the segment
      for (long long q = q0 + ((grp - q0 % CONV_GROUPS) + CONV_GROUPS) % CONV_GROUPS; q < q0 + nk;
           q += CONV_GROUPS) {
        const int kb = kb0 + static_cast<int>(q - q0);
        const int s = static_cast<int>(q % OST);
        const uint32_t ph = static_cast<uint32_t>(q / OST) & 1u;
        if (NORM != kNoNorm) {
          const int r = static_cast<int>(q % RST);
          const uint32_t rph = static_cast<uint32_t>(q / RST) & 1u;
          // the raw tiles have landed
          if (!warp_wait(&ctrl->raw_full[r], rph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
            ok = false;
            break;
          }
          bf16* vec = vecs + r * 3 * VEC;
          if (K - kb * BK < BK) zero_vec_tails(vec, VEC, K - kb * BK);
          const uint32_t vaddr = smem_u32(vec) + c * 16;
          f32x2 g2[4], be2[4] = {}, bi2[4] = {};
          vec_pairs(vaddr, g2);
          if (NORM == kLayerNorm) vec_pairs(vaddr + 2 * VEC, be2);
          if (BIAS_IN) vec_pairs(vaddr + 4 * VEC, bi2);
          const uint32_t xs = smem_u32(raw + r * RAW_BYTES);
          const uint32_t rsm = xs + X_BYTES;
          uint4 xv[RPT], rv[RPT];
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            const int row = rb + CONV_ROWS_PER_PASS * j;
            const uint32_t off = row * 64 + ((c ^ ((row >> 1) & 3)) << 4);
            xv[j] = ld_shared_v4(xs + off);
            rv[j] = ld_shared_v4(rsm + off);
          }
          // the operand into registers (instantiated with and without the
          // residual_out store of the first N column)
          uint4 hi[RPT], lo[RPT];
          auto convert_rows = [&](auto wres_tag) {
            constexpr bool WRES = decltype(wres_tag)::value;
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
              uint4 hres;
              convert8<(NORM == kNoNorm ? kRMSNorm : NORM), BIAS_IN, SPLIT, WRES>(
                  xv[j], rv[j], g2, be2, bi2, mu[j], rs[j], ss[j], hi[j], lo[j], hres);
              if (WRES) {
                const int gm = mrow0 + rb + CONV_ROWS_PER_PASS * j;
                const int k0 = kb * BK + c * 8;
                if (gm < M && k0 < K) {
                  bf16* dst = p.residual_out + static_cast<size_t>(gm) * K + k0;
                  if (store_in_bounds(p, dst, p.residual_out, static_cast<size_t>(M) * K))
                    *reinterpret_cast<uint4*>(dst) = hres;
                }
              }
            }
          };
          if (write_res) convert_rows(BoolC<true>{});
          else convert_rows(BoolC<false>{});
          // The raw slot may take its next copies now, behind a proxy fence: the
          // fence completes this thread's reads of the slot (the conversion has
          // consumed them) before the tensor copies, which write through the
          // async proxy, can be issued against it. (Released right after the
          // loads were issued and with no fence, the next x tile landed before
          // some loads had read the current one: rows of the operand mixed the
          // next k-block's x with this one's residual.) The slot no longer
          // waits for the UMMA to free an operand slot.
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->raw_empty[r]);
          // the UMMA that last read operand slot s is done: store the operand
          if (q >= OST && !warp_wait(&ctrl->empty[s], ph ^ 1u, abortf, p.status, kStatusWaitEmpty, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t as = smem_u32(smem + s * OPB);
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            const int row = rb + CONV_ROWS_PER_PASS * j;
            const uint32_t off = row * 64 + ((c ^ ((row >> 1) & 3)) << 4);
            st_shared_v4(as + off, hi[j]);
            if (SPLIT) st_shared_v4(as + X_BYTES + off, lo[j]);
          }
          fence_proxy_async_smem();
        }
        // this CTA's weight halves (and, without a norm, its activation tile) have landed
        if (!warp_wait(&ctrl->full_w[s], ph, abortf, p.status, kStatusWaitFull, p.wait_ns)) {
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) {   // this CTA's half of slot s is ready for the pair's UMMA
          if (leader) mbar_arrive(&ctrl->conv[s]);
          else mbar_arrive_remote(&ctrl->conv[s], 0);
        }
      }
      if (!ok) {
        if (lane == 0) abort_pair();
        break;
      }
      if (NORM == kRMSNorm) {
        float sst[RPT];
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          float lo_, hi_;
          unpk2(ss[j], lo_, hi_);
          sst[j] = lo_ + hi_;
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 1);
          sst[j] += __shfl_xor_sync(0xffffffffu, sst[j], 2);
        }
        const int b = i & 1;
        // the epilogue of the segment two back has read rs[b]
        if (!warp_wait(&ctrl->efree[b], (static_cast<uint32_t>(i >> 1) & 1) ^ 1, abortf, p.status,
                       kStatusWaitTmemEmpty, p.wait_ns)) {
          if (lane == 0) abort_pair();
          break;
        }
        if (c == 0) {   // this group's sum of h^2 per row over its k-blocks of the segment
#pragma unroll
          for (int j = 0; j < RPT; ++j) ctrl->rs[b][grp][rb + CONV_ROWS_PER_PASS * j] = sst[j];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sfull[b]);
      }
    }
    // the last segment's share (its epilogue has no next segment to wait behind)
    if (EPI_SHARES > 1 && ok && i > 0) epilogue_share(i - 1, pt, pslot, pnseg, 1 + grp);
  }

  // Every role's loop is over and the even CTA's last UMMA has completed (its
  // issuer waited for it): meet the other CTA, then free the pair's TMEM.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- K6
// Fix-up of the pair kernel's split tiles (its stream-K form), launched right
// after it as its programmatic dependent. For split tile ts (tile sk_full + ts
// of the pair raster) the nseg pairs that held its k-blocks each stored, per
// CTA half and slot, 128 rows x 512 fp32 partial sums and the rows' 128
// partial sums of h^2. One CTA per (split tile, half, 16-row group); each
// thread adds the slots of its 8-column chunks in slot order (the result does
// not depend on which pair finished first) and applies the op's epilogue as
// the pair kernel does: the RMSNorm scale from the summed h^2, then bias and
// the QKV split, SwiGLU, GELU or the residual add. The partial sums were
// written just before, so they are read through L2 (ld.global.cg).
namespace k6 {
constexpr int ROWS = 16;                  // rows of a tile half per CTA
constexpr int GROUPS = k4::BM / ROWS;     // 8 CTAs per tile half
constexpr int THREADS = 256;
}  // namespace k6

template <int EPI, int NORM>
__global__ void __launch_bounds__(k6::THREADS) k6_pair_fixup(const OpParams p, int G) {
  using namespace k4;
  pdl_wait();   // every slot of the pair kernel is stored and visible
  pdl_launch_dependents();
  const int M = p.M, K = p.K;
  const int num_m2 = (M + 2 * BM - 1) / (2 * BM);
  const int num_n = (EPI == kEpiSwiGLU) ? (p.I + 255) / 256 : (p.N + BN - 1) / BN;
  const int nkb = (K + BK - 1) / BK;
  const int full = p.sk_full;
  const long long U = static_cast<long long>(num_m2 * num_n - full) * nkb;
  const int ts = blockIdx.x / (2 * k6::GROUPS);
  const int rank = (blockIdx.x / k6::GROUPS) & 1;
  const int rg = blockIdx.x % k6::GROUPS;
  const int first = unit_owner_fast(static_cast<long long>(ts) * nkb, G, U);
  const int last = unit_owner_fast(static_cast<long long>(ts + 1) * nkb - 1, G, U);
  const int nseg = last - first + 1;
  if (nseg < 2) return;   // one pair held the whole tile and ran its epilogue
  int mb2, nb;
  tile_coords(full + ts, num_m2, num_n, mb2, nb);
  const size_t half0 = static_cast<size_t>(ts) * p.max_seg * 2 + rank;
  // 8-column chunks per row (SwiGLU: gate chunks, each with the matching up chunk)
  constexpr int CH = EPI == kEpiSwiGLU ? 32 : 64;
  constexpr int ITEMS = k6::ROWS * CH / k6::THREADS;
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = threadIdx.x + it * k6::THREADS;
    const int row_local = rg * k6::ROWS + idx / CH;
    const int ch = idx % CH;
    const int m = mb2 * 2 * BM + rank * BM + row_local;
    if (m >= M) continue;
    float scale = 1.f;
    if (NORM == kRMSNorm) {
      float tot = 0.f;
      for (int sl = 0; sl < nseg; ++sl)
        tot += __ldcg(p.part_ss + (half0 + static_cast<size_t>(sl) * 2) * BM + row_local);
      scale = 1.f / sqrtf(tot / static_cast<float>(K) + p.eps);
      if (nb == 0 && ch == 0 && p.rstd_out != nullptr) p.rstd_out[m] = scale;
    }
    auto sum8 = [&](int col, float (&v)[8]) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
      for (int sl = 0; sl < nseg; ++sl) {
        const float* src = p.part + ((half0 + static_cast<size_t>(sl) * 2) * BM + row_local) * 512 + col;
        const float4 a = __ldcg(reinterpret_cast<const float4*>(src));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(src + 4));
        v[0] += a.x;
        v[1] += a.y;
        v[2] += a.z;
        v[3] += a.w;
        v[4] += b.x;
        v[5] += b.y;
        v[6] += b.z;
        v[7] += b.w;
      }
    };
    if (EPI == kEpiSwiGLU) {
      const int jj = nb * 256 + ch * 8;
      if (jj < p.I) {
        float g[8], u[8];
        sum8(ch * 8, g);
        sum8(256 + ch * 8, u);
        store_swiglu8(p, m, jj, g, u, scale);
      }
    } else {
      const int n = nb * BN + ch * 8;
      if (n < p.N) {
        float a[8];
        sum8(ch * 8, a);
        store_out8<EPI>(p, m, n, a, scale);
      }
    }
  }
}

}  // namespace fnl
