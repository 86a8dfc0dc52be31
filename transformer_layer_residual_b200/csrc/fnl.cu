// C-ABI host library for the fused pre-norm linear layer (include/fnl.h).
//
// Host responsibilities: argument validation (alignment, sizes, aliasing),
// the handle's device workspace (status word, split-K arrival counters,
// LayerNorm statistics, split-K partials), TMA tensor-map encoding, the M
// regime choice (small-M split-K kernel vs large-M tile kernel) and the
// launches (the LayerNorm statistics kernel chained to the GEMM kernel by
// programmatic dependent launch).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "fnl.h"
#include "k1_stats.cuh"
#include "k2_tile.cuh"
#include "k2_wide.cuh"
#include "k3_splitk.cuh"
#include "k4_pair.cuh"
#include "k5_tp.cuh"

using fnl::bf16;
using fnl::OpParams;

namespace fnlh {
// A plan: which kernel runs a call, in which form, on how many CTAs.
enum class Kern { K3, K2, K2W, K4, K4S };   // K4S: the pair kernel's stream-K form

struct Plan {
  Kern kern = Kern::K3;
  int grid = 1, threads = 0, smem = 0, mpad = 0, stages = 0, max_seg = 1, T = 0, cls = 0, sk = 0;
  int sk_full = 0;   // pair kernel, stream-K: tiles processed whole before the split ones
};

// Key of the shape auto-tuning cache (see tune()).
struct TuneKey {
  int op, norm, mkey, N, K, I;
  bool operator==(const TuneKey& o) const {
    return op == o.op && norm == o.norm && mkey == o.mkey && N == o.N && K == o.K && I == o.I;
  }
};

struct TunedEntry {
  TuneKey key;
  Plan plan;
  float us;        // median time of the plan when it was tuned
  int candidates;  // plans timed
};
}  // namespace fnlh
using fnlh::Kern;
using fnlh::Plan;
using fnlh::TuneKey;

// Encoded TMA descriptors, keyed by what the encoding depends on. A decode
// loop calls with the same pointers every step, so its three maps are encoded
// once; the table is small and replaced round-robin.
struct MapCache {
  struct Entry {
    const void* ptr;
    long long rows, cols;
    int box_rows, box_cols;
    CUtensorMap map;
  };
  static constexpr int kSize = 32;
  Entry e[kSize];
  int used = 0, next = 0;
  const CUtensorMap* find(const void* ptr, long long rows, long long cols, int br, int bc) const {
    for (int i = 0; i < used; ++i)
      if (e[i].ptr == ptr && e[i].rows == rows && e[i].cols == cols && e[i].box_rows == br && e[i].box_cols == bc)
        return &e[i].map;
    return nullptr;
  }
  void put(const void* ptr, long long rows, long long cols, int br, int bc, const CUtensorMap& m) {
    Entry& x = e[next];
    x.ptr = ptr; x.rows = rows; x.cols = cols; x.box_rows = br; x.box_cols = bc; x.map = m;
    next = (next + 1) % kSize;
    if (used < kSize) ++used;
  }
};

struct fnl_handle {
  int device = 0;
  int num_sms = 148;
  fnl_options opt{};
  uint8_t* ws = nullptr;     // device workspace
  size_t ws_bytes = 0;
  std::string err;
  struct Occ {
    int smem, cls, clusters;
  };
  std::vector<Occ> occ;      // resident clusters of the small-M kernel per (shared memory, cluster size)
  MapCache maps;             // encoded tensor maps of recent calls
  std::string plan_text;     // the last call's plan (fnl_last_plan)
  int pairs = 0;             // resident CTA pairs of the pair kernel (0: not queried yet)
  std::vector<fnlh::TunedEntry> tuned;   // shape auto-tuning cache
};

namespace {

// ------------------------------------------------------------------ workspace
// [status 256 B][counters kMaxTiles * 4 B][stats][part_ss][part]
constexpr size_t kStatusBytes = 256;
constexpr int kMaxTiles = 65536;
constexpr size_t kCountersBytes = static_cast<size_t>(kMaxTiles) * 4;
constexpr size_t kFixedBytes = kStatusBytes + kCountersBytes;
// Largest N (rows of W) any entry point accepts: below kMaxTiles 128-row tiles
// and far below INT_MAX, so every index derived from it fits an int.
constexpr int kMaxN = (kMaxTiles - 1) * 128;

// N = (Hq + 2 Hkv) D computed in 64 bits; 0 when a count is not positive or N
// exceeds kMaxN.
int qkv_columns(int Hq, int Hkv, int D) {
  if (Hq <= 0 || Hkv <= 0 || D <= 0) return 0;
  const long long n = (static_cast<long long>(Hq) + 2LL * Hkv) * D;
  return n <= kMaxN ? static_cast<int>(n) : 0;
}

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

fnl_status fail(fnl_handle* h, fnl_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  return s;
}

fnl_status cuda_fail(fnl_handle* h, cudaError_t e, const char* what) {
  return fail(h, FNL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

fnl_status ensure_workspace(fnl_handle* h, cudaStream_t stream, size_t need) {
  if (need <= h->ws_bytes) return FNL_OK;
  cudaError_t e;
  if (h->ws) {
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(h, e, "cudaDeviceSynchronize");
    cudaFree(h->ws);
    h->ws = nullptr;
    h->ws_bytes = 0;
  }
  const size_t bytes = align256(need + need / 4);
  if ((e = cudaMalloc(&h->ws, bytes)) != cudaSuccess) return cuda_fail(h, e, "cudaMalloc(workspace)");
  if ((e = cudaMemset(h->ws, 0, bytes)) != cudaSuccess) return cuda_fail(h, e, "cudaMemset(workspace)");
  h->ws_bytes = bytes;
  return FNL_OK;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

fnl_status get_encoder(fnl_handle* h) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(h, FNL_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  return FNL_OK;
}

// Row-major bf16 [rows, cols] (cols contiguous), box [box_rows, box_cols] with
// the swizzle the UMMA descriptors expect: 128-byte swizzle for 64-wide boxes,
// 64-byte swizzle for 32-wide boxes; out-of-range elements read 0.
// esize 2: bf16; esize 1: e4m3 codes (uint8). The swizzle span is the box's
// row in bytes (128 or 64).
fnl_status encode_map(fnl_handle* h, CUtensorMap* m, const void* ptr, long long rows, long long cols,
                      int box_rows, int box_cols, int esize = 2) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_cols * esize == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = g_encode(m, esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, FNL_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return FNL_OK;
}

// The map of a [rows, cols] operand at ptr, from the handle's cache when the
// same operand was encoded before (h == NULL: always encoded).
fnl_status make_map(fnl_handle* h, CUtensorMap* m, const void* ptr, long long rows, long long cols,
                    int box_rows, int box_cols = 64, int esize = 2) {
  const int key_cols = box_cols * esize;   // the cache key tells the element sizes apart by the box's bytes
  if (h) {
    if (const CUtensorMap* c = h->maps.find(ptr, rows, cols * esize, box_rows, key_cols)) {
      *m = *c;
      return FNL_OK;
    }
  }
  fnl_status st = encode_map(h, m, ptr, rows, cols, box_rows, box_cols, esize);
  if (st == FNL_OK && h) h->maps.put(ptr, rows, cols * esize, box_rows, key_cols, *m);
  return st;
}

// ------------------------------------------------------------------ validation
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

struct Range {
  const void* p;
  size_t bytes;
  const char* name;
};
bool overlap(const Range& a, const Range& b) {
  if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
  return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

enum class Op { QKV, SwiGLU, GELU, Residual };

struct Call {
  Op op;
  cudaStream_t stream;
  const bf16 *x, *residual, *bias_in, *gamma, *beta, *W, *bias;
  bf16* residual_out;
  fnl_norm norm;
  float eps;
  int M, K, N, I, Hq, Hkv, D;
  bf16 *q, *k, *v, *out;
  float *mean_out, *rstd_out;
  bool fp8;                // FP8 W8A8 form: W holds e4m3 codes (1 byte each), w_scale their row scales
  const float* w_scale;
};

// Residual-stream projection: x = a [M, K], residual [M, N], out [M, N]; out
// may be exactly the residual buffer (each element is read, then written, by
// one thread), any other overlap is rejected.
fnl_status validate_residual(fnl_handle* h, const Call& c) {
  if (c.M < 0 || c.K <= 0 || c.N <= 0) return fail(h, FNL_ERR_INVALID_ARG, "need M >= 0, K > 0, N > 0");
  if (c.K % 8 || c.N % 8) return fail(h, FNL_ERR_ALIGNMENT, "K and N must be multiples of 8 (K=%d N=%d)", c.K, c.N);
  if (c.K > 32768) return fail(h, FNL_ERR_UNSUPPORTED, "K=%d exceeds 32768", c.K);
  if (c.N > kMaxN) return fail(h, FNL_ERR_UNSUPPORTED, "N=%d exceeds %d", c.N, kMaxN);
  if ((h->opt.path == FNL_PATH_SPLITK || h->opt.path == FNL_PATH_SPLITK_CLUSTER) && c.M > fnl::k3::MAX_MPAD)
    return fail(h, FNL_ERR_UNSUPPORTED, "forced split-K path needs M <= %d", fnl::k3::MAX_MPAD);
  if (c.M == 0) return FNL_OK;
  if (!c.x || !c.W || !c.residual || !c.out) return fail(h, FNL_ERR_INVALID_ARG, "a, W, residual and out are required");
  const void* p16[] = {c.x, c.W, c.bias, c.residual, c.out};
  for (const void* p : p16)
    if (p && !al16(p)) return fail(h, FNL_ERR_ALIGNMENT, "a bf16 pointer is not 16-byte aligned");
  const size_t MN = static_cast<size_t>(c.M) * c.N * 2;
  const Range out{c.out, MN, "out"};
  const Range ins[] = {{c.x, static_cast<size_t>(c.M) * c.K * 2, "a"},
                       {c.W, static_cast<size_t>(c.N) * c.K * 2, "W"},
                       {c.bias, static_cast<size_t>(c.N) * 2, "bias"}};
  for (const Range& in : ins)
    if (overlap(out, in)) return fail(h, FNL_ERR_ALIAS, "output out overlaps input %s", in.name);
  if (c.out != c.residual && overlap(out, Range{c.residual, MN, "residual"}))
    return fail(h, FNL_ERR_ALIAS, "out overlaps residual without being the same buffer");
  return FNL_OK;
}

fnl_status validate(fnl_handle* h, const Call& c) {
  if (!h) return FNL_ERR_INVALID_ARG;
  if (c.op == Op::Residual) return validate_residual(h, c);
  if (c.norm != FNL_NORM_LAYERNORM && c.norm != FNL_NORM_RMSNORM)
    return fail(h, FNL_ERR_INVALID_ARG, "norm must be FNL_NORM_LAYERNORM or FNL_NORM_RMSNORM");
  if (!(c.eps > 0.f) || c.eps > 1e30f)   // also rejects NaN
    return fail(h, FNL_ERR_INVALID_ARG, "eps must be finite and > 0 (a constant row has zero variance)");
  if (c.M < 0 || c.K <= 0 || c.N <= 0) return fail(h, FNL_ERR_INVALID_ARG, "need M >= 0, K > 0, N > 0");
  if (c.K % 8 || c.N % 8) return fail(h, FNL_ERR_ALIGNMENT, "K and N must be multiples of 8 (K=%d N=%d)", c.K, c.N);
  if (c.K > 32768) return fail(h, FNL_ERR_UNSUPPORTED, "K=%d exceeds 32768", c.K);
  if (c.op == Op::QKV) {
    if (c.Hq <= 0 || c.Hkv <= 0 || c.D <= 0) return fail(h, FNL_ERR_INVALID_ARG, "Hq, Hkv, D must be > 0");
    if (c.Hq % c.Hkv) return fail(h, FNL_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", c.Hq, c.Hkv);
    if (c.D % 8) return fail(h, FNL_ERR_ALIGNMENT, "D must be a multiple of 8 (D=%d)", c.D);
  }
  if (c.op == Op::SwiGLU && (c.I <= 0 || c.I % 8))
    return fail(h, FNL_ERR_ALIGNMENT, "I must be a positive multiple of 8 (I=%d)", c.I);
  if (c.N > kMaxN) return fail(h, FNL_ERR_UNSUPPORTED, "N=%d exceeds %d", c.N, kMaxN);
  if (c.norm == FNL_NORM_RMSNORM && c.beta)
    return fail(h, FNL_ERR_INVALID_ARG, "beta must be NULL for RMSNorm");
  if (c.norm == FNL_NORM_RMSNORM && c.mean_out)
    return fail(h, FNL_ERR_INVALID_ARG, "mean_out must be NULL for RMSNorm (no mean is computed)");
  if (h->opt.path == FNL_PATH_SPLITK && c.M > fnl::k3::MAX_MPAD)
    return fail(h, FNL_ERR_UNSUPPORTED, "forced split-K path needs M <= %d", fnl::k3::MAX_MPAD);
  if (c.fp8) {
    if (c.M > fnl::k3::MAX_MPAD)
      return fail(h, FNL_ERR_UNSUPPORTED, "the FP8 form runs the small-M kernel: M <= %d", fnl::k3::MAX_MPAD);
    if (h->opt.path != FNL_PATH_AUTO && h->opt.path != FNL_PATH_SPLITK && h->opt.path != FNL_PATH_SPLITK_CLUSTER)
      return fail(h, FNL_ERR_UNSUPPORTED, "the FP8 form has no tile-kernel path");
    if (c.K % 16) return fail(h, FNL_ERR_ALIGNMENT, "FP8: K must be a multiple of 16 (K=%d)", c.K);
  }
  if (c.M == 0) return FNL_OK;
  if (c.fp8) {
    if (!c.w_scale) return fail(h, FNL_ERR_INVALID_ARG, "w_scale is required");
    if (!al16(c.w_scale)) return fail(h, FNL_ERR_ALIGNMENT, "w_scale must be 16-byte aligned");
  }
  // required pointers
  if (!c.x || !c.residual || !c.residual_out || !c.gamma || !c.W)
    return fail(h, FNL_ERR_INVALID_ARG, "x, residual, residual_out, gamma and W are required");
  if (c.op == Op::QKV && (!c.q || !c.k || !c.v)) return fail(h, FNL_ERR_INVALID_ARG, "q, k, v are required");
  if (c.op != Op::QKV && !c.out) return fail(h, FNL_ERR_INVALID_ARG, "out is required");
  const void* p16[] = {c.x, c.residual, c.bias_in, c.gamma, c.beta, c.W, c.bias, c.residual_out,
                       c.q, c.k, c.v, c.out};
  for (const void* p : p16)
    if (p && !al16(p)) return fail(h, FNL_ERR_ALIGNMENT, "a bf16 pointer is not 16-byte aligned");
  if ((c.mean_out && !al4(c.mean_out)) || (c.rstd_out && !al4(c.rstd_out)))
    return fail(h, FNL_ERR_ALIGNMENT, "mean_out / rstd_out must be 4-byte aligned");
  // aliasing: outputs vs inputs and vs each other
  const size_t MK = static_cast<size_t>(c.M) * c.K * 2;
  const size_t n_out = c.op == Op::SwiGLU ? static_cast<size_t>(c.I) : static_cast<size_t>(c.N);
  const Range ins[] = {{c.x, MK, "x"},
                            {c.residual, MK, "residual"},
                            {c.bias_in, static_cast<size_t>(c.K) * 2, "bias_in"},
                            {c.gamma, static_cast<size_t>(c.K) * 2, "gamma"},
                            {c.beta, static_cast<size_t>(c.K) * 2, "beta"},
                            {c.W, static_cast<size_t>(c.N) * c.K * (c.fp8 ? 1 : 2), "W"},
                            {c.bias, static_cast<size_t>(c.N) * 2, "bias"},
                       {c.w_scale, static_cast<size_t>(c.N) * 4, "w_scale"}};
  Range outs[6] = {{c.residual_out, MK, "residual_out"},
                   {c.mean_out, static_cast<size_t>(c.M) * 4, "mean_out"},
                   {c.rstd_out, static_cast<size_t>(c.M) * 4, "rstd_out"}};
  size_t n_outs = 3;
  if (c.op == Op::QKV) {
    outs[n_outs++] = {c.q, static_cast<size_t>(c.Hq) * c.M * c.D * 2, "q"};
    outs[n_outs++] = {c.k, static_cast<size_t>(c.Hkv) * c.M * c.D * 2, "k"};
    outs[n_outs++] = {c.v, static_cast<size_t>(c.Hkv) * c.M * c.D * 2, "v"};
  } else {
    outs[n_outs++] = {c.out, static_cast<size_t>(c.M) * n_out * 2, "out"};
  }
  for (size_t i = 0; i < n_outs; ++i) {
    for (const Range& in : ins)
      if (overlap(outs[i], in))
        return fail(h, FNL_ERR_ALIAS, "output %s overlaps input %s", outs[i].name, in.name);
    for (size_t j = i + 1; j < n_outs; ++j)
      if (overlap(outs[i], outs[j]))
        return fail(h, FNL_ERR_ALIAS, "outputs %s and %s overlap", outs[i].name, outs[j].name);
  }
  return FNL_OK;
}

// ------------------------------------------------------------------ launches
// Dynamic shared-memory limit of each kernel per device, as last set by this
// library (the attribute is per function and device, so the table is
// process-wide). set_smem raises a limit only when it is below what the launch
// needs, so a decode loop pays cudaFuncSetAttribute once.
struct AttrEntry {
  int dev;
  const void* fn;
  int smem;
};
constexpr int kMaxAttrs = 256;
AttrEntry g_attrs[kMaxAttrs];
int g_n_attrs = 0;
std::mutex g_attr_mu;

template <typename Kern>
fnl_status set_smem_exact(fnl_handle* h, int dev, Kern kern, int bytes, bool exact) {
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(g_attr_mu);
  AttrEntry* a = nullptr;
  for (int i = 0; i < g_n_attrs; ++i)
    if (g_attrs[i].dev == dev && g_attrs[i].fn == fn) a = &g_attrs[i];
  if (a && (exact ? a->smem == bytes : a->smem >= bytes)) return FNL_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    if (a) a->smem = -1;   // unknown now
    return cuda_fail(h, e, "cudaFuncSetAttribute");
  }
  if (a) a->smem = bytes;
  else if (g_n_attrs < kMaxAttrs) g_attrs[g_n_attrs++] = {dev, fn, bytes};
  return FNL_OK;
}

template <typename Kern>
fnl_status set_smem(fnl_handle* h, Kern kern, int bytes) {
  int dev = 0;
  if (h) dev = h->device;
  else if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  return set_smem_exact(h, dev, kern, bytes, false);
}

template <typename Kern>
fnl_status launch_gemm(fnl_handle* h, Kern kern, int grid, int threads, int smem, bool pdl, cudaStream_t stream,
                       const CUtensorMap& mx, const CUtensorMap& mr, const CUtensorMap& mw, const OpParams& p) {
  fnl_status st = set_smem(h, kern, smem);
  if (st != FNL_OK) return st;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.cls > 0) {   // the small-M kernel's cluster form
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(p.cls);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mx, mr, mw, p);
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the fused GEMM kernel");
  return FNL_OK;
}

template <int EPI, bool SPLIT>
fnl_status dispatch_gemm_p(fnl_handle* h, bool small, bool rms, int grid, int threads, int smem, bool pdl,
                           cudaStream_t stream, const CUtensorMap& mx, const CUtensorMap& mr, const CUtensorMap& mw,
                           const OpParams& p, bool wide, bool pair) {
  using fnl::kLayerNorm;
  using fnl::kRMSNorm;
  if (pair) {
    if (rms)
      return launch_gemm(h, fnl::k4_pair_kernel<EPI, kRMSNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
    return launch_gemm(h, fnl::k4_pair_kernel<EPI, kLayerNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
  }
  if (wide) {
    if (rms)
      return launch_gemm(h, fnl::k2w_tile_kernel<EPI, kRMSNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
    return launch_gemm(h, fnl::k2w_tile_kernel<EPI, kLayerNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
  }
  if (small) {
    if (rms)
      return launch_gemm(h, fnl::k3_splitk_kernel<EPI, kRMSNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
    return launch_gemm(h, fnl::k3_splitk_kernel<EPI, kLayerNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw,
                       p);
  }
  if (rms)
    return launch_gemm(h, fnl::k2_tile_kernel<EPI, kRMSNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
  return launch_gemm(h, fnl::k2_tile_kernel<EPI, kLayerNorm, SPLIT>, grid, threads, smem, pdl, stream, mx, mr, mw, p);
}

// The operand precision (p.split) selects the kernel instantiation: the hi/lo
// split is a template parameter of every GEMM kernel, so their converter loops
// carry no branch on it.
template <int EPI>
fnl_status dispatch_gemm(fnl_handle* h, bool small, bool rms, int grid, int threads, int smem, bool pdl,
                         cudaStream_t stream, const CUtensorMap& mx, const CUtensorMap& mr, const CUtensorMap& mw,
                         const OpParams& p, bool wide = false, bool pair = false) {
  if (p.split)
    return dispatch_gemm_p<EPI, true>(h, small, rms, grid, threads, smem, pdl, stream, mx, mr, mw, p, wide, pair);
  return dispatch_gemm_p<EPI, false>(h, small, rms, grid, threads, smem, pdl, stream, mx, mr, mw, p, wide, pair);
}

// The residual-stream projection: no norm, residual epilogue, one operand rounding.
fnl_status dispatch_residual(fnl_handle* h, bool small, bool wide, bool pair, int grid, int threads, int smem,
                             bool pdl, cudaStream_t stream, const CUtensorMap& mx, const CUtensorMap& mw,
                             const OpParams& p) {
  using fnl::kEpiResidual;
  using fnl::kNoNorm;
  if (pair)
    return launch_gemm(h, fnl::k4_pair_kernel<kEpiResidual, kNoNorm, false>, grid, threads, smem, pdl, stream, mx, mx,
                       mw, p);
  if (wide)
    return launch_gemm(h, fnl::k2w_tile_kernel<kEpiResidual, kNoNorm, false>, grid, threads, smem, pdl, stream, mx, mx,
                       mw, p);
  if (small)
    return launch_gemm(h, fnl::k3_splitk_kernel<kEpiResidual, kNoNorm, false>, grid, threads, smem, pdl, stream, mx,
                       mx, mw, p);
  return launch_gemm(h, fnl::k2_tile_kernel<kEpiResidual, kNoNorm, false>, grid, threads, smem, pdl, stream, mx, mx,
                     mw, p);
}

// The fix-up of the pair kernel's split tiles (stream-K form), a programmatic
// dependent of the pair kernel: one CTA per (split tile, CTA half, 16 rows).
template <int EPI, int NORM>
fnl_status launch_fixup_t(fnl_handle* h, int T, int pairs, cudaStream_t stream, const OpParams& p) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(T) * 2 * fnl::k6::GROUPS);
  cfg.blockDim = dim3(fnl::k6::THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fnl::k6_pair_fixup<EPI, NORM>, p, pairs);
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the pair kernel's fix-up kernel");
  return FNL_OK;
}

fnl_status launch_fixup(fnl_handle* h, int epi, int norm, int T, int pairs, cudaStream_t stream,
                        const OpParams& p) {
  using namespace fnl;
  if (epi == kEpiResidual) return launch_fixup_t<kEpiResidual, kNoNorm>(h, T, pairs, stream, p);
  const bool rms = norm == kRMSNorm;
  switch (epi) {
    case kEpiQKV:
      return rms ? launch_fixup_t<kEpiQKV, kRMSNorm>(h, T, pairs, stream, p)
                 : launch_fixup_t<kEpiQKV, kLayerNorm>(h, T, pairs, stream, p);
    case kEpiSwiGLU:
      return rms ? launch_fixup_t<kEpiSwiGLU, kRMSNorm>(h, T, pairs, stream, p)
                 : launch_fixup_t<kEpiSwiGLU, kLayerNorm>(h, T, pairs, stream, p);
    default:
      return rms ? launch_fixup_t<kEpiGELU, kRMSNorm>(h, T, pairs, stream, p)
                 : launch_fixup_t<kEpiGELU, kLayerNorm>(h, T, pairs, stream, p);
  }
}

fnl_status launch_k1(fnl_handle* h, const Call& c, float2* stats, cudaStream_t stream) {
  const int nvec = c.K / 8;
  const int v = (nvec + fnl::kK1Threads - 1) / fnl::kK1Threads;
  dim3 grid(c.M), block(fnl::kK1Threads);
#define FNL_K1(MAXV)                                                                                     \
  fnl::k1_layernorm_stats<MAXV><<<grid, block, 0, stream>>>(c.x, c.residual, c.bias_in, c.residual_out, \
                                                            stats, c.mean_out, c.rstd_out, c.M, c.K, c.eps)
  if (v <= 1) FNL_K1(1);
  else if (v <= 2) FNL_K1(2);
  else if (v <= 4) FNL_K1(4);
  else if (v <= 8) FNL_K1(8);
  else FNL_K1(16);
#undef FNL_K1
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the LayerNorm statistics kernel");
  return FNL_OK;
}

int round_up(int a, int b) { return (a + b - 1) / b * b; }

// How many clusters of `cls` CTAs of the small-M kernel (with `smem` bytes of
// shared memory each) the GPU runs at once; cached per handle. Every
// instantiation has one CTA per SM, so one stands for all.
int resident_clusters(fnl_handle* h, int smem, int cls) {
  for (const auto& o : h->occ)
    if (o.smem == smem && o.cls == cls) return o.clusters;
  auto kern = fnl::k3_splitk_kernel<fnl::kEpiQKV, fnl::kRMSNorm, false>;
  int n = 0;
  // the occupancy query needs the limit at exactly `smem` (recorded in the table)
  if (set_smem_exact(h, h->device, kern, smem, true) == FNL_OK) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(cls);
    cfg.blockDim = dim3(fnl::k3::NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = static_cast<unsigned>(cls);
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();   // a refused query leaves no sticky error behind
  h->occ.push_back({smem, cls, n});
  return n;
}

int epi_of(const Call& c) {
  return c.op == Op::QKV ? fnl::kEpiQKV : (c.op == Op::SwiGLU ? fnl::kEpiSwiGLU : fnl::kEpiGELU);
}

// FP8 pre-pass: residual_out, statistics outputs, the per-token (mean, rstd,
// s_a, 448 / amax) and the activation codes q8 [M][K] that the GEMM loads.
fnl_status launch_fp8_prepass(fnl_handle* h, const Call& c, float4* stats8, uint8_t* q8, cudaStream_t stream) {
  const int nvec = c.K / 8;
  const int v = (nvec + fnl::kK1Threads - 1) / fnl::kK1Threads;
  const bool rms = c.norm == FNL_NORM_RMSNORM;
  dim3 grid(c.M), block(fnl::kK1Threads);
#define FNL_PP(MAXV)                                                                                               \
  do {                                                                                                             \
    if (rms)                                                                                                       \
      fnl::k1_fp8_prepass<MAXV, true><<<grid, block, 0, stream>>>(c.x, c.residual, c.bias_in, c.gamma, nullptr,   \
                                                                  c.residual_out, stats8, q8, nullptr, c.rstd_out, \
                                                                  c.M, c.K, c.eps);                                \
    else                                                                                                           \
      fnl::k1_fp8_prepass<MAXV, false><<<grid, block, 0, stream>>>(c.x, c.residual, c.bias_in, c.gamma, c.beta,   \
                                                                   c.residual_out, stats8, q8, c.mean_out,         \
                                                                   c.rstd_out,                                     \
                                                                   c.M, c.K, c.eps);                               \
  } while (0)
  if (v <= 1) FNL_PP(1);
  else if (v <= 2) FNL_PP(2);
  else if (v <= 4) FNL_PP(4);
  else if (v <= 8) FNL_PP(8);
  else FNL_PP(16);
#undef FNL_PP
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the FP8 pre-pass kernel");
  return FNL_OK;
}

// The small-M kernel's FP8 form, for each epilogue.
fnl_status dispatch_fp8(fnl_handle* h, int epi, int grid, int threads, int smem, bool pdl, cudaStream_t stream,
                        const CUtensorMap& mx, const CUtensorMap& mr, const CUtensorMap& mw, const OpParams& p) {
  using fnl::kLayerNorm;
  if (epi == fnl::kEpiSwiGLU)
    return launch_gemm(h, fnl::k3_splitk_kernel<fnl::kEpiSwiGLU, kLayerNorm, false, true>, grid, threads, smem, pdl,
                       stream, mx, mr, mw, p);
  if (epi == fnl::kEpiGELU)
    return launch_gemm(h, fnl::k3_splitk_kernel<fnl::kEpiGELU, kLayerNorm, false, true>, grid, threads, smem, pdl,
                       stream, mx, mr, mw, p);
  return launch_gemm(h, fnl::k3_splitk_kernel<fnl::kEpiQKV, kLayerNorm, false, true>, grid, threads, smem, pdl,
                     stream, mx, mr, mw, p);
}

// ------------------------------------------------------------------ plans

// Largest CTA index range of one tile when U units are dealt evenly over grid
// CTAs, tiles of nkb units each: the number of partial-sum slots per tile.
int max_segments(int T, int nkb, int grid) {
  const long long U = static_cast<long long>(T) * nkb;
  int m = 1;
  for (int t = 0; t < T; ++t) {
    const int first = fnl::unit_owner(static_cast<long long>(t) * nkb, grid, U);
    const int last = fnl::unit_owner(static_cast<long long>(t + 1) * nkb - 1, grid, U);
    m = std::max(m, last - first + 1);
  }
  return m;
}

// Plan of kernel `kern` for call c. Small-M kernel: cls_req < 0 applies the
// automatic rule (the cluster form when its clusters cover the GPU and are all
// resident), 0 forces the stream-K form, >= 2 requests that cluster size
// (FNL_ERR_UNSUPPORTED when its clusters cannot all be resident).
// CTA pairs of the pair kernel resident at once (one CTA per SM); cached per handle.
int resident_pairs(fnl_handle* h) {
  if (h->pairs > 0) return h->pairs;
  auto kern = fnl::k4_pair_kernel<fnl::kEpiQKV, fnl::kRMSNorm, false>;
  int n = 0;
  if (set_smem_exact(h, h->device, kern, fnl::k4::SMEM_BYTES, false) == FNL_OK) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(fnl::k4::NUM_THREADS);
    cfg.dynamicSmemBytes = fnl::k4::SMEM_BYTES;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = 2;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  h->pairs = n > 0 ? n : 0;
  return h->pairs;
}

fnl_status plan_kernel(fnl_handle* h, const Call& c, Kern kern, int cls_req, Plan* pl) {
  const int max_ctas = h->opt.max_ctas > 0 ? std::min(h->opt.max_ctas, h->num_sms) : h->num_sms;
  const int nkb = (c.K + 63) / 64;
  Plan q;
  q.kern = kern;
  if (kern == Kern::K3) {
    if (c.M > fnl::k3::MAX_MPAD) return fail(h, FNL_ERR_UNSUPPORTED, "the small-M kernel needs M <= %d", fnl::k3::MAX_MPAD);
    q.mpad = round_up(std::max(c.M, 1), 16);
    q.T = c.op == Op::SwiGLU ? (c.I + 63) / 64 : (c.N + 127) / 128;
    if (q.T > kMaxTiles) return fail(h, FNL_ERR_UNSUPPORTED, "too many W tiles");
    const long long U = static_cast<long long>(q.T) * nkb;
    q.grid = static_cast<int>(std::min<long long>(max_ctas, U));
    const int sb = c.fp8 ? fnl::k3::stage_bytes8(q.mpad) : fnl::k3::stage_bytes(q.mpad);
    q.stages = std::min(c.fp8 ? fnl::k3::MAX_STAGES_FP8 : fnl::k3::MAX_STAGES, (200 * 1024) / sb);
    q.smem = fnl::k3::smem_bytes(q.mpad, q.stages, c.fp8);
    q.threads = fnl::k3::NUM_THREADS;
    if (cls_req >= 2) {
      if (cls_req > 8 || cls_req > nkb || resident_clusters(h, q.smem, cls_req) < q.T)
        return fail(h, FNL_ERR_UNSUPPORTED, "the %d W tiles cannot run at once as clusters of %d CTAs", q.T, cls_req);
      q.cls = cls_req;
    } else if (cls_req < 0 && h->opt.max_ctas == 0) {
      // Cluster form: one W tile per cluster of cls CTAs, each taking 1/cls of
      // its k-blocks, partial sums reduced on chip. Used when the clusters cover
      // the GPU (or every unit of work) and all of them are resident at once;
      // the largest such cluster size (<= 8, <= the k-blocks).
      for (int c_ = std::min({8, h->num_sms / std::max(q.T, 1), nkb}); c_ >= 2 && q.cls == 0; --c_) {
        const bool covers = static_cast<long long>(q.T) * c_ >= std::min<long long>(U, (h->num_sms * 9) / 10);
        if (covers && resident_clusters(h, q.smem, c_) >= q.T) q.cls = c_;
      }
    }
    if (q.cls > 0) q.grid = q.T * q.cls;
    else q.max_seg = max_segments(q.T, nkb, q.grid);
  } else if (c.fp8) {
    return fail(h, FNL_ERR_UNSUPPORTED, "the FP8 form runs the small-M kernel only");
  } else if (kern == Kern::K4 || kern == Kern::K4S) {
    // CTA pairs, 256 tokens x 512 W rows per pair tile, one pair tile at a time per pair
    const int pairs_max = std::min(resident_pairs(h), max_ctas / 2);
    if (pairs_max <= 0) return fail(h, FNL_ERR_UNSUPPORTED, "the pair kernel cannot be resident");
    const int num_m2 = (c.M + 255) / 256;
    const long long tiles = static_cast<long long>(num_m2) *
                            (c.op == Op::SwiGLU ? (c.I + 255) / 256 : (c.N + fnl::k4::BN - 1) / fnl::k4::BN);
    q.grid = 2 * static_cast<int>(std::min<long long>(pairs_max, tiles));
    // Stream-K form: the whole waves stay whole tiles, and the (tile, 32-wide
    // k-block) units of the tiles left over are dealt evenly over all pairs;
    // the fix-up kernel adds the split tiles' partial sums. Measured on B200:
    // 70B QKV at M = 2048 (2.16 waves) 348 us against 396 with whole tiles; at
    // M = 256 (20 tiles, all split) 90 us against 86 for the 128x256 stream-K
    // kernel; with a last wave more than half full, whole tiles win.
    const long long nkb4 = (c.K + fnl::k4::BK - 1) / fnl::k4::BK;
    if (kern == Kern::K4S) {
      if (tiles * nkb4 < pairs_max)
        return fail(h, FNL_ERR_UNSUPPORTED, "the pair kernel's stream-K form needs a unit per pair");
      const long long full = (tiles / pairs_max) * pairs_max;
      if (2 * (tiles - full) > kMaxTiles) return fail(h, FNL_ERR_UNSUPPORTED, "too many W tiles");
      if (full < tiles) {   // (whole waves only: nothing to split, the plain form)
        q.sk = 1;
        q.sk_full = static_cast<int>(full);
        q.T = static_cast<int>(tiles - full);   // the split tiles (partial-sum slots)
        q.grid = 2 * pairs_max;
        q.max_seg = max_segments(q.T, static_cast<int>(nkb4), pairs_max);
      }
    }
    q.cls = 2;
    q.smem = fnl::k4::SMEM_BYTES;
    q.threads = fnl::k4::NUM_THREADS;
  } else {
    const bool wide = kern == Kern::K2W;
    const int num_m = (c.M + 127) / 128;
    const long long tiles = static_cast<long long>(num_m) *
                            (wide ? (c.op == Op::SwiGLU ? (c.I + 255) / 256 : (c.N + fnl::k2w::BN - 1) / fnl::k2w::BN)
                                  : (c.op == Op::SwiGLU ? (c.I + 127) / 128 : (c.N + fnl::k2::BN - 1) / fnl::k2::BN));
    q.grid = static_cast<int>(std::min<long long>(max_ctas, tiles));
    // Fewer 128x256 tiles than CTAs by a fifth or more (e.g. 70B QKV at
    // M = 256: 80 tiles, 148 SMs): stream-K over (tile, k-block) units, so
    // every SM streams weights; partial tiles are summed by their last CTA.
    if (!wide && tiles * 5 <= static_cast<long long>(max_ctas) * 4) {
      q.sk = 1;
      q.T = static_cast<int>(tiles);
      if (q.T > kMaxTiles) return fail(h, FNL_ERR_UNSUPPORTED, "too many W tiles");
      q.grid = static_cast<int>(std::min<long long>(max_ctas, tiles * nkb));
      q.max_seg = max_segments(q.T, nkb, q.grid);
    }
    q.smem = wide ? fnl::k2w::SMEM_BYTES : fnl::k2::SMEM_BYTES;
    q.threads = wide ? fnl::k2w::NUM_THREADS : fnl::k2::NUM_THREADS;
  }
  *pl = q;
  return FNL_OK;
}

// The plan without tuning: the forced path, else M <= 128 -> small-M kernel,
// else the tile shape whose waves of CTAs fit best.
fnl_status default_plan(fnl_handle* h, const Call& c, Plan* pl) {
  switch (h->opt.path) {
    case FNL_PATH_TILE: return plan_kernel(h, c, Kern::K2, -1, pl);
    case FNL_PATH_TILE_WIDE: return plan_kernel(h, c, Kern::K2W, -1, pl);
    case FNL_PATH_TILE_PAIR: return plan_kernel(h, c, Kern::K4, -1, pl);
    case FNL_PATH_TILE_PAIR_SPLIT: return plan_kernel(h, c, Kern::K4S, -1, pl);
    case FNL_PATH_SPLITK: return plan_kernel(h, c, Kern::K3, 0, pl);
    case FNL_PATH_SPLITK_CLUSTER: {
      // the largest cluster size whose clusters are all resident
      const int T = c.op == Op::SwiGLU ? (c.I + 63) / 64 : (c.N + 127) / 128;
      const int nkb = (c.K + 63) / 64;
      for (int c_ = std::min({8, h->num_sms / std::max(T, 1), nkb}); c_ >= 2; --c_) {
        Plan q;
        if (plan_kernel(h, c, Kern::K3, c_, &q) == FNL_OK) {
          *pl = q;
          return FNL_OK;
        }
      }
      return fail(h, FNL_ERR_UNSUPPORTED, "the %d W tiles cannot run at once as clusters of 2..8 CTAs", T);
    }
    default: break;
  }
  if (c.M <= fnl::k3::MAX_MPAD) return plan_kernel(h, c, Kern::K3, -1, pl);
  // three tile shapes: 256 x 512 on CTA pairs (least shared-memory traffic per
  // FLOP), 128 x 512 and 128 x 256 (finer), picked by how well their tiles
  // fill whole waves of CTAs (pairs): per SM, a 128 x 512 tile takes about
  // 1.6x a 128 x 256 tile and a pair tile about 0.9x a 128 x 512 tile
  // (measured on B200 across the prefill shapes)
  const int max_ctas = h->opt.max_ctas > 0 ? std::min(h->opt.max_ctas, h->num_sms) : h->num_sms;
  const int num_m = (c.M + 127) / 128, num_m2 = (c.M + 255) / 256;
  const long long tiles_n = static_cast<long long>(num_m) *
                            (c.op == Op::SwiGLU ? (c.I + 127) / 128 : (c.N + fnl::k2::BN - 1) / fnl::k2::BN);
  const long long tiles_w = static_cast<long long>(num_m) *
                            (c.op == Op::SwiGLU ? (c.I + 255) / 256 : (c.N + fnl::k2w::BN - 1) / fnl::k2w::BN);
  const long long tiles_p = static_cast<long long>(num_m2) *
                            (c.op == Op::SwiGLU ? (c.I + 255) / 256 : (c.N + fnl::k4::BN - 1) / fnl::k4::BN);
  auto waves = [](long long tiles, long long slots) {
    const long long g = std::min<long long>(slots, tiles);
    return static_cast<double>((tiles + g - 1) / g);
  };
  // the stream-K forms (plan_kernel's rules) spread the units evenly: fractional
  // waves, plus the partial-sum exchange
  auto sk_waves = [](long long tiles, long long slots) { return static_cast<double>(tiles) / slots + 0.15; };
  const double t_n =
      tiles_n * 5 <= static_cast<long long>(max_ctas) * 4 ? sk_waves(tiles_n, max_ctas) : waves(tiles_n, max_ctas);
  const double t_w = 1.6 * waves(tiles_w, max_ctas);
  const int pairs = h->opt.max_ctas == 0 ? resident_pairs(h) : 0;
  const double t_p = pairs > 0 ? 1.45 * waves(tiles_p, pairs) : 1e30;
  // The pair kernel's stream-K form once there is a whole wave: the leftover
  // tiles' units spread over all pairs, at about half a tile's time of extra
  // cost (partial-sum stores, the fix-up kernel; 0.1-0.6 measured on B200 at
  // the prefill shapes: 70B QKV at M = 2048, 2.16 waves, 396 -> 348 us)
  const double t_ps = pairs > 0 && tiles_p >= pairs ? 1.45 * (static_cast<double>(tiles_p) / pairs + 0.5) : 1e30;
  const double t_pair = std::min(t_p, t_ps);
  if (t_pair <= t_w && t_pair <= t_n) return plan_kernel(h, c, t_ps < t_p ? Kern::K4S : Kern::K4, -1, pl);
  return plan_kernel(h, c, t_w <= t_n ? Kern::K2W : Kern::K2, -1, pl);
}

size_t stats_bytes_of(const Call& c) {
  // FP8: (mean, rstd, s_a, 448 / amax) per token, then the tokens' e4m3 activation codes
  if (c.fp8) return align256(static_cast<size_t>(c.M) * 16) + align256(static_cast<size_t>(c.M) * c.K);
  const bool ln = c.op != Op::Residual && c.norm == FNL_NORM_LAYERNORM;
  return ln ? align256(static_cast<size_t>(c.M) * 8) : 0;
}
size_t ss_bytes_of(const Plan& q) {
  // pair kernel, stream-K: per (tile, slot, CTA half) 128 rows' partial sums of h^2
  if (q.kern == Kern::K4 || q.kern == Kern::K4S)
    return q.sk ? align256(static_cast<size_t>(q.T) * q.max_seg * 2 * 128 * 4) : 0;
  return q.kern == Kern::K3 && q.cls == 0 ? align256(static_cast<size_t>(q.T) * q.max_seg * q.mpad * 4) : 0;
}
size_t part_bytes_of(const Plan& q) {
  // pair kernel, stream-K: per (tile, slot, CTA half) 128 x 512 fp32 partial sums
  if (q.kern == Kern::K4 || q.kern == Kern::K4S)
    return q.sk ? align256(static_cast<size_t>(q.T) * q.max_seg * 2 * 128 * 512 * 4) : 0;
  if (q.kern == Kern::K3) return q.cls == 0 ? align256(static_cast<size_t>(q.T) * q.max_seg * q.mpad * 128 * 4) : 0;
  if (q.sk) return align256(static_cast<size_t>(q.T) * q.max_seg * fnl::k2::SLOT_FLOATS * 4);
  return 0;
}
size_t workspace_of(const Call& c, const Plan& q) {
  return kFixedBytes + stats_bytes_of(c) + ss_bytes_of(q) + part_bytes_of(q);
}

const char* kern_name(const Plan& q) {
  switch (q.kern) {
    case Kern::K3: return q.cls > 0 ? "small-M split-K kernel, cluster form" : "small-M split-K kernel, stream-K form";
    case Kern::K2: return q.sk ? "128x256 tile kernel, stream-K" : "128x256 tile kernel";
    case Kern::K4:
    case Kern::K4S: return q.sk ? "256x512 CTA-pair kernel, stream-K" : "256x512 CTA-pair kernel";
    default: return "128x512 tile kernel";
  }
}

// Enqueue call c with plan q (the workspace must already hold workspace_of(c, q)).
fnl_status launch_plan(fnl_handle* h, const Call& c, const Plan& q) {
  fnl_status st;
  const bool nonorm = c.op == Op::Residual;   // residual-stream projection: no add, no norm
  const bool rms = !nonorm && c.norm == FNL_NORM_RMSNORM;
  const bool small = q.kern == Kern::K3, wide = q.kern == Kern::K2W,
             pair = q.kern == Kern::K4 || q.kern == Kern::K4S;
  const size_t sb = stats_bytes_of(c), ssb = ss_bytes_of(q);
  uint8_t* ws = h->ws;
  int* status = reinterpret_cast<int*>(ws);
  unsigned* counters = reinterpret_cast<unsigned*>(ws + kStatusBytes);
  float2* stats = reinterpret_cast<float2*>(ws + kFixedBytes);
  float* part_ss = reinterpret_cast<float*>(ws + kFixedBytes + sb);
  float* part = reinterpret_cast<float*>(ws + kFixedBytes + sb + ssb);

  OpParams p{};
  p.M = c.M; p.K = c.K; p.N = c.N; p.I = c.I; p.Hq = c.Hq; p.Hkv = c.Hkv; p.D = c.D; p.eps = c.eps;
  p.x_in = c.x; p.r_in = nonorm ? nullptr : c.residual;
  p.gamma = c.gamma; p.beta = c.beta; p.bias_in = c.bias_in; p.bias = c.bias;
  p.residual_out = nonorm ? nullptr : c.residual_out; p.rstd_out = rms ? c.rstd_out : nullptr; p.stats = stats;
  p.q = c.q; p.k = c.k; p.v = c.v; p.out = c.out;
  p.res_in = nonorm ? c.residual : nullptr;
  if (c.fp8) {   // the pre-pass writes residual_out and the statistics outputs
    p.stats8 = reinterpret_cast<const float4*>(stats);
    p.fp8_rms = rms ? 1 : 0;
    p.w_scale = c.w_scale;
    p.rstd_out = nullptr;
    p.residual_out = nullptr;
    p.beta = rms ? nullptr : c.beta;
  }
  p.part = part; p.part_ss = part_ss; p.counters = counters; p.max_seg = q.max_seg; p.mpad = q.mpad;
  p.stages = q.stages; p.status = status; p.cls = q.cls; p.sk = q.sk; p.sk_full = q.sk_full;
  p.wait_ns = h->opt.wait_ns > 0 ? static_cast<unsigned long long>(h->opt.wait_ns) : FNL_WAIT_NS;
  p.stall = 0;
  if (h->opt.debug_stall_calls > 0) {   // one-shot fault injection for the status-path tests
    p.stall = 1;
    --h->opt.debug_stall_calls;
  }
  // (the residual-stream projection's operand is bf16 already: nothing to split)
  p.split = !nonorm && (h->opt.precision == FNL_PRECISION_SPLIT ||
                        (h->opt.precision == FNL_PRECISION_DEFAULT && c.op == Op::SwiGLU));

  // tensor maps: x and residual tiles are [rows x 64] ([rows x 32] for the
  // 128x512 kernel), W tiles [rows x 64]
  CUtensorMap mx, mr, mw;
  const int act_rows = small ? q.mpad : fnl::k2::BM;
  int w_rows;
  if (small) w_rows = c.op == Op::SwiGLU ? 64 : fnl::k3::BW;
  else if (wide) w_rows = 256;
  else if (pair) w_rows = 128;   // one CTA's half of an N = 256 operand
  else w_rows = c.op == Op::SwiGLU ? 128 : fnl::k2::BN;
  const int box_cols = wide ? fnl::k2w::BK : (pair ? fnl::k4::BK : 64);
  // FP8: the activation operand is the pre-pass's codes (one byte each), after the per-token scales
  uint8_t* q8 = c.fp8 ? ws + kFixedBytes + align256(static_cast<size_t>(c.M) * 16) : nullptr;
  if (c.fp8) {
    if ((st = make_map(h, &mx, q8, c.M, c.K, act_rows, 64, 1)) != FNL_OK) return st;
    mr = mx;   // unused
  } else {
    if ((st = make_map(h, &mx, c.x, c.M, c.K, act_rows, box_cols)) != FNL_OK) return st;
    if (!nonorm && (st = make_map(h, &mr, c.residual, c.M, c.K, act_rows, box_cols)) != FNL_OK) return st;
  }
  if ((st = make_map(h, &mw, c.W, c.N, c.K, w_rows, box_cols, c.fp8 ? 1 : 2)) != FNL_OK) return st;
  // Every GEMM kernel is a programmatic dependent of its predecessor: it
  // streams its first weight tiles before griddepcontrol.wait and touches
  // activations, statistics, workspace and outputs only after it.
  const bool pdl = true;
  // the pair kernel's stream-K form: its split tiles are finished by the fix-up kernel
  const bool fixup = pair && q.sk != 0 && q.T > 0;
  if (nonorm) {
    st = dispatch_residual(h, small, wide, pair, q.grid, q.threads, q.smem, pdl, c.stream, mx, mw, p);
    if (st == FNL_OK && fixup) st = launch_fixup(h, fnl::kEpiResidual, fnl::kNoNorm, q.T, q.grid / 2, c.stream, p);
    return st;
  }
  if (c.fp8) {
    if ((st = launch_fp8_prepass(h, c, reinterpret_cast<float4*>(stats), q8, c.stream)) != FNL_OK) return st;
    return dispatch_fp8(h, epi_of(c), q.grid, q.threads, q.smem, pdl, c.stream, mx, mr, mw, p);
  }
  if (!rms) {
    if ((st = launch_k1(h, c, stats, c.stream)) != FNL_OK) return st;
  }
  const int epi = c.op == Op::QKV ? fnl::kEpiQKV : (c.op == Op::SwiGLU ? fnl::kEpiSwiGLU : fnl::kEpiGELU);
  switch (epi) {
    case fnl::kEpiQKV:
      st = dispatch_gemm<fnl::kEpiQKV>(h, small, rms, q.grid, q.threads, q.smem, pdl, c.stream, mx, mr, mw, p, wide,
                                       pair);
      break;
    case fnl::kEpiSwiGLU:
      st = dispatch_gemm<fnl::kEpiSwiGLU>(h, small, rms, q.grid, q.threads, q.smem, pdl, c.stream, mx, mr, mw, p,
                                          wide, pair);
      break;
    default:
      st = dispatch_gemm<fnl::kEpiGELU>(h, small, rms, q.grid, q.threads, q.smem, pdl, c.stream, mx, mr, mw, p, wide,
                                        pair);
  }
  if (st == FNL_OK && fixup)
    st = launch_fixup(h, epi, rms ? fnl::kRMSNorm : fnl::kLayerNorm, q.T, q.grid / 2, c.stream, p);
  return st;
}

// ------------------------------------------------------------------ tuner
// Shape auto-tuning (TensorRT-LLM 深度工程实践, §2.4 内核自动调优: candidate
// kernels with different tile shapes are run on the target GPU and the fastest
// is kept; trt-llm-deep-dive, 构建阶段详解 "2. 算子选择": GEMMs are chosen by
// micro-benchmark). With fnl_options.tune, the first call of each shape times
// every candidate plan on the call's stream and caches the fastest for the
// handle. A plan depends on M only through the small-M padding (M <= 128) or
// the count of 128-row blocks, so those key the cache together with the op,
// the norm, the operand precision, N and K.

TuneKey tune_key(const Call& c) {
  TuneKey k;
  k.op = static_cast<int>(c.op);
  k.norm = c.op == Op::Residual ? -1 : static_cast<int>(c.norm);
  k.mkey = c.M <= fnl::k3::MAX_MPAD ? round_up(c.M, 16) : 1000 + (c.M + 127) / 128;
  k.N = c.N; k.K = c.K; k.I = c.I;
  return k;
}

// Time one launch of plan q on c.stream after a write of `flush_bytes` at
// `flush` that evicts the operands from L2 (in a model the weights of a layer
// are not L2-resident when its call starts); us of the launch alone.
fnl_status time_once(fnl_handle* h, const Call& c, const Plan& q, void* flush, size_t flush_bytes, int rep,
                     cudaEvent_t e0, cudaEvent_t e1, float* us) {
  if (flush) cudaMemsetAsync(flush, rep & 0xff, flush_bytes, c.stream);
  cudaEventRecord(e0, c.stream);
  fnl_status st = launch_plan(h, c, q);
  cudaEventRecord(e1, c.stream);
  if (st != FNL_OK) return st;
  cudaError_t e = cudaEventSynchronize(e1);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventSynchronize");
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  *us = ms * 1e3f;
  return FNL_OK;
}

// Same kernel, form and grid.
bool same_plan(const Plan& a, const Plan& b) {
  return a.kern == b.kern && a.cls == b.cls && a.sk == b.sk && a.sk_full == b.sk_full && a.grid == b.grid;
}

fnl_status tune(fnl_handle* h, const Call& c, Plan* best) {
  // candidates: every kernel that takes the shape, the small-M kernel in each
  // of its forms (stream-K and every cluster size whose clusters fit)
  Plan cand[12];
  int n = 0;
  Plan q;
  Plan dflt;
  const bool have_dflt = default_plan(h, c, &dflt) == FNL_OK;
  const bool small_ok = c.M <= fnl::k3::MAX_MPAD;
  if (small_ok) {
    if (plan_kernel(h, c, Kern::K3, 0, &q) == FNL_OK) cand[n++] = q;
    for (int cls = 2; cls <= 8 && n < 10; ++cls)
      if (plan_kernel(h, c, Kern::K3, cls, &q) == FNL_OK) cand[n++] = q;
  }
  if (!c.fp8 && plan_kernel(h, c, Kern::K2, -1, &q) == FNL_OK) cand[n++] = q;
  if (!small_ok && plan_kernel(h, c, Kern::K2W, -1, &q) == FNL_OK) cand[n++] = q;
  if (!small_ok && plan_kernel(h, c, Kern::K4, -1, &q) == FNL_OK) cand[n++] = q;
  if (!small_ok && plan_kernel(h, c, Kern::K4S, -1, &q) == FNL_OK) cand[n++] = q;
  h->err.clear();   // refused candidates are not errors of the call
  if (n == 0) return default_plan(h, c, best);
  size_t need = 0;
  for (int i = 0; i < n; ++i) need = std::max(need, workspace_of(c, cand[i]));
  fnl_status st = ensure_workspace(h, c.stream, need);
  if (st != FNL_OK) return st;
  // an L2-sized buffer to write between timed launches (held for this call only)
  int l2 = 0;
  cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, h->device);
  const size_t flush_bytes = static_cast<size_t>(std::max(l2, 1 << 20)) * 2;
  void* flush = nullptr;
  cudaError_t e = cudaMalloc(&flush, flush_bytes);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaMalloc(tuning L2 flush buffer)");
  // One warm-up launch each, then kReps rounds over all candidates (so that a
  // clock that drifts as the GPU heats up is shared by all of them); the
  // median per candidate.
  constexpr int kReps = 5;
  float t[12][kReps];
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if ((e = cudaEventCreate(&e0)) == cudaSuccess) e = cudaEventCreate(&e1);
  if (e != cudaSuccess) st = cuda_fail(h, e, "cudaEventCreate");
  for (int i = 0; i < n && st == FNL_OK; ++i) st = launch_plan(h, c, cand[i]);
  for (int r = 0; r < kReps && st == FNL_OK; ++r)
    for (int i = 0; i < n && st == FNL_OK; ++i) st = time_once(h, c, cand[i], flush, flush_bytes, r, e0, e1, &t[i][r]);
  cudaStreamSynchronize(c.stream);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  cudaFree(flush);
  if (st != FNL_OK) return st;
  int bi = -1, di = -1;
  float bus = 0.f, dus = 0.f;
  for (int i = 0; i < n; ++i) {
    std::sort(t[i], t[i] + kReps);
    const float us = t[i][kReps / 2];
    if (bi < 0 || us < bus) {
      bi = i;
      bus = us;
    }
    if (have_dflt && di < 0 && same_plan(cand[i], dflt)) {
      di = i;
      dus = us;
    }
  }
  // the untuned plan stays unless another is faster by more than the timing noise
  if (di >= 0 && bus > 0.97f * dus) {
    bi = di;
    bus = dus;
  }
  *best = cand[bi];
  h->tuned.push_back({tune_key(c), cand[bi], bus, n});
  char buf[160];
  snprintf(buf, sizeof(buf), "%s, grid %d (tuned: %.1f us, fastest of %d candidates)", kern_name(cand[bi]),
           cand[bi].grid, bus, n);
  h->plan_text = buf;
  return FNL_OK;
}

fnl_status run(fnl_handle* h, const Call& c) {
  fnl_status st = validate(h, c);
  if (st != FNL_OK || c.M == 0) return st;
  if ((st = get_encoder(h)) != FNL_OK) return st;
  cudaError_t e = cudaSetDevice(h->device);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaSetDevice");

  Plan q;
  bool planned = false;
  if (h->opt.tune && h->opt.path == FNL_PATH_AUTO) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(c.stream, &cap);
    const TuneKey key = tune_key(c);
    for (const auto& t : h->tuned)
      if (t.key == key) {
        q = t.plan;
        planned = true;
        char buf[160];
        snprintf(buf, sizeof(buf), "%s, grid %d (tuned plan from the cache: %.1f us, %d candidates)",
                 kern_name(q), q.grid, t.us, t.candidates);
        h->plan_text = buf;
        break;
      }
    // tuning synchronises the stream: never inside a stream capture
    if (!planned && cap == cudaStreamCaptureStatusNone) {
      if ((st = tune(h, c, &q)) != FNL_OK) return st;
      planned = true;
    }
  }
  if (!planned) {
    if ((st = default_plan(h, c, &q)) != FNL_OK) return st;
    char buf[160];
    snprintf(buf, sizeof(buf), "%s, grid %d", kern_name(q), q.grid);
    h->plan_text = buf;
  }
  if ((st = ensure_workspace(h, c.stream, workspace_of(c, q))) != FNL_OK) return st;
  return launch_plan(h, c, q);
}

const bf16* B(const fnl_bf16* p) { return reinterpret_cast<const bf16*>(p); }
bf16* Bm(fnl_bf16* p) { return reinterpret_cast<bf16*>(p); }

}  // namespace

extern "C" {

fnl_status fnl_create(fnl_handle** out, int device, const fnl_options* opt) {
  if (!out) return FNL_ERR_INVALID_ARG;
  *out = nullptr;
  fnl_handle* h = new fnl_handle();
  if (opt) h->opt = *opt;
  if (h->opt.path < FNL_PATH_AUTO || h->opt.path > FNL_PATH_TILE_PAIR_SPLIT || h->opt.max_tokens < 0 || h->opt.max_n < 0 ||
      h->opt.precision < FNL_PRECISION_DEFAULT || h->opt.precision > FNL_PRECISION_SINGLE || h->opt.wait_ns < 0 ||
      h->opt.debug_stall_calls < 0 || h->opt.tune < 0 || h->opt.tune > 1) {
    delete h;
    return FNL_ERR_INVALID_ARG;
  }
  h->device = device;
  cudaError_t e = cudaSetDevice(device);
  if (e != cudaSuccess) {
    delete h;
    return FNL_ERR_CUDA;
  }
  int sms = 0, major = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  if (major != 10) {
    delete h;
    return FNL_ERR_UNSUPPORTED;   // the kernels are built for sm_100a only
  }
  h->num_sms = sms > 0 ? sms : 148;
  // reserve workspace for the declared maxima (small-M partials dominate)
  size_t need = kFixedBytes;
  if (h->opt.max_tokens > 0) need += align256(static_cast<size_t>(h->opt.max_tokens) * 8);
  if (h->opt.max_n > 0) {
    const size_t T = static_cast<size_t>(h->opt.max_n) / 64 + 1;
    const size_t seg = static_cast<size_t>(h->num_sms) / std::max<size_t>(T, 1) + 2;
    need += align256(T * seg * fnl::k3::MAX_MPAD * 4) + align256(T * seg * fnl::k3::MAX_MPAD * 128 * 4);
  }
  fnl_status st = ensure_workspace(h, nullptr, need);
  if (st != FNL_OK) {
    delete h;
    return st;
  }
  *out = h;
  return FNL_OK;
}

fnl_status fnl_destroy(fnl_handle* h) {
  if (!h) return FNL_OK;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  if (h->ws) cudaFree(h->ws);
  delete h;
  return FNL_OK;
}

const char* fnl_status_string(fnl_status s) {
  switch (s) {
    case FNL_OK: return "FNL_OK";
    case FNL_ERR_INVALID_ARG: return "FNL_ERR_INVALID_ARG";
    case FNL_ERR_ALIGNMENT: return "FNL_ERR_ALIGNMENT";
    case FNL_ERR_ALIAS: return "FNL_ERR_ALIAS";
    case FNL_ERR_UNSUPPORTED: return "FNL_ERR_UNSUPPORTED";
    case FNL_ERR_CUDA: return "FNL_ERR_CUDA";
    case FNL_ERR_DEVICE_STATUS: return "FNL_ERR_DEVICE_STATUS";
  }
  return "FNL_ERR_UNKNOWN";
}

const char* fnl_last_error(const fnl_handle* h) { return h ? h->err.c_str() : ""; }

const char* fnl_last_plan(const fnl_handle* h) { return h ? h->plan_text.c_str() : ""; }

fnl_status fnl_check(fnl_handle* h, fnl_stream stream) {
  if (!h) return FNL_ERR_INVALID_ARG;
  cudaSetDevice(h->device);
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
  int status = 0;
  e = cudaMemcpy(&status, h->ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemcpy(status)");
  if (status != 0) {
    // A CTA that gave up never made its split-K arrival, so its tiles' arrival
    // counters are left part-way; clear them with the status word, or every later
    // call would elect the wrong last CTA.
    e = cudaMemset(h->ws, 0, kFixedBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemset(status, counters)");
    return fail(h, FNL_ERR_DEVICE_STATUS,
                "device status %d (1-7: a kernel gave up a bounded wait; 8: a debug build refused an out-of-range "
                "store)", status);
  }
  return FNL_OK;
}

fnl_status fnl_add_norm_qkv(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                            fnl_bf16* residual_out, const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm,
                            float eps, const fnl_bf16* W, const fnl_bf16* bias, int M, int K, int Hq, int Hkv,
                            int D, fnl_bf16* q, fnl_bf16* k, fnl_bf16* v, float* mean_out, float* rstd_out) {
  Call c{};
  c.op = Op::QKV;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = nullptr; c.gamma = B(gamma); c.beta = B(beta);
  c.W = B(W); c.bias = B(bias); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.Hq = Hq; c.Hkv = Hkv; c.D = D;
  c.N = qkv_columns(Hq, Hkv, D);
  c.q = Bm(q); c.k = Bm(k); c.v = Bm(v); c.out = nullptr;
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  if (c.N <= 0 && h) return fail(h, FNL_ERR_INVALID_ARG, "Hq, Hkv, D must be > 0 and (Hq + 2 Hkv) D <= %d", kMaxN);
  return run(h, c);
}

fnl_status fnl_add_norm_swiglu(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                               fnl_bf16* residual_out, const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm,
                               float eps, const fnl_bf16* W, const fnl_bf16* bias, int M, int K, int I,
                               fnl_bf16* out, float* mean_out, float* rstd_out) {
  Call c{};
  c.op = Op::SwiGLU;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = nullptr; c.gamma = B(gamma); c.beta = B(beta);
  c.W = B(W); c.bias = B(bias); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.I = I; c.N = (I > 0 && I <= kMaxN / 2) ? 2 * I : 0;
  c.out = Bm(out);
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  if (c.N <= 0 && h) return fail(h, FNL_ERR_INVALID_ARG, "I must be > 0 and 2 I <= %d", kMaxN);
  return run(h, c);
}

fnl_status fnl_add_bias_norm_gelu(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                                  const fnl_bf16* bias_in, fnl_bf16* residual_out, const fnl_bf16* gamma,
                                  const fnl_bf16* beta, fnl_norm norm, float eps, const fnl_bf16* W,
                                  const fnl_bf16* bias_out, int M, int K, int N, fnl_bf16* out, float* mean_out,
                                  float* rstd_out) {
  Call c{};
  c.op = Op::GELU;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = B(bias_in); c.gamma = B(gamma); c.beta = B(beta);
  c.W = B(W); c.bias = B(bias_out); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.N = N;
  c.out = Bm(out);
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  return run(h, c);
}

fnl_status fnl_add_norm_qkv_fp8(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                                fnl_bf16* residual_out, const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm,
                                float eps, const uint8_t* Wq, const float* w_scale, const fnl_bf16* bias, int M, int K,
                                int Hq, int Hkv, int D, fnl_bf16* q, fnl_bf16* k, fnl_bf16* v, float* mean_out,
                                float* rstd_out) {
  Call c{};
  c.op = Op::QKV;
  c.fp8 = true;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = nullptr; c.gamma = B(gamma); c.beta = B(beta);
  c.W = reinterpret_cast<const bf16*>(Wq); c.w_scale = w_scale; c.bias = B(bias); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.Hq = Hq; c.Hkv = Hkv; c.D = D;
  c.N = qkv_columns(Hq, Hkv, D);
  c.q = Bm(q); c.k = Bm(k); c.v = Bm(v); c.out = nullptr;
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  if (c.N <= 0 && h) return fail(h, FNL_ERR_INVALID_ARG, "Hq, Hkv, D must be > 0 and (Hq + 2 Hkv) D <= %d", kMaxN);
  return run(h, c);
}

fnl_status fnl_add_norm_swiglu_fp8(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                                   fnl_bf16* residual_out, const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm,
                                   float eps, const uint8_t* Wq, const float* w_scale, const fnl_bf16* bias, int M,
                                   int K, int I, fnl_bf16* out, float* mean_out, float* rstd_out) {
  Call c{};
  c.op = Op::SwiGLU;
  c.fp8 = true;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = nullptr; c.gamma = B(gamma); c.beta = B(beta);
  c.W = reinterpret_cast<const bf16*>(Wq); c.w_scale = w_scale; c.bias = B(bias); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.I = I; c.N = (I > 0 && I <= kMaxN / 2) ? 2 * I : 0;
  c.out = Bm(out);
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  if (c.N <= 0 && h) return fail(h, FNL_ERR_INVALID_ARG, "I must be > 0 and 2 I <= %d", kMaxN);
  return run(h, c);
}

fnl_status fnl_add_bias_norm_gelu_fp8(fnl_handle* h, fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                                      const fnl_bf16* bias_in, fnl_bf16* residual_out, const fnl_bf16* gamma,
                                      const fnl_bf16* beta, fnl_norm norm, float eps, const uint8_t* Wq,
                                      const float* w_scale, const fnl_bf16* bias_out, int M, int K, int N,
                                      fnl_bf16* out, float* mean_out, float* rstd_out) {
  Call c{};
  c.op = Op::GELU;
  c.fp8 = true;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = B(bias_in); c.gamma = B(gamma); c.beta = B(beta);
  c.W = reinterpret_cast<const bf16*>(Wq); c.w_scale = w_scale; c.bias = B(bias_out);
  c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.N = N;
  c.out = Bm(out);
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  return run(h, c);
}

fnl_status fnl_tp_allreduce(fnl_handle* h, fnl_stream stream, const fnl_bf16* const* parts, int P, fnl_bf16* out,
                            long long n) {
  if (!h) return FNL_ERR_INVALID_ARG;
  if (P < 1 || P > fnl::kMaxTpRanks || n < 0)
    return fail(h, FNL_ERR_INVALID_ARG, "need 1 <= P <= %d and n >= 0 (P=%d)", fnl::kMaxTpRanks, P);
  if (n == 0) return FNL_OK;
  if (!parts || !out) return fail(h, FNL_ERR_INVALID_ARG, "parts and out are required");
  fnl::TpParts tp{};
  const Range o{out, static_cast<size_t>(n) * 2, "out"};
  if (!al16(out)) return fail(h, FNL_ERR_ALIGNMENT, "out must be 16-byte aligned");
  for (int q = 0; q < P; ++q) {
    if (!parts[q]) return fail(h, FNL_ERR_INVALID_ARG, "parts[%d] is NULL", q);
    if (!al16(parts[q])) return fail(h, FNL_ERR_ALIGNMENT, "parts[%d] must be 16-byte aligned", q);
    if (overlap(o, Range{parts[q], static_cast<size_t>(n) * 2, "part"}))
      return fail(h, FNL_ERR_ALIAS, "out overlaps parts[%d]", q);
    tp.p[q] = B(parts[q]);
  }
  cudaError_t e = cudaSetDevice(h->device);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaSetDevice");
  const long long n8 = std::max<long long>(n / 8, 1);
  const int grid = static_cast<int>(std::min<long long>((n8 + fnl::kTpThreads - 1) / fnl::kTpThreads,
                                                        static_cast<long long>(h->num_sms) * 4));
  fnl::k5_tp_allreduce<<<grid, fnl::kTpThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      tp, P, reinterpret_cast<bf16*>(out), n);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the tensor-parallel all-reduce");
  return FNL_OK;
}

fnl_status fnl_quantize_weight_fp8(fnl_handle* h, fnl_stream stream, const fnl_bf16* W, int N, int K, uint8_t* Wq,
                                   float* w_scale) {
  if (!h) return FNL_ERR_INVALID_ARG;
  if (N < 0 || K <= 0 || K % 8) return fail(h, FNL_ERR_INVALID_ARG, "need N >= 0 and K a positive multiple of 8");
  if (N == 0) return FNL_OK;
  if (!W || !Wq || !w_scale) return fail(h, FNL_ERR_INVALID_ARG, "W, Wq and w_scale are required");
  if (!al16(W) || reinterpret_cast<uintptr_t>(Wq) % 8 || !al4(w_scale))
    return fail(h, FNL_ERR_ALIGNMENT, "W 16-byte, Wq 8-byte and w_scale 4-byte alignment required");
  const Range out{Wq, static_cast<size_t>(N) * K, "Wq"}, sc{w_scale, static_cast<size_t>(N) * 4, "w_scale"};
  const Range in{W, static_cast<size_t>(N) * K * 2, "W"};
  if (overlap(out, in) || overlap(sc, in) || overlap(out, sc)) return fail(h, FNL_ERR_ALIAS, "outputs overlap");
  cudaError_t e = cudaSetDevice(h->device);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaSetDevice");
  fnl::k0_quantize_weight_fp8<<<N, fnl::kK1Threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(B(W), Wq, w_scale,
                                                                                                   N, K);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "launch of the FP8 weight quantiser");
  return FNL_OK;
}

fnl_status fnl_linear_add_residual(fnl_handle* h, fnl_stream stream, const fnl_bf16* a, const fnl_bf16* W,
                                   const fnl_bf16* bias, const fnl_bf16* residual, fnl_bf16* out, int M, int K,
                                   int N) {
  Call c{};
  c.op = Op::Residual;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(a); c.W = B(W); c.bias = B(bias); c.residual = B(residual); c.out = Bm(out);
  c.norm = FNL_NORM_RMSNORM; c.eps = 1.f;   // unused (no norm)
  c.M = M; c.K = K; c.N = N;
  return run(h, c);
}

}  // extern "C"

// ============================================================================
// Allocation-free entry point: fnl_add_norm_qkv_static.
//
// Some callers cannot allocate device memory on the call path: code recorded
// into a CUDA graph (cudaMalloc cannot be captured), latency-critical decode
// loops that must never hit cudaMalloc/cudaFree's implicit device
// synchronisation, and plugins living inside an inference engine that owns all
// device memory through its own static memory plan. fnl_create allocates the
// handle's workspace, so those callers get this handle-free variant of the
// small-M (decode) QKV kernel instead. Its scratch (split-K partial sums, the
// per-tile arrival counters, the LayerNorm statistics and the status word)
// lives in the file-scope array below, which every GPU that loads this
// library holds until the process exits. Nothing here calls cudaMalloc,
// cudaFree or any other allocating routine.
// ============================================================================
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(16) << 20;   // 16 MiB per device
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kStaticMaxDevices] = {};   // device address of g_static_scratch, per device
int g_static_sms[kStaticMaxDevices] = {};

// Once per device, with that device current: resolve the array's device
// address (in host code the symbol is only a host-side stand-in and must not
// be passed to a kernel).
fnl_status static_setup(int dev, void** ptr, int* sms) {
  if (dev < 0 || dev >= kStaticMaxDevices) return FNL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    int major = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return FNL_ERR_CUDA;
    if (major != 10) return FNL_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FNL_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return FNL_ERR_CUDA;
    g_static_ptr[dev] = p;
    g_static_sms[dev] = count > 0 ? count : 148;
  }
  *ptr = g_static_ptr[dev];
  *sms = g_static_sms[dev];
  return FNL_OK;
}

// Argument checks of fnl_add_norm_qkv, without a handle (and without heap use).
fnl_status validate_static(const Call& c) {
  if (c.norm != FNL_NORM_LAYERNORM && c.norm != FNL_NORM_RMSNORM) return FNL_ERR_INVALID_ARG;
  if (!(c.eps > 0.f) || c.eps > 1e30f) return FNL_ERR_INVALID_ARG;
  if (c.M < 0 || c.K <= 0 || c.Hq <= 0 || c.Hkv <= 0 || c.D <= 0 || c.N <= 0) return FNL_ERR_INVALID_ARG;
  if (c.Hq % c.Hkv) return FNL_ERR_INVALID_ARG;
  if (c.K % 8 || c.D % 8) return FNL_ERR_ALIGNMENT;
  if (c.K > 32768 || c.M > fnl::k3::MAX_MPAD) return FNL_ERR_UNSUPPORTED;
  if (c.norm == FNL_NORM_RMSNORM && (c.beta || c.mean_out)) return FNL_ERR_INVALID_ARG;
  if (c.M == 0) return FNL_OK;
  if (!c.x || !c.residual || !c.residual_out || !c.gamma || !c.W || !c.q || !c.k || !c.v)
    return FNL_ERR_INVALID_ARG;
  const void* p16[] = {c.x, c.residual, c.gamma, c.beta, c.W, c.bias, c.residual_out, c.q, c.k, c.v};
  for (const void* p : p16)
    if (p && !al16(p)) return FNL_ERR_ALIGNMENT;
  if ((c.mean_out && !al4(c.mean_out)) || (c.rstd_out && !al4(c.rstd_out))) return FNL_ERR_ALIGNMENT;
  const size_t MK = static_cast<size_t>(c.M) * c.K * 2;
  const Range ins[] = {{c.x, MK, "x"},
                       {c.residual, MK, "residual"},
                       {c.gamma, static_cast<size_t>(c.K) * 2, "gamma"},
                       {c.beta, static_cast<size_t>(c.K) * 2, "beta"},
                       {c.W, static_cast<size_t>(c.N) * c.K * 2, "W"},
                       {c.bias, static_cast<size_t>(c.N) * 2, "bias"}};
  const Range outs[] = {{c.residual_out, MK, "residual_out"},
                        {c.mean_out, static_cast<size_t>(c.M) * 4, "mean_out"},
                        {c.rstd_out, static_cast<size_t>(c.M) * 4, "rstd_out"},
                        {c.q, static_cast<size_t>(c.Hq) * c.M * c.D * 2, "q"},
                        {c.k, static_cast<size_t>(c.Hkv) * c.M * c.D * 2, "k"},
                        {c.v, static_cast<size_t>(c.Hkv) * c.M * c.D * 2, "v"}};
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    for (const Range& in : ins)
      if (overlap(outs[i], in)) return FNL_ERR_ALIAS;
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (overlap(outs[i], outs[j])) return FNL_ERR_ALIAS;
  }
  return FNL_OK;
}

}  // namespace

extern "C" fnl_status fnl_add_norm_qkv_static(fnl_stream stream, const fnl_bf16* x, const fnl_bf16* residual,
                                              fnl_bf16* residual_out, const fnl_bf16* gamma, const fnl_bf16* beta,
                                              fnl_norm norm, float eps, const fnl_bf16* W, const fnl_bf16* bias,
                                              int M, int K, int Hq, int Hkv, int D, fnl_bf16* q, fnl_bf16* k,
                                              fnl_bf16* v, float* mean_out, float* rstd_out) {
  Call c{};
  c.op = Op::QKV;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.x = B(x); c.residual = B(residual); c.bias_in = nullptr; c.gamma = B(gamma); c.beta = B(beta);
  c.W = B(W); c.bias = B(bias); c.residual_out = Bm(residual_out);
  c.norm = norm; c.eps = eps; c.M = M; c.K = K; c.Hq = Hq; c.Hkv = Hkv; c.D = D;
  c.N = qkv_columns(Hq, Hkv, D);
  c.q = Bm(q); c.k = Bm(k); c.v = Bm(v); c.out = nullptr;
  c.mean_out = mean_out; c.rstd_out = rstd_out;
  fnl_status st = validate_static(c);
  if (st != FNL_OK || c.M == 0) return st;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FNL_ERR_CUDA;
  void* scratch = nullptr;
  int sms = 0;
  if ((st = static_setup(dev, &scratch, &sms)) != FNL_OK) return st;
  if ((st = get_encoder(nullptr)) != FNL_OK) return st;

  // small-M split-K plan, the same as fnl_add_norm_qkv's for M <= 128
  const bool rms = c.norm == FNL_NORM_RMSNORM;
  const int nkb = (c.K + 63) / 64;
  const int mpad = round_up(c.M, 16);
  const int T = (c.N + 127) / 128;
  const long long U = static_cast<long long>(T) * nkb;
  const int grid = static_cast<int>(std::min<long long>(sms, U));
  const int stages = std::min(fnl::k3::MAX_STAGES, (200 * 1024) / fnl::k3::stage_bytes(mpad));
  int max_seg = 1;
  for (int t = 0; t < T; ++t) {
    const int first = fnl::unit_owner(static_cast<long long>(t) * nkb, grid, U);
    const int last = fnl::unit_owner(static_cast<long long>(t + 1) * nkb - 1, grid, U);
    max_seg = std::max(max_seg, last - first + 1);
  }
  // scratch layout: [status][counters][stats][partial h^2 sums][partial accumulators]
  const size_t zero_bytes = align256(kStatusBytes + static_cast<size_t>(T) * 4);
  const size_t counter_bytes = zero_bytes - kStatusBytes;
  const size_t stats_bytes = rms ? 0 : align256(static_cast<size_t>(c.M) * 8);
  const size_t ss_bytes = align256(static_cast<size_t>(T) * max_seg * mpad * 4);
  const size_t part_bytes = align256(static_cast<size_t>(T) * max_seg * mpad * 128 * 4);
  if (zero_bytes + stats_bytes + ss_bytes + part_bytes > kStaticScratchBytes) return FNL_ERR_UNSUPPORTED;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  // The array keeps the previous call's contents: the arrival counters must
  // start at zero (the rest is written before it is read). The status word is
  // left alone: it keeps the first failure code until fnl_check_static reads
  // and clears it.
  cudaError_t e = cudaMemsetAsync(base + kStatusBytes, 0, counter_bytes, c.stream);
  if (e != cudaSuccess) return FNL_ERR_CUDA;

  OpParams p{};
  p.M = c.M; p.K = c.K; p.N = c.N; p.I = 0; p.Hq = c.Hq; p.Hkv = c.Hkv; p.D = c.D; p.eps = c.eps;
  p.x_in = c.x; p.r_in = c.residual;
  p.gamma = c.gamma; p.beta = c.beta; p.bias_in = nullptr; p.bias = c.bias;
  p.residual_out = c.residual_out; p.rstd_out = rms ? c.rstd_out : nullptr;
  p.stats = reinterpret_cast<const float2*>(base + zero_bytes);
  p.q = c.q; p.k = c.k; p.v = c.v; p.out = nullptr;
  p.counters = reinterpret_cast<unsigned*>(base + kStatusBytes);
  p.part_ss = reinterpret_cast<float*>(base + zero_bytes + stats_bytes);
  p.part = reinterpret_cast<float*>(base + zero_bytes + stats_bytes + ss_bytes);
  p.max_seg = max_seg; p.mpad = mpad; p.stages = stages; p.split = 0;
  p.status = reinterpret_cast<int*>(base);
  p.wait_ns = FNL_WAIT_NS;
  p.stall = 0;

  CUtensorMap mx, mr, mw;
  if ((st = make_map(nullptr, &mx, c.x, c.M, c.K, mpad)) != FNL_OK) return st;
  if ((st = make_map(nullptr, &mr, c.residual, c.M, c.K, mpad)) != FNL_OK) return st;
  if ((st = make_map(nullptr, &mw, c.W, c.N, c.K, fnl::k3::BW)) != FNL_OK) return st;
  if (!rms && (st = launch_k1(nullptr, c, reinterpret_cast<float2*>(base + zero_bytes), c.stream)) != FNL_OK)
    return st;
  return dispatch_gemm<fnl::kEpiQKV>(nullptr, true, rms, grid, fnl::k3::NUM_THREADS,
                                     fnl::k3::smem_bytes(mpad, stages), !rms, c.stream, mx, mr, mw, p);
}

extern "C" fnl_status fnl_check_static(fnl_stream stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FNL_ERR_CUDA;
  void* scratch = nullptr;
  int sms = 0;
  fnl_status st = static_setup(dev, &scratch, &sms);
  if (st != FNL_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FNL_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FNL_ERR_CUDA;
  if (status == 0) return FNL_OK;
  // clear the status word (the next call clears the arrival counters itself)
  if (cudaMemset(scratch, 0, sizeof(int)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    return FNL_ERR_CUDA;
  return FNL_ERR_DEVICE_STATUS;
}
