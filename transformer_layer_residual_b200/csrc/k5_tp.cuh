// K5: the tensor-parallel all-reduce that feeds the fused op.
//
// With tensor parallelism the output and down projections are split by rows
// (TensorRT-LLM 深度工程实践, §4.1 Tensor Parallelism): each of the P ranks holds
// a partial activation, and their sum is the next fused add + norm +
// projection's x. This kernel forms that sum on one GPU from P buffers that may
// live on other GPUs (peer pointers mapped into this device's address space,
// read over NVLink with plain loads; no cluster multicast anywhere): one pass
// over the n elements, 16-byte loads of every rank's 8 values, an fp32 sum in
// rank order 0..P-1 (so every rank that runs it gets the same bits), one
// rounding to bf16. HBM (or NVLink) bound: (P + 1) n 2 bytes. The kernel never
// waits on another GPU: the caller orders it after every rank's partial is
// complete (a barrier on the host, or stream events).
#pragma once

#include "common.cuh"

namespace fnl {

constexpr int kMaxTpRanks = 16;
constexpr int kTpThreads = 256;

struct TpParts {
  const bf16* p[kMaxTpRanks];
};

__global__ void __launch_bounds__(kTpThreads) k5_tp_allreduce(const __grid_constant__ TpParts parts, int P,
                                                            bf16* __restrict__ out,
                                                            long long n) {
  pdl_launch_dependents();   // the fused op that reads `out` may take its SMs early
  const long long n8 = n >> 3;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long first = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long long i = first; i < n8; i += stride) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int q = 0; q < P; ++q) {
      float f[8];
      unpack8(ldg16(parts.p[q] + i * 8), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += f[e];
    }
    *reinterpret_cast<uint4*>(out + i * 8) = pack8(acc);
  }
  for (long long i = n8 * 8 + first; i < n; i += stride) {   // the last n % 8 elements
    float acc = 0.f;
    for (int q = 0; q < P; ++q) acc += __bfloat162float(parts.p[q][i]);
    out[i] = __float2bfloat16_rn(acc);
  }
}

}  // namespace fnl
