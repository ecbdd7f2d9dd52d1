// k_combine.cu -- gated combination of the three branch outputs.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: the three attention outputs are merged by gate values from a small
// network (sigmoid outputs here, one per head and branch).  "Sparsity is
// Cool: Reverse-Engineering MoBA and NSA", TL;DR / Key claims: unused
// branches are pruned, so a disabled branch is neither read nor added.
//
// Elementwise over [B*Tq*Hq, 64]: each thread handles 8 consecutive head
// dims of one row with 16-byte (bf16) or 2x16-byte (fp32) accesses.
#include "common.cuh"
#include "internal.h"

namespace nsa {

template <typename T>
__global__ void combine_kernel(const float* __restrict__ gates,
                               const T* __restrict__ oc, const T* __restrict__ os,
                               const T* __restrict__ ow, T* __restrict__ out,
                               long nrows, int mask) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // 8-element chunk
  if (i >= nrows * 8) return;
  const long r = i >> 3;
  const float gc = (mask & 1) ? gates[r * 3 + 0] : 0.f;
  const float gs = (mask & 2) ? gates[r * 3 + 1] : 0.f;
  const float gw = (mask & 4) ? gates[r * 3 + 2] : 0.f;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const size_t off = (size_t)i * 8;
  if (mask & 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(gc, to_f32(oc[off + e]), acc[e]);
  }
  if (mask & 2) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(gs, to_f32(os[off + e]), acc[e]);
  }
  if (mask & 4) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(gw, to_f32(ow[off + e]), acc[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) out[off + e] = from_f32<T>(acc[e]);
}

cudaError_t launch_combine(const Dims& d, const float* gates, const void* o_cmp,
                           const void* o_sel, const void* o_swa, void* out,
                           cudaStream_t s) {
  const long nrows = (long)d.B * d.Tq * d.Hq;
  const long n = nrows * 8;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (d.dtype == 1)
    combine_kernel<bf16><<<blocks, threads, 0, s>>>(
        gates, (const bf16*)o_cmp, (const bf16*)o_sel, (const bf16*)o_swa, (bf16*)out,
        nrows, d.branch_mask);
  else
    combine_kernel<float><<<blocks, threads, 0, s>>>(
        gates, (const float*)o_cmp, (const float*)o_sel, (const float*)o_swa,
        (float*)out, nrows, d.branch_mask);
  return cudaGetLastError();
}

}  // namespace nsa
