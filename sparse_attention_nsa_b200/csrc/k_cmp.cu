// k_cmp.cu -- compression branch and block-importance scores.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: COMPRESSION attends to one summary key/value per block; SELECTION
// reuses the compression attention scores to rank blocks.  Here a block is
// visible to query position t once complete (j*l + l - 1 <= t); the
// importance of block j for KV group g is the compression softmax
// probability summed over the G query heads that share the group.
//
// This is the fp32 path (and the path for geometries the tensor-core kernel
// in k_cmp_tc.cu does not tile).  One warp per (sequence, query, KV group).  For each of the G heads the
// warp computes the logits of all visible blocks (lanes over blocks), keeps
// them in shared memory, normalises them in fp32, adds them into the
// group's score row, and forms o_cmp with lanes over the head dimension.
#include "common.cuh"
#include "internal.h"

namespace nsa {

constexpr int kCmpWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kCmpWarps * 32)
cmp_scores_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                  const T* __restrict__ vc, T* __restrict__ o_cmp,
                  float* __restrict__ lse_cmp, float* __restrict__ score, Dims d,
                  int write_o) {
  extern __shared__ float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* logit = sm + (size_t)warp * d.Nc;                       // [Nc]
  float* sacc = sm + (size_t)kCmpWarps * d.Nc + (size_t)warp * d.Nc;  // [Nc]
  float* qs = sm + (size_t)2 * kCmpWarps * d.Nc + warp * 64;     // [64]
  const int tq = blockIdx.x * kCmpWarps + warp;
  const int g = blockIdx.y, b = blockIdx.z;
  if (tq >= d.Tq) return;
  const int t = d.q_off + tq;
  const int nvis = cmp_nvis(d, t);
  const float sl2 = d.scale * kLog2e;
  for (int j = lane; j < d.Nc; j += 32) sacc[j] = 0.f;
  const size_t row = (size_t)d.Hkv * 64;  // elements between consecutive kc rows
  const T* kcb = kc + (size_t)b * d.Nc * row + (size_t)g * 64;
  const T* vcb = vc + (size_t)b * d.Nc * row + (size_t)g * 64;
  for (int hh = 0; hh < d.G; ++hh) {
    const int h = g * d.G + hh;
    const size_t qrow = (((size_t)b * d.Tq + tq) * d.Hq + h) * 64;
    qs[lane] = to_f32(q[qrow + lane]);
    qs[lane + 32] = to_f32(q[qrow + lane + 32]);
    __syncwarp();
    float mx = -INFINITY;
    for (int j = lane; j < nvis; j += 32) {
      const T* kr = kcb + (size_t)j * row;
      float acc = 0.f;
#pragma unroll 16
      for (int e = 0; e < 64; ++e) acc = fmaf(qs[e], to_f32(kr[e]), acc);
      acc *= sl2;
      logit[j] = acc;
      mx = fmaxf(mx, acc);
    }
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < nvis; j += 32) sum += exp2f(logit[j] - mx);
    sum = warp_sum(sum);
    const float inv = nvis > 0 ? 1.f / sum : 0.f;
    for (int j = lane; j < nvis; j += 32) {
      const float p = exp2f(logit[j] - mx) * inv;
      logit[j] = p;
      sacc[j] += p;
    }
    __syncwarp();
    if (write_o) {
      float o0 = 0.f, o1 = 0.f;
      for (int j = 0; j < nvis; ++j) {
        const float p = logit[j];
        o0 = fmaf(p, to_f32(vcb[(size_t)j * row + lane]), o0);
        o1 = fmaf(p, to_f32(vcb[(size_t)j * row + lane + 32]), o1);
      }
      o_cmp[qrow + lane] = from_f32<T>(o0);
      o_cmp[qrow + lane + 32] = from_f32<T>(o1);
    }
    if (lane == 0 && lse_cmp)
      lse_cmp[((size_t)b * d.Tq + tq) * d.Hq + h] =
          nvis > 0 ? (mx + log2f(sum)) * kLn2 : -INFINITY;
    __syncwarp();
  }
  float* srow = score + (((size_t)b * d.Tq + tq) * d.Hkv + g) * d.Nc;
  for (int j = lane; j < d.Nc; j += 32) srow[j] = sacc[j];
}

template <typename T>
static cudaError_t launch_t(const Dims& d, const void* q, const void* kc, const void* vc,
                            void* o_cmp, float* lse, float* score, cudaStream_t s) {
  const size_t smem = ((size_t)2 * kCmpWarps * d.Nc + kCmpWarps * 64) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(cmp_scores_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((d.Tq + kCmpWarps - 1) / kCmpWarps, d.Hkv, d.B);
  cmp_scores_kernel<T><<<grid, kCmpWarps * 32, smem, s>>>(
      (const T*)q, (const T*)kc, (const T*)vc, (T*)o_cmp, lse, score, d,
      o_cmp != nullptr);
  return cudaGetLastError();
}

cudaError_t launch_cmp_scores_simt(const Dims& d, const void* q, const void* kc,
                                   const void* vc, void* o_cmp, float* lse_cmp,
                                   float* score, cudaStream_t s) {
  return d.dtype == 1 ? launch_t<bf16>(d, q, kc, vc, o_cmp, lse_cmp, score, s)
                      : launch_t<float>(d, q, kc, vc, o_cmp, lse_cmp, score, s);
}

}  // namespace nsa
