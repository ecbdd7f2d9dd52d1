// k_compress.cu -- mean-pool compression of keys and values.
//
// "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method / Key claims:
// the compression branch summarises each block of l consecutive tokens by
// the plain mean of its key (and value) rows, instead of NSA's MLP.
//
// One CTA owns one (sequence, block, k or v): the block's l token rows are
// one contiguous l * Hkv * 64-element span, read with 16-byte loads, fully
// coalesced, every load of a thread issued before the first add.  Thread
// (row r0, column chunk c) sums rows r0, r0+R, ... of its chunk in fp64
// (exact for bf16 inputs); the R partial sums per column are then added in
// a fixed order, so the result is deterministic and, for bf16 inputs, the
// exact mean rounded once to the output dtype.
#include "common.cuh"
#include "internal.h"

namespace nsa {

template <typename T>
__global__ void compress_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                T* __restrict__ kc, T* __restrict__ vc, int T_,
                                int Hkv, int l, int stride, int Nc) {
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ double part[];  // [R][row_elems]
  const int row_elems = Hkv * 64;
  const int CPT = row_elems / VEC;  // 16-byte chunks per token row
  const int R = blockDim.x / CPT;   // token rows read in parallel
  const int j = blockIdx.x, b = blockIdx.y, which = blockIdx.z;  // which: 0 keys, 1 values
  const int tid = threadIdx.x;
  const int col = tid % CPT, r0 = tid / CPT;
  const T* src = which == 0 ? k : v;
  T* dst = which == 0 ? kc : vc;
  double acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0;
  const T* base = src + ((size_t)b * T_ + (size_t)j * stride) * row_elems + (size_t)col * VEC;
  // all of this thread's rows are loaded before any is summed
  constexpr int kMaxRows = 8;
  uint4 raw[kMaxRows];
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q) {
    const int r = r0 + q * R;
    raw[q] = r < l ? __ldg(reinterpret_cast<const uint4*>(base + (size_t)r * row_elems))
                   : make_uint4(0u, 0u, 0u, 0u);
  }
  for (int r = r0 + kMaxRows * R; r < l; r += R) {  // blocks longer than kMaxRows * R rows
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(base + (size_t)r * row_elems));
    const T* e = reinterpret_cast<const T*>(&x);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += (double)to_f32(e[i]);
  }
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q) {
    const T* e = reinterpret_cast<const T*>(&raw[q]);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += (double)to_f32(e[i]);
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) part[(size_t)r0 * row_elems + col * VEC + i] = acc[i];
  __syncthreads();
  for (int e = tid; e < row_elems; e += blockDim.x) {
    double sum = 0.0;
    for (int r = 0; r < R; ++r) sum += part[(size_t)r * row_elems + e];
    dst[((size_t)b * Nc + j) * row_elems + e] = from_f64<T>(sum / (double)l);
  }
}

template <typename T>
static cudaError_t launch_compress_t(const Dims& d, const void* k, const void* v,
                                     void* kc, void* vc, cudaStream_t s) {
  if (d.Nc == 0) return cudaSuccess;
  constexpr int VEC = 16 / sizeof(T);
  const int cpt = d.Hkv * 64 / VEC;
  const int R = cpt >= 256 ? 1 : 256 / cpt;
  const int threads = cpt * R;
  const size_t smem = (size_t)R * d.Hkv * 64 * sizeof(double);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(compress_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  compress_kernel<T><<<dim3(d.Nc, d.B, 2), threads, smem, s>>>(
      (const T*)k, (const T*)v, (T*)kc, (T*)vc, d.T, d.Hkv, d.lc, d.dc, d.Nc);
  return cudaGetLastError();
}

cudaError_t launch_compress(const Dims& d, const void* k, const void* v, void* kc,
                            void* vc, cudaStream_t s) {
  return d.dtype == 1 ? launch_compress_t<bf16>(d, k, v, kc, vc, s)
                      : launch_compress_t<float>(d, k, v, kc, vc, s);
}

}  // namespace nsa
