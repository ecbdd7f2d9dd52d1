// k_attn_simt.cu -- selection and sliding-window attention on CUDA cores.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: SELECTION attends to the chosen blocks in raw form; SLIDING WINDOW
// attends to the most recent tokens.  The kernel paragraph there groups the
// queries that share a selection: here one CTA serves one (query, KV group)
// and its G warps, one per query head of the group, read the same key rows.
//
// Each warp runs an fp32 online softmax over its key list in chunks of 32
// keys (one key per lane for the logits, lanes over the head dimension for
// the value accumulation).  This is the fp32 path and the reference-shaped
// first implementation of the bf16 path; the tensor-core kernel replaces it
// for bf16 where its tile geometry applies.
#include "common.cuh"
#include "internal.h"

namespace nsa {

template <typename T>
__device__ __forceinline__ float dot64(const float* qs, const T* kr);

template <>
__device__ __forceinline__ float dot64<float>(const float* qs, const float* kr) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(kr) + c);
    acc = fmaf(qs[4 * c + 0], x.x, acc);
    acc = fmaf(qs[4 * c + 1], x.y, acc);
    acc = fmaf(qs[4 * c + 2], x.z, acc);
    acc = fmaf(qs[4 * c + 3], x.w, acc);
  }
  return acc;
}

template <>
__device__ __forceinline__ float dot64<bf16>(const float* qs, const bf16* kr) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(kr) + c);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p[i]);
      acc = fmaf(qs[8 * c + 2 * i], f.x, acc);
      acc = fmaf(qs[8 * c + 2 * i + 1], f.y, acc);
    }
  }
  return acc;
}

struct OnlineSoftmax {
  float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
};

// Fold keys [s0, s1) of one KV head into the running softmax of this warp.
// qs holds the query row pre-multiplied by scale * log2(e).
template <typename T>
__device__ __forceinline__ void fold_keys(OnlineSoftmax& st, const float* qs,
                                          const T* kb, const T* vb, size_t krow,
                                          int s0, int s1, int lane) {
  for (int base = s0; base < s1; base += 32) {
    const int s = base + lane;
    const bool ok = s < s1;
    const float logit = ok ? dot64<T>(qs, kb + (size_t)s * krow) : -INFINITY;
    const float mn = fmaxf(st.m, warp_max(logit));
    const float alpha = exp2f(st.m - mn);
    const float p = ok ? exp2f(logit - mn) : 0.f;
    st.l = st.l * alpha + warp_sum(p);
    st.o0 *= alpha;
    st.o1 *= alpha;
    const int n = min(32, s1 - base);
    for (int i = 0; i < n; ++i) {
      const float pi = __shfl_sync(0xffffffffu, p, i);
      const T* vr = vb + (size_t)(base + i) * krow;
      st.o0 = fmaf(pi, to_f32(vr[lane]), st.o0);
      st.o1 = fmaf(pi, to_f32(vr[lane + 32]), st.o1);
    }
    st.m = mn;
  }
}

template <typename T, bool SEL>
__global__ void __launch_bounds__(1024)
list_attn_kernel(const T* __restrict__ q, const T* __restrict__ k,
                 const T* __restrict__ v, const int32_t* __restrict__ idx,
                 T* __restrict__ o, float* __restrict__ lse, Dims d, int* err) {
  __shared__ float qs_all[32][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tq = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int h = g * d.G + warp;
  const int t = d.q_off + tq;
  float* qs = qs_all[warp];
  const size_t qrow = (((size_t)b * d.Tq + tq) * d.Hq + h) * 64;
  const float sl2 = d.scale * kLog2e;
  qs[lane] = to_f32(q[qrow + lane]) * sl2;
  qs[lane + 32] = to_f32(q[qrow + lane + 32]) * sl2;
  __syncwarp();
  const size_t krow = (size_t)d.Hkv * 64;
  const T* kb = k + (size_t)b * d.T * krow + (size_t)g * 64;
  const T* vb = v + (size_t)b * d.T * krow + (size_t)g * 64;
  OnlineSoftmax st;
  if (SEL) {
    const int32_t* ir = idx + (((size_t)b * d.Tq + tq) * d.Hkv + g) * d.topk;
    const int cur = t / d.l;
    int prev = -1;
    for (int sidx = 0; sidx < d.topk; ++sidx) {
      const int j = ir[sidx];
      if (j == -1) continue;
      if (j < -1 || j <= prev || j > cur) {  // never read outside the causal range
        if (lane == 0) record_error(err, kDevBadIndex);
        continue;
      }
      prev = j;
      fold_keys<T>(st, qs, kb, vb, krow, j * d.l, min(j * d.l + d.l, t + 1), lane);
    }
  } else {
    fold_keys<T>(st, qs, kb, vb, krow, max(0, t - d.window + 1), t + 1, lane);
  }
  const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
  o[qrow + lane] = from_f32<T>(st.o0 * inv);
  o[qrow + lane + 32] = from_f32<T>(st.o1 * inv);
  if (lane == 0 && lse)
    lse[((size_t)b * d.Tq + tq) * d.Hq + h] =
        st.l > 0.f ? (st.m + log2f(st.l)) * kLn2 : -INFINITY;
}

template <typename T, bool SEL>
static cudaError_t launch_t(const Dims& d, const void* q, const void* k, const void* v,
                            const int32_t* idx, void* o, float* lse, int* err,
                            cudaStream_t s) {
  dim3 grid(d.Tq, d.Hkv, d.B);
  list_attn_kernel<T, SEL><<<grid, d.G * 32, 0, s>>>(
      (const T*)q, (const T*)k, (const T*)v, idx, (T*)o, lse, d, err);
  return cudaGetLastError();
}

cudaError_t launch_sel_fwd_simt(const Dims& d, const void* q, const void* k,
                                const void* v, const int32_t* idx, void* o,
                                float* lse, int* err, cudaStream_t s) {
  return d.dtype == 1 ? launch_t<bf16, true>(d, q, k, v, idx, o, lse, err, s)
                      : launch_t<float, true>(d, q, k, v, idx, o, lse, err, s);
}

cudaError_t launch_swa_fwd_simt(const Dims& d, const void* q, const void* k,
                                const void* v, void* o, float* lse, cudaStream_t s) {
  return d.dtype == 1 ? launch_t<bf16, false>(d, q, k, v, nullptr, o, lse, nullptr, s)
                      : launch_t<float, false>(d, q, k, v, nullptr, o, lse, nullptr, s);
}

}  // namespace nsa
