// common.cuh -- device helpers shared by the libnsa kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nsa {

using bf16 = __nv_bfloat16;

// Codes written to the library's device error word (first writer wins).
enum : int {
  kDevOk = 0,
  kDevTimeout = 1,   // a bounded wait gave up
  kDevBadIndex = 2,  // a block index was out of range / not causal / unsorted
  kDevRange = 3,     // a value exceeded an intermediate format's range
};

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---- programmatic dependent launch -------------------------------------------
// A kernel launched with the programmatic-serialization attribute may start
// while the kernel before it in the stream is still running: it calls
// pdl_wait() before reading anything that kernel wrote (the wait returns
// once that grid has completed and its memory is visible; completion of a
// grid implies completion of the ones before it).  pdl_launch_dependents()
// lets the next kernel's launch begin.  Both are no-ops in a kernel launched
// the ordinary way.  (Used by decode; in the prefill forward, measured on
// B200, early-launched dependents only took SM slots from the window branch
// running beside the chain: 0.307 ms without, 0.315 ms with.)
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }


// ---- scalar load/store in the path dtype, arithmetic in fp32 -------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) {
  return __float2bfloat16_rn(x);
}

// Round a double to bfloat16, nearest-even, on the binary64 bit pattern:
// bfloat16 keeps 7 of the 52 fraction bits, so the low 45 bits are rounded
// away (add half an ulp minus one, plus the kept lsb for ties-to-even) and
// the result, which has 8 significant bits, converts to float exactly.
__device__ __forceinline__ bf16 f64_to_bf16_rne(double x) {
  unsigned long long u = (unsigned long long)__double_as_longlong(x);
  const unsigned long long lsb = (u >> 45) & 1ull;
  u += 0x00000FFFFFFFFFFFull + lsb;
  u &= ~0x00001FFFFFFFFFFFull;
  const float f = (float)__longlong_as_double((long long)u);
  return __float2bfloat16_rz(f);  // exact: f is a bfloat16 value
}

template <typename T> __device__ __forceinline__ T from_f64(double x);
template <> __device__ __forceinline__ float from_f64<float>(double x) {
  return __double2float_rn(x);
}
template <> __device__ __forceinline__ bf16 from_f64<bf16>(double x) {
  return f64_to_bf16_rne(x);
}

// ---- warp reductions -------------------------------------------------------
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Load 64 consecutive path-dtype elements as fp32 into smem/regs helpers.
template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return to_f32(*p); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace nsa
