// k_moba.cu -- MoBA block selection (gate + top-k), feeding the selection
// attention kernels.
//
// "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method (MoBA with
// block 512 and top-k 3) and Key claims; "DeepSeek's Native Sparse
// Attention" newsletter, MoBA section: the context is cut into blocks, a
// top-k gate sends each query to its most relevant past blocks, and causal
// protection keeps the query's own block causal.  Per (query, KV group), one
// warp:
//   cur = t / L.  With cur + 1 <= k every block 0..cur is taken.  Otherwise
//   the gate of each complete past block j < cur is
//     sum over the group's query heads h of q_h . mean(k of block j)
//   (formed as (sum_h q_h) . mean(k of block j)), the k - 1 best gates win
//   (equal gates: lower block first) and the query's own block is added.
// The chosen MoBA blocks (ascending) are written as such and expanded into
// 64-key selection blocks (block m covers 64-key blocks m L/64 .. m L/64 +
// L/64 - 1, the query's own block only up to the query's 64-key block), so
// the selection attention kernels of nsa_sel_attn_fwd / _bwd run MoBA
// unchanged with top-k = k L / 64.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace nsa {

constexpr int kMobaWarps = 8;

template <typename T, int QMAX>
__global__ void __launch_bounds__(kMobaWarps * 32)
moba_select_kernel(const T* __restrict__ q, const T* __restrict__ kc, int32_t* __restrict__ idx_m,
                   int32_t* __restrict__ idx64, Dims d, int L, int n) {
  __shared__ float qsum_s[kMobaWarps][64];
  __shared__ int win_s[kMobaWarps][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long row = (long)blockIdx.x * kMobaWarps + warp;  // (b * Tq + tq) * Hkv + g
  if (row >= (long)d.B * d.Tq * d.Hkv) return;
  const int g = (int)(row % d.Hkv);
  const long bt = row / d.Hkv;
  const int tq = (int)(bt % d.Tq), b = (int)(bt / d.Tq);
  const int t = d.q_off + tq;
  const int cur = t / L;
  int* win = win_s[warp];
  int nsel;
  if (cur + 1 <= n) {
    nsel = cur + 1;
    for (int i = lane; i < nsel; i += 32) win[i] = i;
  } else {
    // q summed over the group's heads (dims lane and lane + 32)
    float s0 = 0.f, s1 = 0.f;
    for (int h = g * d.G; h < (g + 1) * d.G; ++h) {
      const T* qr = q + (((size_t)b * d.Tq + tq) * d.Hq + h) * 64;
      s0 += to_f32(qr[lane]);
      s1 += to_f32(qr[lane + 32]);
    }
    qsum_s[warp][lane] = s0;
    qsum_s[warp][lane + 32] = s1;
    __syncwarp();
    const float* qs = qsum_s[warp];
    // gates of the complete past blocks j < cur, lane j % 32 holds block j
    float gate[QMAX];
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) {
      const int j = lane + 32 * qq;
      float acc = -INFINITY;
      if (j < cur) {
        const T* kr = kc + (((size_t)b * d.Nc + j) * d.Hkv + g) * 64;
        acc = 0.f;
#pragma unroll 16
        for (int e = 0; e < 64; ++e) acc = fmaf(qs[e], to_f32(kr[e]), acc);
      }
      gate[qq] = acc;
    }
    // k - 1 rounds of a warp argmax: largest gate, lower block on ties
    for (int r = 0; r < n - 1; ++r) {
      float bv = -INFINITY;
      int bj = INT_MAX;
#pragma unroll
      for (int qq = 0; qq < QMAX; ++qq) {
        const int j = lane + 32 * qq;
        if (j < cur && (gate[qq] > bv || (gate[qq] == bv && j < bj))) {
          bv = gate[qq];
          bj = j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (ov > bv || (ov == bv && oj < bj)) {
          bv = ov;
          bj = oj;
        }
      }
      if (lane == 0) win[r] = bj;
#pragma unroll
      for (int qq = 0; qq < QMAX; ++qq)
        if (lane + 32 * qq == bj) gate[qq] = -INFINITY;  // taken (or never a candidate)
    }
    if (lane == 0) win[n - 1] = cur;
    nsel = n;
  }
  __syncwarp();
  if (lane == 0) {  // ascending (at most 64 entries, insertion sort)
    for (int i = 1; i < nsel; ++i)
      for (int r = i; r > 0 && win[r - 1] > win[r]; --r) {
        const int x = win[r];
        win[r] = win[r - 1];
        win[r - 1] = x;
      }
  }
  __syncwarp();
  if (idx_m)
    for (int i = lane; i < n; i += 32) idx_m[row * n + i] = i < nsel ? win[i] : -1;
  // expansion into 64-key blocks, causal (at most the query's own 64-key block)
  const int sub = L / 64, tk = n * sub, last = t / 64;
  for (int i = lane; i < tk; i += 32) {
    const int s = i / sub, w = i % sub;
    int j = -1;
    if (s < nsel) {
      const int jj = win[s] * sub + w;
      j = jj <= last ? jj : -1;
    }
    idx64[row * tk + i] = j;
  }
  // the query's own block is the last chosen, so the -1 entries of its cut
  // 64-key blocks come last: the list is ascending and -1 padded as the
  // selection kernels require
}

// MoBA block indices [rows, n] -> 64-key block indices [rows, n L/64]
// (the backward's view of a forward's selection).
__global__ void moba_expand_kernel(const int32_t* __restrict__ idx_m, int32_t* __restrict__ idx64,
                                   Dims d, int L, int n) {
  const long row = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= (long)d.B * d.Tq * d.Hkv) return;
  const int tq = (int)((row / d.Hkv) % d.Tq);
  const int t = d.q_off + tq, last = t / 64;
  const int sub = L / 64, tk = n * sub;
  int32_t* r = idx64 + row * tk;
  int wpos = 0;
  for (int s = 0; s < n; ++s) {
    const int m = idx_m[row * n + s];
    if (m < 0) continue;
    for (int w = 0; w < sub; ++w) {
      const int jj = m * sub + w;
      if (jj <= last && wpos < tk) r[wpos++] = jj;
    }
  }
  for (; wpos < tk; ++wpos) r[wpos] = -1;
}

cudaError_t launch_moba_select(const Dims& d, const void* q, const void* kc, int32_t* idx_m,
                               int32_t* idx64, int L, int n, cudaStream_t s) {
  const long rows = (long)d.B * d.Tq * d.Hkv;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kMobaWarps - 1) / kMobaWarps);
  const int nb = d.T / L;  // complete MoBA blocks: at most nb candidates
  if (d.dtype == 1) {
    if (nb <= 32) moba_select_kernel<bf16, 1><<<blocks, kMobaWarps * 32, 0, s>>>((const bf16*)q, (const bf16*)kc, idx_m, idx64, d, L, n);
    else moba_select_kernel<bf16, 4><<<blocks, kMobaWarps * 32, 0, s>>>((const bf16*)q, (const bf16*)kc, idx_m, idx64, d, L, n);
  } else {
    if (nb <= 32) moba_select_kernel<float, 1><<<blocks, kMobaWarps * 32, 0, s>>>((const float*)q, (const float*)kc, idx_m, idx64, d, L, n);
    else moba_select_kernel<float, 4><<<blocks, kMobaWarps * 32, 0, s>>>((const float*)q, (const float*)kc, idx_m, idx64, d, L, n);
  }
  return cudaGetLastError();
}

cudaError_t launch_moba_expand(const Dims& d, const int32_t* idx_m, int32_t* idx64, int L, int n,
                               cudaStream_t s) {
  const long rows = (long)d.B * d.Tq * d.Hkv;
  if (rows == 0) return cudaSuccess;
  moba_expand_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(idx_m, idx64, d, L, n);
  return cudaGetLastError();
}

}  // namespace nsa
