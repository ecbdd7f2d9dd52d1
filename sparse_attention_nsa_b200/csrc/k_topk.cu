// k_topk.cu -- per-(query, KV group) top-k block selection.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work? (SELECTION): keep the most important blocks in raw form.
// "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method (block 64,
// top-k 16) and Key claims (NSA always includes the first block).
// Rule: cur = t / l.  With at most topk causal blocks every one of them is
// taken; otherwise blocks 0 and cur are forced and the topk - 2 best of
// 1..cur-1 are added, equal scores going to the lower block index.  The
// output is ascending and padded with -1.
//
// One warp per row, no shared memory.  Lane `lane` holds the candidates
// 1 + lane + 32 q in registers as order-preserving integer keys.  A radix
// select finds tau, the (topk-2)-th largest key, bit by bit from the top
// (each step one warp-wide count with redux.sync).  The winners are every
// key above tau plus, among keys equal to tau, the lowest block indices
// (ballots in ascending block order); they are written out in ascending
// order between the forced blocks 0 and cur.
#include "common.cuh"
#include "internal.h"

namespace nsa {

constexpr int kTopkWarps = 8;

// Monotone map of a float to uint32 (larger float -> larger key); NaN -> 0.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int QMAX>
__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ score, int32_t* __restrict__ idx, Dims d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long r = (long)blockIdx.x * kTopkWarps + warp;
  const long nrows = (long)d.B * d.Tq * d.Hkv;
  if (r >= nrows) return;
  const int tq = (int)((r / d.Hkv) % d.Tq);
  const int t = d.q_off + tq;
  const int cur = t / d.l;
  int32_t* out = idx + r * d.topk;
  if (cur + 1 <= d.topk) {
    for (int s = lane; s < d.topk; s += 32) out[s] = s <= cur ? s : -1;
    return;
  }
  // candidates are blocks 1..cur-1 (all complete, so all have scores)
  const float* sr = score + r * d.Nc;
  uint32_t key[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int j = 1 + lane + 32 * q;
    key[q] = j < cur ? order_key(__ldg(sr + j)) : 0u;
  }
  const int K2 = d.topk - 2;
  // tau = the largest value with at least K2 keys >= tau (absent slots are
  // excluded from the counts)
  uint32_t tau = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t tc = tau | (1u << bit);
    unsigned c = 0;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) c += (1 + lane + 32 * q < cur && key[q] >= tc) ? 1u : 0u;
    if ((int)__reduce_add_sync(0xffffffffu, c) >= K2) tau = tc;
  }
  unsigned cg = 0;
#pragma unroll
  for (int q = 0; q < QMAX; ++q) cg += (1 + lane + 32 * q < cur && key[q] > tau) ? 1u : 0u;
  const int need = K2 - (int)__reduce_add_sync(0xffffffffu, cg);  // >= 1 keys equal to tau
  int eq_before = 0, pos = 1;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int j = 1 + lane + 32 * q;
    const bool ok = j < cur;
    const bool eq = ok && key[q] == tau;
    const unsigned em = __ballot_sync(0xffffffffu, eq);
    const bool win = ok && (key[q] > tau || (eq && eq_before + __popc(em & lt) < need));
    const unsigned wm = __ballot_sync(0xffffffffu, win);
    if (win) out[pos + __popc(wm & lt)] = j;
    pos += __popc(wm);
    eq_before += __popc(em);
  }
  if (lane == 0) {
    out[0] = 0;
    out[K2 + 1] = cur;
  }
}

cudaError_t launch_topk(const Dims& d, const float* score, int32_t* idx,
                        cudaStream_t s) {
  const long nrows = (long)d.B * d.Tq * d.Hkv;
  const unsigned blocks = (unsigned)((nrows + kTopkWarps - 1) / kTopkWarps);
  const int q = (d.Nb + 31) / 32;  // candidate slots per lane
  if (q <= 4) topk_kernel<4><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else if (q <= 8) topk_kernel<8><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else if (q <= 16) topk_kernel<16><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else topk_kernel<32><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  return cudaGetLastError();
}

}  // namespace nsa
