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
// One warp per row.  Each of the topk - 2 rounds is a warp arg-max over the
// still-free candidates (lanes stride over blocks), ordered by
// (score desc, index asc); a per-warp bitmap in shared memory records the
// winners, and the ascending list is read back from the bitmap.
#include "common.cuh"
#include "internal.h"

namespace nsa {

constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ score, int32_t* __restrict__ idx, Dims d,
            int words) {
  extern __shared__ uint32_t bits_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* bits = bits_all + (size_t)warp * words;
  const long row = (long)blockIdx.x * kTopkWarps + warp;
  const long nrows = (long)d.B * d.Tq * d.Hkv;
  if (row >= nrows) return;
  const int tq = (int)((row / d.Hkv) % d.Tq);
  const int t = d.q_off + tq;
  const int cur = t / d.l;
  int32_t* out = idx + row * d.topk;
  if (cur + 1 <= d.topk) {
    for (int s = lane; s < d.topk; s += 32) out[s] = s <= cur ? s : -1;
    return;
  }
  const float* sr = score + row * d.Nc;
  for (int w = lane; w < words; w += 32) bits[w] = 0u;
  __syncwarp();
  for (int r = 0; r < d.topk - 2; ++r) {
    float best = -INFINITY;
    int bj = 0x7fffffff;
    for (int j = 1 + lane; j < cur; j += 32) {
      if (bits[j >> 5] & (1u << (j & 31))) continue;
      const float s = sr[j];
      if (s > best || (s == best && j < bj)) {
        best = s;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ob > best || (ob == best && oj < bj)) {
        best = ob;
        bj = oj;
      }
    }
    // every lane holds the same winner; none only if all free scores are NaN
    if (bj == 0x7fffffff) break;
    if (lane == 0) bits[bj >> 5] |= 1u << (bj & 31);
    __syncwarp();
  }
  if (lane == 0) {
    bits[0] |= 1u;
    bits[cur >> 5] |= 1u << (cur & 31);
  }
  __syncwarp();
  // ascending write-out: lanes own 32-block words, prefix count over lanes
  int base = 0;
  for (int w0 = 0; w0 <= (cur >> 5); w0 += 32) {
    const int w = w0 + lane;
    const uint32_t m = w <= (cur >> 5) ? bits[w] : 0u;
    const int c = __popc(m);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - c;
    uint32_t mm = m;
    while (mm) {
      const int bit = __ffs(mm) - 1;
      mm &= mm - 1;
      if (pos < d.topk) out[pos] = w * 32 + bit;
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int p = base + lane; p < d.topk; p += 32) out[p] = -1;
}

cudaError_t launch_topk(const Dims& d, const float* score, int32_t* idx,
                        cudaStream_t s) {
  const long nrows = (long)d.B * d.Tq * d.Hkv;
  const int words = (d.Nb + 31) / 32;
  const size_t smem = (size_t)kTopkWarps * words * sizeof(uint32_t);
  const long blocks = (nrows + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<<<(unsigned)blocks, kTopkWarps * 32, smem, s>>>(score, idx, d, words);
  return cudaGetLastError();
}

}  // namespace nsa
