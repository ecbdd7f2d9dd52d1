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
// One warp per row.  The row's candidate scores are staged in shared
// memory; each lane keeps the best of its own candidates (blocks
// 1 + lane + 32q), each of the topk - 2 rounds is a warp arg-max over those
// lane bests ordered by (score desc, index asc), and only the winning lane
// rescans its candidates.  A per-warp bitmap records the winners and the
// ascending list is read back from it.
#include "common.cuh"
#include "internal.h"

namespace nsa {

constexpr int kTopkWarps = 8;

// Best not-yet-taken candidate of this lane: blocks 1 + lane + 32 q, q < 32,
// below cur, ordered by (score desc, index asc).
__device__ __forceinline__ void lane_best(const float* row, int cur, int lane, uint32_t taken,
                                          float& bv, int& bj) {
  bv = -INFINITY;
  bj = 0x7fffffff;
  for (int q = 0; q < 32; ++q) {
    const int j = 1 + lane + 32 * q;
    if (j >= cur) break;
    if ((taken >> q) & 1u) continue;
    const float v = row[j];
    if (v > bv || (v == bv && j < bj)) {
      bv = v;
      bj = j;
    }
  }
}

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ score, int32_t* __restrict__ idx, Dims d, int words) {
  extern __shared__ uint32_t sm_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* row = reinterpret_cast<float*>(sm_all) + (size_t)warp * (d.Nc + words);
  uint32_t* bits = reinterpret_cast<uint32_t*>(row + d.Nc);
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
  for (int j = lane; j < cur; j += 32) row[j] = sr[j];
  for (int w = lane; w < words; w += 32) bits[w] = 0u;
  __syncwarp();
  uint32_t taken = 0;
  float bv;
  int bj;
  lane_best(row, cur, lane, taken, bv, bj);
  for (int k = 0; k < d.topk - 2; ++k) {
    float wv = bv;
    int wj = bj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, wj, o);
      if (ov > wv || (ov == wv && oj < wj)) {
        wv = ov;
        wj = oj;
      }
    }
    if (wj == 0x7fffffff) break;  // only NaN scores left
    if (lane == ((wj - 1) & 31)) {
      taken |= 1u << ((wj - 1) >> 5);
      lane_best(row, cur, lane, taken, bv, bj);
    }
    if (lane == 0) bits[wj >> 5] |= 1u << (wj & 31);
  }
  __syncwarp();
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
  const size_t smem = (size_t)kTopkWarps * (d.Nc + words) * sizeof(uint32_t);
  const long blocks = (nrows + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<<<(unsigned)blocks, kTopkWarps * 32, smem, s>>>(score, idx, d, words);
  return cudaGetLastError();
}

}  // namespace nsa
