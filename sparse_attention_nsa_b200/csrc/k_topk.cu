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
// One warp per row, no shared memory: the radix select of topk.cuh over the
// row's fp32 scores read straight from global memory.  With a compression
// block or stride other than the selection block ("Sparsity is Cool",
// Method, and "DeepSeek's Native Sparse Attention", COMPRESSION, give block
// size and stride as parameters), the importance of selection block j is
// the sum, in ascending order, of the scores of the compressed blocks whose
// tokens overlap it (compressed block i covers [i dc, i dc + lc), selection
// block j covers [j l, (j + 1) l)); the sum is formed as each candidate's
// key is loaded.
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace nsa {

constexpr int kTopkWarps = 8;

template <int QMAX, bool REMAP>
__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ score, int32_t* __restrict__ idx, Dims d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x * kTopkWarps + warp;  // row within the sequence: tq * Hkv + g
  if (rb >= d.Tq * d.Hkv) return;
  const int t = d.q_off + rb / d.Hkv;
  for (int b = blockIdx.y; b < d.B; b += gridDim.y) {
    const size_t r = (size_t)b * d.Tq * d.Hkv + rb;
    // candidates are blocks 1..cur-1 (all complete, so all have scores)
    const float* row = score + r * d.Nc;
    if (!REMAP) {
      warp_select_blocks<QMAX>(row, t / d.l, d.topk, idx + r * d.topk, lane);
    } else {
      auto remap = [row, &d](int j) {
        const int lo = j * d.l;  // selection block j: tokens [lo, lo + l)
        const int ilo = lo < d.lc ? 0 : (lo - d.lc) / d.dc + 1;
        const int ihi = min((lo + d.l - 1) / d.dc, d.Nc - 1);
        float acc = 0.f;
        for (int i = ilo; i <= ihi; ++i) acc += row[i];
        return acc;
      };
      warp_select_blocks_fn<QMAX>(remap, t / d.l, d.topk, idx + r * d.topk, lane);
    }
  }
}

template <bool REMAP>
static void launch_topk_t(const Dims& d, const float* score, int32_t* idx, dim3 blocks, int q,
                          cudaStream_t s) {
  if (q <= 4) topk_kernel<4, REMAP><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else if (q <= 8) topk_kernel<8, REMAP><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else if (q <= 16) topk_kernel<16, REMAP><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
  else topk_kernel<32, REMAP><<<blocks, kTopkWarps * 32, 0, s>>>(score, idx, d);
}

cudaError_t launch_topk(const Dims& d, const float* score, int32_t* idx,
                        cudaStream_t s) {
  const long rows = (long)d.Tq * d.Hkv;  // per sequence (< 2^31: Tq < 2^24, Hkv <= 128)
  if (rows == 0 || d.B == 0) return cudaSuccess;
  if (rows > INT_MAX - kTopkWarps) return cudaErrorInvalidValue;
  const dim3 blocks((unsigned)((rows + kTopkWarps - 1) / kTopkWarps), (unsigned)min(d.B, 65535));
  const int q = (d.Nb + 31) / 32;  // candidate slots per lane
  if (plain_geometry(d)) launch_topk_t<false>(d, score, idx, blocks, q, s);
  else launch_topk_t<true>(d, score, idx, blocks, q, s);
  return cudaGetLastError();
}

}  // namespace nsa
