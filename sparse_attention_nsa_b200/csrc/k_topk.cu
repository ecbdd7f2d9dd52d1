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

// With cnt, each row also adds its selected blocks to the reverse map's
// per-(chunk of kRevChunkQueries queries, block) counts, cnt[(b Hkv + g) nchunk
// + chunk][block] (zeroed before), so the map needs no counting pass of its
// own (integer sums: the same counts in any order).
template <int QMAX, bool REMAP>
__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ score, int32_t* __restrict__ idx, int* __restrict__ cnt,
            int nchunk, Dims d) {
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
    if (cnt) {
      __syncwarp();  // the row's indices, written by the warp's lanes, are visible to it
      const int32_t* ir = idx + r * d.topk;
      const int tq = rb / d.Hkv, g = rb - tq * d.Hkv, cur = t / d.l;
      int* crow = cnt + (((size_t)b * d.Hkv + g) * nchunk + tq / kRevChunkQueries) * d.Nb;
      for (int s = lane; s < d.topk; s += 32) {
        const int j = ir[s];
        if (j >= 0 && j <= cur && (s == 0 || ir[s - 1] < j)) atomicAdd(crow + j, 1);
      }
    }
  }
}

template <bool REMAP>
static void launch_topk_t(const Dims& d, const float* score, int32_t* idx, int* cnt, int nchunk,
                          dim3 blocks, int q, cudaStream_t s) {
  const int th = kTopkWarps * 32;
  if (q <= 4) topk_kernel<4, REMAP><<<blocks, th, 0, s>>>(score, idx, cnt, nchunk, d);
  else if (q <= 8) topk_kernel<8, REMAP><<<blocks, th, 0, s>>>(score, idx, cnt, nchunk, d);
  else if (q <= 16) topk_kernel<16, REMAP><<<blocks, th, 0, s>>>(score, idx, cnt, nchunk, d);
  else topk_kernel<32, REMAP><<<blocks, th, 0, s>>>(score, idx, cnt, nchunk, d);
}

cudaError_t launch_topk(const Dims& d, const float* score, int32_t* idx, cudaStream_t s,
                        int* rev_counts) {
  const long rows = (long)d.Tq * d.Hkv;  // per sequence (< 2^31: Tq < 2^24, Hkv <= 128)
  if (rows == 0 || d.B == 0) return cudaSuccess;
  if (rows > INT_MAX - kTopkWarps) return cudaErrorInvalidValue;
  const dim3 blocks((unsigned)((rows + kTopkWarps - 1) / kTopkWarps), (unsigned)min(d.B, 65535));
  const int q = (d.Nb + 31) / 32;  // candidate slots per lane
  const int nchunk = (d.Tq + kRevChunkQueries - 1) / kRevChunkQueries;
  if (rev_counts) {
    const cudaError_t e =
        cudaMemsetAsync(rev_counts, 0, revmap_chunk_ints(d) * sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  if (plain_geometry(d)) launch_topk_t<false>(d, score, idx, rev_counts, nchunk, blocks, q, s);
  else launch_topk_t<true>(d, score, idx, rev_counts, nchunk, blocks, q, s);
  return cudaGetLastError();
}

}  // namespace nsa
