// k_decode.cu -- single-token NSA decode, split for HBM bandwidth.
//
// One query per sequence at position T-1 (the pages' method applied to the
// last position: "DeepSeek's Native Sparse Attention", How Does Native
// Sparse Attention Work? -- compression, selection, sliding window, gated
// merge).  Decode reads each cached byte once, so it is bound by HBM; the
// work is split so that all SMs stream:
//   K1  one single-warp CTA per (64-block chunk of the compressed cache,
//       group, sequence): S = Q Kc^T for the G query heads stacked as MMA
//       rows, the chunk's softmax partial (max, sum, P Vc) and the scaled
//       logits for the block scores;
//   K2  one single-warp CTA per (sequence, group, 64-key block) of the
//       window or the selection: TMA-loads that block's K and V and computes
//       the block's unnormalised softmax partial (max, sum, P V).  Window
//       blocks are known up front and start before K1 ends; every selection
//       CTA first computes the group's block scores from K1's logits and the
//       top-k (the same in each), then takes its own slot's block;
//   K3  per (sequence, group): merges the partials of the three branches and
//       applies the gates.
// The head dimension contractions use warp-level mma.sync (m16n8k16, bf16 in,
// fp32 accumulate): with G <= 16 heads per group the row count is 16, below
// the 64/128-row tcgen05 tiles, and the kernel is bandwidth-bound anyway.
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace nsa {
namespace {

using namespace sm100;

constexpr int kPartStride = 66;  // o[64], m (log2 units), l per row
constexpr int kMaxChunks = 16;   // 64-block chunks of the compressed cache (Nc <= 1024)

__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int chunk) {
  return base + (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D += A B, m16n8k16, bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Stage the G query rows of one (sequence, group) as a 16 x 64 bf16 tile
// with the 128-byte swizzle (rows >= G are zero).  32 threads of one warp.
__device__ __forceinline__ void stage_q(uint8_t* qs, const bf16* qrow0, int G, int lane) {
  const uint32_t base = smem_u32(qs);
  for (int e = lane; e < 16 * 8; e += 32) {
    const int row = e >> 3, chunk = e & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < G) v = *reinterpret_cast<const uint4*>(qrow0 + row * 64 + chunk * 8);
    st_shared_v4(swz(base, row, chunk), v.x, v.y, v.z, v.w);
  }
}

// A fragments of the 16 x 64 Q tile for the four 16-wide k steps.
__device__ __forceinline__ void load_qa(uint32_t qa[4][4], uint32_t qbase, int lane) {
  const int mi = lane >> 3;
  const int row = (mi & 1) * 8 + (lane & 7);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) ldsm_x4(qa[kk], swz(qbase, row, 2 * kk + (mi >> 1)));
}

// S[16 x 64] = Q K^T for a 64-row key tile at kbase (keys key0 .. key0+63 of
// the tile); acc[nt] holds n-tile nt (8 keys).
__device__ __forceinline__ void qk_tile(float acc[8][4], const uint32_t qa[4][4], uint32_t kbase,
                                        int key0, int lane) {
  const int mi = lane >> 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    const int key = key0 + 16 * np + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t kb[4];
      ldsm_x4(kb, swz(kbase, key, 2 * kk + (mi & 1)));
      mma16816(acc[2 * np], qa[kk], kb[0], kb[1]);
      mma16816(acc[2 * np + 1], qa[kk], kb[2], kb[3]);
    }
  }
}

// O[16 x 64] += P V for a 64-key tile: P from the S accumulators (bf16),
// V rows key0 .. key0+63 of the tile at vbase.
__device__ __forceinline__ void pv_tile(float o[8][4], const float p[8][4], uint32_t vbase,
                                        int key0, int lane) {
  const int mi = lane >> 3;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
    const int key = key0 + 16 * kk + (mi & 1) * 8 + (lane & 7);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t vb[4];
      ldsm_x4_t(vb, swz(vbase, key, 2 * np + (mi >> 1)));
      mma16816(o[2 * np], a, vb[0], vb[1]);
      mma16816(o[2 * np + 1], a, vb[2], vb[3]);
    }
  }
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

struct DecodeWs {
  float* pcmp;   // [B*Hkv][nchunk][16][66]  compression-branch partials
  float* logit;  // [B*Hkv][16][Nc]          compression logits (log2 units)
  int* idx;      // [B*Hkv][topk]
  float* psel;   // [B*Hkv][topk][16][66]
  float* pswa;   // [B*Hkv][nwin][16][66]
  int nwin;      // window blocks of the decoded position
  int jlo;       // first window block
  int nchunk;    // 64-block chunks of the compressed cache
};

// Softmax partial of one 64-key tile for the 16 MMA rows (rows >= G and
// invisible keys are -inf in p on entry): writes (P V, max, sum) to part in
// the [16][kPartStride] layout; p is replaced by its exponentials.
__device__ __forceinline__ void tile_partial(float p[8][4], uint32_t vbase, float* part,
                                             bool need_o, int lane) {
  const int r0 = lane >> 2, cq = lane & 3;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    mx0 = fmaxf(mx0, fmaxf(p[nt][0], p[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(p[nt][2], p[nt][3]));
  }
  mx0 = quad_max(mx0);
  mx1 = quad_max(mx1);
  const float b0 = mx0 == -INFINITY ? 0.f : mx0, b1 = mx1 == -INFINITY ? 0.f : mx1;
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    p[nt][0] = fast_exp2(p[nt][0] - b0);
    p[nt][1] = fast_exp2(p[nt][1] - b0);
    p[nt][2] = fast_exp2(p[nt][2] - b1);
    p[nt][3] = fast_exp2(p[nt][3] - b1);
    l0 += p[nt][0] + p[nt][1];
    l1 += p[nt][2] + p[nt][3];
  }
  l0 = quad_sum(l0);
  l1 = quad_sum(l1);
  if (need_o) {
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    pv_tile(o, p, vbase, 0, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      part[r0 * kPartStride + nt * 8 + 2 * cq] = o[nt][0];
      part[r0 * kPartStride + nt * 8 + 2 * cq + 1] = o[nt][1];
      part[(r0 + 8) * kPartStride + nt * 8 + 2 * cq] = o[nt][2];
      part[(r0 + 8) * kPartStride + nt * 8 + 2 * cq + 1] = o[nt][3];
    }
  }
  if (cq == 0) {
    part[r0 * kPartStride + 64] = mx0;
    part[r0 * kPartStride + 65] = l0;
    part[(r0 + 8) * kPartStride + 64] = mx1;
    part[(r0 + 8) * kPartStride + 65] = l1;
  }
}

// ---- K1: compression branch over one 64-block chunk of the compressed cache --------
// One single-warp CTA per (chunk, group, sequence), so every SM streams the
// compressed cache: S = Q Kc^T for the G heads of the group (rows of the
// m16n8k16 MMA), the chunk's softmax partial (max, sum, P Vc) for the
// compression branch, and the scaled logits for the block scores.
__global__ void __launch_bounds__(32)
decode_cmp_chunk_kernel(const __grid_constant__ CUtensorMap tm_kc,
                        const __grid_constant__ CUtensorMap tm_vc, const bf16* __restrict__ q,
                        Dims d, DecodeWs ws, int need_o, int* err) {
  __shared__ __align__(1024) uint8_t kv[2 * 8192];
  __shared__ __align__(1024) uint8_t qs[2048];
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  const int lane = threadIdx.x;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int bg = b * d.Hkv + g;
  const int t = d.T - 1;
  const int nvis = min((t + 1) / d.l, d.Nc);  // complete blocks
  pdl_launch_dependents();
  if (lane == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    abort_s = 0;
  }
  __syncwarp();
  if (lane == 0) {
    mbar_expect_tx(&bar, (need_o ? 2u : 1u) * 8192u);
    tma_load_3d(kv, &tm_kc, &bar, 0, g, b * d.Nc + c * 64);
    if (need_o) tma_load_3d(kv + 8192, &tm_vc, &bar, 0, g, b * d.Nc + c * 64);
  }
  stage_q(qs, q + ((size_t)b * d.Hq + (size_t)g * d.G) * 64, d.G, lane);
  fence_proxy_async_smem();
  __syncwarp();
  uint32_t qa[4][4];
  load_qa(qa, smem_u32(qs), lane);
  if (!wait_bar(&bar, 0, (volatile int*)&abort_s, err)) {
    drain_bar(&bar, 0);  // let the copies land before the CTA exits
    return;
  }
  float s[8][4];
  qk_tile(s, qa, smem_u32(kv), 0, lane);
  const int r0 = lane >> 2, cq = lane & 3;
  const float sl2 = d.scale * kLog2e;
  float* lg = ws.logit + (size_t)bg * 16 * d.Nc;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = c * 64 + nt * 8 + 2 * cq + (e & 1);
      const int row = r0 + (e >> 1) * 8;
      const bool vis = j < nvis && row < d.G;
      s[nt][e] = vis ? s[nt][e] * sl2 : -INFINITY;
      if (row < d.G && j < d.Nc) lg[(size_t)row * d.Nc + j] = s[nt][e];
    }
  tile_partial(s, smem_u32(kv + 8192), ws.pcmp + ((size_t)bg * ws.nchunk + c) * 16 * kPartStride,
               need_o != 0, lane);
}

// ---- the block selection of one (sequence, group), by one warp ----------------------
// lse of each head row from the compression chunk partials, block scores
// score_j = sum over the group's heads of exp2(logit - lse2), then the warp
// radix select of topk.cuh.  Every load of a step is issued before any is
// used (fixed trip counts, predicated).
template <int QMAX>
__device__ __forceinline__ void decode_select(const Dims& d, const DecodeWs& ws, int bg, int lane,
                                              float* score, int* idx, float* lse2s) {
  const int t = d.T - 1;
  const int cur = t / d.l;
  const int nvis = min((t + 1) / d.l, d.Nc);
  if (lane < 16) {
    float M = -INFINITY, L = 0.f;
    if (lane < d.G) {
      const float* part =
          ws.pcmp + (size_t)bg * ws.nchunk * 16 * kPartStride + lane * kPartStride;
      float m[kMaxChunks], l[kMaxChunks];
#pragma unroll
      for (int c = 0; c < kMaxChunks; ++c) {
        const bool ok = c < ws.nchunk;
        m[c] = ok ? part[(size_t)c * 16 * kPartStride + 64] : -INFINITY;
        l[c] = ok ? part[(size_t)c * 16 * kPartStride + 65] : 0.f;
      }
#pragma unroll
      for (int c = 0; c < kMaxChunks; ++c) M = fmaxf(M, m[c]);
#pragma unroll
      for (int c = 0; c < kMaxChunks; ++c)
        if (m[c] != -INFINITY) L += fast_exp2(m[c] - M) * l[c];
    }
    lse2s[lane] = L > 0.f ? M + __log2f(L) : INFINITY;  // no visible block: scores 0
  }
  __syncwarp();
  const float* lg = ws.logit + (size_t)bg * 16 * d.Nc;
  for (int j0 = 0; j0 < QMAX * 32; j0 += 128) {
    float x[4][16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + 32 * q + lane;
#pragma unroll
      for (int r = 0; r < 16; ++r)
        x[q][r] = (r < d.G && j < nvis) ? lg[(size_t)r * d.Nc + j] : -INFINITY;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float sc = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < d.G) sc += fast_exp2(x[q][r] - lse2s[r]);
      if (j0 + 32 * q < QMAX * 32) score[j0 + 32 * q + lane] = sc;
    }
  }
  __syncwarp();
  warp_select_blocks<QMAX>(score, cur, d.topk, idx, lane);
  __syncwarp();
}

// ---- K2: one 64-key block of the window or the selection ------------------------------
template <int QMAX>
__global__ void __launch_bounds__(32)
decode_block_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const bf16* __restrict__ q, Dims d, DecodeWs ws, int32_t* __restrict__ idx_out,
                    int do_sel, int do_swa, int* err) {
  __shared__ __align__(1024) uint8_t kv[2 * 8192];
  __shared__ __align__(1024) uint8_t qs[2048];
  __shared__ float score_s[QMAX * 32];
  __shared__ int idx_s[64];
  __shared__ float lse2_s[16];
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  const int lane = threadIdx.x;
  const int u = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int bg = b * d.Hkv + g;
  const int t = d.T - 1;
  const int cur = t / d.l;
  pdl_launch_dependents();
  // which block and branch: window blocks are known before the selection, so
  // their loads start before K1 has finished; a selected block inside the
  // window gets its own CTA (the two branches mask it differently)
  int j, sel_slot = -1;
  bool win = false;
  if (u < ws.nwin) {
    if (!do_swa) {
      pdl_wait();  // completion of this grid implies completion of the ones before
      return;
    }
    j = ws.jlo + u;
    win = true;
  } else {
    pdl_wait();
    if (!do_sel) return;
    // every selection CTA of the (sequence, group) runs the same selection
    // (no kernel boundary between the scores and their use); slot 0 stores it
    const int m = u - ws.nwin;
    decode_select<QMAX>(d, ws, bg, lane, score_s, idx_s, lse2_s);
    if (m == 0)
      for (int s = lane; s < d.topk; s += 32) {
        ws.idx[(size_t)bg * d.topk + s] = idx_s[s];
        if (idx_out) idx_out[(size_t)bg * d.topk + s] = idx_s[s];
      }
    j = idx_s[m];
    if (j < 0) return;
    if (j > cur) {  // never read a non-causal block
      if (lane == 0) record_error(err, kDevBadIndex);
      return;
    }
    sel_slot = m;
  }
  if (lane == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    abort_s = 0;
  }
  __syncwarp();
  if (lane == 0) {
    mbar_expect_tx(&bar, 2 * 8192u);
    tma_load_3d(kv, &tm_k, &bar, 0, g, b * d.T + j * 64);
    tma_load_3d(kv + 8192, &tm_v, &bar, 0, g, b * d.T + j * 64);
  }
  stage_q(qs, q + ((size_t)b * d.Hq + (size_t)g * d.G) * 64, d.G, lane);
  fence_proxy_async_smem();
  __syncwarp();
  uint32_t qa[4][4];
  load_qa(qa, smem_u32(qs), lane);
  if (!wait_bar(&bar, 0, (volatile int*)&abort_s, err)) {
    drain_bar(&bar, 0);  // let the copies land before the CTA exits
    return;
  }
  float s[8][4];
  qk_tile(s, qa, smem_u32(kv), 0, lane);
  const int r0 = lane >> 2, cq = lane & 3;
  const float sl2 = d.scale * kLog2e;
  for (int br = 0; br < 2; ++br) {
    const bool is_sel = br == 0;
    if (is_sel ? sel_slot < 0 : !win) continue;
    const int lo = is_sel ? 0 : max(0, t - d.window + 1);
    float p[8][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 64 + nt * 8 + 2 * cq + (e & 1);
        const bool vis = key <= t && key >= lo;
        p[nt][e] = vis ? s[nt][e] * sl2 : -INFINITY;
        if (e < 2) mx0 = fmaxf(mx0, p[nt][e]);
        else mx1 = fmaxf(mx1, p[nt][e]);
      }
    mx0 = quad_max(mx0);
    mx1 = quad_max(mx1);
    const float b0 = mx0 == -INFINITY ? 0.f : mx0, b1 = mx1 == -INFINITY ? 0.f : mx1;
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      p[nt][0] = fast_exp2(p[nt][0] - b0);
      p[nt][1] = fast_exp2(p[nt][1] - b0);
      p[nt][2] = fast_exp2(p[nt][2] - b1);
      p[nt][3] = fast_exp2(p[nt][3] - b1);
      l0 += p[nt][0] + p[nt][1];
      l1 += p[nt][2] + p[nt][3];
    }
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    pv_tile(o, p, smem_u32(kv + 8192), 0, lane);
    float* part = is_sel ? ws.psel + ((size_t)bg * d.topk + sel_slot) * 16 * kPartStride
                         : ws.pswa + ((size_t)bg * ws.nwin + u) * 16 * kPartStride;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      part[r0 * kPartStride + nt * 8 + 2 * cq] = o[nt][0];
      part[r0 * kPartStride + nt * 8 + 2 * cq + 1] = o[nt][1];
      part[(r0 + 8) * kPartStride + nt * 8 + 2 * cq] = o[nt][2];
      part[(r0 + 8) * kPartStride + nt * 8 + 2 * cq + 1] = o[nt][3];
    }
    if (cq == 0) {
      part[r0 * kPartStride + 64] = mx0;
      part[r0 * kPartStride + 65] = l0;
      part[(r0 + 8) * kPartStride + 64] = mx1;
      part[(r0 + 8) * kPartStride + 65] = l1;
    }
  }
  if (win) pdl_wait();  // completion of this grid implies completion of the ones before
}

// ---- K3: merge the partials of each branch and apply the gates ------------------------
// One warp per query head.  The slots of all three branches (compression
// chunks, selected blocks, window blocks) are one list: lanes read the
// slots' (max, sum) in parallel, the warp reduces them per branch, then the
// slots' 64-wide partial outputs are folded in 16 at a time with every load
// of a batch issued before any is used.
__global__ void __launch_bounds__(32)
decode_merge_kernel(const float* __restrict__ gates, bf16* __restrict__ out, Dims d,
                    DecodeWs ws) {
  // one single-warp CTA per (sequence and group, head): small enough to be
  // resident beside the block kernel's CTAs and wait there (PDL)
  const int bg = blockIdx.x;
  const int row = blockIdx.y, lane = threadIdx.x;
  pdl_wait();
  const int b = bg / d.Hkv, g = bg % d.Hkv;
  const int h = g * d.G + row;
  const int t = d.T - 1;
  const int cur = t / d.l;
  const int* sel = ws.idx + (size_t)bg * d.topk;
  const float* grow = gates + ((size_t)b * d.Hq + h) * 3;
  const int nc = (d.branch_mask & 1) ? ws.nchunk : 0;
  const int nsel = (d.branch_mask & 2) ? d.topk : 0;
  const int nw = (d.branch_mask & 4) ? ws.nwin : 0;
  const int ns = nc + nsel + nw;
  auto slot_ptr = [&](int s) -> const float* {
    if (s < nc) return ws.pcmp + ((size_t)bg * ws.nchunk + s) * 16 * kPartStride + row * kPartStride;
    s -= nc;
    if (s < nsel) return ws.psel + ((size_t)bg * d.topk + s) * 16 * kPartStride + row * kPartStride;
    s -= nsel;
    return ws.pswa + ((size_t)bg * ws.nwin + s) * 16 * kPartStride + row * kPartStride;
  };
  auto slot_branch = [&](int s) { return s < nc ? 0 : s < nc + nsel ? 1 : 2; };
  auto slot_valid = [&](int s) {  // a selected slot holds a partial only for a real block
    if (s < nc || s >= nc + nsel) return true;
    const int j = sel[s - nc];
    return j >= 0 && j <= cur;
  };
  // Two rounds of loads: every slot's (m, l) and the selected indices at
  // once (lane L holds slots L + 32 k), then the partial rows 16 slots at a
  // time.  Slots past ns or not holding a partial get weight 0.
  constexpr int kMaxSlots = 128;
  float m[kMaxSlots / 32], l[kMaxSlots / 32];
  int br[kMaxSlots / 32];
#pragma unroll
  for (int k = 0; k < kMaxSlots / 32; ++k) {
    const int sl = lane + 32 * k;
    const bool in = sl < ns;
    const float* pr = slot_ptr(in ? sl : 0);  // inside the workspace
    br[k] = in ? slot_branch(sl) : 3;
    m[k] = in ? pr[64] : -INFINITY;
    l[k] = in ? pr[65] : 0.f;
  }
#pragma unroll
  for (int k = 0; k < kMaxSlots / 32; ++k)
    if (br[k] < 3 && !slot_valid(lane + 32 * k)) m[k] = -INFINITY;
  float M0 = -INFINITY, M1 = -INFINITY, M2 = -INFINITY;
#pragma unroll
  for (int k = 0; k < kMaxSlots / 32; ++k) {
    M0 = fmaxf(M0, br[k] == 0 ? m[k] : -INFINITY);
    M1 = fmaxf(M1, br[k] == 1 ? m[k] : -INFINITY);
    M2 = fmaxf(M2, br[k] == 2 ? m[k] : -INFINITY);
  }
  M0 = warp_max(M0);
  M1 = warp_max(M1);
  M2 = warp_max(M2);
  float L0 = 0.f, L1 = 0.f, L2 = 0.f;
  float fw[kMaxSlots / 32];
#pragma unroll
  for (int k = 0; k < kMaxSlots / 32; ++k) {
    const float Mb = br[k] == 0 ? M0 : br[k] == 1 ? M1 : M2;
    fw[k] = (br[k] < 3 && m[k] != -INFINITY) ? fast_exp2(m[k] - Mb) : 0.f;
    if (br[k] == 0) L0 += fw[k] * l[k];
    else if (br[k] == 1) L1 += fw[k] * l[k];
    else if (br[k] == 2) L2 += fw[k] * l[k];
  }
  float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f, a20 = 0.f, a21 = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxSlots / 32; ++k) {
    if (32 * k >= ns) break;
    {
      constexpr int i0 = 0;  // all 32 slots of this group of loads in flight together
      float fs[32], x0[32], x1[32];
      int bs[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int i = i0 + q;
        fs[q] = __shfl_sync(0xffffffffu, fw[k], i);
        bs[q] = __shfl_sync(0xffffffffu, br[k], i);
        const bool use = 32 * k + i < ns && fs[q] != 0.f;
        const float* pr = slot_ptr(use ? 32 * k + i : 0);
        x0[q] = use ? pr[lane] : 0.f;
        x1[q] = use ? pr[lane + 32] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float w0 = bs[q] == 0 ? fs[q] : 0.f, w1 = bs[q] == 1 ? fs[q] : 0.f,
                    w2 = bs[q] == 2 ? fs[q] : 0.f;
        a00 = fmaf(w0, x0[q], a00);
        a01 = fmaf(w0, x1[q], a01);
        a10 = fmaf(w1, x0[q], a10);
        a11 = fmaf(w1, x1[q], a11);
        a20 = fmaf(w2, x0[q], a20);
        a21 = fmaf(w2, x1[q], a21);
      }
    }
  }
  L0 = warp_sum(L0);
  L1 = warp_sum(L1);
  L2 = warp_sum(L2);
  const float g0 = L0 > 0.f ? grow[0] / L0 : 0.f, g1 = L1 > 0.f ? grow[1] / L1 : 0.f,
              g2 = L2 > 0.f ? grow[2] / L2 : 0.f;
  bf16* o = out + ((size_t)b * d.Hq + h) * 64;
  o[lane] = __float2bfloat16_rn(g0 * a00 + g1 * a10 + g2 * a20);
  o[lane + 32] = __float2bfloat16_rn(g0 * a01 + g1 * a11 + g2 * a21);
}

int window_blocks(const Dims& d, int* jlo) {
  const int t = d.T - 1;
  *jlo = max(0, t - d.window + 1) / d.l;
  return t / d.l - *jlo + 1;
}

}  // namespace

// Decode with the split kernels applies to bf16, block 64, G <= 16 heads per
// group (the 16 MMA rows), up to 1024 compressed blocks (the top-k warp's
// registers) and one query.
bool decode_split_eligible(const Dims& d) {
  if (!(d.Tq == 1 && d.dtype == 1 && d.l == 64 && plain_geometry(d) && d.D == 64 && d.G <= 16 &&
        d.Nc <= 1024 &&
        tmap_encode_fn() != nullptr))
    return false;
  int jlo = 0;
  const int slots = (d.Nc + 63) / 64 + d.topk + window_blocks(d, &jlo);
  return slots <= 128;  // the merge holds up to 128 partial slots per row
}

namespace {
size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

size_t decode_split_ws_bytes(const Dims& d) {
  int jlo;
  const int nwin = window_blocks(d, &jlo);
  const size_t bgn = (size_t)d.B * d.Hkv;
  const size_t nchunk = (size_t)(d.Nc + 63) / 64;
  return al256(bgn * nchunk * 16 * kPartStride * 4) + al256(bgn * 16 * (size_t)d.Nc * 4) +
         al256(bgn * d.topk * 4) + al256(bgn * d.topk * 16 * kPartStride * 4) +
         al256(bgn * nwin * 16 * kPartStride * 4);
}

// K1 (chunks of the compressed cache) -> K2 (block scores and top-k, then
// the selected and window blocks) -> K3 (merge, gates), chained with
// programmatic dependent launch: each kernel's prologue overlaps the tail of
// the previous one, and every CTA of a dependent kernel waits for its
// predecessor before it exits, so completion is transitive.
cudaError_t launch_decode_split(const Dims& d, const void* q, const void* kcache,
                                const void* vcache, const void* kc, const void* vc,
                                const float* gates, void* out, int32_t* idx_out, void* ws_ptr,
                                int* err, cudaStream_t s) {
  DecodeWs ws;
  ws.nwin = window_blocks(d, &ws.jlo);
  ws.nchunk = (d.Nc + 63) / 64;
  const size_t bgn = (size_t)d.B * d.Hkv;
  char* w = (char*)ws_ptr;
  ws.pcmp = (float*)w;
  w += al256(bgn * ws.nchunk * 16 * kPartStride * 4);
  ws.logit = (float*)w;
  w += al256(bgn * 16 * (size_t)d.Nc * 4);
  ws.idx = (int*)w;
  w += al256(bgn * d.topk * 4);
  ws.psel = (float*)w;
  w += al256(bgn * d.topk * 16 * kPartStride * 4);
  ws.pswa = (float*)w;
  const bool cmp = d.branch_mask & 1, sel = d.branch_mask & 2, swa = d.branch_mask & 4;
  CUtensorMap mkc{}, mvc{}, mk, mv;
  const bool k1 = d.Nc > 0 && (cmp || sel);
  if (k1) {
    if (!make_tmap_bf16(&mkc, kc, d.Hkv, (long)d.B * d.Nc, 1, 64) ||
        !make_tmap_bf16(&mvc, vc, d.Hkv, (long)d.B * d.Nc, 1, 64))
      return cudaErrorInvalidValue;
  }
  if (!make_tmap_bf16(&mk, kcache, d.Hkv, (long)d.B * d.T, 1, 64) ||
      !make_tmap_bf16(&mv, vcache, d.Hkv, (long)d.B * d.T, 1, 64))
    return cudaErrorInvalidValue;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  const bf16* qb = (const bf16*)q;
  if (k1) {
    decode_cmp_chunk_kernel<<<dim3(ws.nchunk, d.Hkv, d.B), 32, 0, s>>>(mkc, mvc, qb, d, ws,
                                                                      cmp ? 1 : 0, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (sel || swa) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ws.nwin + d.topk, d.Hkv, d.B);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    const int ds = sel ? 1 : 0, dw = swa ? 1 : 0;
    cudaError_t e =
        d.Nc <= 512
            ? cudaLaunchKernelEx(&cfg, decode_block_kernel<16>, mk, mv, qb, d, ws, idx_out, ds, dw, err)
            : cudaLaunchKernelEx(&cfg, decode_block_kernel<32>, mk, mv, qb, d, ws, idx_out, ds, dw, err);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)bgn, (unsigned)d.G);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  bf16* ob = (bf16*)out;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel, gates, ob, d, ws);
}

}  // namespace nsa
