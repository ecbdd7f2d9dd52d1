// k_decode.cu -- single-token NSA decode, split for HBM bandwidth.
//
// One query per sequence at position T-1 (the pages' method applied to the
// last position: "DeepSeek's Native Sparse Attention", How Does Native
// Sparse Attention Work? -- compression, selection, sliding window, gated
// merge).  Decode reads each cached byte once, so it is bound by HBM; the
// work is split so that all SMs stream:
//   K1  one CTA per (sequence, KV group): the compressed keys/values of the
//       sequence (TMA), S = Q Kc^T for the G query heads stacked as MMA rows,
//       softmax, block scores (summed over the group), o_cmp = P Vc, and the
//       top-k selection with forced first/current blocks;
//   K2  one single-warp CTA per (sequence, group, 64-key block) of the
//       window or the selection: TMA-loads that block's K and V, computes
//       the block's unnormalised softmax partial (max, sum, P V) for each
//       branch the block belongs to;
//   K3  per (sequence, group): merges the partials of each branch and applies
//       the gates.
// The head dimension contractions use warp-level mma.sync (m16n8k16, bf16 in,
// fp32 accumulate): with G <= 16 heads per group the row count is 16, below
// the 64/128-row tcgen05 tiles, and the kernel is bandwidth-bound anyway.
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace nsa {
namespace {

using namespace sm100;

constexpr int kPartStride = 66;  // o[64], m (log2 units), l per row

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

// Programmatic dependent launch: the next kernel in the stream may start its
// prologue early; it waits for this grid's completion (and memory) with
// griddepcontrol.wait before touching this grid's outputs.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// (score desc, block asc): does (va, ia) come before (vb, ib)?
__device__ __forceinline__ bool goes_first(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
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
  float* ocmp;   // [B*Hkv][16][64]
  int* idx;      // [B*Hkv][topk]
  float* psel;   // [B*Hkv][topk][16][66]
  float* pswa;   // [B*Hkv][nwin][16][66]
  int nwin;      // window blocks of the decoded position
  int jlo;       // first window block
};

// ---- K1: compression branch, block scores, top-k --------------------------------------
constexpr int kK1Threads = 256;

__global__ void __launch_bounds__(kK1Threads, 1)
decode_cmp_topk_kernel(const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_vc, const bf16* __restrict__ q,
                       Dims d, DecodeWs ws, int32_t* __restrict__ idx_out, int need_o,
                       int need_idx, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int ncp = (d.Nc + 63) & ~63;  // compressed rows staged (64-row TMA boxes)
  // region 0 holds the staged Kc and Vc, later the per-warp o_cmp partials
  const size_t r0_bytes = max((size_t)ncp * 256, (size_t)8 * 16 * 64 * 4);
  uint8_t* kcs = smem;
  uint8_t* vcs = kcs + (size_t)ncp * 128;
  uint8_t* qs = smem + r0_bytes;
  float* red = (float*)(qs + 2048);             // [8 warps][16 rows]
  float* rowM = red + 8 * 16;                   // [16]
  float* rowL = rowM + 16;                      // [16]
  float* score = rowL + 16;                     // [ncp]
  uint32_t* bits = (uint32_t*)(score + ncp);    // [(Nb+31)/32]
  float* sort_v = (float*)(bits + (d.Nb + 31) / 32 + 2);  // [512]
  int* sort_i = (int*)(sort_v + 512);                      // [512]
  uint64_t* bar = (uint64_t*)(((uintptr_t)(sort_i + 512) + 7) & ~(uintptr_t)7);
  volatile int* abort_flag = (volatile int*)(bar + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.x;
  const int b = bg / d.Hkv, g = bg % d.Hkv;
  const int t = d.T - 1;
  const int nvis = min((t + 1) / d.l, d.Nc);
  const int nchunks = ncp / 64;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_barrier_init();
    *abort_flag = 0;
  }
  pdl_launch_dependents();
  __syncthreads();
  if (threadIdx.x == 0 && nchunks > 0) {
    mbar_expect_tx(&bar[0], (uint32_t)nchunks * 8192u);
    for (int c = 0; c < nchunks; ++c)
      tma_load_3d(kcs + c * 8192, &tm_kc, &bar[0], 0, g, b * d.Nc + c * 64);
    if (need_o) {
      mbar_expect_tx(&bar[1], (uint32_t)nchunks * 8192u);
      for (int c = 0; c < nchunks; ++c)
        tma_load_3d(vcs + c * 8192, &tm_vc, &bar[1], 0, g, b * d.Nc + c * 64);
    }
  }
  if (warp == 0) stage_q(qs, q + ((size_t)b * d.Hq + (size_t)g * d.G) * 64, d.G, lane);
  fence_proxy_async_smem();
  __syncthreads();
  const uint32_t qbase = smem_u32(qs);
  const int r0 = lane >> 2, cq = lane & 3;  // fragment row (and r0 + 8), column pair
  const float sl2 = d.scale * kLog2e;
  const int key0 = warp * 64;               // this warp's 64 compressed blocks
  const bool active = key0 < ncp && nvis > 0;
  float s[8][4];
  bool ok = true;
  if (nchunks > 0) ok = wait_bar_warp(&bar[0], 0, abort_flag, err);
  if (active && ok) {
    uint32_t qa[4][4];
    load_qa(qa, qbase, lane);
    qk_tile(s, qa, smem_u32(kcs), key0, lane);
  } else {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
  }
  // scale, mask (block visible, row is a real head), row max
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = key0 + nt * 8 + 2 * cq + (e & 1);
      const int row = r0 + (e >> 1) * 8;
      const bool vis = active && j < nvis && row < d.G;
      s[nt][e] = vis ? s[nt][e] * sl2 : -INFINITY;
      if (e < 2) mx0 = fmaxf(mx0, s[nt][e]);
      else mx1 = fmaxf(mx1, s[nt][e]);
    }
  mx0 = quad_max(mx0);
  mx1 = quad_max(mx1);
  if (cq == 0) {
    red[warp * 16 + r0] = mx0;
    red[warp * 16 + r0 + 8] = mx1;
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    float m = -INFINITY;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w * 16 + threadIdx.x]);
    rowM[threadIdx.x] = m;
  }
  __syncthreads();
  const float M0 = rowM[r0], M1 = rowM[r0 + 8];
  const float b0 = M0 == -INFINITY ? 0.f : M0, b1 = M1 == -INFINITY ? 0.f : M1;
  float sm0 = 0.f, sm1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    s[nt][0] = fast_exp2(s[nt][0] - b0);
    s[nt][1] = fast_exp2(s[nt][1] - b0);
    s[nt][2] = fast_exp2(s[nt][2] - b1);
    s[nt][3] = fast_exp2(s[nt][3] - b1);
    sm0 += s[nt][0] + s[nt][1];
    sm1 += s[nt][2] + s[nt][3];
  }
  sm0 = quad_sum(sm0);
  sm1 = quad_sum(sm1);
  if (cq == 0) {
    red[warp * 16 + r0] = sm0;
    red[warp * 16 + r0 + 8] = sm1;
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    float l = 0.f;
    for (int w = 0; w < 8; ++w) l += red[w * 16 + threadIdx.x];
    rowL[threadIdx.x] = l;
  }
  __syncthreads();
  const float i0 = rowL[r0] > 0.f ? 1.f / rowL[r0] : 0.f;
  const float i1 = rowL[r0 + 8] > 0.f ? 1.f / rowL[r0 + 8] : 0.f;
  // normalised probabilities; block scores = sum over the group's heads
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    s[nt][0] *= i0;
    s[nt][1] *= i0;
    s[nt][2] *= i1;
    s[nt][3] *= i1;
    float c0 = s[nt][0] + s[nt][2], c1 = s[nt][1] + s[nt][3];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      c0 += __shfl_xor_sync(0xffffffffu, c0, off);
      c1 += __shfl_xor_sync(0xffffffffu, c1, off);
    }
    if (r0 == 0 && key0 < ncp) {
      score[key0 + nt * 8 + 2 * cq] = c0;
      score[key0 + nt * 8 + 2 * cq + 1] = c1;
    }
  }
  // o_cmp = P Vc: each warp its 64 blocks, then a sum over warps
  if (need_o) {
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    const bool okv = nchunks > 0 && wait_bar_warp(&bar[1], 0, abort_flag, err);
    if (active && okv) pv_tile(o, s, smem_u32(vcs), key0, lane);
    __syncthreads();  // every warp is done with Kc and Vc: reuse region 0
    float* part = (float*)smem;  // [8 warps][16][64]
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      part[(warp * 16 + r0) * 64 + nt * 8 + 2 * cq] = o[nt][0];
      part[(warp * 16 + r0) * 64 + nt * 8 + 2 * cq + 1] = o[nt][1];
      part[(warp * 16 + r0 + 8) * 64 + nt * 8 + 2 * cq] = o[nt][2];
      part[(warp * 16 + r0 + 8) * 64 + nt * 8 + 2 * cq + 1] = o[nt][3];
    }
    __syncthreads();
    float* dst = ws.ocmp + (size_t)bg * 16 * 64;
    for (int e = threadIdx.x; e < 16 * 64; e += kK1Threads) {
      float acc = 0.f;
      for (int w = 0; w < 8; ++w) acc += part[w * 16 * 64 + e];
      dst[e] = acc;
    }
  } else {
    __syncthreads();
  }
  // top-k over blocks 1..cur-1 (forced: 0 and cur).  Each warp sorts the
  // candidates among its 64 blocks by (score desc, block asc) with a bitonic
  // network in registers and shuffles; warp 0 then merges the eight sorted
  // lists, taking the best head topk - 2 times.
  if (need_idx) {
    int* out = ws.idx + (size_t)bg * d.topk;
    int32_t* out2 = idx_out ? idx_out + (size_t)bg * d.topk : nullptr;
    const int cur = t / d.l;
    const int K2 = d.topk - 2;
    if (cur + 1 <= d.topk) {
      for (int k = threadIdx.x; k < d.topk; k += kK1Threads) {
        out[k] = k <= cur ? k : -1;
        if (out2) out2[k] = out[k];
      }
    } else {
      float v[2];
      int ix[2];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const int j = key0 + lane + 32 * sl;
        const bool c = j >= 1 && j < cur && j < ncp;
        v[sl] = c ? score[j] : -INFINITY;
        ix[sl] = c ? j : INT_MAX;
      }
      for (int size = 2; size <= 64; size <<= 1) {
        for (int jj = size >> 1; jj > 0; jj >>= 1) {
          if (jj == 32) {  // the pair is held by one lane: (lane, lane + 32)
            const bool dir = (lane & size) == 0;
            const bool f = goes_first(v[0], ix[0], v[1], ix[1]);
            if (f != dir) {
              const float tv = v[0];
              const int ti = ix[0];
              v[0] = v[1];
              ix[0] = ix[1];
              v[1] = tv;
              ix[1] = ti;
            }
          } else {
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
              const int e = lane + 32 * sl;
              const float pv = __shfl_xor_sync(0xffffffffu, v[sl], jj);
              const int pi = __shfl_xor_sync(0xffffffffu, ix[sl], jj);
              const bool lower = (e & jj) == 0;
              const bool dir = (e & size) == 0;
              const bool self_first = goes_first(v[sl], ix[sl], pv, pi);
              const bool keep = lower ? (dir == self_first) : (dir != self_first);
              if (!keep) {
                v[sl] = pv;
                ix[sl] = pi;
              }
            }
          }
        }
      }
      float* cand_v = sort_v + warp * 64;
      int* cand_i = sort_i + warp * 64;
      cand_v[lane] = v[0];
      cand_i[lane] = ix[0];
      cand_v[lane + 32] = v[1];
      cand_i[lane + 32] = ix[1];
      __syncthreads();
      if (warp == 0) {
        const int words = (d.Nb + 31) / 32;
        for (int w = lane; w < words; w += 32) bits[w] = 0u;
        __syncwarp();
        int head = 0;  // lanes 0..7: position in warp `lane`'s sorted list
        for (int k = 0; k < K2; ++k) {
          float hv = -INFINITY;
          int hi = INT_MAX;
          if (lane < 8 && head < 64) {
            hv = sort_v[lane * 64 + head];
            hi = sort_i[lane * 64 + head];
          }
          float wv = hv;
          int wi = hi, wl = lane;
#pragma unroll
          for (int off = 4; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, wi, off);
            const int ol = __shfl_xor_sync(0xffffffffu, wl, off);
            if (goes_first(ov, oi, wv, wi)) {
              wv = ov;
              wi = oi;
              wl = ol;
            }
          }
          wv = __shfl_sync(0xffffffffu, wv, 0);
          wi = __shfl_sync(0xffffffffu, wi, 0);
          wl = __shfl_sync(0xffffffffu, wl, 0);
          if (wi == INT_MAX) break;
          if (lane == wl) ++head;
          if (lane == 0) bits[wi >> 5] |= 1u << (wi & 31);
        }
        __syncwarp();
        if (lane == 0) {
          bits[0] |= 1u;
          bits[cur >> 5] |= 1u << (cur & 31);
        }
        __syncwarp();
        int base = 0;
        for (int w0 = 0; w0 <= (cur >> 5); w0 += 32) {
          const int w = w0 + lane;
          const uint32_t m = w <= (cur >> 5) ? bits[w] : 0u;
          const int c = __popc(m);
          int incl = c;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
          }
          int pos = base + incl - c;
          uint32_t mm = m;
          while (mm) {
            const int bit = __ffs(mm) - 1;
            mm &= mm - 1;
            if (pos < d.topk) {
              out[pos] = w * 32 + bit;
              if (out2) out2[pos] = w * 32 + bit;
            }
            ++pos;
          }
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
        for (int p = base + lane; p < d.topk; p += 32) {
          out[p] = -1;
          if (out2) out2[p] = -1;
        }
      }
    }
  }
}

// ---- K2: one 64-key block of the window or the selection ------------------------------
__global__ void __launch_bounds__(32)
decode_block_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const bf16* __restrict__ q, Dims d, DecodeWs ws, int do_sel, int do_swa,
                    int* err) {
  __shared__ __align__(1024) uint8_t kv[2 * 8192];
  __shared__ __align__(1024) uint8_t qs[2048];
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  const int lane = threadIdx.x;
  const int u = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int bg = b * d.Hkv + g;
  const int t = d.T - 1;
  const int cur = t / d.l;
  const int* sel = ws.idx + (size_t)bg * d.topk;
  pdl_launch_dependents();
  // which block, and which branches it serves here; window blocks are known
  // before the selection, so their loads start before K1 has finished
  int j, sel_slot = -1;
  bool win = false;
  if (u < ws.nwin) {
    if (!do_swa) return;
    j = ws.jlo + u;
    win = true;
  } else {
    if (!do_sel) return;
    pdl_wait();
    const int m = u - ws.nwin;
    j = sel[m];
    if (j < 0) return;
    if (j > cur) {  // never read a non-causal block
      if (lane == 0) record_error(err, kDevBadIndex);
      return;
    }
    if (do_swa && j >= ws.jlo) return;  // its window CTA covers the selection too
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
  if (win && do_sel) {  // is this window block also selected?
    pdl_wait();
    for (int m = 0; m < d.topk; ++m)
      if (sel[m] == j) sel_slot = m;
  }
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
}

// ---- K3: merge the partials of each branch and apply the gates ------------------------
// One warp per query head: lanes read the slots' (max, sum) in parallel, the
// warp reduces them, then every slot's 64-wide partial output is folded in.
__global__ void decode_merge_kernel(const float* __restrict__ gates, bf16* __restrict__ out,
                                    Dims d, DecodeWs ws) {
  const int bg = blockIdx.x;
  const int row = threadIdx.x >> 5, lane = threadIdx.x & 31;  // one warp per head
  pdl_wait();
  if (row >= d.G) return;
  const int b = bg / d.Hkv, g = bg % d.Hkv;
  const int h = g * d.G + row;
  const int t = d.T - 1;
  const int cur = t / d.l;
  const int* sel = ws.idx + (size_t)bg * d.topk;
  const float* grow = gates + ((size_t)b * d.Hq + h) * 3;
  float acc0 = 0.f, acc1 = 0.f;
  for (int br = 0; br < 2; ++br) {
    const bool is_sel = br == 0;
    if (!(d.branch_mask & (is_sel ? 2 : 4))) continue;
    const int n = is_sel ? d.topk : ws.nwin;
    const float* base = (is_sel ? ws.psel + (size_t)bg * d.topk * 16 * kPartStride
                                : ws.pswa + (size_t)bg * ws.nwin * 16 * kPartStride) +
                        row * kPartStride;
    float M = -INFINITY;
    for (int m = lane; m < n; m += 32) {
      const bool ok = !is_sel || (sel[m] >= 0 && sel[m] <= cur);
      if (ok) M = fmaxf(M, base[(size_t)m * 16 * kPartStride + 64]);
    }
    M = warp_max(M);
    float L = 0.f, o0 = 0.f, o1 = 0.f;
    for (int m0 = 0; m0 < n; m0 += 32) {
      const int m = m0 + lane;
      float f = 0.f;
      if (m < n) {
        const bool ok = !is_sel || (sel[m] >= 0 && sel[m] <= cur);
        const float mm = ok ? base[(size_t)m * 16 * kPartStride + 64] : -INFINITY;
        f = mm == -INFINITY ? 0.f : fast_exp2(mm - M);
        L += f * base[(size_t)m * 16 * kPartStride + 65];
      }
      const int cnt = min(32, n - m0);
      // loads of every slot are issued together (all addresses are inside
      // the workspace); slots without a partial get weight 0 and their
      // (possibly stale) values are discarded by the select
#pragma unroll 8
      for (int i = 0; i < cnt; ++i) {
        const float fi = __shfl_sync(0xffffffffu, f, i);
        const float* pr = base + (size_t)(m0 + i) * 16 * kPartStride;
        const float x0 = pr[lane], x1 = pr[lane + 32];
        o0 = fi != 0.f ? fmaf(fi, x0, o0) : o0;
        o1 = fi != 0.f ? fmaf(fi, x1, o1) : o1;
      }
    }
    L = warp_sum(L);
    const float gi = grow[is_sel ? 1 : 2] * (L > 0.f ? 1.f / L : 0.f);
    acc0 = fmaf(gi, o0, acc0);
    acc1 = fmaf(gi, o1, acc1);
  }
  if (d.branch_mask & 1) {
    const float* oc = ws.ocmp + ((size_t)bg * 16 + row) * 64;
    acc0 = fmaf(grow[0], oc[lane], acc0);
    acc1 = fmaf(grow[0], oc[lane + 32], acc1);
  }
  bf16* o = out + ((size_t)b * d.Hq + h) * 64;
  o[lane] = __float2bfloat16_rn(acc0);
  o[lane + 32] = __float2bfloat16_rn(acc1);
}

int window_blocks(const Dims& d, int* jlo) {
  const int t = d.T - 1;
  *jlo = max(0, t - d.window + 1) / d.l;
  return t / d.l - *jlo + 1;
}

size_t k1_smem(const Dims& d) {
  const int ncp = (d.Nc + 63) & ~63;
  const size_t r0_bytes = ((size_t)ncp * 256 > 32768) ? (size_t)ncp * 256 : 32768;
  return r0_bytes + 2048 + (8 * 16 + 32) * 4 + (size_t)ncp * 4 + ((d.Nb + 31) / 32 + 2) * 4 +
         512 * 8 + 64 + 1024 + 64;
}

}  // namespace

// Decode with the split kernels applies to bf16, block 64, G <= 16 heads per
// group, up to 512 compressed blocks (the K1 tile) and one query.
bool decode_split_eligible(const Dims& d) {
  return d.Tq == 1 && d.dtype == 1 && d.l == 64 && d.D == 64 && d.G <= 16 && d.Nc <= 512 &&
         tmap_encode_fn() != nullptr;
}

size_t decode_split_ws_bytes(const Dims& d) {
  int jlo;
  const int nwin = window_blocks(d, &jlo);
  const size_t bgn = (size_t)d.B * d.Hkv;
  auto a = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return a(bgn * 16 * 64 * 4) + a(bgn * d.topk * 4) + a(bgn * d.topk * 16 * kPartStride * 4) +
         a(bgn * nwin * 16 * kPartStride * 4);
}

cudaError_t launch_decode_split(const Dims& d, const void* q, const void* kcache,
                                const void* vcache, const void* kc, const void* vc,
                                const float* gates, void* out, int32_t* idx_out, void* ws_ptr,
                                int* err, cudaStream_t s) {
  DecodeWs ws;
  ws.nwin = window_blocks(d, &ws.jlo);
  const size_t bgn = (size_t)d.B * d.Hkv;
  auto a = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* w = (char*)ws_ptr;
  ws.ocmp = (float*)w;
  w += a(bgn * 16 * 64 * 4);
  ws.idx = (int*)w;
  w += a(bgn * d.topk * 4);
  ws.psel = (float*)w;
  w += a(bgn * d.topk * 16 * kPartStride * 4);
  ws.pswa = (float*)w;
  const bool cmp = d.branch_mask & 1, sel = d.branch_mask & 2, swa = d.branch_mask & 4;
  CUtensorMap mkc{}, mvc{}, mk, mv;
  if (d.Nc > 0 && (cmp || sel)) {
    if (!make_tmap_bf16(&mkc, kc, d.Hkv, (long)d.B * d.Nc, 1, 64) ||
        !make_tmap_bf16(&mvc, vc, d.Hkv, (long)d.B * d.Nc, 1, 64))
      return cudaErrorInvalidValue;
  }
  if (!make_tmap_bf16(&mk, kcache, d.Hkv, (long)d.B * d.T, 1, 64) ||
      !make_tmap_bf16(&mv, vcache, d.Hkv, (long)d.B * d.T, 1, 64))
    return cudaErrorInvalidValue;
  if (cmp || sel) {
    const size_t smem = k1_smem(d);
    cudaError_t e = cudaFuncSetAttribute(decode_cmp_topk_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_cmp_topk_kernel<<<(unsigned)bgn, kK1Threads, smem, s>>>(
        mkc, mvc, (const bf16*)q, d, ws, idx_out, cmp ? 1 : 0, sel ? 1 : 0, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  if (sel || swa) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ws.nwin + d.topk, d.Hkv, d.B);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    const bf16* qb = (const bf16*)q;
    const int ds = sel ? 1 : 0, dw = swa ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_block_kernel, mk, mv, qb, d, ws, ds, dw, err);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)bgn);
  cfg.blockDim = dim3(d.G * 32);
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  bf16* ob = (bf16*)out;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel, gates, ob, d, ws);
}

}  // namespace nsa
