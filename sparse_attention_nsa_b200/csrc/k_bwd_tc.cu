// k_bwd_tc.cu -- backward pass 1 (dQ, query-stationary) of the selection and
// sliding-window branches on the sm_100a tensor cores.
//
// "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method / Key claims:
// the selection backward runs a query-stationary pass for dQ first, then a
// key-stationary pass for dK/dV over the reverse block->query map.  This is
// the first pass.  Per row r = (token t, head h) and key s:
//   P = exp(scale q.k_s - lse_r),  dP = dO_r . v_s,
//   dS = P (dP - delta_r),  dq_r += scale * sum_s dS k_s,
// with delta_r = dO_r . o_r, written here for the second pass.
//
// Tiling follows the forward kernel: a CTA owns 128 rows = 128/G
// consecutive tokens x the G heads of one KV group and walks the ascending
// union of its tokens' selected blocks (or the contiguous window blocks).
// Per 64-key block, with K and V staged by TMA:
//   S  = Q K^T  and  dP = dO V^T     (tcgen05, M128 N64 K64, fp32 in TMEM)
//   row threads: P, dS (bf16) into TMEM
//   dQ += dS K                        (tcgen05, dS the TMEM A operand,
//                                      K read MN-major, fp32 in TMEM)
// Q comes by TMA; dO (fp32 in memory) is rounded to bf16 by the row
// threads into the same 128-byte-swizzled layout.  The row threads release
// S/dP as soon as they have loaded them, so the next block's MMAs overlap
// this block's arithmetic; dS is single-buffered.
// TMEM columns (256 per CTA): S [0,64), dP [64,128), dQ [128,192),
// dS [192,224).  Warp roles (192 threads): warps 0-3 rows, warp 4 MMA issue
// and TMEM owner, warp 5 TMA producer.
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace nsa {
namespace {

using namespace sm100;

constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = kKeys * 64 * 2;
constexpr uint32_t kQBytes = kRows * 64 * 2;

constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128, kColDS = 192;

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_DO = OFF_Q + kQBytes;
constexpr uint32_t OFF_KV = OFF_DO + kQBytes;
constexpr uint32_t OFF_BAR = OFF_KV + kStages * 2 * kTileBytes;

struct Bars {
  uint64_t q;       // Q landed (TMA)
  uint64_t dorows;  // the 128 row threads have staged dO
  uint64_t full[kStages];
  uint64_t empty[kStages];  // dQ MMA of the block in that stage done
  uint64_t s;       // S and dP of the current block are in TMEM
  uint64_t sfree;   // the 128 row threads have loaded them
  uint64_t ds;      // the 128 row threads have written dS
  uint64_t fin;
};
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr uint32_t OFF_LIST = OFF_MISC + 16;

__host__ __device__ inline int tokens_per_tile(int G) { return kRows / G; }

__host__ __device__ inline size_t list_ints(const Dims& d) {
  const int words = (d.Nb + 31) / 32;
  return (size_t)d.Nb + words + (size_t)tokens_per_tile(d.G) * (d.topk + 1);
}

template <bool SEL>
__global__ void __launch_bounds__(kThreads, 2)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const bf16* __restrict__ o,
                 const float* __restrict__ lse, const float* __restrict__ dO,
                 const int32_t* __restrict__ idx, float* __restrict__ dq,
                 float* __restrict__ delta, Dims d, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  uint32_t* tmem_slot = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  int* nblk_s = (int*)(smem + OFF_MISC + 8);
  int* blk = (int*)(smem + OFF_LIST);
  const int words = (d.Nb + 31) / 32;
  uint32_t* bits = (uint32_t*)(blk + d.Nb);
  int* toks = (int*)(bits + words);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int TQ = tokens_per_tile(d.G);
  const int tile = gridDim.x - 1 - blockIdx.x;  // heavy (late) tiles first
  const int t0 = tile * TQ;
  const int g = blockIdx.y, b = blockIdx.z;
  const int nvalid = min(TQ, d.Tq - t0);
  const int pos0 = d.q_off + t0;

  if (tid == 0) {
    mbar_init(&bars->q, 1);
    mbar_init(&bars->dorows, 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->s, 1);
    mbar_init(&bars->sfree, 128);
    mbar_init(&bars->ds, 128);
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  if (warp == 4) tmem_alloc(tmem_slot, 256);
  if (warp == 5 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }

  // ---- block list (as in the forward kernel) ---------------------------------------
  if (SEL) {
    for (int w = tid; w < words; w += kThreads) bits[w] = 0u;
    __syncthreads();
    for (int tl = tid; tl < TQ; tl += kThreads) {
      int* lst = toks + tl * (d.topk + 1);
      int cnt = 0;
      if (tl < nvalid) {
        const int t = pos0 + tl;
        const int cur = t / d.l;
        const int32_t* ir = idx + (((size_t)b * d.Tq + t0 + tl) * d.Hkv + g) * d.topk;
        int prev = -1;
        for (int s = 0; s < d.topk; ++s) {
          const int j = ir[s];
          if (j == -1) continue;
          if (j < -1 || j <= prev || j > cur) {  // never read a non-causal block
            record_error(err, kDevBadIndex);
            continue;
          }
          prev = j;
          lst[cnt++] = j;
          atomicOr(&bits[j >> 5], 1u << (j & 31));
        }
      }
      lst[cnt] = INT_MAX;
    }
    __syncthreads();
    if (warp == 0) {
      int base = 0;
      for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        uint32_t m = w < words ? bits[w] : 0u;
        const int c = __popc(m);
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        int pos = base + incl - c;
        while (m) {
          const int bit = __ffs(m) - 1;
          m &= m - 1;
          blk[pos++] = w * 32 + bit;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) *nblk_s = base;
    }
  } else if (tid == 0) {
    const int tlast = pos0 + nvalid - 1;
    const int jlo = max(0, pos0 - d.window + 1) / d.l;
    const int jhi = tlast / d.l;
    blk[0] = jlo;
    *nblk_s = jhi - jlo + 1;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *nblk_s;
  const int blk0 = blk[0];

  if (warp == 5) {
    // ---- TMA producer --------------------------------------------------------------
    if (lane == 0) {
      mbar_expect_tx(&bars->q, kQBytes);
      tma_load_3d(smem + OFF_Q, &tm_q, &bars->q, 0, g * d.G, b * d.Tq + t0);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % kStages;
        if (i >= kStages &&
            !wait_bar(&bars->empty[st], ((i / kStages) & 1) ^ 1, abort_flag, err))
          break;
        const int j = SEL ? blk[i] : blk0 + i;
        const int row = b * d.T + j * kKeys;
        uint8_t* kv = smem + OFF_KV + st * 2 * kTileBytes;
        mbar_expect_tx(&bars->full[st], 2 * kTileBytes);
        tma_load_3d(kv, &tm_k, &bars->full[st], 0, g, row);
        tma_load_3d(kv + kTileBytes, &tm_v, &bars->full[st], 0, g, row);
        issued = i + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before exit
        drain_bar(&bars->q, 0);
        for (int i = max(0, issued - kStages); i < issued; ++i)
          drain_bar(&bars->full[i % kStages], (i / kStages) & 1);
      }
    }
  } else if (warp == 4) {
    // ---- MMA issue: S, dP of block i, then dQ of block i-1 ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, false, false);
      constexpr uint32_t idesc_q = idesc_bf16(kRows, 64, false, true);
      const uint32_t q_addr = smem_u32(smem + OFF_Q), do_addr = smem_u32(smem + OFF_DO);
      bool ok = wait_bar(&bars->q, 0, abort_flag, err) &&
                wait_bar(&bars->dorows, 0, abort_flag, err);
      auto issue_dq = [&](int i) -> bool {
        // dS of block i (TMEM) times K of block i read MN-major
        if (!wait_bar(&bars->ds, i & 1, abort_flag, err)) return false;
        tc_fence_after();
        const int st = i % kStages;
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + kColDQ, tmem + kColDS + kk * 8, desc_sw128(k_addr + kk * 2048, 8192),
                      idesc_q, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[st]);  // frees the stage and the dS columns
        return true;
      };
      for (int i = 0; ok && i < n; ++i) {
        // S and dP are single-buffered: the rows must have loaded block i-1's
        if (i >= 1 && !wait_bar(&bars->sfree, (i - 1) & 1, abort_flag, err)) break;
        const int st = i % kStages;
        if (!wait_bar(&bars->full[st], (i / kStages) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
        const uint32_t v_addr = k_addr + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kColS, desc_sw128(q_addr + kk * 32, 16), desc_sw128(k_addr + kk * 32, 16),
                   idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kColDP, desc_sw128(do_addr + kk * 32, 16),
                   desc_sw128(v_addr + kk * 32, 16), idesc_s, kk > 0);
        mma_commit(&bars->s);
        if (i >= 1 && !issue_dq(i - 1)) break;
        if (i == n - 1) issue_dq(i);
      }
      // every MMA issued must finish before TMEM is released
      mma_commit(&bars->fin);
      drain_bar(&bars->fin, 0);
    }
  } else {
    // ---- rows: thread r owns query row r -----------------------------------------------
    const int r = tid;
    const int tl = r / d.G, hh = r % d.G;
    const bool valid = tl < nvalid;
    const int t = pos0 + tl;
    const size_t row = ((size_t)b * d.Tq + t0 + tl) * d.Hq + (size_t)g * d.G + hh;
    const uint32_t lane_tmem = tmem + ((uint32_t)(warp * 32) << 16);
    float dl = 0.f, lse2 = -INFINITY;
    {  // delta = dO . o, and dO rounded to bf16 into the swizzled A tile
      const uint32_t drow = smem_u32(smem + OFF_DO) + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (valid) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(dO + row * 64) + 2 * c);
          const float4 a2 = __ldg(reinterpret_cast<const float4*>(dO + row * 64) + 2 * c + 1);
          const uint4 ou = __ldg(reinterpret_cast<const uint4*>(o + row * 64) + c);
          const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ou);
          const float2 o0 = __bfloat1622float2(op[0]), o1 = __bfloat1622float2(op[1]);
          const float2 o2 = __bfloat1622float2(op[2]), o3 = __bfloat1622float2(op[3]);
          dl = fmaf(a.x, o0.x, fmaf(a.y, o0.y, fmaf(a.z, o1.x, fmaf(a.w, o1.y, dl))));
          dl = fmaf(a2.x, o2.x, fmaf(a2.y, o2.y, fmaf(a2.z, o3.x, fmaf(a2.w, o3.y, dl))));
          w[0] = pack_bf16(a.x, a.y);
          w[1] = pack_bf16(a.z, a.w);
          w[2] = pack_bf16(a2.x, a2.y);
          w[3] = pack_bf16(a2.z, a2.w);
        }
        st_shared_v4(drow + ((uint32_t)(c ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
      }
      if (valid) {
        delta[row] = dl;
        lse2 = lse[row] * kLog2e;
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->dorows);
    }
    const int lo = SEL ? 0 : max(0, t - d.window + 1);
    const int* lst = SEL ? toks + tl * (d.topk + 1) : nullptr;
    int ptr = 0;
    int nxt = SEL && valid ? lst[0] : INT_MAX;
    const float sl2 = d.scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int j = SEL ? blk[i] : blk0 + i;
      const int k0 = j * kKeys;
      bool rowsel = valid && k0 <= t && lse2 != -INFINITY;
      if (SEL) {
        const bool hit = nxt == j;
        if (hit) nxt = lst[++ptr];
        rowsel = rowsel && hit;
      } else {
        rowsel = rowsel && (k0 + kKeys - 1 >= lo);
      }
      if (!wait_bar_warp(&bars->s, i & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t dsk[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float sv[32], pv[32];
        tmem_ld32(lane_tmem + kColS + 32u * h2, sv);
        tmem_ld32(lane_tmem + kColDP + 32u * h2, pv);
        tmem_wait_ld();
        if (h2 == 1) {  // S and dP of this block are in registers: release them
          tc_fence_before();
          mbar_arrive(&bars->sfree);
        }
        if (rowsel) {
          const bool part = !((k0 + kKeys - 1 <= t) && (k0 >= lo));
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int key = k0 + 32 * h2 + c;
            float p0 = fast_exp2(fmaf(sv[c], sl2, -lse2));
            float p1 = fast_exp2(fmaf(sv[c + 1], sl2, -lse2));
            if (part) {
              if (key > t || key < lo) p0 = 0.f;
              if (key + 1 > t || key + 1 < lo) p1 = 0.f;
            }
            dsk[16 * h2 + c / 2] = pack_bf16(p0 * (pv[c] - dl), p1 * (pv[c + 1] - dl));
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) dsk[16 * h2 + c] = 0u;
        }
      }
      // the dQ MMA of block i-1 reads the dS columns: wait for it
      if (i >= 1) {
        if (!wait_bar_warp(&bars->empty[(i - 1) % kStages], ((i - 1) / kStages) & 1, abort_flag,
                           err)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32u(lane_tmem + kColDS, dsk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds);
    }
    // epilogue: dq += scale * dQ (fp32, accumulated across branches)
    float acc[64];
    bool have = false;
    if (ok && n > 0) have = wait_bar_warp(&bars->fin, 0, abort_flag, err);
    if (have) {
      tc_fence_after();
      tmem_ld32(lane_tmem + kColDQ, acc);
      tmem_ld32(lane_tmem + kColDQ + 32u, acc + 32);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] = 0.f;
    }
    tc_fence_before();
    if (valid && have) {
      float4* dst = reinterpret_cast<float4*>(dq + row * 64);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float4 x = dst[c];
        x.x = fmaf(acc[4 * c], d.scale, x.x);
        x.y = fmaf(acc[4 * c + 1], d.scale, x.y);
        x.z = fmaf(acc[4 * c + 2], d.scale, x.z);
        x.w = fmaf(acc[4 * c + 3], d.scale, x.w);
        dst[c] = x;
      }
    }
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <bool SEL>
cudaError_t launch_dq_tc_t(const Dims& d, const void* q, const void* k, const void* v,
                           const int32_t* idx, const void* o, const float* lse, const float* dO,
                           float* dq, float* delta, int* err, cudaStream_t s) {
  const int TQ = tokens_per_tile(d.G);
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16(&mq, q, d.Hq, (long)d.B * d.Tq, d.G, TQ) ||
      !make_tmap_bf16(&mk, k, d.Hkv, (long)d.B * d.T, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, (long)d.B * d.T, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = OFF_LIST + list_ints(d) * sizeof(int) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel<SEL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.Tq + TQ - 1) / TQ, d.Hkv, d.B);
  bwd_dq_tc_kernel<SEL><<<grid, kThreads, smem, s>>>(mq, mk, mv, (const bf16*)o, lse, dO, idx, dq,
                                                     delta, d, err);
  return cudaGetLastError();
}

}  // namespace

// Tensor-core dQ applies to bf16, 64-key blocks, head dim 64, G dividing 128.
bool dq_tc_eligible(const Dims& d, int mode) {
  return mode != 2 && d.dtype == 1 && d.l == kKeys && d.D == 64 && d.G >= 1 &&
         kRows % d.G == 0 && d.Nb <= 4096 && tmap_encode_fn() != nullptr;
}

cudaError_t launch_dq_tc(const Dims& d, int mode, const void* q, const void* k, const void* v,
                         const int32_t* idx, const void* o, const float* lse, const float* dO,
                         float* dq, float* delta, int* err, cudaStream_t s) {
  return mode == 0 ? launch_dq_tc_t<true>(d, q, k, v, idx, o, lse, dO, dq, delta, err, s)
                   : launch_dq_tc_t<false>(d, q, k, v, idx, o, lse, dO, dq, delta, err, s);
}

}  // namespace nsa
