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
// dS [192,224).  Warp roles (320 threads, two CTAs per SM): warps 0-7 rows
// (warps w and w + 4 share the rows of TMEM lane quarter w, warp w the
// first 32 keys of every block and warp w + 4 the last 32: P = exp(S - lse)
// needs no statistics shared between them), warp 8 MMA issue and TMEM
// owner, warp 9 TMA producer.
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
constexpr int kThreads = 320;  // 8 row warps, the MMA warp, the TMA warp
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
  // single-pass variant only
  uint64_t pfree;   // dV/dK MMAs of a block pair done: P / dS tiles free
  uint64_t kvfull;  // dV/dK of a block pair are in TMEM
  uint64_t kvfree;  // the 128 epilogue threads have loaded them
};
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr uint32_t OFF_LIST = OFF_MISC + 16;

// Shared-memory layout of the single-pass (atomic) variant: three K/V
// stages, then the P and dS tiles of a pair of blocks (each 128 rows x 64
// keys, 128-byte swizzle: P of block 2m, P of block 2m+1 (fp16), dS of 2m,
// dS of 2m+1 (bf16)), the dO lo tile (bf16: dO - bf16(dO)) and the dO tile
// in fp16, then the barriers and the block list.
constexpr int kAtStages = 3;
constexpr uint32_t AT_OFF_P = OFF_KV + kAtStages * 2 * kTileBytes;
constexpr uint32_t AT_OFF_DOL = AT_OFF_P + 4 * kQBytes;
constexpr uint32_t AT_OFF_DOH = AT_OFF_DOL + kQBytes;
constexpr uint32_t AT_OFF_BAR = AT_OFF_DOH + kQBytes;
constexpr uint32_t AT_OFF_MISC = AT_OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr uint32_t AT_OFF_LIST = AT_OFF_MISC + 16;
constexpr int kAtThreads = 448;  // plus 4 epilogue warps
constexpr uint32_t kColDV = 256, kColDK = 320;  // TMEM columns of a pair's dV / dK

__host__ __device__ inline int tokens_per_tile(int G) { return kRows / G; }

__host__ __device__ inline size_t list_ints(const Dims& d) {
  const int words = (d.Nb + 31) / 32;
  return (size_t)d.Nb + words + (size_t)tokens_per_tile(d.G) * (d.topk + 1);
}

// MODE 0 selection, 1 window, 2 compression (keys = the compressed cache;
// key c is visible to the query at t when its block is complete:
// c d + l - 1 <= t).
//
// ATOMIC (selection only): the single-pass query-stationary backward that
// "Sparsity is Cool", Method, sets against the two-pass one: the same pass
// also forms each block's dK and dV from this tile's rows and adds them to
// dk / dv with atomics.  dK and dV sum over many rows, so they need what
// the two-pass kernel needs: dP = V (dO_hi + dO_lo)^T to about fp32 (dS =
// P (dP - delta) cancels when the softmax is peaked) and dV in fp16.  The
// row threads write P (fp16) and dS (bf16) of each union block into shared
// memory as well; once two blocks' tiles are there (or the last block is),
// one MMA per gradient covers both blocks' 128 keys:
//   dV = P^T dO (fp16), dK = dS^T Q (bf16)  (M128 N64 K128: A the P / dS
//   tiles read MN-major, the second block's tiles 16 KB after the first's;
//   B the dO (fp16) / Q tiles read MN-major), fp32 in TMEM [256, 384);
// warps 10-13 (thread = key of the pair) load them and add them to dk, dv
// with float4 atomics (so dk / dv depend on the order the atomics land in:
// equal to the two-pass results up to fp32 rounding, not bit for bit).
template <int MODE, bool ATOMIC = false>
__global__ void __launch_bounds__(ATOMIC ? kAtThreads : kThreads, ATOMIC ? 1 : 2)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const bf16* __restrict__ o,
                 const float* __restrict__ lse, const float* __restrict__ dO,
                 const int32_t* __restrict__ idx, float* __restrict__ dq,
                 float* __restrict__ delta, Dims d, int* err, float* __restrict__ dk_at = nullptr,
                 float* __restrict__ dv_at = nullptr) {
  constexpr bool SEL = MODE == 0;
  constexpr int NST = ATOMIC ? kAtStages : kStages;
  constexpr uint32_t O_BAR = ATOMIC ? AT_OFF_BAR : OFF_BAR;
  constexpr uint32_t O_MISC = ATOMIC ? AT_OFF_MISC : OFF_MISC;
  constexpr uint32_t O_LIST = ATOMIC ? AT_OFF_LIST : OFF_LIST;
  constexpr uint32_t TMEM_COLS = ATOMIC ? 512 : 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + O_BAR);
  const int nkeys = MODE == 2 ? d.Nc : d.T;  // key rows per sequence
  uint32_t* tmem_slot = (uint32_t*)(smem + O_MISC);
  volatile int* abort_flag = (volatile int*)(smem + O_MISC + 4);
  int* nblk_s = (int*)(smem + O_MISC + 8);
  int* blk = (int*)(smem + O_LIST);
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
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->s, 1);
    mbar_init(&bars->sfree, 256);
    mbar_init(&bars->ds, 256);
    mbar_init(&bars->fin, 1);
    mbar_init(&bars->pfree, 1);
    mbar_init(&bars->kvfull, 1);
    mbar_init(&bars->kvfree, 128);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  if (warp == 8) tmem_alloc(tmem_slot, TMEM_COLS);
  if (warp == 9 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }

  // ---- block list (as in the forward kernel) ---------------------------------------
  if (SEL) {
    for (int w = tid; w < words; w += blockDim.x) bits[w] = 0u;
    __syncthreads();
    for (int tl = tid; tl < TQ; tl += blockDim.x) {
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
    if (MODE == 1) {
      const int jlo = max(0, pos0 - d.window + 1) / d.l;
      blk[0] = jlo;
      *nblk_s = tlast / d.l - jlo + 1;
    } else {  // compressed keys 0 .. (tlast + 1) / l - 1, in 64-key chunks
      const int cmax = cmp_nvis(d, tlast) - 1;
      blk[0] = 0;
      *nblk_s = cmax < 0 ? 0 : cmax / kKeys + 1;
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *nblk_s;
  const int blk0 = blk[0];

  if (warp == 9) {
    // ---- TMA producer --------------------------------------------------------------
    if (lane == 0) {
      mbar_expect_tx(&bars->q, kQBytes);
      tma_load_3d(smem + OFF_Q, &tm_q, &bars->q, 0, g * d.G, b * d.Tq + t0);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % NST;
        if (i >= NST &&
            !wait_bar(&bars->empty[st], ((i / NST) & 1) ^ 1, abort_flag, err))
          break;
        const int j = SEL ? blk[i] : blk0 + i;
        const int row = b * nkeys + j * kKeys;
        uint8_t* kv = smem + OFF_KV + st * 2 * kTileBytes;
        mbar_expect_tx(&bars->full[st], 2 * kTileBytes);
        tma_load_3d(kv, &tm_k, &bars->full[st], 0, g, row);
        tma_load_3d(kv + kTileBytes, &tm_v, &bars->full[st], 0, g, row);
        issued = i + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before exit
        drain_bar(&bars->q, 0);
        for (int i = max(0, issued - NST); i < issued; ++i)
          drain_bar(&bars->full[i % NST], (i / NST) & 1);
      }
    }
  } else if (warp == 8) {
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
        const int st = i % NST;
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + kColDQ, tmem + kColDS + kk * 8, desc_sw128(k_addr + kk * 2048, 8192),
                      idesc_q, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[st]);  // frees the stage and the dS columns
        if constexpr (ATOMIC) {
          if ((i & 1) || i == n - 1) {  // blocks 2m and 2m+1 (or the last alone)
            const int pi = i >> 1;
            if (pi >= 1 && !wait_bar(&bars->kvfree, (pi - 1) & 1, abort_flag, err)) return false;
            tc_fence_after();
            constexpr uint32_t idesc_kv = idesc_bf16(128, 64, true, true);  // A, B MN-major
            constexpr uint32_t idesc_v16 = idesc_f16(128, 64, true, true);  // dV: fp16
            const uint32_t p_addr = smem_u32(smem + AT_OFF_P), s_addr = p_addr + 2 * kQBytes;
            const uint32_t doh_addr = smem_u32(smem + AT_OFF_DOH);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // K = the tile's 128 rows, 16 at a time
              mma_bf16(tmem + kColDV, desc_sw128(p_addr + kk * 2048, kQBytes),
                       desc_sw128(doh_addr + kk * 2048, 8192), idesc_v16, kk > 0);
              mma_bf16(tmem + kColDK, desc_sw128(s_addr + kk * 2048, kQBytes),
                       desc_sw128(q_addr + kk * 2048, 8192), idesc_kv, kk > 0);
            }
            mma_commit(&bars->pfree);
            mma_commit(&bars->kvfull);
          }
        }
        return true;
      };
      for (int i = 0; ok && i < n; ++i) {
        // S and dP are single-buffered: the rows must have loaded block i-1's
        if (i >= 1 && !wait_bar(&bars->sfree, (i - 1) & 1, abort_flag, err)) break;
        const int st = i % NST;
        if (!wait_bar(&bars->full[st], (i / NST) & 1, abort_flag, err)) break;
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
        if constexpr (ATOMIC) {  // dO lo: dP to about fp32 for dS = P (dP - delta)
          const uint32_t dol_addr = smem_u32(smem + AT_OFF_DOL);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColDP, desc_sw128(dol_addr + kk * 32, 16),
                     desc_sw128(v_addr + kk * 32, 16), idesc_s, 1u);
        }
        mma_commit(&bars->s);
        if (i >= 1 && !issue_dq(i - 1)) break;
        if (i == n - 1) issue_dq(i);
      }
      // every MMA issued must finish before TMEM is released
      mma_commit(&bars->fin);
      drain_bar(&bars->fin, 0);
    }
  } else if (ATOMIC && warp >= 10) {
    // ---- single pass: dK / dV of each block pair into dk, dv with atomics --------------
    const int k = 32 * (warp & 3) + lane;  // key of the pair (TMEM lane k)
    const uint32_t lane_tmem = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int npairs = (n + 1) / 2;
    for (int pi = 0; pi < npairs; ++pi) {
      if (!wait_bar_warp(&bars->kvfull, pi & 1, abort_flag, err)) break;
      const int bi = 2 * pi + (k >> 6);
      const int key = bi < n ? blk[bi] * kKeys + (k & 63) : nkeys;
      const size_t krow = (((size_t)b * nkeys + min(key, nkeys - 1)) * d.Hkv + g) * 64;
#pragma unroll 1
      for (int hc = 0; hc < 2; ++hc) {  // columns [32 hc, 32 hc + 32) of dV and dK
        tc_fence_after();
        float av[32], ak[32];
        tmem_ld32(lane_tmem + kColDV + 32u * hc, av);
        tmem_ld32(lane_tmem + kColDK + 32u * hc, ak);
        tmem_wait_ld();
        if (hc == 1) {  // both halves loaded: the next pair's MMAs may overwrite them
          tc_fence_before();
          mbar_arrive(&bars->kvfree);
        }
        if (key >= nkeys) continue;
        float4* pv4 = reinterpret_cast<float4*>(dv_at + krow + 32 * hc);
        float4* pk4 = reinterpret_cast<float4*>(dk_at + krow + 32 * hc);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          atomicAdd(pv4 + c, make_float4(av[4 * c], av[4 * c + 1], av[4 * c + 2], av[4 * c + 3]));
          atomicAdd(pk4 + c, make_float4(ak[4 * c] * d.scale, ak[4 * c + 1] * d.scale,
                                         ak[4 * c + 2] * d.scale, ak[4 * c + 3] * d.scale));
        }
      }
    }
  } else if (warp < 8) {
    // ---- rows: thread r owns query row r; warps w and w + 4 share row r = 32 (w % 4) +
    // lane (TMEM lane quarter w % 4), warp w taking keys 0..31 of every block and warp
    // w + 4 keys 32..63 (P needs no per-block statistics here: lse is known) ------------
    const int qw = warp & 3, ch = warp >> 2;
    const int r = 32 * qw + lane;
    const int tl = r / d.G, hh = r % d.G;
    const bool valid = tl < nvalid;
    const int t = pos0 + tl;
    const size_t row = ((size_t)b * d.Tq + t0 + tl) * d.Hq + (size_t)g * d.G + hh;
    const uint32_t lane_tmem = tmem + ((uint32_t)(qw * 32) << 16);
    float* row_lse2 = (float*)(toks + (SEL ? TQ * (d.topk + 1) : 0));  // [128], then delta [128]
    float* row_dl = row_lse2 + kRows;
    float dl = 0.f, lse2 = -INFINITY;
    if (ch == 0) {  // delta = dO . o, and dO rounded to bf16 into the swizzled A tile
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
          if constexpr (ATOMIC) {
            const float x[8] = {a.x, a.y, a.z, a.w, a2.x, a2.y, a2.z, a2.w};
            uint32_t wl[4], wh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float h0 = __bfloat162float(__float2bfloat16_rn(x[2 * e]));
              const float h1 = __bfloat162float(__float2bfloat16_rn(x[2 * e + 1]));
              wl[e] = pack_bf16(x[2 * e] - h0, x[2 * e + 1] - h1);
              wh[e] = pack_f16(x[2 * e], x[2 * e + 1]);
            }
            const uint32_t sw = (uint32_t)(c ^ (r & 7)) << 4;
            const uint32_t base = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u + sw;
            st_shared_v4(smem_u32(smem + AT_OFF_DOL) + base, wl[0], wl[1], wl[2], wl[3]);
            st_shared_v4(smem_u32(smem + AT_OFF_DOH) + base, wh[0], wh[1], wh[2], wh[3]);
          }
        } else if constexpr (ATOMIC) {
          const uint32_t sw = (uint32_t)(c ^ (r & 7)) << 4;
          const uint32_t base = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u + sw;
          st_shared_v4(smem_u32(smem + AT_OFF_DOL) + base, 0u, 0u, 0u, 0u);
          st_shared_v4(smem_u32(smem + AT_OFF_DOH) + base, 0u, 0u, 0u, 0u);
        }
        st_shared_v4(drow + ((uint32_t)(c ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
      }
      if (valid) {
        delta[row] = dl;
        lse2 = lse[row] * kLog2e;
      }
      row_lse2[r] = lse2;
      row_dl[r] = dl;
      fence_proxy_async_smem();
      mbar_arrive(&bars->dorows);  // also publishes lse2 and delta of the row
    }
    bool ok = true;
    if (ch == 1) {
      ok = wait_bar_warp(&bars->dorows, 0, abort_flag, err);
      lse2 = row_lse2[r];
      dl = row_dl[r];
    }
    const int lo = MODE == 1 ? max(0, t - d.window + 1) : 0;
    const int khi = MODE == 2 ? cmp_nvis(d, t) - 1 : t;  // last visible key
    const int* lst = SEL ? toks + tl * (d.topk + 1) : nullptr;
    int ptr = 0;
    int nxt = SEL && valid ? lst[0] : INT_MAX;
    const float sl2 = d.scale * kLog2e;
    const float nl2 = -lse2;
    for (int i = 0; ok && i < n; ++i) {
      const int j = SEL ? blk[i] : blk0 + i;
      const int k0 = j * kKeys + 32 * ch;  // this warp's first key of the block
      bool rowsel = valid && k0 <= khi && lse2 != -INFINITY;
      if (SEL) {
        const bool hit = nxt == j;
        if (hit) nxt = lst[++ptr];
        rowsel = rowsel && hit;
      } else {
        rowsel = rowsel && (k0 + 31 >= lo);
      }
      if (!wait_bar_warp(&bars->s, i & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool any = __any_sync(0xffffffffu, rowsel);
      uint32_t dsk[16];
      uint32_t ppk[ATOMIC ? 16 : 1];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {  // 16 keys at a time
        float sv[16], pv[16];
        if (any) {
          tmem_ld16(lane_tmem + kColS + 32u * ch + 16u * h2, sv);
          tmem_ld16(lane_tmem + kColDP + 32u * ch + 16u * h2, pv);
          tmem_wait_ld();
        }
        if (h2 == 1) {  // S and dP of this block are in registers: release them
          tc_fence_before();
          mbar_arrive(&bars->sfree);
        }
        if (rowsel) {
          const bool part = !((k0 + 31 <= khi) && (k0 >= lo));
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const int key = k0 + 16 * h2 + c;
            float p0 = fast_exp2(fmaf(sv[c], sl2, nl2));
            float p1 = fast_exp2(fmaf(sv[c + 1], sl2, nl2));
            if (part) {
              if (key > khi || key < lo) p0 = 0.f;
              if (key + 1 > khi || key + 1 < lo) p1 = 0.f;
            }
            dsk[8 * h2 + c / 2] = pack_bf16(p0 * (pv[c] - dl), p1 * (pv[c + 1] - dl));
            if constexpr (ATOMIC) ppk[8 * h2 + c / 2] = pack_f16(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            dsk[8 * h2 + c] = 0u;
            if constexpr (ATOMIC) ppk[8 * h2 + c] = 0u;
          }
        }
      }
      if constexpr (ATOMIC) {
        // P and dS of this row's 32 keys for the pair's dV / dK MMAs: chunks
        // 4 ch .. 4 ch + 3 of row r of the tiles of half i & 1 (the pair's
        // previous MMAs must be done with them)
        const int hf = i & 1;
        if (hf == 0 && i >= 2) {
          if (!wait_bar_warp(&bars->pfree, ((i >> 1) - 1) & 1, abort_flag, err)) {
            ok = false;
            break;
          }
        }
        const uint32_t line = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
        const uint32_t pa = smem_u32(smem + AT_OFF_P) + hf * kQBytes + line;
        const uint32_t sa = pa + 2 * kQBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t sw = (uint32_t)((4 * ch + c) ^ (r & 7)) << 4;
          st_shared_v4(pa + sw, ppk[4 * c], ppk[4 * c + 1], ppk[4 * c + 2], ppk[4 * c + 3]);
          st_shared_v4(sa + sw, dsk[4 * c], dsk[4 * c + 1], dsk[4 * c + 2], dsk[4 * c + 3]);
          if (hf == 0 && i == n - 1) {  // a last block alone: its pair half is zero
            st_shared_v4(pa + kQBytes + sw, 0u, 0u, 0u, 0u);
            st_shared_v4(sa + kQBytes + sw, 0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();  // the MMA reads the tiles through the async proxy
      }
      // the dQ MMA of block i-1 reads the dS columns: wait for it
      if (i >= 1) {
        if (!wait_bar_warp(&bars->empty[(i - 1) % NST], ((i - 1) / NST) & 1, abort_flag,
                           err)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st16u(lane_tmem + kColDS + 16u * ch, dsk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds);
    }
    // epilogue: dq += scale * dQ (fp32, accumulated across branches), this
    // warp's 32 of the row's 64 columns
    float acc[32];
    bool have = false;
    if (ok && n > 0) have = wait_bar_warp(&bars->fin, 0, abort_flag, err);
    if (have) {
      tc_fence_after();
      tmem_ld32(lane_tmem + kColDQ + 32u * ch, acc);
      tmem_wait_ld();
    }
    tc_fence_before();
    if (valid && have) {
      float4* dst = reinterpret_cast<float4*>(dq + row * 64 + 32 * ch);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
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
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---- pass 2: dK, dV, key-stationary, on tensor cores --------------------------------
// One CTA per (pair of 64-key blocks j0 = 2p, j1 = 2p+1, KV group, sequence):
// M = 128 keys.  The query rows that attend those keys are streamed in
// tiles of 128 rows, copied by four gather warps with cp.async straight into
// 128-byte-swizzled Q and dO tiles (dO already split into fp16 hi + lo in
// memory), kNBuf tiles deep.  Selection: while both blocks' reverse-map
// lists have rows, a tile takes 64 rows of j0's list (they reach only the
// first 64 keys) and 64 of j1's (the last 64), so each key warp has 64 rows
// of work per tile; the rest of the longer list follows in full tiles.
// Window: the contiguous range of tokens whose windows reach the pair.  Per
// tile:
//   S^T = K Q^T                    (bf16, M128 N128 K64, fp32 in TMEM)
//   dP^T = V (dO_hi + dO_lo)^T     (fp16, M128 N128 K64, fp32 in TMEM)
//   key threads: P^T (fp16), dS^T (bf16) into TMEM (one thread per key)
//   dV += P^T dO_hi                (fp16, M128 N64 K128, A from TMEM, B the
//                                   gathered dO tile read MN-major)
//   dK += dS^T Q                   (bf16, likewise)
// Precision: dS = P (dP - delta) subtracts two nearly equal numbers when the
// softmax is peaked, so dP must keep about fp32 accuracy: dO enters it as an
// fp16 pair hi + lo (dO = hi + lo to 2^-22), against V converted exactly
// from bf16 to fp16 in shared memory.  dV sums P dO over many rows, so both
// factors are fp16 (2^-11); dK takes dS in bf16 (2^-9; the rounding errors
// of independent rows add in quadrature).  A V or dO element beyond fp16's
// range (|x| > 65504) is recorded as a range error.  The sums over rows
// accumulate in fp32 in TMEM.
// TMEM (512 columns, one CTA per SM): S^T [0,128), dP^T [128,256),
// dV [256,320), dK [320,384), P^T [384,448), dS^T [448,512).
// Warps: 0-7 key threads and epilogue (warps w and w + 4 share TMEM lane
// quarter w: keys 32w .. 32w+31; warp w takes the 32-row chunks 0 and 2 of
// every tile, warp w + 4 chunks 1 and 3, so that an interleaved tile gives
// each warp one chunk of work), 8 S^T/dP^T issue and TMEM owner (and the
// K/V TMA), 9 dV/dK issue (its 16 MMAs per tile overlap the next tile's
// S^T/dP^T and key-thread work), 10-13 row gather (warp 10 + c fills rows
// 32c .. 32c+31).
constexpr int kKvThreads = 448;
constexpr int kKeyThreads = 256;
constexpr int kCmpShares = 16;  // row shares of a compression-branch key pair
constexpr int kNBuf = 3;        // row-tile buffers
constexpr uint32_t kKTile2 = 128 * 64 * 2;  // 128 keys x 64 dims, bf16
constexpr uint32_t kRowTile = 128 * 64 * 2;
constexpr int kNoKey = 0x40000000;  // first visible key of a row that reaches none

constexpr uint32_t kvColS = 0, kvColDP = 128, kvColDV = 256, kvColDK = 320, kvColP = 384,
                   kvColDS = 448;

// Per tile row r: the keys it reaches among the pair's first 64 (h = 0) and
// last 64 (h = 1) are those with absolute index in [klo[h][r], klo[h][r] +
// span[h][r]]; nlse2 = -lse * log2(e), ndelta = -delta.
struct KvRowInfo {
  float nlse2[128];
  float ndelta[128];
  int klo[2][128];
  int span[2][128];
  int chunk[4];  // bit h: some row of rows 32c .. 32c+31 reaches a key of half h
};

constexpr uint32_t KV_OFF_K = 0;
constexpr uint32_t KV_OFF_V = KV_OFF_K + kKTile2;
constexpr uint32_t KV_OFF_Q = KV_OFF_V + kKTile2;                // kNBuf buffers each:
constexpr uint32_t KV_OFF_DO = KV_OFF_Q + kNBuf * kRowTile;      //   Q, dO hi, dO lo (bf16)
constexpr uint32_t KV_OFF_DOL = KV_OFF_DO + kNBuf * kRowTile;
constexpr uint32_t KV_OFF_INFO = KV_OFF_DOL + kNBuf * kRowTile;  // kNBuf x KvRowInfo
constexpr uint32_t KV_OFF_BAR = KV_OFF_INFO + ((kNBuf * sizeof(KvRowInfo) + 15) / 16) * 16;

struct KvBars {
  uint64_t kv;                 // K and V of the pair landed (TMA)
  uint64_t vready;             // 256 key threads converted V to fp16
  uint64_t gathered[kNBuf];    // 128 gather threads filled row buffer u % kNBuf
  uint64_t s;                  // S^T and dP^T of the current tile are in TMEM
  uint64_t sfree;              // 128 key threads loaded them
  uint64_t p;                  // 128 key threads wrote P^T and dS^T
  uint64_t bfree[kNBuf];       // dV / dK MMAs of the tile in row buffer u % kNBuf done
  uint64_t sdone;              // every S^T / dP^T MMA done (unwinding)
  uint64_t fin;
};
constexpr uint32_t KV_OFF_MISC = KV_OFF_BAR + ((sizeof(KvBars) + 15) / 16) * 16;
constexpr uint32_t KV_SMEM = KV_OFF_MISC + 16;
static_assert(KV_SMEM + 1024 <= 227 * 1024, "dK/dV kernel shared memory");

// Row r of tile u of a CTA's row sequence -> (list, index within that list's
// rows) for the selection branch.  R0, R1: rows (tokens x G) of j0's and
// j1's lists; nI = tiles that take 64 rows of each.
__device__ __forceinline__ long sel_tile_row(int u, int r, long R0, long R1, int nI, int* which) {
  if (u < nI) {
    *which = r >> 6;
    const long rix = (long)u * 64 + (r & 63);
    return rix < (r < 64 ? R0 : R1) ? rix : -1;
  }
  const bool first = R0 > R1;  // the longer list continues in full tiles
  *which = first ? 0 : 1;
  const long rix = (long)nI * 64 + (long)(u - nI) * 128 + r;
  return rix < (first ? R0 : R1) ? rix : -1;
}

// MODE 0 selection, 1 window, 2 compression.  With nseg > 1 (compression:
// every later query sees a compressed key, so one pair has all the rows)
// the CTA blockIdx.x = pair * nseg + seg takes the seg-th share of the
// pair's row tiles and stores its partial dK/dV in part[seg] instead of
// accumulating; a reduction kernel sums the shares in order.
template <int MODE>
__global__ void __launch_bounds__(kKvThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const bf16* __restrict__ q, const float* __restrict__ lse,
                   const float* __restrict__ delta, const __half* __restrict__ dO_hi,
                   const __half* __restrict__ dO_lo, const int* __restrict__ offsets,
                   const int* __restrict__ list, float* __restrict__ dk, float* __restrict__ dv,
                   float* __restrict__ part, int nseg, Dims d, int* err) {
  constexpr bool SEL = MODE == 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  KvBars* bars = (KvBars*)(smem + KV_OFF_BAR);
  KvRowInfo* info = (KvRowInfo*)(smem + KV_OFF_INFO);
  uint32_t* tmem_slot = (uint32_t*)(smem + KV_OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + KV_OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int pr = blockIdx.x / nseg, seg = blockIdx.x % nseg, g = blockIdx.y, b = blockIdx.z;
  const int nkeys = MODE == 2 ? d.Nc : d.T;
  const int j0 = 2 * pr;
  const int kbase = j0 * kKeys;  // first key of the pair

  // the rows of this CTA
  long R0 = 0, R1 = 0;
  int nI = 0, tq_lo = 0, ntok = 0;
  const int* l0 = nullptr;
  const int* l1 = nullptr;
  int ntiles_all;
  if (SEL) {
    const size_t bg = (size_t)b * d.Hkv + g;
    const int* off = offsets + bg * (d.Nb + 1);
    l0 = list + bg * (size_t)d.Tq * d.topk + off[j0];
    R0 = (long)(off[j0 + 1] - off[j0]) * d.G;
    if (j0 + 1 < d.Nb) {
      l1 = list + bg * (size_t)d.Tq * d.topk + off[j0 + 1];
      R1 = (long)(off[j0 + 2] - off[j0 + 1]) * d.G;
    }
    const long h0 = (R0 + 63) / 64, h1 = (R1 + 63) / 64;
    nI = (int)min(h0, h1);
    const long rest = (R0 > R1 ? R0 : R1) - (long)nI * 64;
    ntiles_all = nI + (int)((max(rest, 0L) + 127) / 128);
  } else {
    if (MODE == 1) {
      const int t_lo = kbase, t_hi = min(kbase + 2 * kKeys - 1 + d.window - 1, d.T - 1);
      tq_lo = max(0, t_lo - d.q_off);
      ntok = max(0, t_hi - d.q_off - tq_lo + 1);
    } else {  // every query from the one that completes compressed block kbase on
      tq_lo = max(0, kbase * d.dc + d.lc - 1 - d.q_off);
      ntok = max(0, d.Tq - tq_lo);
    }
    ntiles_all = (int)(((long)ntok * d.G + 127) / 128);
  }
  const int tps = (ntiles_all + nseg - 1) / nseg;  // tiles per share
  const int u0 = seg * tps;
  const int ntiles = max(0, min(tps, ntiles_all - u0));

  if (tid == 0) {
    mbar_init(&bars->kv, 1);
    mbar_init(&bars->vready, kKeyThreads);
    for (int i = 0; i < kNBuf; ++i) {
      mbar_init(&bars->gathered[i], 128);
      mbar_init(&bars->bfree[i], 1);
    }
    mbar_init(&bars->s, 1);
    mbar_init(&bars->sfree, kKeyThreads);
    mbar_init(&bars->p, kKeyThreads);
    mbar_init(&bars->sdone, 1);
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  if (warp == 8) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 10) {
    // ---- row gather: warp 10 + w fills rows 32w .. 32w+31 of each tile ------------------
    // Thread gr looks up row gr's token (one iteration ahead: the list entry
    // of the next tile is loaded while this tile's copies go out).  The Q and
    // dO rows go by cp.async (16 bytes each, zero-filled for an absent row),
    // lane L copying 16-byte chunk L % 8 of rows 4i + L / 8 of the warp's 32,
    // so each instruction covers four whole 128-byte rows; a tile is handed
    // to the MMA side one iteration after its copies were issued, once they
    // have landed.
    const int gr = tid - 320;
    const int ch = lane & 7;
    auto row_of = [&](int u, int* which, int* hh) -> int {  // query index or -1
      const int uu = u0 + u;
      if (SEL) {
        const long rix = sel_tile_row(uu, gr, R0, R1, nI, which);
        if (rix < 0) return -1;
        *hh = (int)(rix % d.G);
        return (*which ? l1 : l0)[rix / d.G];
      }
      *which = 0;
      const long rix = (long)uu * 128 + gr;
      *hh = (int)(rix % d.G);
      const long ti = rix / d.G;
      return ti < ntok ? tq_lo + (int)ti : -1;
    };
    int wh_n = 0, hh_n = 0;
    int tq_n = ntiles > 0 ? row_of(0, &wh_n, &hh_n) : -1;
    bool ok = true;
    for (int u = 0; u < ntiles; ++u) {
      const int bu = u % kNBuf;
      if (u >= kNBuf &&
          !wait_bar(&bars->bfree[bu], ((u - kNBuf) / kNBuf) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      const int tq = tq_n, which = wh_n, hh = hh_n;
      if (u + 1 < ntiles) tq_n = row_of(u + 1, &wh_n, &hh_n);  // issued now, used next iteration
      const bool okr = tq >= 0 && tq < d.Tq;
      const size_t row = ((size_t)b * d.Tq + (okr ? tq : 0)) * d.Hq + (size_t)g * d.G + hh;
      const uint32_t qb = smem_u32(smem + KV_OFF_Q + bu * kRowTile);
      const uint32_t hb = smem_u32(smem + KV_OFF_DO + bu * kRowTile);
      const uint32_t lb = smem_u32(smem + KV_OFF_DOL + bu * kRowTile);
      const unsigned long long rowc = okr ? (unsigned long long)row : ~0ull;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 4 * i + (lane >> 3);  // row of the warp's 32
        const unsigned long long rw = __shfl_sync(0xffffffffu, rowc, rr);
        const int r = 32 * (warp - 10) + rr;  // row of the tile
        const uint32_t off = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
                             ((uint32_t)(ch ^ (r & 7)) << 4);
        const bool present = rw != ~0ull;
        const size_t src = (present ? (size_t)rw : 0) * 64 + 8 * ch;
        const uint32_t nb = present ? 16u : 0u;
        cp_async16(qb + off, q + src, nb);
        cp_async16(hb + off, dO_hi + src, nb);
        cp_async16(lb + off, dO_lo + src, nb);
      }
      cp_async_commit();
      float l2 = -INFINITY, dl = 0.f;
      if (okr) {
        l2 = __ldg(lse + row) * kLog2e;
        dl = __ldg(delta + row);
      }
      // visible keys of this row among the pair's two halves
      const int t = d.q_off + (okr ? tq : 0);
      const bool live = okr && l2 != -INFINITY;
      int lo0 = kNoKey, lo1 = kNoKey, sp0 = 0, sp1 = 0;
      if (live) {
        if (SEL) {
          if (which == 0) {
            lo0 = 0;
            sp0 = t;
          } else {
            lo1 = 0;
            sp1 = t;
          }
        } else if (MODE == 1) {
          lo0 = lo1 = max(0, t - d.window + 1);
          sp0 = sp1 = t - lo0;
        } else {
          const int khi = cmp_nvis(d, t) - 1;  // last complete compressed block
          if (khi >= 0) {
            lo0 = lo1 = 0;
            sp0 = sp1 = khi;
          }
        }
      }
      KvRowInfo& in = info[bu];
      in.nlse2[gr] = -l2;
      in.ndelta[gr] = -dl;
      in.klo[0][gr] = lo0;
      in.span[0][gr] = sp0;
      in.klo[1][gr] = lo1;
      in.span[1][gr] = sp1;
      // rows 32c .. 32c+31 are this warp's: flag the halves they reach
      const int kb0 = kbase, kb1 = kbase + kKeys;
      const bool r0 = lo0 <= kb0 + kKeys - 1 && lo0 + sp0 >= kb0;
      const bool r1 = lo1 <= kb1 + kKeys - 1 && lo1 + sp1 >= kb1;
      const unsigned m0 = __ballot_sync(0xffffffffu, r0), m1 = __ballot_sync(0xffffffffu, r1);
      if (lane == 0) in.chunk[warp - 10] = (m0 ? 1 : 0) | (m1 ? 2 : 0);
      if (u >= 1) {
        cp_async_wait<1>();        // tile u - 1 has landed
        fence_proxy_async_smem();  // the MMAs read it through the async proxy
        mbar_arrive(&bars->gathered[(u - 1) % kNBuf]);
      }
    }
    cp_async_wait<0>();  // no copy outlives the CTA
    if (ok && ntiles > 0) {
      fence_proxy_async_smem();
      mbar_arrive(&bars->gathered[(ntiles - 1) % kNBuf]);
    }
  } else if (warp == 8) {
    // ---- S^T / dP^T issue (and the pair's K/V by TMA) ---------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_st = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_dp = idesc_f16(128, 128, false, false);
      const uint32_t k_addr = smem_u32(smem + KV_OFF_K), v_addr = smem_u32(smem + KV_OFF_V);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_expect_tx(&bars->kv, 2 * kKTile2);
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(smem + KV_OFF_K + h * kTileBytes, &tm_k, &bars->kv, 0, g, b * nkeys + kbase + h * kKeys);
        tma_load_3d(smem + KV_OFF_V + h * kTileBytes, &tm_v, &bars->kv, 0, g, b * nkeys + kbase + h * kKeys);
      }
      const bool ok = wait_bar(&bars->kv, 0, abort_flag, err) &&
                      (ntiles == 0 || wait_bar(&bars->vready, 0, abort_flag, err));
      for (int u = 0; ok && u < ntiles; ++u) {
        const int bu = u % kNBuf;
        if (!wait_bar(&bars->gathered[bu], (u / kNBuf) & 1, abort_flag, err)) break;
        // S^T / dP^T are single-buffered: the key threads must have loaded tile u-1's
        if (u >= 1 && !wait_bar(&bars->sfree, (u - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + KV_OFF_Q + bu * kRowTile);
        const uint32_t do_addr = smem_u32(smem + KV_OFF_DO + bu * kRowTile);
        const uint32_t dol_addr = smem_u32(smem + KV_OFF_DOL + bu * kRowTile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kvColS, desc_sw128(k_addr + kk * 32, 16), desc_sw128(q_addr + kk * 32, 16),
                   idesc_st, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kvColDP, desc_sw128(v_addr + kk * 32, 16), desc_sw128(do_addr + kk * 32, 16),
                   idesc_dp, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dO lo: dP^T keeps about fp32 accuracy
          mma_bf16(tmem + kvColDP, desc_sw128(v_addr + kk * 32, 16),
                   desc_sw128(dol_addr + kk * 32, 16), idesc_dp, 1u);
        mma_commit(&bars->s);
      }
      mma_commit(&bars->sdone);
      drain_bar(&bars->sdone, 0);
      if (!ok) drain_bar(&bars->kv, 0);
    }
  } else if (warp == 9) {
    // ---- dV += P^T dO, dK += dS^T Q issue ----------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_kv = idesc_bf16(128, 64, false, true);  // A in TMEM, B MN-major
      constexpr uint32_t idesc_v16 = idesc_f16(128, 64, false, true);   // dV: fp16 P^T, dO
      for (int u = 0; u < ntiles; ++u) {
        // A operands in TMEM; the gathered tiles read MN-major: K dimension = rows
        if (!wait_bar(&bars->p, u & 1, abort_flag, err)) break;
        tc_fence_after();
        const int bu = u % kNBuf;
        const uint32_t q_addr = smem_u32(smem + KV_OFF_Q + bu * kRowTile);
        const uint32_t do_addr = smem_u32(smem + KV_OFF_DO + bu * kRowTile);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_ts(tmem + kvColDV, tmem + kvColP + kk * 8,
                      desc_sw128(do_addr + kk * 2048, 8192), idesc_v16, acc);
          mma_bf16_ts(tmem + kvColDK, tmem + kvColDS + kk * 8,
                      desc_sw128(q_addr + kk * 2048, 8192), idesc_kv, acc);
        }
        mma_commit(&bars->bfree[bu]);  // frees the row buffer and the P^T / dS^T columns
      }
      mma_commit(&bars->fin);
      drain_bar(&bars->fin, 0);
    }
  } else {
    // ---- key threads: key kbase + k (TMEM lane k), k = 32 (warp % 4) + lane -----------
    const int k = 32 * (warp & 3) + lane;
    const int csel = warp >> 2;  // this warp's chunks: csel and csel + 2
    const int key = kbase + k;
    const int half = k >> 6;  // which block of the pair
    const uint32_t lane_tmem = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = d.scale * kLog2e;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    if (ntiles > 0) {
      // V of the pair (bf16, landed by TMA) -> fp16 in place, for dP^T
      ok = wait_bar_warp(&bars->kv, 0, abort_flag, err);
      if (ok) {
        uint4* vv = reinterpret_cast<uint4*>(smem + KV_OFF_V);
        bool range_ok = true;
        for (int i = tid; i < (int)(kKTile2 / 16); i += kKeyThreads) {
          uint4 x = vv[i];
          uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            range_ok = range_ok && fabsf(f.x) <= 65504.f && fabsf(f.y) <= 65504.f;
            w[e] = pack_f16(f.x, f.y);
          }
          vv[i] = x;
        }
        if (!range_ok) record_error(err, kDevRange);
        fence_proxy_async_smem();  // the MMA reads V through the async proxy
        mbar_arrive(&bars->vready);
      }
    }
    int dirty = 3;  // bit i: P^T / dS^T columns of chunk csel + 2i may hold nonzero values
    for (int u = 0; u < ntiles; ++u) {
      const KvRowInfo& in = info[u % kNBuf];
      if (!wait_bar_warp(&bars->s, u & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      bool stop = false;
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {  // 32 rows at a time, in halves of 16
        const int c = csel + 2 * i;
        const bool any = (in.chunk[c] >> half) & 1;  // warp-uniform
        if (!any) {
          if (i == 1) {  // nothing to load: release S^T / dP^T now
            tc_fence_before();
            mbar_arrive(&bars->sfree);
          }
          if (!((dirty >> i) & 1)) continue;  // columns already zero
        }
        if (u >= 1 && (dirty & 4) == 0) {
          // P^T / dS^T (TMEM): the dV/dK MMAs of tile u-1 must have read them
          // (waited for before this warp's first store of the tile; bit 2 of
          // dirty records that it has been)
          if (!wait_bar_warp(&bars->bfree[(u - 1) % kNBuf], ((u - 1) / kNBuf) & 1, abort_flag,
                             err)) {
            stop = true;
            if (any && i == 1) mbar_arrive(&bars->sfree);
            break;
          }
          tc_fence_after();
        }
        dirty |= 4;
        if (!any) {
          uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            tmem_st8u(lane_tmem + kvColP + 16u * c + 8u * hf, z);
            tmem_st8u(lane_tmem + kvColDS + 16u * c + 8u * hf, z);
          }
          dirty &= ~(1 << i);
          continue;
        }
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          float sv[16], pv[16];
          tmem_ld16(lane_tmem + kvColS + 32u * c + 16u * hf, sv);
          tmem_ld16(lane_tmem + kvColDP + 32u * c + 16u * hf, pv);
          tmem_wait_ld();
          if (i == 1 && hf == 1) {  // S^T and dP^T of this tile are in registers: release them
            tc_fence_before();
            mbar_arrive(&bars->sfree);
          }
          uint32_t pp[8], dd[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int r = 32 * c + 16 * hf + e;
            const int2 lo = *reinterpret_cast<const int2*>(&in.klo[half][r]);
            const int2 sp = *reinterpret_cast<const int2*>(&in.span[half][r]);
            const uint64_t nl = *reinterpret_cast<const uint64_t*>(&in.nlse2[r]);
            const uint64_t nd = *reinterpret_cast<const uint64_t*>(&in.ndelta[r]);
            const float2 x = f2_unpack(f2_fma(f2_pack(sv[e], sv[e + 1]), sl2x2, nl));
            const bool v0 = (unsigned)(key - lo.x) <= (unsigned)sp.x;
            const bool v1 = (unsigned)(key - lo.y) <= (unsigned)sp.y;
            const float p0 = v0 ? fast_exp2(x.x) : 0.f;
            const float p1 = v1 ? fast_exp2(x.y) : 0.f;
            const uint64_t pq = f2_pack(p0, p1);
            const float2 ds = f2_unpack(f2_mul(pq, f2_add(f2_pack(pv[e], pv[e + 1]), nd)));
            pp[e / 2] = pack_f16(p0, p1);
            dd[e / 2] = pack_bf16(ds.x, ds.y);
          }
          tmem_st8u(lane_tmem + kvColP + 16u * c + 8u * hf, pp);
          tmem_st8u(lane_tmem + kvColDS + 16u * c + 8u * hf, dd);
        }
        dirty |= 1 << i;
      }
      dirty &= 3;
      if (stop) {
        ok = false;
        break;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p);
    }
    // epilogue: dv += dV (warps 0-3), dk += scale * dK (warps 4-7) for this key
    bool have = false;
    if (ok && ntiles > 0) have = wait_bar_warp(&bars->fin, 0, abort_flag, err);
    float a[32];
    const size_t krow = ((size_t)b * nkeys + key) * d.Hkv * 64 + (size_t)g * 64;
    const bool kin = key < nkeys;
    const size_t nk_all = (size_t)d.B * nkeys * d.Hkv * 64;  // one share of dK (or dV)
    const bool isk = csel == 1;
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {  // columns [32h, 32h + 32) of dV or dK
      if (have) {
        tc_fence_after();
        tmem_ld32(lane_tmem + (isk ? kvColDK : kvColDV) + 32u * h, a);
        tmem_wait_ld();
      }
      const float sc = isk ? d.scale : 1.f;
      if (MODE == 2 && kin) {  // this share's partial (zeros when it had no rows)
        float* dst = part + ((size_t)seg * 2 + (isk ? 0 : 1)) * nk_all + krow + 32 * h;
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(dst + c) =
              have ? make_float4(a[c] * sc, a[c + 1] * sc, a[c + 2] * sc, a[c + 3] * sc)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      } else if (have && kin) {
        float* dst = (isk ? dk : dv) + krow + 32 * h;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          float4 x = *reinterpret_cast<float4*>(dst + c);
          x.x = fmaf(a[c], sc, x.x);
          x.y = fmaf(a[c + 1], sc, x.y);
          x.z = fmaf(a[c + 2], sc, x.z);
          x.w = fmaf(a[c + 3], sc, x.w);
          *reinterpret_cast<float4*>(dst + c) = x;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dO (fp32) split into an fp16 pair for the gathered dK/dV tiles: hi = dO
// rounded to nearest even, lo = (dO - hi) rounded likewise; n a multiple
// of 8.  A finite element beyond fp16's range is recorded as a range error.
__global__ void dO_split_f16_kernel(const float* __restrict__ src, __half* __restrict__ hi,
                                    __half* __restrict__ lo, size_t n, int* err) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  const float4 a = *reinterpret_cast<const float4*>(src + i);
  const float4 c = *reinterpret_cast<const float4*>(src + i + 4);
  const float x[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
  uint32_t h[4], l[4];
  bool range_ok = true;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float h0 = __half2float(__float2half_rn(x[2 * e]));
    const float h1 = __half2float(__float2half_rn(x[2 * e + 1]));
    range_ok = range_ok && fabsf(x[2 * e]) <= 65504.f && fabsf(x[2 * e + 1]) <= 65504.f;
    h[e] = pack_f16(h0, h1);
    l[e] = pack_f16(x[2 * e] - h0, x[2 * e + 1] - h1);
  }
  if (!range_ok) record_error(err, kDevRange);
  *reinterpret_cast<uint4*>(hi + i) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(lo + i) = make_uint4(l[0], l[1], l[2], l[3]);
}

// dk += sum over shares of part[s][0], dv += sum of part[s][1], in share order.
__global__ void dkdv_share_sum_kernel(const float* __restrict__ part, float* __restrict__ dk,
                                      float* __restrict__ dv, size_t n, int nseg) {
  const size_t e = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= n) return;
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  for (int s = 0; s < nseg; ++s) {
    const float4 x = *reinterpret_cast<const float4*>(part + (size_t)(2 * s) * n + e);
    const float4 y = *reinterpret_cast<const float4*>(part + (size_t)(2 * s + 1) * n + e);
    sk.x += x.x; sk.y += x.y; sk.z += x.z; sk.w += x.w;
    sv.x += y.x; sv.y += y.y; sv.z += y.z; sv.w += y.w;
  }
  float4* pk = reinterpret_cast<float4*>(dk + e);
  float4* pv = reinterpret_cast<float4*>(dv + e);
  float4 a = *pk, c = *pv;
  a.x += sk.x; a.y += sk.y; a.z += sk.z; a.w += sk.w;
  c.x += sv.x; c.y += sv.y; c.z += sv.z; c.w += sv.w;
  *pk = a;
  *pv = c;
}

template <int MODE>
cudaError_t launch_dkdv_tc_t(const Dims& d, const void* q, const void* k, const void* v,
                             const float* lse, const float* delta, const float* dO,
                             void* dO16, const int* offsets, const int* list, float* dk,
                             float* dv, float* part, int* err, cudaStream_t s, bool ready) {
  const int nkeys = MODE == 2 ? d.Nc : d.T;
  const int nchunk = (nkeys + kKeys - 1) / kKeys;
  const int npairs = (nchunk + 1) / 2;
  if (npairs == 0) return cudaSuccess;
  const size_t nel = (size_t)d.B * d.Tq * d.Hq * 64;
  if (!ready)
    dO_split_f16_kernel<<<(unsigned)((nel / 8 + 255) / 256), 256, 0, s>>>(
        dO, (__half*)dO16, (__half*)dO16 + nel, nel, err);
  const int nseg = MODE == 2 ? kCmpShares : 1;
  CUtensorMap mk, mv;
  if (!make_tmap_bf16(&mk, k, d.Hkv, (long)d.B * nkeys, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, (long)d.B * nkeys, 1, kKeys))
    return cudaErrorInvalidValue;
  // 512 TMEM columns per CTA: ask for enough shared memory that a second CTA
  // never shares the SM (it would wait in tcgen05.alloc)
  const size_t smem = KV_SMEM + 1024 > 120 * 1024 ? KV_SMEM + 1024 : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_dkdv_tc_kernel<MODE><<<dim3(npairs * nseg, d.Hkv, d.B), kKvThreads, smem, s>>>(
      mk, mv, (const bf16*)q, lse, delta, (const __half*)dO16, (const __half*)dO16 + nel, offsets,
      list, dk, dv, part, nseg, d, err);
  e = cudaGetLastError();
  if (e != cudaSuccess || MODE != 2) return e;
  const size_t n = (size_t)d.B * nkeys * d.Hkv * 64;
  dkdv_share_sum_kernel<<<(unsigned)((n / 4 + 255) / 256), 256, 0, s>>>(part, dk, dv, n, nseg);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_dq_tc_t(const Dims& d, const void* q, const void* k, const void* v,
                           const int32_t* idx, const void* o, const float* lse, const float* dO,
                           float* dq, float* delta, int* err, cudaStream_t s) {
  const int TQ = tokens_per_tile(d.G);
  const long key_rows = (long)d.B * (MODE == 2 ? d.Nc : d.T);
  if (key_rows == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16(&mq, q, d.Hq, (long)d.B * d.Tq, d.G, TQ) ||
      !make_tmap_bf16(&mk, k, d.Hkv, key_rows, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, key_rows, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = OFF_LIST + (list_ints(d) + 2 * kRows) * sizeof(int) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel<MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.Tq + TQ - 1) / TQ, d.Hkv, d.B);
  bwd_dq_tc_kernel<MODE><<<grid, kThreads, smem, s>>>(mq, mk, mv, (const bf16*)o, lse, dO, idx,
                                                      dq, delta, d, err);
  return cudaGetLastError();
}

}  // namespace

// Tensor-core dQ applies to bf16, 64-key blocks, head dim 64, G dividing 128,
// for every branch alike.
bool dq_tc_eligible(const Dims& d, int /*mode*/) {
  return d.dtype == 1 && d.l == kKeys && d.D == 64 && d.G >= 1 && kRows % d.G == 0 &&
         d.Nb <= 4096 && tmap_encode_fn() != nullptr;
}

// Tensor-core dK/dV: the same geometry (key-stationary over pairs of blocks).
bool dkdv_tc_eligible(const Dims& d, int mode) { return dq_tc_eligible(d, mode); }

size_t dkdv_cmp_part_bytes(const Dims& d) {
  return (size_t)kCmpShares * 2 * d.B * d.Nc * d.Hkv * 64 * sizeof(float);
}

cudaError_t launch_dkdv_tc(const Dims& d, int mode, const void* q, const void* k, const void* v,
                           const float* lse, const float* delta, const float* dO, void* dO16,
                           const int* offsets, const int* list, float* dk, float* dv, float* part,
                           int* err, cudaStream_t s, bool dO16_ready) {
  void* o16 = dO16;
  const bool r = dO16_ready;
  if (mode == 0)
    return launch_dkdv_tc_t<0>(d, q, k, v, lse, delta, dO, o16, offsets, list, dk, dv, part, err, s, r);
  if (mode == 1)
    return launch_dkdv_tc_t<1>(d, q, k, v, lse, delta, dO, o16, offsets, list, dk, dv, part, err, s, r);
  return launch_dkdv_tc_t<2>(d, q, k, v, lse, delta, dO, o16, offsets, list, dk, dv, part, err, s, r);
}

// The single-pass selection backward: dQ as launch_dq_tc (mode 0), dK and
// dV added into dk, dv by atomics in the same kernel.
cudaError_t launch_sel_bwd_atomic(const Dims& d, const void* q, const void* k, const void* v,
                                  const int32_t* idx, const void* o, const float* lse,
                                  const float* dO, float* dq, float* delta, float* dk, float* dv,
                                  int* err, cudaStream_t s) {
  const int TQ = tokens_per_tile(d.G);
  if ((long)d.B * d.T == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16(&mq, q, d.Hq, (long)d.B * d.Tq, d.G, TQ) ||
      !make_tmap_bf16(&mk, k, d.Hkv, (long)d.B * d.T, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, (long)d.B * d.T, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = AT_OFF_LIST + (list_ints(d) + 2 * kRows) * sizeof(int) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel<0, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.Tq + TQ - 1) / TQ, d.Hkv, d.B);
  bwd_dq_tc_kernel<0, true><<<grid, kAtThreads, smem, s>>>(
      mq, mk, mv, (const bf16*)o, lse, dO, idx, dq, delta, d, err, dk, dv);
  return cudaGetLastError();
}

cudaError_t launch_dq_tc(const Dims& d, int mode, const void* q, const void* k, const void* v,
                         const int32_t* idx, const void* o, const float* lse, const float* dO,
                         float* dq, float* delta, int* err, cudaStream_t s) {
  return mode == 0   ? launch_dq_tc_t<0>(d, q, k, v, idx, o, lse, dO, dq, delta, err, s)
         : mode == 1 ? launch_dq_tc_t<1>(d, q, k, v, idx, o, lse, dO, dq, delta, err, s)
                     : launch_dq_tc_t<2>(d, q, k, v, idx, o, lse, dO, dq, delta, err, s);
}

}  // namespace nsa
