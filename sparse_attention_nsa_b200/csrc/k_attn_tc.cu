// k_attn_tc.cu -- selection and sliding-window attention on the sm_100a
// tensor cores (tcgen05 + TMEM, TMA-staged K/V blocks), bf16 in, fp32
// softmax and accumulation.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: SELECTION attends to the top-scoring blocks in raw form, SLIDING
// WINDOW to the most recent tokens; the kernel paragraph groups the queries
// that share a sparse selection so reads stay contiguous.  Here the queries
// of one KV group are the unit: a CTA owns 128 query rows = 128/G
// consecutive tokens x the G heads of one KV group (head-stacking gives the
// MMA its M = 128), and walks a list of 64-key blocks:
//   selection: the ascending union of the blocks its tokens selected; a row
//              whose token did not select a block gets P = 0 for it;
//   window   : the contiguous blocks that intersect any row's window.
// The K and V tile of a block is loaded once per CTA by TMA and serves all
// 128 rows.
//
// Per block:  S = Q K^T   (tcgen05, M=128 N=64 K=64, into TMEM)
//             softmax rows in fp32 (one thread per row, exp2 on MUFU)
//             P (bf16, into TMEM) ;  O += P V  (tcgen05, accumulated in TMEM)
// P is relative to a per-row reference max that moves only when a block's
// max exceeds it by more than 2^8; then the row's O is rescaled in TMEM.
// Q and P are A operands read from TMEM, so the only shared-memory traffic
// per block is the TMA write of K and V and the MMAs' reads of them: with
// N = 64 tiles, A operands in shared memory would make the MMAs wait on
// shared-memory bandwidth rather than on the tensor pipe.
// TMEM columns (256 per CTA): S double buffer [0,128), O [128,192),
// Q [192,224) (bf16 pairs per 32-bit column).  P of block i overwrites the
// first 32 columns of the S buffer it was computed from, so writing P never
// waits for an earlier P*V; instead the S MMA that next fills that buffer is
// issued only once the P*V reading it has completed (MMAs of different
// accumulators may overlap in the pipe).
// Warp roles (224 threads): warps 0-3 load Q, softmax and epilogue; warp 4
// issues the S MMAs and owns TMEM; warp 6 issues the P*V MMAs; warp 5 is the
// TMA producer.  Each tcgen05.mma, commit and barrier wait costs its issuing
// thread tens of cycles (measured in place: about 80 per MMA, 100 per
// commit or satisfied wait), so one thread issuing both kinds is the
// critical path once the softmax is short.  S is double-buffered, K/V sit
// in a 6-stage ring.  Two CTAs fit per SM (TMEM).
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace nsa {

cudaError_t launch_sel_fwd_simt(const Dims& d, const void* q, const void* k,
                                const void* v, const int32_t* idx, void* o,
                                float* lse, int* err, cudaStream_t s);
cudaError_t launch_swa_fwd_simt(const Dims& d, const void* q, const void* k,
                                const void* v, void* o, float* lse, cudaStream_t s);

namespace {

using namespace sm100;

constexpr int kRows = 128;   // query rows per CTA (M)
constexpr int kKeys = 64;    // keys per block (N of S, K of P*V)
constexpr int kStages = 6;   // K/V ring depth
constexpr int kThreads = 224;
constexpr uint32_t kTileBytes = kKeys * 64 * 2;  // one K or V block, bf16

// TMEM column map
constexpr uint32_t kColS = 0;    // two S buffers of 64 fp32 columns
constexpr uint32_t kColO = 128;  // O, 64 fp32 columns
constexpr uint32_t kColQ = 192;  // Q rows, 64 bf16 in 32 columns

constexpr uint32_t OFF_KV = 0;  // stage s: K, then V
constexpr uint32_t OFF_BAR = OFF_KV + kStages * 2 * kTileBytes;

struct Bars {
  uint64_t q;      // the 128 row threads have written Q into TMEM
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s[2];
  // p[i & 1]: the 128 row threads have written P of block i.  Two barriers,
  // because a warp may finish block i+1 before another finishes block i.
  uint64_t p[2];
  uint64_t fin;
};
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;  // tmem, abort, nblk
constexpr uint32_t OFF_LIST = OFF_MISC + 16;

__host__ __device__ inline int tokens_per_tile(int G) { return kRows / G; }

__host__ __device__ inline size_t list_ints(const Dims& d) {
  const int words = (d.Nb + 31) / 32;
  return (size_t)d.Nb + words + (size_t)tokens_per_tile(d.G) * (d.topk + 1);
}

// The gated combination (EpilogueFuse) is fused into the epilogue of the
// branch that runs last in a forward, with o_own unrounded; o_own itself is
// stored only when `o` is not null.
using Fuse = EpilogueFuse;

template <bool SEL, bool FUSE>
__global__ void __launch_bounds__(kThreads, 2)
attn_tc_kernel(const bf16* __restrict__ qg, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, bf16* __restrict__ o,
               float* __restrict__ lse, const int32_t* __restrict__ idx, Dims d, int* err,
               Fuse fz) {
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
  const int pos0 = d.q_off + t0;  // key position of the tile's first query

  if (tid == 0) {
    mbar_init(&bars->q, 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s[i], 1);
      mbar_init(&bars->p[i], 128);
    }
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  if (warp == 4) tmem_alloc(tmem_slot, 256);
  if (warp == 5 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }

  // ---- block list ------------------------------------------------------------
  if (SEL) {
    for (int w = tid; w < words; w += kThreads) bits[w] = 0u;
    __syncthreads();
    // one thread per token: validate and copy its selection, mark the union
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
    if (warp == 0) {  // compact the bitmap into an ascending list
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
    // ---- TMA producer -----------------------------------------------------------
    if (lane == 0) {
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
        for (int i = max(0, issued - kStages); i < issued; ++i)
          drain_bar(&bars->full[i % kStages], (i / kStages) & 1);
      }
    }
  } else if (warp == 4) {
    // ---- S = Q K^T issue --------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, false, false);
      bool ok = wait_bar(&bars->q, 0, abort_flag, err);
      tc_fence_after();
      for (int i = 0; ok && i < n; ++i) {
        const int st = i % kStages;
        // S buffer i&1 holds P of block i-2: its P*V (hence its softmax) must
        // be complete; the commit that frees that block's K/V stage says so
        if (i >= 2 &&
            !wait_bar(&bars->empty[(i - 2) % kStages], ((i - 2) / kStages) & 1, abort_flag, err))
          break;
        if (!wait_bar(&bars->full[st], (i / kStages) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
        const uint32_t d_tmem = tmem + kColS + (uint32_t)(i & 1) * 64u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(d_tmem, tmem + kColQ + kk * 8, desc_sw128(k_addr + kk * 32, 16), idesc_s,
                      kk > 0);
        mma_commit(&bars->s[i & 1]);
      }
    }
  } else if (warp == 6) {
    // ---- O += P V issue -----------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16(kRows, 64, false, true);
      for (int i = 0; i < n; ++i) {
        if (!wait_bar(&bars->p[i & 1], (i >> 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const int st = i % kStages;
        const uint32_t v_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes + kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + kColO, tmem + kColS + (uint32_t)(i & 1) * 64u + kk * 8,
                      desc_sw128(v_addr + kk * 2048, 8192), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        // frees the K/V stage and the P columns; O is complete up to block i
        mma_commit(&bars->empty[st]);
      }
      // every P*V must finish before the epilogue reads O; every S MMA has
      // finished before the P it fed was written
      mma_commit(&bars->fin);
      drain_bar(&bars->fin, 0);
    }
  } else {
    // ---- softmax and epilogue: thread r owns query row r -------------------------
    // O accumulates in TMEM (the MMA adds P*V of every block).  P is taken
    // relative to a per-row reference max `mref` that only moves when the
    // block max exceeds it by more than 2^8, so P <= 256; when it moves for
    // some row of a warp, the warp rescales its O rows in TMEM once the
    // previous P*V has landed.
    const int r = tid;
    const int tl = r / d.G, hh = r % d.G;
    const bool valid = tl < nvalid;
    const int t = pos0 + tl;
    const uint32_t lane_tmem = tmem + ((uint32_t)(warp * 32) << 16);
    {  // this row of Q into TMEM (zeros past the last query)
      uint32_t qv[32];
      if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(
            qg + (((size_t)b * d.Tq + t0 + tl) * d.Hq + (size_t)g * d.G + hh) * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = __ldg(src + c);
          qv[4 * c] = u.x;
          qv[4 * c + 1] = u.y;
          qv[4 * c + 2] = u.z;
          qv[4 * c + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) qv[c] = 0u;
      }
      tmem_st32u(lane_tmem + kColQ, qv);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->q);
    }
    const int lo = SEL ? 0 : max(0, t - d.window + 1);  // first key of the row
    const int* lst = SEL ? toks + tl * (d.topk + 1) : nullptr;
    int ptr = 0;
    int nxt = SEL && valid ? lst[0] : INT_MAX;  // next block this row selected
    float mref = -INFINITY, lsum = 0.f;
    const float sl2 = d.scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int j = SEL ? blk[i] : blk0 + i;
      const int k0 = j * kKeys;
      bool rowsel = valid && k0 <= t;
      if (SEL) {
        // the union list is ascending and contains every block of the row's
        // list, so the row's next selected block is never below j
        const bool hit = nxt == j;
        if (hit) nxt = lst[++ptr];  // consumed only at the next hit
        rowsel = rowsel && hit;
      } else {
        rowsel = rowsel && (k0 + kKeys - 1 >= lo);
      }
      if (!wait_bar_warp(&bars->s[i & 1], (i >> 1) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[64];
      tmem_ld32(lane_tmem + kColS + (uint32_t)(i & 1) * 64u, sv);
      tmem_ld32(lane_tmem + kColS + (uint32_t)(i & 1) * 64u + 32u, sv + 32);
      tmem_wait_ld();
      float ms = -INFINITY;  // block max, scaled to log2 units
      if (rowsel) {
        if (!((k0 + kKeys - 1 <= t) && (k0 >= lo))) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (k0 + c > t || k0 + c < lo) sv[c] = -INFINITY;
        }
        // instruction-bound: three-input max, scale and sums on fp32 pairs
        float m0 = sv[0], m1 = sv[1], m2 = sv[2], m3 = sv[3];
#pragma unroll
        for (int c = 4; c < 64; c += 8) {
          m0 = fmax3(m0, sv[c], sv[c + 4]);
          m1 = fmax3(m1, sv[c + 1], sv[c + 5]);
          m2 = fmax3(m2, sv[c + 2], sv[c + 6]);
          m3 = fmax3(m3, sv[c + 3], sv[c + 7]);
        }
        ms = fmaxf(fmax3(m0, m1, m2), m3) * sl2;
      }
      const bool grow = rowsel && ms > mref + 8.f;
      const bool resc = grow && mref != -INFINITY;
      float f = 1.f;  // factor for this row's O (blocks before i)
      if (grow) {
        if (resc) {
          f = fast_exp2(mref - ms);
          lsum *= f;
        }
        mref = ms;
      }
      uint32_t pk[32];
      if (rowsel) {
        const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mref, -mref);
        uint64_t r01 = f2_pack(0.f, 0.f), r23 = r01;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float2 x01 = f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), sc2, nm2));
          const float2 x23 = f2_unpack(f2_fma(f2_pack(sv[c + 2], sv[c + 3]), sc2, nm2));
          const float p0 = fast_exp2(x01.x), p1 = fast_exp2(x01.y);
          const float p2 = fast_exp2(x23.x), p3 = fast_exp2(x23.y);
          r01 = f2_add(r01, f2_pack(p0, p1));
          r23 = f2_add(r23, f2_pack(p2, p3));
          pk[c / 2] = pack_bf16(p0, p1);
          pk[c / 2 + 1] = pack_bf16(p2, p3);
        }
        const float2 a01 = f2_unpack(r01), a23 = f2_unpack(r23);
        lsum += (a01.x + a01.y) + (a23.x + a23.y);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      if (__any_sync(0xffffffffu, resc)) {  // resc implies i > 0
        // O holds P*V of blocks 0..i-1: wait for the last one (its commit
        // frees that block's K/V stage), then rescale rows.  The next phase
        // of that barrier needs the P*V of block i-1+kStages, so the parity
        // below cannot alias.
        if (!wait_bar_warp(&bars->empty[(i - 1) % kStages], ((i - 1) / kStages) & 1, abort_flag,
                           err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float ov[32];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          tmem_ld32(lane_tmem + kColO + 32u * h2, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] *= f;
          tmem_st32(lane_tmem + kColO + 32u * h2, ov);
        }
      }
      tmem_st32u(lane_tmem + kColS + (uint32_t)(i & 1) * 64u, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p[i & 1]);
    }
    float acc[64];
    bool have_o = false;
    // every MMA of this CTA has completed once `fin` (committed after the
    // last P*V) fires
    if (ok && n > 0) have_o = wait_bar_warp(&bars->fin, 0, abort_flag, err);
    if (have_o) {
      tc_fence_after();
      tmem_ld32(lane_tmem + kColO, acc);
      tmem_ld32(lane_tmem + kColO + 32u, acc + 32);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] = 0.f;
    }
    tc_fence_before();
    if (valid) {
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      const int h = g * d.G + hh;
      const size_t row = ((size_t)b * d.Tq + t0 + tl) * d.Hq + h;
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] *= inv;
      if (o) {
        uint4* dst = reinterpret_cast<uint4*>(o + row * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 u;
          u.x = pack_bf16(acc[8 * c + 0], acc[8 * c + 1]);
          u.y = pack_bf16(acc[8 * c + 2], acc[8 * c + 3]);
          u.z = pack_bf16(acc[8 * c + 4], acc[8 * c + 5]);
          u.w = pack_bf16(acc[8 * c + 6], acc[8 * c + 7]);
          dst[c] = u;
        }
      }
      if (FUSE) {
        const float gw = fz.gates[row * 3 + fz.own_gate];
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] *= gw;
#pragma unroll
        for (int br = 0; br < 2; ++br) {
          if (!fz.other[br]) continue;
          const float gb = fz.gates[row * 3 + fz.other_gate[br]];
          const uint4* src = reinterpret_cast<const uint4*>((const bf16*)fz.other[br] + row * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 u = src[c];
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(pb[e]);
              acc[8 * c + 2 * e] = fmaf(gb, f.x, acc[8 * c + 2 * e]);
              acc[8 * c + 2 * e + 1] = fmaf(gb, f.y, acc[8 * c + 2 * e + 1]);
            }
          }
        }
        uint4* dst = reinterpret_cast<uint4*>((bf16*)fz.out + row * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 u;
          u.x = pack_bf16(acc[8 * c + 0], acc[8 * c + 1]);
          u.y = pack_bf16(acc[8 * c + 2], acc[8 * c + 3]);
          u.z = pack_bf16(acc[8 * c + 4], acc[8 * c + 5]);
          u.w = pack_bf16(acc[8 * c + 6], acc[8 * c + 7]);
          dst[c] = u;
        }
      }
      if (lse) lse[row] = lsum > 0.f ? (mref + log2f(lsum)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---- host side ------------------------------------------------------------------------
bool tc_eligible(const Dims& d) {
  return d.dtype == 1 && d.l == kKeys && d.D == 64 && d.G >= 1 && kRows % d.G == 0 &&
         d.Nb <= 4096 && tmap_encode_fn() != nullptr;
}

template <bool SEL, bool FUSE>
cudaError_t launch_tc(const Dims& d, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* o, float* lse, int* err, const Fuse& fz,
                      cudaStream_t s) {
  const int TQ = tokens_per_tile(d.G);
  CUtensorMap mk, mv;
  if (!make_tmap_bf16(&mk, k, d.Hkv, (long)d.B * d.T, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, (long)d.B * d.T, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = OFF_LIST + list_ints(d) * sizeof(int) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<SEL, FUSE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d.Tq + TQ - 1) / TQ, d.Hkv, d.B);
  attn_tc_kernel<SEL, FUSE><<<grid, kThreads, smem, s>>>((const bf16*)q, mk, mv, (bf16*)o, lse,
                                                        idx, d, err,
                                                        fz);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sel_fwd(const Dims& d, const void* q, const void* k, const void* v,
                           const int32_t* idx, void* o, float* lse, int* err,
                           cudaStream_t s) {
  if (tc_eligible(d)) return launch_tc<true, false>(d, q, k, v, idx, o, lse, err, Fuse{}, s);
  return launch_sel_fwd_simt(d, q, k, v, idx, o, lse, err, s);
}

cudaError_t launch_swa_fwd(const Dims& d, const void* q, const void* k, const void* v,
                           void* o, float* lse, cudaStream_t s) {
  if (tc_eligible(d)) return launch_tc<false, false>(d, q, k, v, nullptr, o, lse, nullptr, Fuse{}, s);
  return launch_swa_fwd_simt(d, q, k, v, o, lse, s);
}

bool swa_combine_fusable(const Dims& d) { return tc_eligible(d); }

cudaError_t launch_swa_fwd_combine(const Dims& d, const void* q, const void* k, const void* v,
                                   void* o_swa, float* lse_swa, const float* gates,
                                   const void* o_cmp, const void* o_sel, void* out,
                                   cudaStream_t s) {
  Fuse fz{gates,
          {(d.branch_mask & 1) ? o_cmp : nullptr, (d.branch_mask & 2) ? o_sel : nullptr},
          {0, 1},
          2,
          out};
  return launch_tc<false, true>(d, q, k, v, nullptr, o_swa, lse_swa, nullptr, fz, s);
}

cudaError_t launch_sel_fwd_combine(const Dims& d, const void* q, const void* k, const void* v,
                                   const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                                   const float* gates, const void* o_cmp, const void* o_swa,
                                   void* out, cudaStream_t s) {
  Fuse fz{gates,
          {(d.branch_mask & 1) ? o_cmp : nullptr, (d.branch_mask & 4) ? o_swa : nullptr},
          {0, 2},
          1,
          out};
  return launch_tc<true, true>(d, q, k, v, idx, o_sel, lse_sel, err, fz, s);
}

}  // namespace nsa
