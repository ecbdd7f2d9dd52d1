// k_sel_bm.cu -- selection attention, block-major: each key block is read
// once per work unit and meets exactly the queries that selected it.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: SELECTION attends, per query and KV group, to the top-n blocks in
// raw form; the kernel paragraph's point is that the queries sharing a
// block should be served from one load of it.  The query-tiled kernel
// (k_attn_tc.cu) walks the union of a tile's blocks, and with independent
// selections that union is nearly the whole causal prefix: its MMAs and its
// per-block softmax pass run about Nb / topk times the selected work.  Here
// the iteration is inverted.  The reverse map (block -> the queries that
// chose it, k_bwd.cu) is cut into work units of at most kSeg tiles; a
// persistent CTA takes units in turn, loads the unit's K and V block by TMA
// once, gathers 128 query rows per tile (128/G queries x the G heads of the
// group) and computes each row's softmax over the block on its own:
//     m_s = max_c S[c],  l_s = sum_c 2^(S[c] - m_s),  O_s = (P V) / l_s,
//     lse_s = ln 2 * (m_s + log2 l_s)                 (S in log2 units)
// for the row's slot s (the block's rank in the row's selection).  Each
// row's partials are then merged exactly (sel_merge_kernel):
//     lse = log sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) O_s,
// the split-softmax identity; the merge also applies the gates.  Every MMA
// row and every exponential belongs to a selected (query, block) pair, at
// the price of one fp16 partial row (128 B) and one float per (query, head,
// slot) written and read back.
//
// Per tile (M = 128 rows, N = 64 keys):
//   gather warps: the tile's list entries into a ring
//   softmax warpgroup: the tile's Q rows (cp.async, 128B swizzle), two of
//   its tiles ahead
//   S = Q K^T  (tcgen05, K by TMA)
//   softmax warpgroup: block max, P = 2^(S - m) (bf16, into TMEM over S), l
//   O = P V    (tcgen05, P from TMEM, V MN-major)
//   epilogue warpgroup: O / l -> the rows' partial slots (fp16), lse_s
// Warp specialisation (512 threads, one CTA per SM): the exponentials are
// the bound, so the two softmax warpgroups (even / odd tiles) do little
// else but copy their own Q rows; the epilogue warpgroup reads O and
// stores, two warps read the list entries, and two single-thread roles issue
// the S MMAs (and the K/V TMA) and the P*V MMAs.
// TMEM (512 columns): softmax warpgroup x owns [256 x, 256 x + 256): two
// S/P buffers of 64 columns, then two O buffers of 64.
#include <atomic>
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace nsa {
namespace {

using namespace sm100;

constexpr int kRows = 128;       // rows per tile (M)
constexpr int kKeys = 64;        // keys per block
constexpr int kSeg = 4;          // tiles per work unit (unit sizes 1 .. kSeg: four classes)
constexpr int kThreads = 512;
constexpr int kQBufs = 8;        // Q tiles in shared memory (copied kQBufs tiles ahead)
constexpr int kERing = 16;       // list-entry ring (tiles)
constexpr int kMRing = 8;        // row-statistics ring (tiles)
constexpr int kMaxUnits = 256;   // units per CTA (the grid grows past that)
constexpr int kMaxSortedGroups = 1024;  // (sequence, group) pairs whose units are dealt by size
constexpr uint32_t kTileBytes = kKeys * 64 * 2;  // one K or V block, bf16
constexpr uint32_t kQBytes = kRows * 64 * 2;

constexpr int kKvStages = 3;     // K/V blocks in shared memory (units)

// warp roles
constexpr int kWarpEpi = 8;      // warps 8-11
constexpr int kWarpS = 12, kWarpPV = 13, kWarpGather = 14;  // gather: warps 14-15

constexpr uint32_t OFF_KV = 0;                                    // kKvStages x (K, V)
constexpr uint32_t OFF_Q = OFF_KV + kKvStages * 2 * kTileBytes;   // kQBufs Q tiles
constexpr uint32_t OFF_STG = OFF_Q + kQBufs * kQBytes;            // 4 KB per epilogue warp
constexpr uint32_t OFF_ERING = OFF_STG + kRows * 128;             // kERing x 128 list entries
constexpr uint32_t OFF_MRING = OFF_ERING + kERing * kRows * 4;    // kMRing x 128 x (m, l, slot)
constexpr uint32_t OFF_UNITS = OFF_MRING + kMRing * kRows * 16;   // kMaxUnits int4
constexpr int kMaxTiles = kMaxUnits * kSeg;
constexpr uint32_t OFF_TLIST = OFF_UNITS + kMaxUnits * 16;       // kMaxTiles uint16: unit << 2 | tile
constexpr uint32_t OFF_BAR = OFF_TLIST + kMaxTiles * 2;

struct Bars {
  uint64_t kvfull[kKvStages];
  uint64_t kvfree[kKvStages];  // every P*V of the unit in that stage is done
  uint64_t qfull[kQBufs];      // the softmax warpgroup's Q copies of the tile landed
  uint64_t efull[kERing];      // the tile's list entries are in the ring
  uint64_t efree[kERing];      // the softmax warpgroup is done with the tile's entries
  uint64_t s[2][2];            // [warpgroup][buffer]: S is in TMEM
  uint64_t p[2][2];            // the warpgroup wrote P over it
  uint64_t spfree[2][2];       // the P*V that read that P is done
  uint64_t o[2][2];            // O is in TMEM
  uint64_t ofree[2][2];        // the epilogue loaded that O
  uint64_t mfull[kMRing];      // the tile's row statistics are in the ring
  uint64_t fin;                // every P*V of the CTA is done
  uint64_t sfin;               // every S MMA of the CTA is done
};
// tmem, abort, ntiles, units, four class bases, unit total
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 48;
static_assert(kSeg == 4, "four unit-size classes");
static_assert(kMRing * kRows * 16 >= 4 * kMaxSortedGroups * 4, "class prefixes fit the row ring");
static_assert(kERing * kRows * 4 >= 16 * 4 * 4, "scan scratch fits the entry ring");

__host__ __device__ inline int tile_tokens(int G) { return kRows / G; }

// A CTA's unit k (shared memory): x = sequence << 20 | group << 13 | block,
// y, z = first and end list position, w = global unit index; y == z for a
// slot past its group's unit count.
__device__ __forceinline__ int u_b(int4 u) { return u.x >> 20; }
__device__ __forceinline__ int u_g(int4 u) { return (u.x >> 13) & 127; }
__device__ __forceinline__ int u_j(int4 u) { return u.x & 8191; }

__global__ void __launch_bounds__(kThreads, 1)
sel_bm_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const bf16* __restrict__ q, const int* __restrict__ list,
              const int4* __restrict__ units, const int* __restrict__ ucount, int umax,
              __half* __restrict__ part_o, float* __restrict__ part_lse, Dims d, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  int4* us = (int4*)(smem + OFF_UNITS);
  int* ering = (int*)(smem + OFF_ERING);
  float4* mring = (float4*)(smem + OFF_MRING);
  uint32_t* tmem_slot = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int TQ = tile_tokens(d.G);
  const int lgG = __ffs(d.G) - 1;  // G is a power of two (it divides 128)
  const int BG = d.B * d.Hkv;
  const int nU = BG * umax;
  const int4* ucls = reinterpret_cast<const int4*>(ucount);  // class sizes per (sequence, group)
  const size_t list_stride = (size_t)d.Tq * d.topk;  // list entries per (sequence, group)

  if (tid == 0) {
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&bars->kvfull[s], 1);
      mbar_init(&bars->kvfree[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      for (int x = 0; x < 2; ++x) {
        mbar_init(&bars->s[x][s], 1);
        mbar_init(&bars->p[x][s], kRows);
        mbar_init(&bars->spfree[x][s], 1);
        mbar_init(&bars->o[x][s], 1);
        mbar_init(&bars->ofree[x][s], kRows);
      }
    }
    for (int s = 0; s < kQBufs; ++s) mbar_init(&bars->qfull[s], kRows);
    for (int s = 0; s < kERing; ++s) {
      mbar_init(&bars->efull[s], 64);
      mbar_init(&bars->efree[s], kRows);
    }
    for (int s = 0; s < kMRing; ++s) mbar_init(&bars->mfull[s], kRows);
    mbar_init(&bars->fin, 1);
    mbar_init(&bars->sfin, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  // This CTA's units.  Each group's units come sorted by size (kSeg tiles,
  // then tails of kSeg-1 .. 1 tiles); with at most kMaxSortedGroups groups
  // the CTAs deal the globally sorted sequence (class by class, groups in
  // order) in a snake: CTA c takes positions c, 2 grid - 1 - c, 2 grid + c,
  // ..., so every CTA gets nearly the same number of tiles.  With more
  // groups, CTA c takes unit slots c, c + grid, ... of the groups' arrays.
  int* misc = (int*)(smem + OFF_MISC);  // [3] units of this CTA, [4..7] class bases, [8] total
  const bool dealt = BG <= kMaxSortedGroups;
  const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
  int* pre = (int*)(smem + OFF_MRING);  // [4][BG] per class: its units in the groups before
  if (dealt) {
    // exclusive scan over the groups of the four class sizes (two groups a thread)
    int* wsum = (int*)(smem + OFF_ERING);  // 16 warps x 4, scratch before the ring is used
    const int g0 = 2 * tid, g1 = 2 * tid + 1;
    const int4 v0 = g0 < BG ? __ldg(ucls + g0) : make_int4(0, 0, 0, 0);
    const int4 v1 = g1 < BG ? __ldg(ucls + g1) : make_int4(0, 0, 0, 0);
    int inc[4] = {v0.x + v1.x, v0.y + v1.y, v0.z + v1.z, v0.w + v1.w};
    const int own[4] = {inc[0], inc[1], inc[2], inc[3]};
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int y = __shfl_up_sync(0xffffffffu, inc[c], o);
        if (lane >= o) inc[c] += y;
      }
    if (lane == 31)
#pragma unroll
      for (int c = 0; c < 4; ++c) wsum[warp * 4 + c] = inc[c];
    __syncthreads();
    int ex[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      int base = 0, all = 0;
      for (int w2 = 0; w2 < kThreads / 32; ++w2) {
        const int x = wsum[w2 * 4 + c];
        base += w2 < warp ? x : 0;
        all += x;
      }
      ex[c] = base + inc[c] - own[c];
      if (tid == 0) misc[4 + c] = all;  // class total, turned into bases below
    }
    const int v0c[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (g0 < BG) pre[c * BG + g0] = ex[c];
      if (g1 < BG) pre[c * BG + g1] = ex[c] + v0c[c];
    }
    __syncthreads();
    if (tid == 0) {
      int at = 0;
      for (int c = 0; c < 4; ++c) {
        const int n = misc[4 + c];
        misc[4 + c] = at;
        at += n;
      }
      misc[8] = at;
      const int F = at / grid, rem = at - F * grid;
      const int posF = (F & 1) ? grid - 1 - bid : bid;
      misc[3] = F + (posF < rem ? 1 : 0);  // <= ceil(nU / grid) <= kMaxUnits
    }
  } else if (tid == 0) {
    misc[3] = bid < nU ? (nU - bid + grid - 1) / grid : 0;  // <= kMaxUnits (host sizes the grid)
  }
  __syncthreads();
  const int nk = misc[3];
  for (int k = tid; k < nk; k += kThreads) {
    int bg, local;
    bool live = true;
    if (dealt) {
      const int sp = k * grid + ((k & 1) ? grid - 1 - bid : bid);
      const int c = sp < misc[5] ? 0 : sp < misc[6] ? 1 : sp < misc[7] ? 2 : 3;
      const int r = sp - misc[4 + c];
      const int* pc = pre + c * BG;
      int a = 0, z = BG - 1;  // the last group with pc[a] <= r
      while (a < z) {
        const int mid = (a + z + 1) >> 1;
        if (pc[mid] <= r) a = mid;
        else z = mid - 1;
      }
      bg = a;
      const int4 n = __ldg(ucls + bg);  // the group's units of the classes before c come first
      local = (c > 0 ? n.x : 0) + (c > 1 ? n.y : 0) + (c > 2 ? n.z : 0) + (r - pc[a]);
    } else {
      const int U = bid + k * grid;
      bg = U / umax;
      local = U - bg * umax;
      const int4 n = __ldg(ucls + bg);
      live = local < n.x + n.y + n.z + n.w;
    }
    int4 e = make_int4(0, 0, 0, 0);
    if (live) {
      const int4 x = __ldg(units + (size_t)bg * umax + local);
      const int b = bg / d.Hkv;
      e = make_int4((b << 20) | ((bg - b * d.Hkv) << 13) | x.x, x.y, x.z, 0);
    }
    us[k] = e;
  }
  if (warp == kWarpS) tmem_alloc(tmem_slot, 512);
  if (warp == kWarpS && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  // The CTA's tiles in order (tile i = entry i: unit k, tile t of it), so
  // the roles index tiles instead of walking the unit list: thread k < nk
  // counts unit k's tiles, a block scan places them.
  uint16_t* tl = (uint16_t*)(smem + OFF_TLIST);
  int* ntiles_s = (int*)(smem + OFF_MISC + 8);
  {
    int* wsum = (int*)(smem + OFF_ERING);  // scratch before the ring is used
    const int4 u = tid < nk ? us[tid] : make_int4(0, 0, 0, 0);
    const int cnt = u.z > u.y ? (u.z - u.y + TQ - 1) / TQ : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += wsum[w2];
    if (tid == kThreads - 1) *ntiles_s = base + incl;
    for (int t2 = 0; t2 < cnt; ++t2) tl[base + incl - cnt + t2] = (uint16_t)((tid << 2) | t2);
    __syncthreads();
  }
  const int ntiles = *ntiles_s;
  auto tile_pos = [&](int it, int4& u, int& p) {  // unit and first list position of tile it
    const int e = tl[it];
    u = us[e >> 2];
    p = u.y + (e & 3) * TQ;
  };
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kWarpGather) {
    // ---- list entries of each tile into the ring: warp 14 + h, rows [64 h, 64 h + 64)
    // Lane L copies (4-byte cp.async) the entries of rows 64 h + L + 32 k of
    // tile i + kEAhead while tile i's are published, so kEAhead list reads
    // are in flight at a time.
    constexpr int kEAhead = 4;
    const int h = warp - kWarpGather;
    const uint32_t ering_s = smem_u32(ering);
    auto fetch = [&](int it) {  // one cp.async group
      const uint32_t dst = ering_s + (uint32_t)(((it & (kERing - 1)) * kRows + 64 * h + lane) * 4);
      if (it >= ntiles) {
        st_shared_u32(dst, (uint32_t)-2);
        st_shared_u32(dst + 128, (uint32_t)-2);
      } else {
        int4 u;
        int p0;
        tile_pos(it, u, p0);
        const int* lst = list + (size_t)(u_b(u) * d.Hkv + u_g(u)) * list_stride;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int pos = p0 + ((64 * h + lane + 32 * k) >> lgG);
          if (pos < u.z)
            cp_async4(dst + 128 * k, lst + pos);
          else
            st_shared_u32(dst + 128 * k, (uint32_t)-1);
        }
      }
      cp_async_commit();
    };
    for (int j = 0; j < kEAhead; ++j) fetch(j);
    for (int i = 0; i < ntiles; ++i) {
      const int ia = i + kEAhead;
      // ring slot ia % kERing held tile ia - kERing's entries
      if (ia >= kERing && !wait_bar_warp(&bars->efree[ia & (kERing - 1)],
                                         ((ia / kERing) - 1) & 1, abort_flag, err))
        break;
      fetch(ia);
      cp_async_wait<kEAhead>();  // tile i's group has landed
      __syncwarp();
      mbar_arrive(&bars->efull[i & (kERing - 1)]);
    }
    cp_async_wait<0>();  // no copy outlives the CTA
  } else if (warp == kWarpS) {
    // ---- S = Q K^T ----------------------------------------------------------------------
    // This thread also loads each unit's K/V block by TMA, two units ahead:
    // after the S MMAs of unit kv it refills the stage of unit kv - 1, whose
    // P*Vs finished tiles ago.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, false, false);
      int kv = 0, i = 0, nload = 0, kl = 0;  // units loaded; next unit index to load
      bool ok = true;
      auto load_next = [&]() -> bool {  // K/V of the next non-empty unit, if any
        while (kl < nk && us[kl].y >= us[kl].z) ++kl;
        if (kl >= nk) return true;
        const int st = nload % kKvStages;
        if (nload >= kKvStages &&
            !wait_bar(&bars->kvfree[st], ((nload / kKvStages) - 1) & 1, abort_flag, err))
          return false;
        const int4 u = us[kl];
        const int row = u_b(u) * d.T + u_j(u) * kKeys;
        uint8_t* kvp = smem + OFF_KV + st * 2 * kTileBytes;
        mbar_expect_tx(&bars->kvfull[st], 2 * kTileBytes);
        tma_load_3d(kvp, &tm_k, &bars->kvfull[st], 0, u_g(u), row);
        tma_load_3d(kvp + kTileBytes, &tm_v, &bars->kvfull[st], 0, u_g(u), row);
        ++nload;
        ++kl;
        return true;
      };
      ok = load_next() && load_next();
      for (int k = 0; ok && k < nk; ++k) {
        const int4 u = us[k];
        if (u.y >= u.z) continue;
        const int st = kv % kKvStages;
        if (!wait_bar(&bars->kvfull[st], (kv / kKvStages) & 1, abort_flag, err)) break;
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
        for (int p = u.y; p < u.z; p += TQ, ++i) {
          const int x = i & 1, bf = (i >> 1) & 1;
          // the S/P buffer is free once the P*V of its previous tile (i-4) is done
          if (!wait_bar(&bars->qfull[i % kQBufs], (i / kQBufs) & 1, abort_flag, err) ||
              (i >= 4 && !wait_bar(&bars->spfree[x][bf], ((i >> 2) - 1) & 1, abort_flag, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + OFF_Q + (i % kQBufs) * kQBytes);
          const uint32_t d_tmem = tmem + (uint32_t)(x * 256 + bf * 64);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d_tmem, desc_sw128(q_addr + kk * 32, 16), desc_sw128(k_addr + kk * 32, 16),
                     idesc_s, kk > 0);
          mma_commit(&bars->s[x][bf]);
        }
        ++kv;
        if (ok) ok = load_next();
      }
      mma_commit(&bars->sfin);
      drain_bar(&bars->sfin, 0);
      if (*abort_flag) {  // let the K/V copies already issued land before exit
        for (int x = max(0, nload - kKvStages); x < nload; ++x)
          drain_bar(&bars->kvfull[x % kKvStages], (x / kKvStages) & 1);
      }
    }
  } else if (warp == kWarpPV) {
    // ---- O = P V --------------------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16(kRows, 64, false, true);
      int kv = 0, i = 0;
      bool ok = true;
      for (int k = 0; ok && k < nk; ++k) {
        const int4 u = us[k];
        if (u.y >= u.z) continue;
        const int st = kv % kKvStages;
        if (!wait_bar(&bars->kvfull[st], (kv / kKvStages) & 1, abort_flag, err)) break;
        const uint32_t v_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes + kTileBytes);
        for (int p = u.y; p < u.z; p += TQ, ++i) {
          const int x = i & 1, bf = (i >> 1) & 1;
          // the O buffer is free once the epilogue has loaded its previous tile's O
          if (!wait_bar(&bars->p[x][bf], (i >> 2) & 1, abort_flag, err) ||
              (i >= 4 && !wait_bar(&bars->ofree[x][bf], ((i >> 2) - 1) & 1, abort_flag, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sp = tmem + (uint32_t)(x * 256 + bf * 64);
          const uint32_t ob = tmem + (uint32_t)(x * 256 + 128 + bf * 64);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(ob, sp + kk * 8, desc_sw128(v_addr + kk * 2048, 8192), idesc_o,
                        kk > 0 ? 1u : 0u);
          mma_commit(&bars->o[x][bf]);
          mma_commit(&bars->spfree[x][bf]);
        }
        if (ok) mma_commit(&bars->kvfree[kv % kKvStages]);  // the unit's K/V stage is free
        ++kv;
      }
      mma_commit(&bars->fin);
      drain_bar(&bars->fin, 0);
    }
  } else if (warp < kWarpEpi) {
    // ---- softmax warpgroup x = warp / 4: tiles i with i % 2 == x, row r --------------
    // The warpgroup also copies its tiles' Q rows, kQBufs tiles (four of its
    // own) ahead, far enough for the copies' latency (L2 misses: the partial
    // stores stream through L2): warp w moves rows [32 w, 32 w + 32), lane L
    // chunk L % 8 of rows 32 w + L / 8 + 4 k, so each cp.async instruction
    // covers four whole rows.  Tile i+2's copies are published before tile
    // i's softmax, so its S MMA runs under these exponentials.
    const int x = warp >> 2;
    const int r = tid - x * kRows;
    const uint32_t lane_tmem = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(x * 256);
    const float sl2 = d.scale * kLog2e;
    const int hh = r & (d.G - 1);
    auto copy_q = [&](int it) -> bool {  // one cp.async group
      if (it < ntiles) {
        if (!wait_bar_warp(&bars->efull[it & (kERing - 1)], (it / kERing) & 1, abort_flag, err))
          return false;
        int4 u;
        int p0;
        tile_pos(it, u, p0);
        const int* er = ering + (it & (kERing - 1)) * kRows + (warp & 3) * 32;
        int ev[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ev[k] = er[(lane >> 3) + 4 * k];
        const uint32_t qa = smem_u32(smem + OFF_Q + (it % kQBufs) * kQBytes);
        const int c = lane & 7;
        const bf16* qg =
            q + ((size_t)u_b(u) * d.Tq * d.Hq + (size_t)u_g(u) * d.G) * 64 + c * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = (warp & 3) * 32 + (lane >> 3) + 4 * k;
          const bf16* src = qg + ((size_t)(max(ev[k], 0) >> 6) * d.Hq + (rr & (d.G - 1))) * 64;
          cp_async16(qa + (uint32_t)rr * 128u + ((uint32_t)(c ^ (rr & 7)) << 4), src,
                     ev[k] >= 0 ? 16u : 0u);
        }
      }
      cp_async_commit();
      return true;
    };
    auto publish_q = [&](int it) {  // the copies of tile it landed: kQBufs/2 - 2 newer groups
      cp_async_wait<kQBufs / 2 - 2>();
      fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
      mbar_arrive(&bars->qfull[it % kQBufs]);
    };
    {  // this warpgroup's first kQBufs / 2 tiles: x, x + 2, ...
      bool ok0 = true;
      for (int j = 0; ok0 && j < kQBufs / 2; ++j) ok0 = copy_q(x + 2 * j);
      if (ok0 && x < ntiles) {  // tile x: all but the kQBufs/2 - 1 newer groups
        cp_async_wait<kQBufs / 2 - 1>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->qfull[x % kQBufs]);
      }
    }
    for (int i = x; i < ntiles; i += 2) {
      const int bf = (i >> 1) & 1;
      if (!wait_bar_warp(&bars->efull[i & (kERing - 1)], (i / kERing) & 1, abort_flag, err)) break;
      const int e = ering[(i & (kERing - 1)) * kRows + r];
      if (!wait_bar_warp(&bars->s[x][bf], (i >> 2) & 1, abort_flag, err)) break;
      if (i + 2 < ntiles) publish_q(i + 2);
      // tile i+kQBufs's Q into the buffer tile i's S MMA has finished
      // reading; the copies are in flight under this tile's softmax
      if (!copy_q(i + kQBufs)) break;
      const int4 u = us[tl[i] >> 2];
      const bool valid = e >= 0;
      const int tq = max(e, 0) >> 6;
      const int tpos = d.q_off + tq;
      const int k0 = u_j(u) * kKeys;
      tc_fence_after();
      float sv[64];
      tmem_ld32(lane_tmem + (uint32_t)(bf * 64), sv);
      tmem_ld32(lane_tmem + (uint32_t)(bf * 64 + 32), sv + 32);
      tmem_wait_ld();
      uint32_t pk[32];
      float mx = 0.f, l = 0.f;
      // some row of the warp is in its own block: keys after t are masked
      const bool own = __any_sync(0xffffffffu, valid && tpos < k0 + kKeys - 1);
      if (valid) {
        if (own) {
          const int lim = tpos - k0;
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
        }
        // the row is instruction-bound: three-input max, and the scale and
        // the running sums on fp32 pairs (one instruction per two columns)
        float m0 = sv[0], m1 = sv[1], m2 = sv[2], m3 = sv[3];
#pragma unroll
        for (int c = 4; c < 64; c += 8) {
          m0 = fmax3(m0, sv[c], sv[c + 4]);
          m1 = fmax3(m1, sv[c + 1], sv[c + 5]);
          m2 = fmax3(m2, sv[c + 2], sv[c + 6]);
          m3 = fmax3(m3, sv[c + 3], sv[c + 7]);
        }
        mx = fmaxf(fmax3(m0, m1, m2), m3) * sl2;  // key k0 <= t: finite
        const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mx, -mx);
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
        l = (a01.x + a01.y) + (a23.x + a23.y);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      tmem_st32u(lane_tmem + (uint32_t)(bf * 64), pk);  // P over the first 32 columns of S
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p[x][bf]);
      // the row's statistics and partial slot for the epilogue
      uint32_t slot = UINT_MAX;
      if (valid)
        slot = (uint32_t)((((size_t)u_b(u) * d.Tq + tq) * d.Hq + (size_t)u_g(u) * d.G + hh) *
                              d.topk +
                          (e & 63));
      mring[(i & (kMRing - 1)) * kRows + r] = make_float4(mx, l, __uint_as_float(slot), 0.f);
      mbar_arrive(&bars->mfull[i & (kMRing - 1)]);
      mbar_arrive(&bars->efree[i & (kERing - 1)]);  // tile i's entries are no longer read
    }
    cp_async_wait<0>();  // no copy outlives the CTA
  } else {
    // ---- epilogue warpgroup: O / l of row r to its partial slot, every tile ----------
    const int r = tid - kWarpEpi * 32;
    const uint32_t lane_tmem = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t stg = smem_u32(smem + OFF_STG) + (uint32_t)(warp - kWarpEpi) * 4096u;
    const uint32_t mine = stg + (uint32_t)lane * 128u;
    for (int i = 0; i < ntiles; ++i) {
      const int x = i & 1, bf = (i >> 1) & 1;
      if (!wait_bar_warp(&bars->mfull[i & (kMRing - 1)], (i / kMRing) & 1, abort_flag, err)) break;
      const float4 st = mring[(i & (kMRing - 1)) * kRows + r];
      const uint32_t slot = __float_as_uint(st.z);
      if (!wait_bar_warp(&bars->o[x][bf], (i >> 2) & 1, abort_flag, err)) break;
      tc_fence_after();
      const float inv = slot != UINT_MAX ? __fdividef(1.f, st.y) : 0.f;  // l in [1, 64]
      float ov[64];
      tmem_ld32(lane_tmem + (uint32_t)(x * 256 + 128 + bf * 64), ov);
      tmem_ld32(lane_tmem + (uint32_t)(x * 256 + 128 + bf * 64 + 32), ov + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->ofree[x][bf]);
      // fp16 partials: 11 significant bits, so the merge of up to topk of
      // them adds well under the output's own bf16 rounding.  A partial
      // beyond fp16's range (|v| > 65504) becomes inf, which the merge
      // reports (its output is then not finite).
      const uint64_t inv2 = f2_pack(inv, inv);
      uint32_t hv[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float2 v = f2_unpack(f2_mul(f2_pack(ov[c], ov[c + 1]), inv2));
        hv[c / 2] = pack_f16(v.x, v.y);
      }
      __syncwarp();  // the previous tile's staging reads are done
#pragma unroll
      for (int c = 0; c < 8; ++c)  // fp16 into the staging row, chunks XOR-swizzled by row
        st_shared_v4(mine + ((uint32_t)(c ^ (lane & 7)) << 4), hv[4 * c], hv[4 * c + 1],
                     hv[4 * c + 2], hv[4 * c + 3]);
      if (slot != UINT_MAX) __stcs(part_lse + slot, (st.x + __log2f(st.y)) * kLn2);
      __syncwarp();
      // four whole rows per store instruction; loads first so their latencies overlap
      const int c = lane & 7;
      uint32_t sl[8];
      uint4 w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sl[k] = __shfl_sync(0xffffffffu, slot, (lane >> 3) + 4 * k);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = (lane >> 3) + 4 * k;
        w[k] = ld_shared_v4(stg + (uint32_t)rr * 128u + ((uint32_t)(c ^ (rr & 7)) << 4));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (sl[k] != UINT_MAX)  // streaming: the partials must not evict Q and K/V from L2
          __stcs(reinterpret_cast<uint4*>(part_o + (size_t)sl[k] * 64) + c, w[k]);
    }
  }
  __syncthreads();
  if (warp == kWarpS) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// A slot holds a partial exactly when the reverse map listed it: a causal
// block index above the previous entry (the reverse map's rule).
__device__ __forceinline__ bool slot_used(const int32_t* ir, int s, int cur) {
  const int j = ir[s];
  return j >= 0 && j <= cur && (s == 0 || ir[s - 1] < j);
}

// Merge of a row's slot partials (8 threads per row, 8 head dims each), then
// the row's selection output, lse, and with FUSE the gated combination.
// Lane `sub` of a row owns slots sub, sub + 8, ...: it reads their indices
// and lse values, the row's max and weights are exchanged by shuffles, and
// every lane then reads its 16 bytes of each used slot, 8 slots in flight.
constexpr int kMergeSlots = 8;  // slots per lane: topk <= 64
template <bool FUSE>
__global__ void __launch_bounds__(256)
sel_merge_kernel(const int32_t* __restrict__ idx, const __half* __restrict__ part_o,
                 const float* __restrict__ part_lse, bf16* __restrict__ o_sel,
                 float* __restrict__ lse_sel, Dims d, EpilogueFuse fz, int* err) {
  const size_t nrows = (size_t)d.B * d.Tq * d.Hq;
  const size_t row0 = (size_t)blockIdx.x * 32 + (threadIdx.x >> 3);
  const bool live = row0 < nrows;  // every lane stays for the shuffles
  const size_t row = live ? row0 : nrows - 1;
  const int sub = threadIdx.x & 7;
  const int lane = threadIdx.x & 31, gbase = lane & ~7;
  const size_t bt = row / d.Hq;
  const int h = (int)(row - bt * d.Hq);
  const int tq = (int)(bt % d.Tq);
  const int cur = (d.q_off + tq) / d.l;
  const int32_t* ir = idx + (bt * d.Hkv + h / d.G) * d.topk;
  const float* ls = part_lse + row * d.topk;
  // the first 8 slots' partials and the slots' lse values are read with the
  // indices, not after them (an unused slot's bytes are read but dropped: its
  // weight is 0), so a row's loads wait for one memory latency, not three
  const uint4* po = reinterpret_cast<const uint4*>(part_o + row * d.topk * 64) + sub;
  uint4 u0[8];
#pragma unroll
  for (int q2 = 0; q2 < 8; ++q2)
    if (q2 < d.topk) u0[q2] = po[q2 * 8];
  float wk[kMergeSlots];
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    const int s = sub + 8 * k;
    wk[k] = s < d.topk ? ls[s] : -INFINITY;
  }
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    const int s = sub + 8 * k;
    if (!(s < d.topk && slot_used(ir, s, cur))) wk[k] = -INFINITY;
    m = fmaxf(m, wk[k]);
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
  float L = 0.f;
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    wk[k] = wk[k] == -INFINITY ? 0.f : expf(wk[k] - m);
    L += wk[k];
  }
  L += __shfl_xor_sync(0xffffffffu, L, 1);
  L += __shfl_xor_sync(0xffffffffu, L, 2);
  L += __shfl_xor_sync(0xffffffffu, L, 4);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    if (8 * k >= d.topk) break;
    uint4 u[8];
#pragma unroll
    for (int q2 = 0; q2 < 8; ++q2)
      if (8 * k + q2 < d.topk) u[q2] = k == 0 ? u0[q2] : po[(8 * k + q2) * 8];
#pragma unroll
    for (int q2 = 0; q2 < 8; ++q2) {
      if (8 * k + q2 >= d.topk) break;
      const float w = __shfl_sync(0xffffffffu, wk[k], gbase + q2);
      if (w == 0.f) continue;  // unused slot: its memory is not a partial
      const __half2* pb = reinterpret_cast<const __half2*>(&u[q2]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(pb[e]);
        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
      }
    }
  }
  if (!live) return;
  // the weights are at most 1, so the sum is finite unless a partial that
  // contributes to it overflowed fp16 (or the inputs were not finite)
  bool finite = true;
#pragma unroll
  for (int c = 0; c < 8; ++c) finite = finite && fabsf(acc[c]) <= FLT_MAX;
  if (!finite) record_error(err, kDevRange);
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] *= inv;
  if (o_sel) {
    uint4 w;
    w.x = pack_bf16(acc[0], acc[1]);
    w.y = pack_bf16(acc[2], acc[3]);
    w.z = pack_bf16(acc[4], acc[5]);
    w.w = pack_bf16(acc[6], acc[7]);
    reinterpret_cast<uint4*>(o_sel + row * 64)[sub] = w;
  }
  if (lse_sel && sub == 0) lse_sel[row] = L > 0.f ? m + logf(L) : -INFINITY;
  if (FUSE) {
    const float gw = fz.gates[row * 3 + fz.own_gate];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= gw;
#pragma unroll
    for (int br = 0; br < 2; ++br) {
      if (!fz.other[br]) continue;
      const float gb = fz.gates[row * 3 + fz.other_gate[br]];
      const uint4 u = reinterpret_cast<const uint4*>((const bf16*)fz.other[br] + row * 64)[sub];
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(pb[e]);
        acc[2 * e] = fmaf(gb, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(gb, f.y, acc[2 * e + 1]);
      }
    }
    uint4 w;
    w.x = pack_bf16(acc[0], acc[1]);
    w.y = pack_bf16(acc[2], acc[3]);
    w.z = pack_bf16(acc[4], acc[5]);
    w.w = pack_bf16(acc[6], acc[7]);
    reinterpret_cast<uint4*>((bf16*)fz.out + row * 64)[sub] = w;
  }
}

// ---- host side ---------------------------------------------------------------------------
int units_per_group(const Dims& d) {
  const int tpu = kSeg * tile_tokens(d.G);
  return d.Nb + (int)(((long)d.Tq * d.topk + tpu - 1) / tpu);
}

// workspace layout, each part 256-byte aligned
struct BmCarve {
  size_t chunk, offsets, cursor, list, units, ucount, part_o, part_lse, total;
};
BmCarve bm_carve(const Dims& d) {
  BmCarve c{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t o = at;
    at += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t bg = (size_t)d.B * d.Hkv;
  const size_t slots = (size_t)d.B * d.Tq * d.Hq * d.topk;
  c.chunk = take(revmap_chunk_ints(d) * 4);
  c.offsets = take(bg * (d.Nb + 1) * 4);
  c.cursor = take(bg * d.Nb * 4);
  c.list = take(bg * d.Tq * d.topk * 4);
  c.units = take(bg * units_per_group(d) * sizeof(int4));
  c.ucount = take(bg * sizeof(int4));  // four unit-class sizes per (sequence, group)
  c.part_o = take(slots * 64 * 2);
  c.part_lse = take(slots * 4);
  c.total = at;
  return c;
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

}  // namespace

namespace {
std::atomic<cudaEvent_t> g_ev_start{nullptr}, g_ev_stop{nullptr};
}  // namespace

void set_sel_bm_events(cudaEvent_t start, cudaEvent_t stop) {
  g_ev_start.store(start);
  g_ev_stop.store(stop);
}

bool sel_bm_eligible(const Dims& d) {
  return d.dtype == 1 && d.l == kKeys && d.D == 64 && d.G >= 1 && kRows % d.G == 0 &&
         d.Tq >= 1 && d.Nb >= 1 && d.Nb <= 8192 && d.B < 2048 && d.Hkv <= 128 &&
         d.Tq < (1 << 24) &&
         (size_t)d.B * d.Tq * d.Hq * d.topk < (size_t)UINT_MAX &&  // 32-bit slot numbers
         tmap_encode_fn() != nullptr;
}

size_t sel_bm_ws_bytes(const Dims& d) { return bm_carve(d).total; }

cudaError_t launch_sel_bm_prep(const Dims& d, const int32_t* idx, int* err, void* ws,
                               cudaStream_t s, bool counted) {
  const BmCarve c = bm_carve(d);
  char* w = (char*)ws;
  return launch_revmap_units(d, idx, (int*)(w + c.chunk), (int*)(w + c.offsets),
                             (int*)(w + c.cursor), (int*)(w + c.list), (int4*)(w + c.units),
                             (int*)(w + c.ucount), kSeg * tile_tokens(d.G), tile_tokens(d.G),
                             units_per_group(d), err, s, counted);
}

int* sel_bm_rev_counts(const Dims& d, void* ws) {
  return (int*)((char*)ws + bm_carve(d).chunk);
}

cudaError_t launch_sel_bm(const Dims& d, const void* q, const void* k, const void* v,
                          const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                          const EpilogueFuse* fz, void* ws, cudaStream_t s) {
  const cudaError_t e = launch_sel_bm_prep(d, idx, err, ws, s);
  if (e != cudaSuccess) return e;
  return launch_sel_bm_run(d, q, k, v, idx, o_sel, lse_sel, err, fz, ws, s);
}

cudaError_t launch_sel_bm_run(const Dims& d, const void* q, const void* k, const void* v,
                              const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                              const EpilogueFuse* fz, void* ws, cudaStream_t s) {
  const BmCarve c = bm_carve(d);
  char* w = (char*)ws;
  int* list = (int*)(w + c.list);
  int4* units = (int4*)(w + c.units);
  int* ucount = (int*)(w + c.ucount);
  __half* part_o = (__half*)(w + c.part_o);
  float* part_lse = (float*)(w + c.part_lse);
  const int umax = units_per_group(d);
  cudaError_t e = cudaSuccess;
  CUtensorMap mk, mv;
  if (!make_tmap_bf16(&mk, k, d.Hkv, (long)d.B * d.T, 1, kKeys) ||
      !make_tmap_bf16(&mv, v, d.Hkv, (long)d.B * d.T, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = SMEM_BYTES + 1024;
  e = cudaFuncSetAttribute(sel_bm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long nU = (long)d.B * d.Hkv * umax;
  const long grid = std::max(std::min(nU, (long)sm_count()), (nU + kMaxUnits - 1) / kMaxUnits);
  const cudaEvent_t ev0 = g_ev_start.load(), ev1 = g_ev_stop.load();
  if (ev0 && (e = cudaEventRecord(ev0, s)) != cudaSuccess) return e;
  sel_bm_kernel<<<(unsigned)grid, kThreads, smem, s>>>(mk, mv, (const bf16*)q, list, units, ucount,
                                                       umax, part_o, part_lse, d, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ev1 && (e = cudaEventRecord(ev1, s)) != cudaSuccess) return e;
  const size_t nrows = (size_t)d.B * d.Tq * d.Hq;
  const unsigned mgrid = (unsigned)((nrows + 31) / 32);
  if (fz)
    sel_merge_kernel<true><<<mgrid, 256, 0, s>>>(idx, part_o, part_lse, (bf16*)o_sel, lse_sel, d,
                                                 *fz, err);
  else
    sel_merge_kernel<false><<<mgrid, 256, 0, s>>>(idx, part_o, part_lse, (bf16*)o_sel, lse_sel,
                                                  d, EpilogueFuse{}, err);
  return cudaGetLastError();
}

}  // namespace nsa
