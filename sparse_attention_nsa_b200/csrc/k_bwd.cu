// k_bwd.cu -- NSA backward: gated combination, selection (two passes over
// a reverse block->query map), sliding window and compression branches.
//
// "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method / Key claims:
// each query attends to its own selected subset of keys, so the usual
// key-stationary FlashAttention backward does not apply directly; the study
// runs a query-stationary pass for dQ and then a key-stationary pass for
// dK/dV over a reconstructed reverse key->query mapping, which beats a
// single pass with atomics because keys are shared by many queries.  The
// same two-pass shape serves the window and compression branches, whose
// reverse maps are plain ranges.  No gradient flows through the top-k.
//
// Math per branch (rows r = (token t, head h), keys s):
//   P = exp(scale q.k_s - lse), delta_r = dO_r . o_r,
//   dS = P (dO_r . v_s - delta_r),  dq += scale dS k_s,
//   dk_s += scale dS q_r,  dv_s += P dO_r.
// Gradients are fp32 and accumulated (+=) so the branches can be summed;
// every element is written by one thread in a fixed order (deterministic).
#include "common.cuh"
#include "internal.h"

namespace nsa {

enum BwdMode { kBwdSel = 0, kBwdSwa = 1, kBwdCmp = 2 };

// ---- gated combination ---------------------------------------------------------
// dgates[r, i] = dout_r . o_i,r (enabled branches, else 0); dO_i = gate_i dout.
// 8 consecutive values of a row as fp32 (one 16-byte load for bf16, two for fp32)
__device__ __forceinline__ void load8(const bf16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 c = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
}

// Eight threads per row, eight values each: every load of the row (dout and
// the enabled branches' outputs) is issued before any is used, the three dot
// products are reduced over the row's eight lanes.
struct Half3 {
  __half* p[3];  // per branch: the fp16 pair's hi half (lo follows nel later), or null
};

template <typename T>
__global__ void __launch_bounds__(256)
gate_bwd_kernel(const float* __restrict__ gates, const T* __restrict__ dout,
                const T* __restrict__ oc, const T* __restrict__ os, const T* __restrict__ ow,
                float* __restrict__ dgates, float* __restrict__ dOc, float* __restrict__ dOs,
                float* __restrict__ dOw, long nrows, int mask, Half3 h16, int* err) {
  const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long row0 = t >> 3;
  const int sub = (int)(t & 7);
  const bool live = row0 < nrows;  // every lane stays for the shuffles
  const long row = live ? row0 : nrows - 1;
  const size_t base = (size_t)row * 64 + 8 * sub;
  const T* br[3] = {oc, os, ow};
  float* dst[3] = {dOc, dOs, dOw};
  float g[8], x[3][8];
  load8(dout + base, g);
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    if ((mask >> i) & 1) load8(br[i] + base, x[i]);
    else
#pragma unroll
      for (int e = 0; e < 8; ++e) x[i][e] = 0.f;
  }
  float gi[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) gi[i] = ((mask >> i) & 1) ? gates[row * 3 + i] : 0.f;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    float dg = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dg = fmaf(g[e], x[i][e], dg);
    dg += __shfl_xor_sync(0xffffffffu, dg, 1);
    dg += __shfl_xor_sync(0xffffffffu, dg, 2);
    dg += __shfl_xor_sync(0xffffffffu, dg, 4);
    if (!live) continue;
    if (dst[i]) {
      float4* o = reinterpret_cast<float4*>(dst[i] + base);
      o[0] = make_float4(gi[i] * g[0], gi[i] * g[1], gi[i] * g[2], gi[i] * g[3]);
      o[1] = make_float4(gi[i] * g[4], gi[i] * g[5], gi[i] * g[6], gi[i] * g[7]);
    }
    if (h16.p[i]) {  // the same fp32 values as the fp16 pair hi + lo
      uint32_t hw[4], lw[4];
      bool range_ok = true;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = gi[i] * g[2 * e], x1 = gi[i] * g[2 * e + 1];
        const float h0 = __half2float(__float2half_rn(x0));
        const float h1 = __half2float(__float2half_rn(x1));
        range_ok = range_ok && fabsf(x0) <= 65504.f && fabsf(x1) <= 65504.f;
        const __half2 hh = __floats2half2_rn(h0, h1);
        const __half2 ll = __floats2half2_rn(x0 - h0, x1 - h1);
        hw[e] = *reinterpret_cast<const uint32_t*>(&hh);
        lw[e] = *reinterpret_cast<const uint32_t*>(&ll);
      }
      if (!range_ok) record_error(err, kDevRange);
      const size_t nel = (size_t)nrows * 64;
      *reinterpret_cast<uint4*>(h16.p[i] + base) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(h16.p[i] + nel + base) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    if (sub == 0) dgates[row * 3 + i] = ((mask >> i) & 1) ? dg : 0.f;
  }
}

// Two 64-wide dot products of shared-memory rows a, c with global rows x, y
// (16-byte loads).
template <typename T>
__device__ __forceinline__ void dot2_64(const float* a, const float* c, const T* x, const T* y,
                                        float& ax, float& cy);
template <>
__device__ __forceinline__ void dot2_64<bf16>(const float* a, const float* c, const bf16* x,
                                              const bf16* y, float& ax, float& cy) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 ux = __ldg(reinterpret_cast<const uint4*>(x) + k);
    const uint4 uy = __ldg(reinterpret_cast<const uint4*>(y) + k);
    const __nv_bfloat162* px = reinterpret_cast<const __nv_bfloat162*>(&ux);
    const __nv_bfloat162* py = reinterpret_cast<const __nv_bfloat162*>(&uy);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fx = __bfloat1622float2(px[i]), fy = __bfloat1622float2(py[i]);
      s0 = fmaf(a[8 * k + 2 * i], fx.x, s0);
      s0 = fmaf(a[8 * k + 2 * i + 1], fx.y, s0);
      s1 = fmaf(c[8 * k + 2 * i], fy.x, s1);
      s1 = fmaf(c[8 * k + 2 * i + 1], fy.y, s1);
    }
  }
  ax = s0;
  cy = s1;
}
template <>
__device__ __forceinline__ void dot2_64<float>(const float* a, const float* c, const float* x,
                                               const float* y, float& ax, float& cy) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 fx = __ldg(reinterpret_cast<const float4*>(x) + k);
    const float4 fy = __ldg(reinterpret_cast<const float4*>(y) + k);
    s0 = fmaf(a[4 * k], fx.x, fmaf(a[4 * k + 1], fx.y, fmaf(a[4 * k + 2], fx.z, fmaf(a[4 * k + 3], fx.w, s0))));
    s1 = fmaf(c[4 * k], fy.x, fmaf(c[4 * k + 1], fy.y, fmaf(c[4 * k + 2], fy.z, fmaf(c[4 * k + 3], fy.w, s1))));
  }
  ax = s0;
  cy = s1;
}

// ---- pass 1: dQ, query-stationary ----------------------------------------------
// One CTA per (sequence, query, KV group), one warp per head of the group.
// Also writes delta_r = dO_r . o_r for the key-stationary pass.
template <typename T, int MODE>
__global__ void __launch_bounds__(1024)
dq_kernel(const T* __restrict__ q, const T* __restrict__ keys, const T* __restrict__ vals,
          const int32_t* __restrict__ idx, const T* __restrict__ o, const float* __restrict__ lse,
          const float* __restrict__ dO, float* __restrict__ dq, float* __restrict__ delta, Dims d,
          int* err) {
  __shared__ float qs_all[32][64];
  __shared__ float ds_all[32][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tq = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int h = g * d.G + warp;
  const int t = d.q_off + tq;
  const size_t row = ((size_t)b * d.Tq + tq) * d.Hq + h;
  float* qs = qs_all[warp];
  float* dos = ds_all[warp];
  const float sl2 = d.scale * kLog2e;
  qs[lane] = to_f32(q[row * 64 + lane]) * sl2;
  qs[lane + 32] = to_f32(q[row * 64 + lane + 32]) * sl2;
  const float d0 = dO[row * 64 + lane], d1 = dO[row * 64 + lane + 32];
  dos[lane] = d0;
  dos[lane + 32] = d1;
  const float dl = warp_sum(d0 * to_f32(o[row * 64 + lane]) + d1 * to_f32(o[row * 64 + lane + 32]));
  if (lane == 0) delta[row] = dl;
  __syncwarp();
  const float lse2 = lse[row] * kLog2e;
  float a0 = 0.f, a1 = 0.f;  // dq / scale, dims lane and lane + 32
  if (lse2 != -INFINITY) {
    // key rows of this KV head: raw keys (sel, swa) or compressed keys (cmp)
    const int nrow_keys = MODE == kBwdCmp ? d.Nc : d.T;
    const size_t krow = (size_t)d.Hkv * 64;
    const T* kb = keys + (size_t)b * nrow_keys * krow + (size_t)g * 64;
    const T* vb = vals + (size_t)b * nrow_keys * krow + (size_t)g * 64;
    auto fold = [&](int s0, int s1) {
      for (int base = s0; base < s1; base += 32) {
        const int s = base + lane;
        float ds = 0.f;
        if (s < s1) {
          float qk, dv;
          dot2_64<T>(qs, dos, kb + (size_t)s * krow, vb + (size_t)s * krow, qk, dv);
          const float p = exp2f(qk - lse2);
          ds = p * (dv - dl);
        }
        const int nk = min(32, s1 - base);
        for (int i = 0; i < nk; ++i) {
          const float dsi = __shfl_sync(0xffffffffu, ds, i);
          const T* kr = kb + (size_t)(base + i) * krow;
          a0 = fmaf(dsi, to_f32(kr[lane]), a0);
          a1 = fmaf(dsi, to_f32(kr[lane + 32]), a1);
        }
      }
    };
    if (MODE == kBwdSel) {
      const int32_t* ir = idx + (((size_t)b * d.Tq + tq) * d.Hkv + g) * d.topk;
      const int cur = t / d.l;
      int prev = -1;
      for (int sidx = 0; sidx < d.topk; ++sidx) {
        const int j = ir[sidx];
        if (j == -1) continue;
        if (j < -1 || j <= prev || j > cur) {
          if (lane == 0) record_error(err, kDevBadIndex);
          continue;
        }
        prev = j;
        fold(j * d.l, min(j * d.l + d.l, t + 1));
      }
    } else if (MODE == kBwdSwa) {
      fold(max(0, t - d.window + 1), t + 1);
    } else {
      fold(0, cmp_nvis(d, t));
    }
  }
  dq[row * 64 + lane] += a0 * d.scale;
  dq[row * 64 + lane + 32] += a1 * d.scale;
}

// ---- reverse block -> query map (selection) -------------------------------------
// For each (sequence, KV group) and block j: offsets[j] .. offsets[j+1] index
// the ascending list of the queries tq that selected j.  Built without
// global atomics in three steps over chunks of kRevChunk consecutive
// queries: (1) per chunk, a shared-memory histogram of the blocks chosen;
// (2) per (sequence, group), the per-block totals, their exclusive scan
// (offsets) and each chunk's first position per block; (3) per chunk, one
// warp walks the queries in ascending order, 32 at a time, and places each
// selection at its block's running position plus its rank among the lanes
// that chose the same block.  A selection counts when it is a real,
// causal block that does not repeat or go back (the forward's rule).
constexpr int kRevChunk = kRevChunkQueries;
constexpr int kMaxUnitClasses = 4;  // work-unit sizes of 1 .. 4 tiles

__device__ __forceinline__ bool rev_valid(const int32_t* ir, int s, int cur) {
  const int j = ir[s];
  return j >= 0 && j <= cur && (s == 0 || ir[s - 1] < j);
}

__global__ void __launch_bounds__(kRevChunk)
rev_chunk_count_kernel(const int32_t* __restrict__ idx, int* __restrict__ chunk, Dims d,
                       int* err, int* __restrict__ totals) {
  extern __shared__ int hist[];  // [Nb]
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int nchunk = gridDim.x;
  for (int j = threadIdx.x; j < d.Nb; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  const int tq = c * kRevChunk + threadIdx.x;
  if (tq < d.Tq) {
    const int32_t* ir = idx + (((size_t)b * d.Tq + tq) * d.Hkv + g) * d.topk;
    const int cur = (d.q_off + tq) / d.l;
    int prev = -1;
    for (int s = 0; s < d.topk; ++s) {
      if (rev_valid(ir, s, cur)) atomicAdd(&hist[ir[s]], 1);
      if (err) {  // the forward's rule: -1 or a causal block above the last one
        const int j = ir[s];
        if (j == -1) continue;
        if (j < -1 || j <= prev || j > cur) record_error(err, kDevBadIndex);
        else prev = j;
      }
    }
  }
  __syncthreads();
  if (totals) {  // per-(sequence, group) totals only: the order inside a list is free
    int* tot = totals + ((size_t)b * d.Hkv + g) * d.Nb;
    for (int j = threadIdx.x; j < d.Nb; j += blockDim.x)
      if (hist[j]) atomicAdd(tot + j, hist[j]);
    return;
  }
  int* out = chunk + (((size_t)b * d.Hkv + g) * nchunk + c) * d.Nb;
  for (int j = threadIdx.x; j < d.Nb; j += blockDim.x) out[j] = hist[j];
}

// one CTA per (sequence, group); chunk[c][j] becomes chunk c's first list
// position for block j
__global__ void __launch_bounds__(1024)
rev_chunk_scan_kernel(int* __restrict__ chunk, int* __restrict__ offsets, Dims d, int nchunk,
                      int4* __restrict__ units, int* __restrict__ ucount, int* __restrict__ cursor,
                      int tpu, int tq, int umax) {
  extern __shared__ int tot[];  // [Nb]; with units [Nb + 1] offsets, then [kMaxUnitClasses][Nb]
  __shared__ int wsum[32];
  __shared__ int4 wsum4[32];
  __shared__ int cbase[kMaxUnitClasses];
  __shared__ int utotal;
  const int bg = blockIdx.x;
  int* cc = chunk + (size_t)bg * nchunk * d.Nb;
  // each block's counts over the chunks -> the chunks' first positions
  // within it: P lanes of a warp share a block (P a power of two, so a
  // group never straddles warps), each sums a contiguous range of chunks,
  // a shuffle scan over the group places the ranges
  int P = 1;
  while (P < 32 && P * 2 * d.Nb <= (int)blockDim.x && P < nchunk) P *= 2;
  const int sub = threadIdx.x & (P - 1);
  const int c0 = (int)((long)nchunk * sub / P), c1 = (int)((long)nchunk * (sub + 1) / P);
  for (int jb = 0; jb < d.Nb; jb += (int)blockDim.x / P) {
    const int j = jb + (int)threadIdx.x / P;
    const bool ok = j < d.Nb;
    int part = 0;
    if (ok)
      for (int c = c0; c < c1; ++c) part += cc[(size_t)c * d.Nb + j];
    int incl = part;
    for (int o = 1; o < P; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o, P);
      if (sub >= o) incl += y;
    }
    if (ok) {
      int run = incl - part;
      for (int c = c0; c < c1; ++c) {
        const int v = cc[(size_t)c * d.Nb + j];
        cc[(size_t)c * d.Nb + j] = run;
        run += v;
      }
      if (sub == P - 1) tot[j] = incl;
    }
  }
  __syncthreads();
  // exclusive scan of tot over j: each thread a contiguous range
  const int per = (d.Nb + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per, hi = min(lo + per, d.Nb);
  int sum = 0;
  for (int j = lo; j < hi; ++j) sum += tot[j];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) / 32;
    int w = lane < nw ? wsum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    wsum[lane] = wi - w;  // exclusive over warps
  }
  __syncthreads();
  int run = wsum[warp] + incl - sum;
  int* off = offsets + (size_t)bg * (d.Nb + 1);
  for (int j = lo; j < hi; ++j) {
    const int t = tot[j];
    tot[j] = run;
    off[j] = run;
    run += t;
  }
  if (threadIdx.x == blockDim.x - 1) {
    off[d.Nb] = run;
    if (units) tot[d.Nb] = run;  // with units tot holds Nb + 1 offsets
  }
  __syncthreads();
  for (int x = threadIdx.x; x < nchunk * d.Nb; x += blockDim.x) cc[x] += tot[x % d.Nb];
  if (!units) return;
  // Work units of at most tpu list entries (tpu = kseg tiles of tq entries):
  // block j's list [off[j], off[j+1]) in consecutive pieces.  The group's
  // units are written sorted by size, so that the kernel can deal them out
  // evenly: class 0 = units of kseg tiles (block order; a block's full units,
  // then its tail if that also has kseg tiles), class c = the tails of
  // kseg - c tiles (block order).  ucls[bg][c] = the class sizes.
  // tq and tpu are powers of two (shifts, not divisions); the offsets are
  // read from shared memory (tot[0 .. Nb])
  const int lq = __ffs(tq) - 1, lpu = __ffs(tpu) - 1;
  const int kseg = tpu >> lq;  // <= kMaxUnitClasses
  const int* offs = tot;
  auto block_counts = [&](int j, int4& n) {
    const int len = offs[j + 1] - offs[j];
    const int nf = len >> lpu, rem = len - (nf << lpu);
    const int tc = rem ? (rem + tq - 1) >> lq : 0;  // tail tiles, 0 = no tail
    int a[kMaxUnitClasses] = {nf + (tc == kseg ? 1 : 0), 0, 0, 0};
    if (tc > 0 && tc < kseg) a[kseg - tc] = 1;
    n = make_int4(a[0], a[1], a[2], a[3]);
  };
  int4 mine = make_int4(0, 0, 0, 0);
  for (int j = lo; j < hi; ++j) {
    int4 n;
    block_counts(j, n);
    mine.x += n.x;
    mine.y += n.y;
    mine.z += n.z;
    mine.w += n.w;
  }
  int4 incl4 = mine;
#pragma unroll
  for (int o2 = 1; o2 < 32; o2 <<= 1) {
    const int ax = __shfl_up_sync(0xffffffffu, incl4.x, o2);
    const int ay = __shfl_up_sync(0xffffffffu, incl4.y, o2);
    const int az = __shfl_up_sync(0xffffffffu, incl4.z, o2);
    const int aw = __shfl_up_sync(0xffffffffu, incl4.w, o2);
    if (lane >= o2) {
      incl4.x += ax;
      incl4.y += ay;
      incl4.z += az;
      incl4.w += aw;
    }
  }
  __syncthreads();  // wsum and tot are reused below
  if (lane == 31) wsum4[warp] = incl4;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) / 32;
    const int4 w = lane < nw ? wsum4[lane] : make_int4(0, 0, 0, 0);
    int4 wi = w;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const int ax = __shfl_up_sync(0xffffffffu, wi.x, o2);
      const int ay = __shfl_up_sync(0xffffffffu, wi.y, o2);
      const int az = __shfl_up_sync(0xffffffffu, wi.z, o2);
      const int aw = __shfl_up_sync(0xffffffffu, wi.w, o2);
      if (lane >= o2) {
        wi.x += ax;
        wi.y += ay;
        wi.z += az;
        wi.w += aw;
      }
    }
    wsum4[lane] = make_int4(wi.x - w.x, wi.y - w.y, wi.z - w.z, wi.w - w.w);  // exclusive
    if (lane == 31) {
      reinterpret_cast<int4*>(ucount)[bg] = wi;  // class sizes
      cbase[0] = 0;
      cbase[1] = wi.x;
      cbase[2] = wi.x + wi.y;
      cbase[3] = wi.x + wi.y + wi.z;
      utotal = wi.x + wi.y + wi.z + wi.w;
    }
  }
  __syncthreads();
  // pre[c][j] = the units of class c before block j
  int* pre = tot + d.Nb + 1;  // [kMaxUnitClasses][Nb]
  {
    const int4 w = wsum4[warp];
    int4 at = make_int4(w.x + incl4.x - mine.x, w.y + incl4.y - mine.y, w.z + incl4.z - mine.z,
                        w.w + incl4.w - mine.w);
    for (int j = lo; j < hi; ++j) {
      cursor[(size_t)bg * d.Nb + j] = offs[j];
      pre[j] = at.x;
      pre[d.Nb + j] = at.y;
      pre[2 * d.Nb + j] = at.z;
      pre[3 * d.Nb + j] = at.w;
      int4 n;
      block_counts(j, n);
      at.x += n.x;
      at.y += n.y;
      at.z += n.z;
      at.w += n.w;
    }
  }
  __syncthreads();
  // unit p of class c, rank r in its class, belongs to the last block j
  // with pre[c][j] <= r (a block with none shares its prefix with the next)
  int4* ub = units + (size_t)bg * umax;
  for (int p = threadIdx.x; p < utotal; p += blockDim.x) {
    const int c = p < cbase[1] ? 0 : p < cbase[2] ? 1 : p < cbase[3] ? 2 : 3;
    const int r = p - cbase[c];
    const int* pc = pre + c * d.Nb;
    int a = 0, z = d.Nb - 1;
    while (a < z) {
      const int mid = (a + z + 1) >> 1;
      if (pc[mid] <= r) a = mid;
      else z = mid - 1;
    }
    const int nf = (offs[a + 1] - offs[a]) >> lpu;
    const int k = c == 0 ? r - pc[a] : nf;  // the tail follows the full units
    const int p0 = offs[a] + (k << lpu);
    ub[p] = make_int4(a, p0, min(p0 + tpu, offs[a + 1]), 0);
  }
}

// The list fill of the forward (entries query << 6 | slot, topk <= 64) and
// of the backward (entries query): per chunk of kRevChunk queries, one
// thread per query, a block's entries in ascending query order from the
// chunk's scanned first position for that block, so the lists are the same
// on every run.  Warp w marks in bits[w][j] the lanes whose query chose
// block j (atomicOr: the result does not depend on the order of the
// updates); thread j turns the warps' counts into each warp's first
// position; a (query, slot) pair lands at pos[w][j] + the number of lower
// lanes of its warp that chose j.
constexpr int kRevWarps = kRevChunk / 32;
template <bool SLOT>
__global__ void __launch_bounds__(kRevChunk)
rev_fill_kernel(const int32_t* __restrict__ idx, const int* __restrict__ chunk,
                int* __restrict__ list, Dims d) {
  extern __shared__ int sm[];  // bits[kRevWarps][Nb], pos[kRevWarps][Nb]
  unsigned* bits = reinterpret_cast<unsigned*>(sm);
  int* pos = sm + kRevWarps * d.Nb;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int nchunk = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bg = (size_t)b * d.Hkv + g;
  for (int x = threadIdx.x; x < kRevWarps * d.Nb; x += blockDim.x) bits[x] = 0u;
  __syncthreads();
  const int tq = c * kRevChunk + threadIdx.x;
  const bool q_ok = tq < d.Tq;
  const int32_t* ir = idx + (((size_t)b * d.Tq + (q_ok ? tq : 0)) * d.Hkv + g) * d.topk;
  const int cur = (d.q_off + tq) / d.l;
  unsigned* mine = bits + warp * d.Nb;
  if (q_ok)
    for (int s = 0; s < d.topk; ++s)
      if (rev_valid(ir, s, cur)) atomicOr(&mine[ir[s]], 1u << lane);
  __syncthreads();
  const int* base = chunk + (bg * nchunk + c) * d.Nb;
  for (int j = threadIdx.x; j < d.Nb; j += blockDim.x) {
    int run = base[j];
#pragma unroll
    for (int w = 0; w < kRevWarps; ++w) {
      pos[w * d.Nb + j] = run;
      run += __popc(bits[w * d.Nb + j]);
    }
  }
  __syncthreads();
  int* lst = list + bg * (size_t)d.Tq * d.topk;
  const unsigned lt = (1u << lane) - 1u;
  const int* mpos = pos + warp * d.Nb;
  if (q_ok)
    for (int s = 0; s < d.topk; ++s)
      if (rev_valid(ir, s, cur)) {
        const int j = ir[s];
        lst[mpos[j] + __popc(mine[j] & lt)] = SLOT ? ((tq << 6) | s) : tq;
      }
}

cudaError_t launch_rev_fill(const Dims& d, bool slot, const int32_t* idx, const int* chunk,
                            int* list, int nchunk, cudaStream_t s) {
  const size_t smem = 2 * (size_t)kRevWarps * d.Nb * sizeof(int);
  auto kern = slot ? rev_fill_kernel<true> : rev_fill_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nchunk, d.Hkv, d.B), kRevChunk, smem, s>>>(idx, chunk, list, d);
  return cudaGetLastError();
}

// ---- pass 2: dK, dV, key-stationary ----------------------------------------------
// One CTA per (sequence, KV group, 64-key block); thread (key, quarter) owns
// 16 head dims of that key's dk and dv.  Query rows are streamed in batches
// of 32 through shared memory, in ascending query order.
constexpr int kKB = 64;     // keys per CTA
constexpr int kRB = 32;     // query rows per batch

template <typename T, int MODE>
__global__ void __launch_bounds__(256)
dkdv_kernel(const T* __restrict__ q, const T* __restrict__ keys, const T* __restrict__ vals,
            const float* __restrict__ lse, const float* __restrict__ delta,
            const float* __restrict__ dO, const int* __restrict__ offsets,
            const int* __restrict__ list, float* __restrict__ dk, float* __restrict__ dv,
            Dims d) {
  __shared__ float qsm[kRB][64];
  __shared__ float dosm[kRB][64];
  __shared__ float lse_s[kRB], del_s[kRB];
  __shared__ int pos_s[kRB];
  const int tid = threadIdx.x;
  const int kl = tid >> 2, qd = tid & 3;  // key in chunk, quarter of dims
  const int g = blockIdx.y, b = blockIdx.z;
  const int nrow_keys = MODE == kBwdCmp ? d.Nc : d.T;
  // selection: chunk c of selection block j (a block of l keys spans
  // ceil(l / 64) chunks); window / compression: plain 64-key chunks
  const int nsub = (d.l + kKB - 1) / kKB;
  const int j = MODE == kBwdSel ? (int)blockIdx.x / nsub : (int)blockIdx.x;
  const int csub = MODE == kBwdSel ? (int)blockIdx.x % nsub : 0;
  const int s = MODE == kBwdSel ? j * d.l + csub * kKB + kl : j * kKB + kl;  // key index
  const bool key_ok = s < nrow_keys && (MODE != kBwdSel || csub * kKB + kl < d.l);
  const size_t krow = (size_t)d.Hkv * 64;
  float kr[16], vr[16], dka[16], dva[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    kr[e] = key_ok ? to_f32(keys[((size_t)b * nrow_keys + s) * krow + g * 64 + qd * 16 + e]) : 0.f;
    vr[e] = key_ok ? to_f32(vals[((size_t)b * nrow_keys + s) * krow + g * 64 + qd * 16 + e]) : 0.f;
    dka[e] = 0.f;
    dva[e] = 0.f;
  }
  const float sl2 = d.scale * kLog2e;
  // query tokens (as query indices tq) contributing to this key block
  int n_tok = 0, tq_lo = 0;
  const int* lst = nullptr;
  if (MODE == kBwdSel) {
    const size_t bg = (size_t)b * d.Hkv + g;
    const int o0 = offsets[bg * (d.Nb + 1) + j], o1 = offsets[bg * (d.Nb + 1) + j + 1];
    n_tok = o1 - o0;
    lst = list + bg * (size_t)d.Tq * d.topk + o0;
  } else if (MODE == kBwdSwa) {
    const int t_lo = j * kKB, t_hi = min(j * kKB + kKB - 1 + d.window - 1, d.T - 1);
    tq_lo = max(0, t_lo - d.q_off);
    n_tok = max(0, t_hi - d.q_off - tq_lo + 1);
  } else {
    const int t_lo = (j * kKB) * d.dc + d.lc - 1;  // first query that sees the chunk
    tq_lo = max(0, t_lo - d.q_off);
    n_tok = max(0, d.Tq - tq_lo);
  }
  const long n_rows = (long)n_tok * d.G;
  for (long r0 = 0; r0 < n_rows; r0 += kRB) {
    const int nr = (int)min((long)kRB, n_rows - r0);
    __syncthreads();
    // load the batch: row = (token-in-list, head), token-major
    for (int e = tid; e < nr * 64; e += 256) {
      const int rr = e >> 6, c = e & 63;
      const long rix = r0 + rr;
      const int ti = (int)(rix / d.G), hh = (int)(rix % d.G);
      int tq = MODE == kBwdSel ? lst[ti] : tq_lo + ti;
      const bool tq_ok = tq >= 0 && tq < d.Tq;
      if (!tq_ok) tq = 0;
      const size_t row = ((size_t)b * d.Tq + tq) * d.Hq + g * d.G + hh;
      qsm[rr][c] = tq_ok ? to_f32(q[row * 64 + c]) : 0.f;
      dosm[rr][c] = tq_ok ? dO[row * 64 + c] : 0.f;
      if (c == 0) {
        lse_s[rr] = tq_ok ? lse[row] * kLog2e : -INFINITY;
        del_s[rr] = tq_ok ? delta[row] : 0.f;
        pos_s[rr] = d.q_off + tq;
      }
    }
    __syncthreads();
    for (int rr = 0; rr < nr; ++rr) {
      float qk = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        qk = fmaf(qsm[rr][qd * 16 + e], kr[e], qk);
        dp = fmaf(dosm[rr][qd * 16 + e], vr[e], dp);
      }
      qk += __shfl_xor_sync(0xffffffffu, qk, 1);
      qk += __shfl_xor_sync(0xffffffffu, qk, 2);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 2);
      const int t = pos_s[rr];
      bool vis;
      if (MODE == kBwdSel) vis = s <= t;
      else if (MODE == kBwdSwa) vis = s <= t && s >= t - d.window + 1;
      else vis = s * d.dc + d.lc - 1 <= t;
      vis = vis && key_ok && lse_s[rr] != -INFINITY;
      const float p = vis ? exp2f(qk * sl2 - lse_s[rr]) : 0.f;
      const float ds = p * (dp - del_s[rr]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        dva[e] = fmaf(p, dosm[rr][qd * 16 + e], dva[e]);
        dka[e] = fmaf(ds, qsm[rr][qd * 16 + e], dka[e]);
      }
    }
  }
  if (key_ok) {
    float* dkr = dk + ((size_t)b * nrow_keys + s) * krow + g * 64 + qd * 16;
    float* dvr = dv + ((size_t)b * nrow_keys + s) * krow + g * 64 + qd * 16;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      dkr[e] += dka[e] * d.scale;
      dvr[e] += dva[e];
    }
  }
}

// Mean-pool backward: compressed block c covers tokens [c dc, c dc + lc), so
// dk[t] += sum over the blocks c covering t of dkc[c] / lc (ascending c),
// same for dv; tokens that no complete block covers get nothing.
__global__ void pool_bwd_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc,
                                float* __restrict__ dk, float* __restrict__ dv, Dims d) {
  // four consecutive values a thread (16-byte loads and stores)
  const long e4 = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long row4 = (long)d.Hkv * 16;
  const long n4 = (long)d.B * d.T * row4;
  if (e4 >= n4) return;
  const long c4 = e4 % row4;
  const long tok = e4 / row4;  // b * T + t
  const int t = (int)(tok % d.T);
  const int b = (int)(tok / d.T);
  const int chi = min(t / d.dc, d.Nc - 1);                       // last block starting <= t
  const int clo = t < d.lc ? 0 : (t - d.lc) / d.dc + 1;          // first block ending after t
  if (clo > chi) return;
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  for (int jc = clo; jc <= chi; ++jc) {
    const size_t src = ((size_t)b * d.Nc + jc) * row4 + c4;
    const float4 a = reinterpret_cast<const float4*>(dkc)[src];
    const float4 v = reinterpret_cast<const float4*>(dvc)[src];
    sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
    sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
  }
  const float inv = 1.f / (float)d.lc;
  float4* pk = reinterpret_cast<float4*>(dk) + e4;
  float4* pv = reinterpret_cast<float4*>(dv) + e4;
  float4 ok = *pk, ov = *pv;
  ok.x += sk.x * inv; ok.y += sk.y * inv; ok.z += sk.z * inv; ok.w += sk.w * inv;
  ov.x += sv.x * inv; ov.y += sv.y * inv; ov.z += sv.z * inv; ov.w += sv.w * inv;
  *pk = ok;
  *pv = ov;
}

// ---- launchers ----------------------------------------------------------------------
cudaError_t launch_gate_bwd(const Dims& d, const float* gates, const void* dout,
                            const void* o_cmp, const void* o_sel, const void* o_swa,
                            float* dgates, float* dOc, float* dOs, float* dOw, cudaStream_t s,
                            void* const* h16, int* err) {
  Half3 hp{{nullptr, nullptr, nullptr}};
  if (h16)
    for (int i = 0; i < 3; ++i) hp.p[i] = (__half*)h16[i];
  const long nrows = (long)d.B * d.Tq * d.Hq;
  const unsigned blocks = (unsigned)((nrows * 8 + 255) / 256);
  if (d.dtype == 1)
    gate_bwd_kernel<bf16><<<blocks, 256, 0, s>>>(gates, (const bf16*)dout, (const bf16*)o_cmp,
                                                 (const bf16*)o_sel, (const bf16*)o_swa, dgates,
                                                 dOc, dOs, dOw, nrows, d.branch_mask, hp, err);
  else
    gate_bwd_kernel<float><<<blocks, 256, 0, s>>>(gates, (const float*)dout, (const float*)o_cmp,
                                                  (const float*)o_sel, (const float*)o_swa,
                                                  dgates, dOc, dOs, dOw, nrows, d.branch_mask, hp,
                                                  err);
  return cudaGetLastError();
}

template <typename T, int MODE>
static cudaError_t dq_t(const Dims& d, const void* q, const void* keys, const void* vals,
                        const int32_t* idx, const void* o, const float* lse, const float* dO,
                        float* dq, float* delta, int* err, cudaStream_t s) {
  dq_kernel<T, MODE><<<dim3(d.Tq, d.Hkv, d.B), d.G * 32, 0, s>>>(
      (const T*)q, (const T*)keys, (const T*)vals, idx, (const T*)o, lse, dO, dq, delta, d, err);
  return cudaGetLastError();
}

cudaError_t launch_dq(const Dims& d, int mode, const void* q, const void* keys, const void* vals,
                      const int32_t* idx, const void* o, const float* lse, const float* dO,
                      float* dq, float* delta, int* err, cudaStream_t s) {
  if (dq_tc_eligible(d, mode))
    return launch_dq_tc(d, mode, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
  if (d.dtype == 1) {
    if (mode == kBwdSel) return dq_t<bf16, kBwdSel>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
    if (mode == kBwdSwa) return dq_t<bf16, kBwdSwa>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
    return dq_t<bf16, kBwdCmp>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
  }
  if (mode == kBwdSel) return dq_t<float, kBwdSel>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
  if (mode == kBwdSwa) return dq_t<float, kBwdSwa>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
  return dq_t<float, kBwdCmp>(d, q, keys, vals, idx, o, lse, dO, dq, delta, err, s);
}

size_t revmap_chunk_ints(const Dims& d) {
  return (size_t)d.B * d.Hkv * ((d.Tq + kRevChunk - 1) / kRevChunk) * d.Nb;
}

cudaError_t launch_revmap(const Dims& d, const int32_t* idx, int* chunk, int* offsets,
                          int* list, cudaStream_t s) {
  const int nchunk = (d.Tq + kRevChunk - 1) / kRevChunk;
  if (nchunk == 0 || d.Nb == 0) return cudaSuccess;
  const size_t nb_bytes = (size_t)d.Nb * sizeof(int);
  rev_chunk_count_kernel<<<dim3(nchunk, d.Hkv, d.B), kRevChunk, nb_bytes, s>>>(idx, chunk, d,
                                                                              nullptr, nullptr);
  rev_chunk_scan_kernel<<<d.B * d.Hkv, 1024, nb_bytes, s>>>(chunk, offsets, d, nchunk, nullptr,
                                                           nullptr, nullptr, 0, 1, 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_rev_fill(d, false, idx, chunk, list, nchunk, s);
}

cudaError_t launch_revmap_units(const Dims& d, const int32_t* idx, int* chunk, int* offsets,
                                int* cursor, int* list, int4* units, int* ucount, int tpu, int tq,
                                int umax, int* err, cudaStream_t s, bool counted) {
  if (tq < 1 || (tq & (tq - 1)) || (tpu & (tpu - 1)) || tpu < tq || tpu / tq > kMaxUnitClasses)
    return cudaErrorInvalidValue;  // powers of two, at most four tiles a unit
  const int nchunk = (d.Tq + kRevChunk - 1) / kRevChunk;
  if (nchunk == 0 || d.Nb == 0) return cudaSuccess;
  const size_t nb_bytes = (size_t)d.Nb * sizeof(int);
  // per-(chunk, block) counts -> each chunk's first position per block, the
  // offsets and the work units -> the entries in ascending query order
  if (!counted)
    rev_chunk_count_kernel<<<dim3(nchunk, d.Hkv, d.B), kRevChunk, nb_bytes, s>>>(idx, chunk, d,
                                                                                err, nullptr);
  rev_chunk_scan_kernel<<<d.B * d.Hkv, 1024, (kMaxUnitClasses + 1) * nb_bytes + sizeof(int), s>>>(
      chunk, offsets, d, nchunk, units, ucount, cursor, tpu, tq, umax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_rev_fill(d, true, idx, chunk, list, nchunk, s);
}

template <typename T, int MODE>
static cudaError_t dkdv_t(const Dims& d, const void* q, const void* keys, const void* vals,
                          const float* lse, const float* delta, const float* dO,
                          const int* offsets, const int* list, float* dk, float* dv,
                          cudaStream_t s) {
  const int nkeys = MODE == kBwdCmp ? d.Nc : d.T;
  const int nblk = MODE == kBwdSel ? d.Nb * ((d.l + kKB - 1) / kKB) : (nkeys + kKB - 1) / kKB;
  if (nblk == 0) return cudaSuccess;
  dkdv_kernel<T, MODE><<<dim3(nblk, d.Hkv, d.B), 256, 0, s>>>(
      (const T*)q, (const T*)keys, (const T*)vals, lse, delta, dO, offsets, list, dk, dv, d);
  return cudaGetLastError();
}

cudaError_t launch_dkdv(const Dims& d, int mode, const void* q, const void* keys,
                        const void* vals, const float* lse, const float* delta, const float* dO,
                        void* dO16, const int* offsets, const int* list, float* dk, float* dv,
                        float* part, int* err, cudaStream_t s, bool dO16_ready) {
  if (dkdv_tc_eligible(d, mode))
    return launch_dkdv_tc(d, mode, q, keys, vals, lse, delta, dO, dO16, offsets, list, dk, dv,
                          part, err, s, dO16_ready);
  if (d.dtype == 1) {
    if (mode == kBwdSel) return dkdv_t<bf16, kBwdSel>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
    if (mode == kBwdSwa) return dkdv_t<bf16, kBwdSwa>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
    return dkdv_t<bf16, kBwdCmp>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
  }
  if (mode == kBwdSel) return dkdv_t<float, kBwdSel>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
  if (mode == kBwdSwa) return dkdv_t<float, kBwdSwa>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
  return dkdv_t<float, kBwdCmp>(d, q, keys, vals, lse, delta, dO, offsets, list, dk, dv, s);
}

cudaError_t launch_pool_bwd(const Dims& d, const float* dkc, const float* dvc, float* dk,
                            float* dv, cudaStream_t s) {
  const long n4 = d.Nc == 0 ? 0 : (long)d.B * d.T * d.Hkv * 16;
  if (n4 == 0) return cudaSuccess;
  pool_bwd_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(dkc, dvc, dk, dv, d);
  return cudaGetLastError();
}

}  // namespace nsa
