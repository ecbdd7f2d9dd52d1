// k_cmp_mlp.cu -- parametric compression (NSA's original compressor) and its
// gradient, on the sm_100a tensor cores.
//
// "DeepSeek's Native Sparse Attention", COMPRESSION: a small neural layer
// summarises each block into one key and one value; "Sparsity is Cool",
// Method and Key claims: the study swaps it for mean-pooling (its special
// case here).  The layer is one linear map over the block's l rows of 64
// values flattened in token order, weights shared by every head and block:
//   kc[b, j, g, :] = sum_{i<l} k[b, j d + i, g, :] Wk[i]      (Wk[i] = rows
//   vc[b, j, g, :] = sum_{i<l} v[b, j d + i, g, :] Wv[i]       i*64 .. i*64+63)
// Each is a GEMM whose contraction runs over the block's rows:
//   forward  D[j, n]       += A_i[j, e] W_i[e, n]    M = 128 blocks, N = 64,
//            K = 64 per token offset i; A_i's rows are the tokens j d + i,
//            gathered by cp.async straight from k / v.
//   dW       dW[(i, e), n] += X[q, (i, e)] dXc[q, n]  M = 128 rows (i, e) of
//            two offsets, N = 64, K = every (sequence, block, group) q, split
//            over CTAs and summed in a fixed order.
//   dA       dA[q, (i, e)]  = dXc[q, n] W[(i, e), n]  M = 128 blocks q, N = 64
//            per offset i, K = 64.
// The raw rows' gradient sums dA over the blocks covering each token in block
// order (deterministic, no atomics).  The upstream dXc (fp32) enters the MMAs
// as a bf16 pair hi + lo, so it is carried to about 16 bits.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace nsa {
namespace {

using namespace sm100;

constexpr int kMlpThreads = 160;  // warps 0-3 operands + epilogue, warp 4 MMA + TMEM
constexpr int kMlpStages = 3;
constexpr uint32_t kRowTile = 128 * 64 * 2;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kW64 = 64 * 64 * 2;       // 64 rows x 64 bf16

struct MlpBars {
  uint64_t full[kMlpStages];
  uint64_t empty[kMlpStages];
  uint64_t fin;
  uint64_t dfull[2];  // dA: the offset's D buffer is in TMEM
  uint64_t dfree[2];  // dA: the epilogue threads have read it
};
constexpr uint32_t kBarBytes = ((sizeof(MlpBars) + 15) / 16) * 16;

// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz_off(int r, int c) {
  return (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u + ((uint32_t)(c ^ (r & 7)) << 4);
}

// 8 fp32 -> bf16 hi and lo (f - hi), packed
__device__ __forceinline__ void split8(const float* src, uint32_t h[4], uint32_t lo[4]) {
  const float4 p0 = *reinterpret_cast<const float4*>(src);
  const float4 p1 = *reinterpret_cast<const float4*>(src + 4);
  const float f[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float h0 = __bfloat162float(__float2bfloat16_rn(f[2 * e]));
    const float h1 = __bfloat162float(__float2bfloat16_rn(f[2 * e + 1]));
    h[e] = pack_bf16(h0, h1);
    lo[e] = pack_bf16(f[2 * e] - h0, f[2 * e + 1] - h1);
  }
}

// dkc, dvc (fp32 [nq, 64]) -> bf16 pairs hi[2][nq][64], lo[2][nq][64] (keys, values), the
// operands of the dW and dA GEMMs; 8 values a thread
__global__ void cmp_mlp_split_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc,
                                     bf16* __restrict__ hi, bf16* __restrict__ lo, long n8) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * n8) return;
  const int which = (int)(e / n8);
  const long o = e - which * n8;
  uint32_t h[4], l[4];
  split8((which ? dvc : dkc) + o * 8, h, l);
  reinterpret_cast<uint4*>(hi)[e] = make_uint4(h[0], h[1], h[2], h[3]);
  reinterpret_cast<uint4*>(lo)[e] = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void setup(MlpBars* bars, volatile int* abort_flag) {
  for (int s = 0; s < kMlpStages; ++s) {
    mbar_init(&bars->full[s], 128);
    mbar_init(&bars->empty[s], 1);
  }
  mbar_init(&bars->fin, 1);
  for (int s = 0; s < 2; ++s) {
    mbar_init(&bars->dfull[s], 1);
    mbar_init(&bars->dfree[s], 128);
  }
  fence_barrier_init();
  fence_proxy_async_smem();
  *abort_flag = 0;
}

// this thread's TMEM row (lane 32 w + lane) as 64 fp32 columns from `col`
__device__ __forceinline__ void load_row64(uint32_t tmem, int warp, uint32_t col, float a[64]) {
  const uint32_t at = tmem + ((uint32_t)(warp * 32) << 16) + col;
  tmem_ld32(at, a);
  tmem_ld32(at + 32u, a + 32);
  tmem_wait_ld();
}

// ---- forward: kc or vc of 128 compressed blocks of one (sequence, group) -------------
// Stage u (token offset u): A [128 blocks x 64] = rows j d + u, K-major; W[u] [64 e x 64 n]
// read MN-major (n contiguous).  D: TMEM [0, 64).  With S > 1 CTAs per tile (too few
// tiles to fill the GPU), CTA z takes the offsets [z L / S, (z + 1) L / S) and writes
// its fp32 partial sum for cmp_mlp_fwd_reduce_kernel to add in order.
constexpr uint32_t MF_STAGE = kRowTile + kW64;
constexpr uint32_t MF_OFF_BAR = kMlpStages * MF_STAGE;
constexpr uint32_t MF_SMEM = MF_OFF_BAR + kBarBytes + 16;

__global__ void __launch_bounds__(kMlpThreads, 1)
cmp_mlp_fwd_kernel(const bf16* __restrict__ k, const bf16* __restrict__ v,
                   const bf16* __restrict__ wk, const bf16* __restrict__ wv, bf16* __restrict__ kc,
                   bf16* __restrict__ vc, float* __restrict__ part, int S, Dims d, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  MlpBars* bars = (MlpBars*)(smem + MF_OFF_BAR);
  uint32_t* tmem_slot = (uint32_t*)(smem + MF_OFF_BAR + kBarBytes);
  volatile int* abort_flag = (volatile int*)(smem + MF_OFF_BAR + kBarBytes + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int j0 = blockIdx.x * 128, g = blockIdx.y;
  const int z = (int)blockIdx.z % S, bw = (int)blockIdx.z / S;
  const int b = bw >> 1, which = bw & 1;  // 0 keys, 1 values
  const bf16* x = which ? v : k;
  const bf16* w = which ? wv : wk;
  const int u0 = (int)(((long)d.lc * z) / S);
  const int L = (int)(((long)d.lc * (z + 1)) / S) - u0;  // this CTA's offsets u0 + [0, L)
  if (tid == 0) setup(bars, abort_flag);
  if (warp == 4) tmem_alloc(tmem_slot, 64);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // lane copies chunk lane % 8 of rows 32 warp + 4 q8 + lane / 8
    const int ch = lane & 7;
    bool ok = true;
    for (int u = 0; u < L; ++u) {
      const int st = u % kMlpStages;
      if (u >= kMlpStages &&
          !wait_bar_warp(&bars->empty[st], ((u - kMlpStages) / kMlpStages) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      const uint32_t a = smem_u32(smem + st * MF_STAGE), aw = a + kRowTile;
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        const int r = 32 * warp + 4 * q8 + (lane >> 3);
        const int j = j0 + r;
        const bool present = j < d.Nc;
        const size_t row =
            ((size_t)b * d.T + (present ? (size_t)j * d.dc + u0 + u : 0)) * d.Hkv + g;
        cp_async16(a + swz_off(r, ch), x + row * 64 + 8 * ch, present ? 16u : 0u);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {  // W[u]: 64 rows x 8 chunks
        const int idx = tid + 128 * m, e = idx >> 3, c = idx & 7;
        cp_async16(aw + swz_off(e, c), w + ((size_t)(u0 + u) * 64 + e) * 64 + 8 * c, 16u);
      }
      cp_async_commit();
      if (u >= 1) {
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->full[(u - 1) % kMlpStages]);
      }
    }
    cp_async_wait<0>();
    if (ok && L > 0) {
      fence_proxy_async_smem();
      mbar_arrive(&bars->full[(L - 1) % kMlpStages]);
    }
    // epilogue: thread r stores compressed block j0 + r
    const bool have = ok && wait_bar_warp(&bars->fin, 0, abort_flag, err);
    if (have) {
      tc_fence_after();
      float a[64];
      load_row64(tmem, warp, 0u, a);
      const int j = j0 + tid;
      const size_t row = ((size_t)b * d.Nc + j) * d.Hkv + g;
      if (j < d.Nc && S > 1) {
        float4* dst = reinterpret_cast<float4*>(
            part + (((size_t)z * 2 + which) * d.B * d.Nc * d.Hkv + row) * 64);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          dst[c] = make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
      } else if (j < d.Nc) {
        bf16* dst = (which ? vc : kc) + row * 64;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 o;
          o.x = pack_bf16(a[8 * c], a[8 * c + 1]);
          o.y = pack_bf16(a[8 * c + 2], a[8 * c + 3]);
          o.z = pack_bf16(a[8 * c + 4], a[8 * c + 5]);
          o.w = pack_bf16(a[8 * c + 6], a[8 * c + 7]);
          *reinterpret_cast<uint4*>(dst + 8 * c) = o;
        }
      }
    }
    tc_fence_before();
  } else if (lane == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);  // A K-major, B MN-major
    for (int u = 0; u < L; ++u) {
      const int st = u % kMlpStages;
      if (!wait_bar(&bars->full[st], (u / kMlpStages) & 1, abort_flag, err)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + st * MF_STAGE), aw = a + kRowTile;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem, desc_sw128(a + kk * 32, 16), desc_sw128(aw + kk * 2048, 8192), idesc,
                 (u > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars->empty[st]);
    }
    mma_commit(&bars->fin);
    drain_bar(&bars->fin, 0);
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// kc / vc = bf16(sum of the S partial sums in order z = 0, 1, ...), 4 values a thread
__global__ void cmp_mlp_fwd_reduce_kernel(const float* __restrict__ part, bf16* __restrict__ kc,
                                          bf16* __restrict__ vc, int S, long n4) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * n4) return;
  const int which = (int)(e / n4);
  const long o = e - which * n4;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int z = 0; z < S; ++z) {
    const float4 p = reinterpret_cast<const float4*>(part)[((long)z * 2 + which) * n4 + o];
    a.x += p.x;
    a.y += p.y;
    a.z += p.z;
    a.w += p.w;
  }
  uint2 h;
  h.x = pack_bf16(a.x, a.y);
  h.y = pack_bf16(a.z, a.w);
  reinterpret_cast<uint2*>(which ? vc : kc)[o] = h;
}

// ---- dW: rows (i, e) of token offsets i = 2m, 2m + 1 against a range of blocks q --------
// Stage: X [64 K rows q][two 64-wide atoms: offsets 2m, 2m + 1] read MN-major (the second
// atom 8 KB after the first), dXc hi, lo [64 q][64 n] read MN-major.  D: TMEM [0, 64).
// Every operand arrives by cp.async, two stages ahead of the MMAs.
// CTA z of S takes the chunks u = z, z + S, ...; with S > 1 it writes its partial sum
// to part[z] for a fixed-order reduction.
constexpr uint32_t MW_STAGE = 4 * kW64;
constexpr uint32_t MW_OFF_BAR = kMlpStages * MW_STAGE;
constexpr uint32_t MW_SMEM = MW_OFF_BAR + kBarBytes + 16;

__global__ void __launch_bounds__(kMlpThreads, 1)
cmp_mlp_dw_kernel(const bf16* __restrict__ xk, const bf16* __restrict__ xv,
                  const bf16* __restrict__ ghi, const bf16* __restrict__ glo,
                  float* __restrict__ dwk, float* __restrict__ dwv, float* __restrict__ part,
                  Dims d, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  MlpBars* bars = (MlpBars*)(smem + MW_OFF_BAR);
  uint32_t* tmem_slot = (uint32_t*)(smem + MW_OFF_BAR + kBarBytes);
  volatile int* abort_flag = (volatile int*)(smem + MW_OFF_BAR + kBarBytes + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int m = blockIdx.x, which = blockIdx.y, z = blockIdx.z, S = gridDim.z;
  const bf16* x = which ? xv : xk;
  const long nq = (long)d.B * d.Nc * d.Hkv;  // contraction length
  const bf16* gh = ghi + which * nq * 64;
  const bf16* gl = glo + which * nq * 64;
  const int nchunk = (int)((nq + 63) / 64);
  const int mine = nchunk > z ? (nchunk - z + S - 1) / S : 0;
  if (tid == 0) setup(bars, abort_flag);
  if (warp == 4) tmem_alloc(tmem_slot, 64);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    bool ok = true;
    auto issue = [&](int it) {  // chunk it's operands into its stage, one cp.async group
      const int st = it % kMlpStages;
      const long u = z + (long)it * S;
      const uint32_t a0 = smem_u32(smem + st * MW_STAGE), a1 = a0 + kW64;
      const uint32_t bh = a1 + kW64, bl = bh + kW64;
      // X: 64 K rows x 2 atoms x 8 chunks = 1024 chunks, 8 per thread
#pragma unroll
      for (int t8 = 0; t8 < 8; ++t8) {
        const int idx = tid + 128 * t8;
        const int atom = idx >> 9, r = (idx >> 3) & 63, c = idx & 7;
        const long q = u * 64 + r;
        const int i = 2 * m + atom;
        const bool present = q < nq && i < d.lc;
        size_t row = 0;
        if (present) {  // q = (b Nc + j) Hkv + g
          const int g = (int)(q % d.Hkv);
          const long bj = q / d.Hkv;
          const int j = (int)(bj % d.Nc), b = (int)(bj / d.Nc);
          row = ((size_t)b * d.T + (size_t)j * d.dc + i) * d.Hkv + g;
        }
        cp_async16((atom ? a1 : a0) + swz_off(r, c), x + row * 64 + 8 * c, present ? 16u : 0u);
      }
      // dXc hi, lo rows: 64 rows x 8 chunks each, 4 + 4 per thread
#pragma unroll
      for (int t4 = 0; t4 < 4; ++t4) {
        const int idx = tid + 128 * t4, r = idx >> 3, c = idx & 7;
        const long q = u * 64 + r;
        const bool present = q < nq;
        const size_t off = (size_t)(present ? q : 0) * 64 + 8 * c;
        cp_async16(bh + swz_off(r, c), gh + off, present ? 16u : 0u);
        cp_async16(bl + swz_off(r, c), gl + off, present ? 16u : 0u);
      }
      cp_async_commit();
    };
    // chunks 0 and 1 in flight before the loop; chunk it + 2 issued once chunk it landed
    for (int it = 0; it < 2 && it < mine; ++it) issue(it);
    for (int it = 0; it < mine; ++it) {
      if (it + 1 < mine) cp_async_wait<1>();
      else cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&bars->full[it % kMlpStages]);
      const int nx = it + 2;
      if (nx < mine) {
        if (nx >= kMlpStages &&
            !wait_bar_warp(&bars->empty[nx % kMlpStages], ((nx - kMlpStages) / kMlpStages) & 1,
                           abort_flag, err)) {
          ok = false;
          break;
        }
        issue(nx);
      }
    }
    cp_async_wait<0>();  // no copy outlives the CTA
    // epilogue: thread r holds row (i, e) = (2m + r / 64, r % 64) of dW
    const bool have = ok && mine > 0 && wait_bar_warp(&bars->fin, 0, abort_flag, err);
    const int i = 2 * m + (tid >> 6), e = tid & 63;
    float a[64];
    if (have) {
      tc_fence_after();
      load_row64(tmem, warp, 0u, a);
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) a[c] = 0.f;
    }
    tc_fence_before();
    if (i < d.lc) {
      const size_t wrow = ((size_t)i * 64 + e) * 64;
      float* dst = S > 1 ? part + ((size_t)(z * 2 + which) * d.lc * 64) * 64 + wrow
                         : (which ? dwv : dwk) + wrow;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        reinterpret_cast<float4*>(dst)[c] =
            make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
    }
  } else if (lane == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 64, true, true);  // A, B MN-major
    for (int it = 0; it < mine; ++it) {
      const int st = it % kMlpStages;
      if (!wait_bar(&bars->full[st], (it / kMlpStages) & 1, abort_flag, err)) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + st * MW_STAGE);
      const uint32_t bh = a0 + 2 * kW64, bl = bh + kW64;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // K = 64 blocks, 16 at a time
        mma_bf16(tmem, desc_sw128(a0 + kk * 2048, kW64), desc_sw128(bh + kk * 2048, 8192), idesc,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_bf16(tmem, desc_sw128(a0 + kk * 2048, kW64), desc_sw128(bl + kk * 2048, 8192), idesc,
                 1u);
      }
      mma_commit(&bars->empty[st]);
    }
    mma_commit(&bars->fin);
    drain_bar(&bars->fin, 0);
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// dW = sum over the S partial sums in order z = 0, 1, ...
__global__ void cmp_mlp_dw_reduce_kernel(const float* __restrict__ part, float* __restrict__ dwk,
                                         float* __restrict__ dwv, int S, long n) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * n) return;
  const int which = (int)(e / n);
  const long o = e % n;
  float s = 0.f;
  for (int z = 0; z < S; ++z) s += part[((size_t)z * 2 + which) * n + o];
  (which ? dwv : dwk)[o] = s;
}

// ---- dA: per 128 blocks q and each offset i, dA_i = dXc W_i^T into a scratch ------------
// A: dXc hi, lo [128 q][64 n] K-major, staged once; B stage: W_i [64 e][64 n] K-major.
// D_i: TMEM [64 (i & 1), + 64), double-buffered so offset i's epilogue overlaps i + 1's MMA.
// CTA z of gridDim.z takes the offsets [z L / Z, (z + 1) L / Z) (outputs do not overlap).
constexpr uint32_t MA_OFF_W = 2 * kRowTile;
constexpr uint32_t MA_OFF_BAR = MA_OFF_W + kMlpStages * kW64;
constexpr uint32_t MA_SMEM = MA_OFF_BAR + kBarBytes + 16;

__global__ void __launch_bounds__(kMlpThreads, 1)
cmp_mlp_da_kernel(const bf16* __restrict__ ghi, const bf16* __restrict__ glo,
                  const bf16* __restrict__ wk, const bf16* __restrict__ wv,
                  float* __restrict__ dak, float* __restrict__ dav, Dims d, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  MlpBars* bars = (MlpBars*)(smem + MA_OFF_BAR);
  uint32_t* tmem_slot = (uint32_t*)(smem + MA_OFF_BAR + kBarBytes);
  volatile int* abort_flag = (volatile int*)(smem + MA_OFF_BAR + kBarBytes + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int which = blockIdx.y;
  const bf16* w = which ? wv : wk;
  float* da = which ? dav : dak;
  const long nq = (long)d.B * d.Nc * d.Hkv;
  const bf16* gh = ghi + which * nq * 64;
  const bf16* gl = glo + which * nq * 64;
  const long q = (long)blockIdx.x * 128 + tid;  // this thread's row (warps 0-3)
  const int Z = (int)gridDim.z, z = (int)blockIdx.z;
  const int u0 = (int)(((long)d.lc * z) / Z);
  const int L = (int)(((long)d.lc * (z + 1)) / Z) - u0;  // this CTA's offsets u0 + [0, L)
  if (tid == 0) setup(bars, abort_flag);
  if (warp == 4) tmem_alloc(tmem_slot, 128);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    const uint32_t ah = smem_u32(smem), al = ah + kRowTile;
    // A (once, with W_0's group): row r = dXc[q] as the bf16 pair, 8 + 8 chunks per thread
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const bool present = q < nq;
      const size_t off = (size_t)(present ? q : 0) * 64 + 8 * c;
      cp_async16(ah + swz_off(tid, c), gh + off, present ? 16u : 0u);
      cp_async16(al + swz_off(tid, c), gl + off, present ? 16u : 0u);
    }
    auto issue = [&](int u) {  // W of offset u into its stage, one cp.async group
      const uint32_t wb = smem_u32(smem + MA_OFF_W + (u % kMlpStages) * kW64);
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        const int idx = tid + 128 * m4, e = idx >> 3, c = idx & 7;
        cp_async16(wb + swz_off(e, c), w + ((size_t)(u0 + u) * 64 + e) * 64 + 8 * c, 16u);
      }
      cp_async_commit();
    };
    for (int u = 0; u < 2 && u < L; ++u) issue(u);
    // offset u's stage is published once it landed; the epilogue of offset u - 1 follows
    for (int u = 0; u <= L; ++u) {
      if (u < L) {
        if (u + 1 < L) cp_async_wait<1>();
        else cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->full[u % kMlpStages]);
        const int nx = u + 2;
        if (nx < L) {
          if (nx >= kMlpStages &&
              !wait_bar_warp(&bars->empty[nx % kMlpStages], ((nx - kMlpStages) / kMlpStages) & 1,
                             abort_flag, err))
            break;
          issue(nx);
        }
      }
      if (u >= 1) {
        const int pu = u - 1, bu = pu & 1;
        if (!wait_bar_warp(&bars->dfull[bu], (pu >> 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        float a[64];
        load_row64(tmem, warp, 64u * bu, a);
        tc_fence_before();
        mbar_arrive(&bars->dfree[bu]);
        if (q < nq) {
          float4* dst = reinterpret_cast<float4*>(da + ((size_t)q * d.lc + u0 + pu) * 64);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
        }
      }
    }
    cp_async_wait<0>();  // no copy outlives the CTA
  } else if (lane == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);  // A, B K-major
    const uint32_t ah = smem_u32(smem), al = ah + kRowTile;
    for (int u = 0; u < L; ++u) {
      const int st = u % kMlpStages, bu = u & 1;
      if (!wait_bar(&bars->full[st], (u / kMlpStages) & 1, abort_flag, err)) break;
      // D buffer bu last held offset u - 2, which the epilogue must have read
      if (u >= 2 && !wait_bar(&bars->dfree[bu], ((u - 2) >> 1) & 1, abort_flag, err)) break;
      tc_fence_after();
      const uint32_t wb = smem_u32(smem + MA_OFF_W + st * kW64);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // K = 64 n, 16 at a time
        mma_bf16(tmem + 64u * bu, desc_sw128(ah + kk * 32, 16), desc_sw128(wb + kk * 32, 16),
                 idesc, kk > 0 ? 1u : 0u);
        mma_bf16(tmem + 64u * bu, desc_sw128(al + kk * 32, 16), desc_sw128(wb + kk * 32, 16),
                 idesc, 1u);
      }
      mma_commit(&bars->empty[st]);
      mma_commit(&bars->dfull[bu]);
    }
    mma_commit(&bars->fin);
    drain_bar(&bars->fin, 0);
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// dx[b, t, g, :] += sum over the blocks j covering t, ascending, of
// dA[(b Nc + j) Hkv + g, t - j d, :]  (4 values a thread)
__global__ void cmp_mlp_gather_kernel(const float* __restrict__ dak, const float* __restrict__ dav,
                                      float* __restrict__ dk, float* __restrict__ dv, Dims d) {
  const long e4 = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long n4 = (long)d.B * d.T * d.Hkv * 16;
  if (e4 >= n4) return;
  const int c4 = (int)(e4 & 15), g = (int)((e4 >> 4) % d.Hkv);
  const long tok = (e4 >> 4) / d.Hkv;
  const int t = (int)(tok % d.T), b = (int)(tok / d.T);
  const int chi = min(t / d.dc, d.Nc - 1);
  const int clo = t < d.lc ? 0 : (t - d.lc) / d.dc + 1;
  if (clo > chi) return;
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  for (int j = clo; j <= chi; ++j) {
    const size_t src = ((((size_t)b * d.Nc + j) * d.Hkv + g) * d.lc + (t - j * d.dc)) * 16 + c4;
    const float4 a = reinterpret_cast<const float4*>(dak)[src];
    const float4 v = reinterpret_cast<const float4*>(dav)[src];
    sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
    sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
  }
  float4* pk = reinterpret_cast<float4*>(dk) + e4;
  float4* pv = reinterpret_cast<float4*>(dv) + e4;
  float4 ok = *pk, ov = *pv;
  ok.x += sk.x; ok.y += sk.y; ok.z += sk.z; ok.w += sk.w;
  ov.x += sv.x; ov.y += sv.y; ov.z += sv.z; ov.w += sv.w;
  *pk = ok;
  *pv = ov;
}

// CTAs per output tile when the tiles alone would leave SMs idle: about `ctas`
// CTAs in all, at most one per unit of the split dimension
int split_for(long tiles, long units, long ctas) {
  long s = ctas / (tiles > 0 ? tiles : 1);
  if (s > units) s = units;
  return s < 1 ? 1 : (int)s;
}
// the forward's fp32 partial sums cost traffic and every dA CTA stages its
// dkc tile: one CTA per SM; dW splits for two CTAs per SM (measured: dW
// 26 -> 18 us at the 340M shape, dA 17 -> 18 us, so dA stays at one)
int fwd_splits(const Dims& d) {
  return split_for((long)((d.Nc + 127) / 128) * d.Hkv * 2 * d.B, d.lc, 148);
}
int da_splits(const Dims& d) {
  return split_for(((long)d.B * d.Nc * d.Hkv + 127) / 128 * 2, d.lc, 148);
}
int dw_splits(const Dims& d) {
  const long nq = (long)d.B * d.Nc * d.Hkv;
  return split_for(((long)d.lc + 1) / 2 * 2, (nq + 63) / 64, 296);
}

}  // namespace

bool cmp_mlp_eligible(const Dims& d) { return d.dtype == 1 && d.D == 64; }

size_t cmp_mlp_fwd_ws_bytes(const Dims& d) {
  const int S = fwd_splits(d);
  return S > 1 ? (size_t)S * 2 * d.B * d.Nc * d.Hkv * 64 * sizeof(float) : 0;
}

// backward workspace: dA scratch [2][nq][l][64] fp32, the dW partial sums, the
// upstream gradient's bf16 pairs hi, lo [2][nq][64] each (each part 256-byte aligned)
struct BwdWs {
  size_t da, part, hi, lo, total;
};
BwdWs bwd_ws(const Dims& d) {
  const size_t nq = (size_t)d.B * d.Nc * d.Hkv;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  BwdWs w{};
  w.da = 0;
  w.part = al(2 * nq * d.lc * 64 * sizeof(float));
  const int S = dw_splits(d);
  w.hi = w.part + al(S > 1 ? (size_t)S * 2 * d.lc * 64 * 64 * sizeof(float) : 0);
  w.lo = w.hi + al(2 * nq * 64 * sizeof(bf16));
  w.total = w.lo + al(2 * nq * 64 * sizeof(bf16));
  return w;
}

size_t cmp_mlp_bwd_ws_bytes(const Dims& d) { return bwd_ws(d).total; }

cudaError_t launch_cmp_mlp_fwd(const Dims& d, const void* k, const void* v, const void* wk,
                               const void* wv, void* kc, void* vc, void* ws, int* err,
                               cudaStream_t s) {
  if (d.Nc == 0) return cudaSuccess;
  const int smem = (int)(MF_SMEM + 1024);
  cudaError_t e =
      cudaFuncSetAttribute(cmp_mlp_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int S = fwd_splits(d);
  cmp_mlp_fwd_kernel<<<dim3((d.Nc + 127) / 128, d.Hkv, 2 * d.B * S), kMlpThreads, smem, s>>>(
      (const bf16*)k, (const bf16*)v, (const bf16*)wk, (const bf16*)wv, (bf16*)kc, (bf16*)vc,
      (float*)ws, S, d, err);
  e = cudaGetLastError();
  if (e != cudaSuccess || S == 1) return e;
  const long n4 = (long)d.B * d.Nc * d.Hkv * 16;
  cmp_mlp_fwd_reduce_kernel<<<(unsigned)((2 * n4 + 255) / 256), 256, 0, s>>>(
      (const float*)ws, (bf16*)kc, (bf16*)vc, S, n4);
  return cudaGetLastError();
}

cudaError_t launch_cmp_mlp_bwd(const Dims& d, const void* k, const void* v, const void* wk,
                               const void* wv, const float* dkc, const float* dvc, float* dk,
                               float* dv, float* dwk, float* dwv, void* ws, int* err,
                               cudaStream_t s) {
  const size_t wbytes = (size_t)d.lc * 64 * 64 * sizeof(float);
  if (d.Nc == 0) {
    cudaError_t e = cudaMemsetAsync(dwk, 0, wbytes, s);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(dwv, 0, wbytes, s);
  }
  const int smw = (int)(MW_SMEM + 1024), sma = (int)(MA_SMEM + 1024);
  cudaError_t e =
      cudaFuncSetAttribute(cmp_mlp_dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smw);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(cmp_mlp_da_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sma);
  if (e != cudaSuccess) return e;
  const long nq = (long)d.B * d.Nc * d.Hkv;
  const BwdWs L = bwd_ws(d);
  float* dak = (float*)((char*)ws + L.da);
  float* dav = dak + (size_t)nq * d.lc * 64;
  float* part = (float*)((char*)ws + L.part);
  bf16* ghi = (bf16*)((char*)ws + L.hi);
  bf16* glo = (bf16*)((char*)ws + L.lo);
  const long n8 = nq * 8;
  cmp_mlp_split_kernel<<<(unsigned)((2 * n8 + 255) / 256), 256, 0, s>>>(dkc, dvc, ghi, glo, n8);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int S = dw_splits(d);
  cmp_mlp_dw_kernel<<<dim3((d.lc + 1) / 2, 2, S), kMlpThreads, smw, s>>>(
      (const bf16*)k, (const bf16*)v, ghi, glo, dwk, dwv, part, d, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (S > 1) {
    const long n = (long)d.lc * 64 * 64;
    cmp_mlp_dw_reduce_kernel<<<(unsigned)((2 * n + 255) / 256), 256, 0, s>>>(part, dwk, dwv, S,
                                                                             n);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cmp_mlp_da_kernel<<<dim3((unsigned)((nq + 127) / 128), 2, da_splits(d)), kMlpThreads, sma, s>>>(
      ghi, glo, (const bf16*)wk, (const bf16*)wv, dak, dav, d, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long n4 = (long)d.B * d.T * d.Hkv * 16;
  cmp_mlp_gather_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(dak, dav, dk, dv, d);
  return cudaGetLastError();
}

}  // namespace nsa
