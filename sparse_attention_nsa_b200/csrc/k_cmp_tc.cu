// k_cmp_tc.cu -- compression branch and block-importance scores on the
// sm_100a tensor cores (tcgen05 + TMEM, TMA-staged compressed blocks).
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work?: COMPRESSION attends to one summary key/value per block; SELECTION
// ranks blocks by reusing the compression attention scores.  The score of
// block j for KV group g is the compression softmax probability summed over
// the G heads of the group, so it needs the final (normalised)
// probabilities of every head: the kernel makes two passes over the
// compressed keys of its 128 rows (128/G tokens x the G heads of one group):
//   pass 1  S = Q Kc^T chunk by chunk (64 compressed blocks per chunk),
//           running row max and sum of exponentials;
//   pass 2  S again (with at most two chunks, re-read from TMEM rather than
//           recomputed), P = exp(S - m) / l exactly normalised, the G heads of
//           each token summed with warp shuffles into the block scores, and
//           (unless only scores are wanted) P in bf16 through swizzled smem
//           into O += P Vc, accumulated directly in TMEM.
// A block is visible to query t once complete: j*l + l - 1 <= t.
// Warp roles as in the attention kernel: warps 0-3 one row per thread,
// warp 4 MMA issue / TMEM owner, warp 5 TMA producer.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace nsa {

cudaError_t launch_cmp_scores_simt(const Dims& d, const void* q, const void* kc,
                                   const void* vc, void* o_cmp, float* lse_cmp,
                                   float* score, cudaStream_t s);

namespace {

using namespace sm100;

constexpr int kRows = 128;
constexpr int kChunk = 64;  // compressed blocks per chunk
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = kChunk * 64 * 2;
constexpr uint32_t kQBytes = kRows * 64 * 2;
constexpr uint32_t kPBytes = kRows * kChunk * 2;

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + kQBytes;
constexpr uint32_t OFF_P = OFF_KV + kStages * 2 * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_P + 2 * kPBytes;

struct Bars {
  uint64_t q;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s[2];
  uint64_t sfree[2];
  uint64_t p[2];
  uint64_t pfree[2];
  uint64_t odone;
};
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr uint32_t kSmemBytes = OFF_MISC + 16 + 1024;

// One reduce-scatter step over v[0, 2H): a lane with `upper` set keeps
// columns [H, 2H), its partner (lane ^ off) the lower ones; each adds the
// partner's copy of the half it keeps, leaving it in v[0, H).
template <int H>
__device__ __forceinline__ void reduce_half(float* v, int upper, int off) {
#pragma unroll
  for (int c = 0; c < H; ++c) {
    const float send = upper ? v[c] : v[c + H];
    const float keep = upper ? v[c + H] : v[c];
    v[c] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

template <bool WITH_O>
__global__ void __launch_bounds__(kThreads, 2)
cmp_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
              const __grid_constant__ CUtensorMap tm_vc, bf16* __restrict__ o_cmp,
              float* __restrict__ lse, float* __restrict__ score, Dims d, int* err, bool vec4) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  uint32_t* tmem_slot = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int TQ = kRows / d.G;
  const int tile = gridDim.x - 1 - blockIdx.x;
  const int t0 = tile * TQ;
  const int g = blockIdx.y, b = blockIdx.z;
  const int nvalid = min(TQ, d.Tq - t0);
  const int pos0 = d.q_off + t0;
  const int nvis_max = nvalid > 0 ? cmp_nvis(d, pos0 + nvalid - 1) : 0;  // of the tile's last token
  const int n = (nvis_max + kChunk - 1) / kChunk;
  // with at most two chunks both S tiles stay in TMEM: pass 2 re-reads them
  // instead of recomputing, and each chunk's Kc and Vc are loaded once
  const bool res = n <= 2;
  const int nload = res ? n : 2 * n;

  if (tid == 0) {
    mbar_init(&bars->q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s[i], 1);
      mbar_init(&bars->sfree[i], 128);
      mbar_init(&bars->p[i], 128);
      mbar_init(&bars->pfree[i], 1);
    }
    mbar_init(&bars->odone, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    *abort_flag = 0;
  }
  if (warp == 4) tmem_alloc(tmem_slot, 256);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 5) {
    if (lane == 0) {  // ---- TMA producer: Q, pass-1 Kc chunks, pass-2 Kc(+Vc) chunks
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kc);
      mbar_expect_tx(&bars->q, kQBytes);
      tma_load_3d(smem + OFF_Q, &tm_q, &bars->q, 0, g * d.G, b * d.Tq + t0);
      int issued = 0;
      for (int u = 0; u < nload; ++u) {
        const int st = u % kStages;
        if (u >= kStages && !wait_bar(&bars->empty[st], ((u / kStages) & 1) ^ 1, abort_flag, err))
          break;
        const int i = u < n ? u : u - n;
        const bool with_v = WITH_O && (res || u >= n);
        uint8_t* kv = smem + OFF_KV + st * 2 * kTileBytes;
        const int row = b * d.Nc + i * kChunk;
        mbar_expect_tx(&bars->full[st], with_v ? 2 * kTileBytes : kTileBytes);
        tma_load_3d(kv, &tm_kc, &bars->full[st], 0, g, row);
        if (with_v) tma_load_3d(kv + kTileBytes, &tm_vc, &bars->full[st], 0, g, row);
        issued = u + 1;
      }
      if (*abort_flag) {
        drain_bar(&bars->q, 0);
        for (int u = max(0, issued - kStages); u < issued; ++u)
          drain_bar(&bars->full[u % kStages], (u / kStages) & 1);
      }
    }
  } else if (warp == 4) {
    if (lane == 0) {  // ---- MMA issue
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kChunk, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(kRows, 64, false, true);
      const uint32_t q_addr = smem_u32(smem + OFF_Q);
      bool ok = wait_bar(&bars->q, 0, abort_flag, err);
      auto do_pv = [&](int i) -> bool {
        if (!wait_bar(&bars->p[i & 1], (i >> 1) & 1, abort_flag, err)) return false;
        tc_fence_after();
        const int st = (res ? i : n + i) % kStages;
        const uint32_t v_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes + kTileBytes);
        const uint32_t p_addr = smem_u32(smem + OFF_P + (i & 1) * kPBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 128u, desc_sw128(p_addr + kk * 32, 16),
                   desc_sw128(v_addr + kk * 2048, 8192), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->pfree[i & 1]);
        mma_commit(&bars->empty[st]);
        return true;
      };
      for (int u = 0; ok && u < nload; ++u) {
        const int st = u % kStages;
        if (!wait_bar(&bars->full[st], (u / kStages) & 1, abort_flag, err)) break;
        if (u >= 2 && !wait_bar(&bars->sfree[u & 1], ((u - 2) >> 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + OFF_KV + st * 2 * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + (uint32_t)(u & 1) * 64u, desc_sw128(q_addr + kk * 32, 16),
                   desc_sw128(k_addr + kk * 32, 16), idesc_s, kk > 0);
        mma_commit(&bars->s[u & 1]);
        if ((u < n && !res) || !WITH_O) mma_commit(&bars->empty[st]);
        if (WITH_O && !res && u - 1 >= n && !do_pv(u - 1 - n)) {
          ok = false;
          break;
        }
      }
      if (ok && WITH_O && res)
        for (int i = 0; ok && i + 1 < n; ++i) ok = do_pv(i);
      if (ok && WITH_O && n > 0) ok = do_pv(n - 1);
      mma_commit(&bars->odone);  // fires when every MMA above has completed
      drain_bar(&bars->odone, 0);
    }
  } else {
    // ---- one thread per query row
    const int r = tid;
    const int tl = r / d.G, hh = r % d.G;
    const bool valid = tl < nvalid;
    const int t = pos0 + tl;
    const int nvis = valid ? cmp_nvis(d, t) : 0;
    const float sl2 = d.scale * kLog2e;
    const uint32_t lane_tmem = tmem + ((uint32_t)(warp * 32) << 16);
    float m = -INFINITY, lsum = 0.f;
    float mu0 = -INFINITY, mu1 = -INFINITY;  // with both chunks resident: their reference maxima
    bool ok = true;
    float sv[64];
    // pass 1: row statistics.  With both chunks resident in TMEM the
    // exponentials (relative to the running max m_u after chunk u) are
    // written back over S, so pass 2 only rescales them by 2^(m_u - m) / l.
    for (int u = 0; u < n; ++u) {
      if (!wait_bar_warp(&bars->s[u & 1], (u >> 1) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld32(lane_tmem + (uint32_t)(u & 1) * 64u, sv);
      tmem_ld32(lane_tmem + (uint32_t)(u & 1) * 64u + 32u, sv + 32);
      tmem_wait_ld();
      if (!res) {
        tc_fence_before();
        mbar_arrive(&bars->sfree[u & 1]);
      }
      const int j0 = u * kChunk;
      if (j0 < nvis) {
        if (j0 + kChunk > nvis) {
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = j0 + c < nvis ? sv[c] : -INFINITY;
        }
        float m0 = sv[0], m1 = sv[1], m2 = sv[2], m3 = sv[3];
#pragma unroll
        for (int c = 4; c < 64; c += 8) {
          m0 = fmax3(m0, sv[c], sv[c + 4]);
          m1 = fmax3(m1, sv[c + 1], sv[c + 5]);
          m2 = fmax3(m2, sv[c + 2], sv[c + 6]);
          m3 = fmax3(m3, sv[c + 3], sv[c + 7]);
        }
        const float mn = fmaxf(m, fmaxf(fmax3(m0, m1, m2), m3) * sl2);  // column 0 is visible
        const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mn, -mn);
        uint64_t r2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), sc2, nm2));
          sv[c] = fast_exp2(x.x);
          sv[c + 1] = fast_exp2(x.y);
          r2 = f2_add(r2, f2_pack(sv[c], sv[c + 1]));
        }
        const float2 rs = f2_unpack(r2);
        lsum = lsum * fast_exp2(m - mn) + (rs.x + rs.y);
        m = mn;
        if (u == 0) mu0 = mn;
        else mu1 = mn;
      }
      // tcgen05.st is warp-collective: every lane stores (a row that sees
      // none of this chunk stores its raw S, which pass 2 never reads)
      if (res) {
        tmem_st32(lane_tmem + (uint32_t)u * 64u, sv);
        tmem_st32(lane_tmem + (uint32_t)u * 64u + 32u, sv + 32);
      }
    }
    if (res) tmem_wait_st();
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    float* srow = score + (((size_t)b * d.Tq + t0 + tl) * d.Hkv + g) * d.Nc;
    const int per = 64 / d.G;  // score columns written by each head-lane of a token
    // pass 2: normalised probabilities, block scores, P for the value MMA
    for (int i = 0; ok && i < n; ++i) {
      const int u = res ? i : n + i;
      if (!res && !wait_bar_warp(&bars->s[u & 1], (u >> 1) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld32(lane_tmem + (uint32_t)(u & 1) * 64u, sv);
      tmem_ld32(lane_tmem + (uint32_t)(u & 1) * 64u + 32u, sv + 32);
      tmem_wait_ld();
      if (!res) {
        tc_fence_before();
        mbar_arrive(&bars->sfree[u & 1]);
      }
      const int j0 = i * kChunk;
      if (j0 >= nvis) {
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = 0.f;
      } else if (res) {  // stored 2^(s - m_i): masked columns are already 0
        const float fac = fast_exp2((i == 0 ? mu0 : mu1) - m) * inv;
        const uint64_t f2 = f2_pack(fac, fac);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = f2_unpack(f2_mul(f2_pack(sv[c], sv[c + 1]), f2));
          sv[c] = x.x;
          sv[c + 1] = x.y;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          sv[c] = j0 + c < nvis ? fast_exp2(fmaf(sv[c], sl2, -m)) * inv : 0.f;
      }
      if (WITH_O) {
        if (i >= 2 && !wait_bar_warp(&bars->pfree[i & 1], ((i - 2) >> 1) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        const uint32_t pb = smem_u32(smem + OFF_P + (i & 1) * kPBytes) + (uint32_t)(r >> 3) * 1024u +
                            (uint32_t)(r & 7) * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(pb + ((uint32_t)(c ^ (r & 7)) << 4), pack_bf16(sv[8 * c], sv[8 * c + 1]),
                       pack_bf16(sv[8 * c + 2], sv[8 * c + 3]),
                       pack_bf16(sv[8 * c + 4], sv[8 * c + 5]),
                       pack_bf16(sv[8 * c + 6], sv[8 * c + 7]));
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p[i & 1]);
      }
      // sum the G heads of each token (consecutive lanes) in fp32 with a
      // reduce-scatter: each step halves the columns a lane keeps and adds
      // the partner lane's copy of them, so head hh ends with the sums of
      // columns [hh*per, (hh+1)*per) in sv[0, per)
      if (d.G >= 2) reduce_half<32>(sv, hh & (32 / per), 32 / per);
      if (d.G >= 4) reduce_half<16>(sv, hh & (16 / per), 16 / per);
      if (d.G >= 8) reduce_half<8>(sv, hh & (8 / per), 8 / per);
      if (d.G >= 16) reduce_half<4>(sv, hh & (4 / per), 4 / per);
      if (d.G >= 32) reduce_half<2>(sv, hh & (2 / per), 2 / per);
      if (valid) {
        const int jb = j0 + hh * per;
        if (vec4) {  // 16-byte groups, each wholly inside or outside [0, Nc)
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            if (c < per && jb + c < d.Nc)
              *reinterpret_cast<float4*>(srow + jb + c) =
                  make_float4(sv[c], sv[c + 1], sv[c + 2], sv[c + 3]);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < per && jb + c < d.Nc) srow[jb + c] = sv[c];
        }
      }
    }
    if (valid) {  // blocks beyond the last chunk are not visible to this tile
      if (vec4)
        for (int j = n * kChunk + 4 * hh; j < d.Nc; j += 4 * d.G)
          *reinterpret_cast<float4*>(srow + j) = make_float4(0.f, 0.f, 0.f, 0.f);
      else
        for (int j = n * kChunk + hh; j < d.Nc; j += d.G) srow[j] = 0.f;
    }
    float ov[64];
    const bool have_o = WITH_O && ok && n > 0 &&
                        wait_bar_warp(&bars->odone, 0, abort_flag, err);
    if (have_o) {
      tc_fence_after();
      tmem_ld32(lane_tmem + 128u, ov);
      tmem_ld32(lane_tmem + 160u, ov + 32);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) ov[c] = 0.f;
    }
    tc_fence_before();
    if (valid) {
      const size_t row = ((size_t)b * d.Tq + t0 + tl) * d.Hq + g * d.G + hh;
      if (WITH_O) {
        uint4* dst = reinterpret_cast<uint4*>(o_cmp + row * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 w4;
          w4.x = pack_bf16(ov[8 * c + 0], ov[8 * c + 1]);
          w4.y = pack_bf16(ov[8 * c + 2], ov[8 * c + 3]);
          w4.z = pack_bf16(ov[8 * c + 4], ov[8 * c + 5]);
          w4.w = pack_bf16(ov[8 * c + 6], ov[8 * c + 7]);
          dst[c] = w4;
        }
      }
      if (lse) lse[row] = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <bool WITH_O>
cudaError_t launch_cmp_tc(const Dims& d, const void* q, const void* kc, const void* vc,
                          void* o_cmp, float* lse, float* score, int* err, cudaStream_t s) {
  const int TQ = kRows / d.G;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16(&mq, q, d.Hq, (long)d.B * d.Tq, d.G, TQ) ||
      !make_tmap_bf16(&mk, kc, d.Hkv, (long)d.B * d.Nc, 1, kChunk))
    return cudaErrorInvalidValue;
  if (WITH_O) {
    if (!make_tmap_bf16(&mv, vc, d.Hkv, (long)d.B * d.Nc, 1, kChunk)) return cudaErrorInvalidValue;
  } else {
    mv = mk;
  }
  cudaError_t e = cudaFuncSetAttribute(cmp_tc_kernel<WITH_O>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((d.Tq + TQ - 1) / TQ, d.Hkv, d.B);
  // score rows in 16-byte groups when every group is aligned: Nc % 4 == 0,
  // a head-lane's run of 64 / G columns a multiple of 4, an aligned base
  const bool vec4 = d.Nc % 4 == 0 && d.G <= 16 && ((uintptr_t)score & 15) == 0;
  cmp_tc_kernel<WITH_O><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, (bf16*)o_cmp, lse, score,
                                                          d, err, vec4);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cmp_scores(const Dims& d, const void* q, const void* kc, const void* vc,
                              void* o_cmp, float* lse_cmp, float* score, int* err,
                              cudaStream_t s) {
  const bool tc = d.dtype == 1 && d.Nc > 0 && kRows % d.G == 0 &&
                  tmap_encode_fn() != nullptr;
  if (!tc) return launch_cmp_scores_simt(d, q, kc, vc, o_cmp, lse_cmp, score, s);
  if (o_cmp) return launch_cmp_tc<true>(d, q, kc, vc, o_cmp, lse_cmp, score, err, s);
  return launch_cmp_tc<false>(d, q, kc, vc, nullptr, lse_cmp, score, err, s);
}

}  // namespace nsa
