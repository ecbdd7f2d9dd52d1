// topk.cuh -- per-(query, KV group) block selection by one warp.
//
// "DeepSeek's Native Sparse Attention", How Does Native Sparse Attention
// Work? (SELECTION); "Sparsity is Cool: Reverse-Engineering MoBA and NSA",
// Method (block 64, top-k 16) and Key claims (the first block is always
// kept).  Rule: cur = t / l.  With at most topk causal blocks every one of
// them is taken; otherwise blocks 0 and cur are forced and the topk - 2 best
// of 1..cur-1 are added, equal scores going to the lower block index.  The
// output is ascending and padded with -1.
//
// Lane `lane` holds the candidates 1 + lane + 32 q in registers as
// order-preserving integer keys.  A radix select finds tau, the (topk-2)-th
// largest key, bit by bit from the top (each step one warp-wide count with
// redux.sync), stopping early once exactly topk-2 keys lie at or above the
// prefix found so far.  The winners are every key above tau plus, among keys equal
// to tau, the lowest block indices (ballots in ascending block order).
#pragma once

#include <cstdint>

namespace nsa {

// Monotone map of a float to uint32 (larger float -> larger key); NaN -> 0.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// score(j) gives the importance of selection block j for j in 1..cur-1;
// QMAX * 32 must cover cur.  All 32 lanes call; out receives topk entries.
template <int QMAX, typename Score>
__device__ __forceinline__ void warp_select_blocks_fn(Score score, int cur, int topk,
                                                      int32_t* out, int lane) {
  if (cur + 1 <= topk) {
    for (int s = lane; s < topk; s += 32) out[s] = s <= cur ? s : -1;
    return;
  }
  uint32_t key[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int j = 1 + lane + 32 * q;
    key[q] = j < cur ? order_key(score(j)) : 0u;
  }
  const int K2 = topk - 2;
  // tau = the largest value with at least K2 keys >= tau.  Absent slots hold
  // key 0 and every threshold tried is >= 1, so they never count.  The bits
  // all candidates share are tau's from the start (every key is >= that
  // prefix); the search walks down from the highest bit in which two
  // candidates differ and stops as soon as exactly K2 keys are >= tau:
  // those are the winners whatever the lower bits of tau.
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll
  for (int q = 0; q < QMAX; ++q)
    if (1 + lane + 32 * q < cur) {
      kand &= key[q];
      kor |= key[q];
    }
  kand = __reduce_and_sync(0xffffffffu, kand);
  kor = __reduce_or_sync(0xffffffffu, kor);
  const uint32_t diff = kand ^ kor;
  int bit = diff ? 31 - __clz(diff) : -1;
  uint32_t tau = bit >= 0 ? kand & ~((2u << bit) - 1u) : kand;  // bit 31: 2u << 31 == 0
  for (; bit >= 0; --bit) {
    const uint32_t tc = tau | (1u << bit);
    unsigned c = 0;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) c += key[q] >= tc ? 1u : 0u;
    const int cnt = (int)__reduce_add_sync(0xffffffffu, c);
    if (cnt >= K2) tau = tc;
    if (cnt == K2) break;
  }
  unsigned cg = 0;
#pragma unroll
  for (int q = 0; q < QMAX; ++q) cg += (1 + lane + 32 * q < cur && key[q] > tau) ? 1u : 0u;
  const int need = K2 - (int)__reduce_add_sync(0xffffffffu, cg);  // >= 1 keys equal to tau
  int eq_before = 0, pos = 1;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int j = 1 + lane + 32 * q;
    const bool ok = j < cur;
    const bool eq = ok && key[q] == tau;
    const unsigned em = __ballot_sync(0xffffffffu, eq);
    const bool win = ok && (key[q] > tau || (eq && eq_before + __popc(em & lt) < need));
    const unsigned wm = __ballot_sync(0xffffffffu, win);
    if (win) out[pos + __popc(wm & lt)] = j;
    pos += __popc(wm);
    eq_before += __popc(em);
  }
  if (lane == 0) {
    out[0] = 0;
    out[K2 + 1] = cur;
  }
}

// score[j] for j in 1..cur-1 readable (global or shared memory).
template <int QMAX>
__device__ __forceinline__ void warp_select_blocks(const float* score, int cur, int topk,
                                                   int32_t* out, int lane) {
  warp_select_blocks_fn<QMAX>([score](int j) { return score[j]; }, cur, topk, out, lane);
}

}  // namespace nsa
