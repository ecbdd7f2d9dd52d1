// internal.h -- launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace nsa {

// Validated, derived problem sizes (see nsa.h for the meaning of each).
struct Dims {
  int B, T, Tq, Hq, Hkv, D, G;
  int l;       // selection block size l'
  int lc;      // compression block size l
  int dc;      // compression stride d
  int Nc;      // complete compressed blocks: (T - lc) / dc + 1 (0 if T < lc)
  int Nb;      // selection blocks: ceil(T / l)
  int topk;
  int window;
  float scale;
  int dtype;   // 0 f32, 1 bf16
  int branch_mask;
  int q_off;   // position of query 0: T - Tq
};

// Compressed blocks complete at position t: block c covers tokens
// [c dc, c dc + lc) and is visible to the query at t once c dc + lc - 1 <= t.
__host__ __device__ inline int cmp_nvis(const Dims& d, int t) {
  if (t + 1 < d.lc) return 0;
  const int n = (t + 1 - d.lc) / d.dc + 1;
  return n < d.Nc ? n : d.Nc;
}

// Compression block = stride = selection block: compressed block j scores
// selection block j directly (no remap of the scores).
__host__ __device__ inline bool plain_geometry(const Dims& d) {
  return d.lc == d.l && d.dc == d.l;
}

// MoBA (k_moba.cu): gate + top-k per (query, KV group) over MoBA blocks of
// L tokens (d.lc = d.dc = L pooled into kc; d.l = 64), writing the chosen
// blocks (idx_m, may be NULL) and their 64-key blocks (idx64, top-k n L/64).
cudaError_t launch_moba_select(const Dims& d, const void* q, const void* kc, int32_t* idx_m,
                               int32_t* idx64, int L, int n, cudaStream_t s);
cudaError_t launch_moba_expand(const Dims& d, const int32_t* idx_m, int32_t* idx64, int L, int n,
                               cudaStream_t s);

// Each launcher enqueues on `s` and returns the launch status.  `err` is
// the device error word (may be NULL).
cudaError_t launch_compress(const Dims& d, const void* k, const void* v,
                            void* kc, void* vc, cudaStream_t s);
cudaError_t launch_cmp_scores(const Dims& d, const void* q, const void* kc,
                              const void* vc, void* o_cmp, float* lse_cmp,
                              float* score, int* err, cudaStream_t s);
// Queries per chunk of the reverse map (its count, scan and fill passes).
constexpr int kRevChunkQueries = 256;
// rev_counts (optional, revmap_chunk_ints(d) ints): also produce the block-major
// reverse map's per-(chunk, block) counts, so its own count pass is skipped
// (launch_sel_bm_prep with counted = true).
cudaError_t launch_topk(const Dims& d, const float* score, int32_t* idx, cudaStream_t s,
                        int* rev_counts = nullptr);
cudaError_t launch_sel_fwd(const Dims& d, const void* q, const void* k,
                           const void* v, const int32_t* idx, void* o,
                           float* lse, int* err, cudaStream_t s);
cudaError_t launch_swa_fwd(const Dims& d, const void* q, const void* k,
                           const void* v, void* o, float* lse, cudaStream_t s);
// window branch with the gated combination fused into its epilogue (bf16
// tensor-core path); o_swa may be NULL (not stored)
bool swa_combine_fusable(const Dims& d);
cudaError_t launch_swa_fwd_combine(const Dims& d, const void* q, const void* k, const void* v,
                                   void* o_swa, float* lse_swa, const float* gates,
                                   const void* o_cmp, const void* o_sel, void* out,
                                   cudaStream_t s);
// selection branch with the gated combination fused into its epilogue;
// o_sel may be NULL (not stored)
cudaError_t launch_sel_fwd_combine(const Dims& d, const void* q, const void* k, const void* v,
                                   const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                                   const float* gates, const void* o_cmp, const void* o_swa,
                                   void* out, cudaStream_t s);
// Gated combination fused into an attention epilogue: out = gate_own * o +
// sum over the non-NULL other[i] of gate(other_gate[i]) * other[i]; gate i of
// a row is gates[row * 3 + i] in the order (cmp, sel, swa); bf16 rows of 64.
struct EpilogueFuse {
  const float* gates;
  const void* other[2];
  int other_gate[2];
  int own_gate;
  void* out;
};
// block-major selection (k_sel_bm.cu): reverse map, per-(query, slot)
// partials, merge; fz (may be NULL) fuses the gated combination into the
// merge.  ws: sel_bm_ws_bytes(d) bytes, 256-byte aligned.  o_sel and
// lse_sel may be NULL (not stored).
bool sel_bm_eligible(const Dims& d);
// CUDA events recorded on the launching stream right before and after the
// block-major selection kernel of every later call (profiling; null: off)
void set_sel_bm_events(cudaEvent_t start, cudaEvent_t stop);
size_t sel_bm_ws_bytes(const Dims& d);
cudaError_t launch_sel_bm(const Dims& d, const void* q, const void* k, const void* v,
                          const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                          const EpilogueFuse* fz, void* ws, cudaStream_t s);
// launch_sel_bm in two steps: the reverse map and work units (prep), then the
// block-major kernel and the merge (run), so that other work can be ordered
// between them
cudaError_t launch_sel_bm_prep(const Dims& d, const int32_t* idx, int* err, void* ws,
                               cudaStream_t s, bool counted = false);
// where launch_sel_bm_prep expects the counts of a counted top-k
int* sel_bm_rev_counts(const Dims& d, void* ws);
cudaError_t launch_sel_bm_run(const Dims& d, const void* q, const void* k, const void* v,
                              const int32_t* idx, void* o_sel, float* lse_sel, int* err,
                              const EpilogueFuse* fz, void* ws, cudaStream_t s);
cudaError_t launch_combine(const Dims& d, const float* gates, const void* o_cmp,
                           const void* o_sel, const void* o_swa, void* out,
                           cudaStream_t s);

// ---- backward (k_bwd.cu); mode 0 selection, 1 window, 2 compression ----
// h16[i] (optional): also write branch i's dO as the fp16 pair the tensor-core
// dK/dV kernel takes (hi at h16[i], lo nel halves after it, nel = B Tq Hq 64),
// so that kernel can skip its own split (launch_dkdv with dO16_ready)
cudaError_t launch_gate_bwd(const Dims& d, const float* gates, const void* dout,
                            const void* o_cmp, const void* o_sel, const void* o_swa,
                            float* dgates, float* dOc, float* dOs, float* dOw, cudaStream_t s,
                            void* const* h16 = nullptr, int* err = nullptr);
cudaError_t launch_dq(const Dims& d, int mode, const void* q, const void* keys,
                      const void* vals, const int32_t* idx, const void* o, const float* lse,
                      const float* dO, float* dq, float* delta, int* err, cudaStream_t s);
// tensor-core dQ pass (k_bwd_tc.cu); modes 0 selection, 1 window
bool dq_tc_eligible(const Dims& d, int mode);
// single-pass selection backward (dQ query-stationary, dK / dV by atomics in
// the same kernel); tensor-core geometry as dq_tc_eligible(d, 0)
cudaError_t launch_sel_bwd_atomic(const Dims& d, const void* q, const void* k, const void* v,
                                  const int32_t* idx, const void* o, const float* lse,
                                  const float* dO, float* dq, float* delta, float* dk, float* dv,
                                  int* err, cudaStream_t s);
cudaError_t launch_dq_tc(const Dims& d, int mode, const void* q, const void* keys,
                         const void* vals, const int32_t* idx, const void* o, const float* lse,
                         const float* dO, float* dq, float* delta, int* err, cudaStream_t s);
// chunk: workspace of revmap_chunk_ints(d) ints
size_t revmap_chunk_ints(const Dims& d);
cudaError_t launch_revmap(const Dims& d, const int32_t* idx, int* chunk, int* offsets,
                          int* list, cudaStream_t s);
// the same map for the block-major selection forward: entries are
// query << 6 | slot, in ascending query order within a block's list (the
// same lists on every run), indices that break the forward's rule are
// reported in err, and per (sequence, group) the lists are cut into work
// units of at most tpu entries (units[bg * umax + u] = (block, first, end)
// for u < ucount[bg]).  cursor: B * Hkv * Nb ints (each block's first
// position).
// Reverse map of the forward's selection plus its work units: per (sequence,
// group) at most umax units of at most tpu = k * tq list entries (k <= 4
// tiles of tq entries), written sorted by size (units of k tiles first, then
// tails of k - 1, ..., 1 tiles, each class in block order); ucount holds the
// four class sizes of each (sequence, group) as an int4.
// counted: chunk already holds the per-(chunk, block) counts (a counted
// launch_topk), so the count pass is skipped.
cudaError_t launch_revmap_units(const Dims& d, const int32_t* idx, int* chunk, int* offsets,
                                int* cursor, int* list, int4* units, int* ucount, int tpu, int tq,
                                int umax, int* err, cudaStream_t s, bool counted = false);
// dO16: scratch of 2*B*Tq*Hq*64 16-bit values (the tensor-core path splits
// dO into an fp16 pair hi, lo there)
// dO16_ready: dO16 already holds dO's fp16 pair (written by launch_gate_bwd)
cudaError_t launch_dkdv(const Dims& d, int mode, const void* q, const void* keys,
                        const void* vals, const float* lse, const float* delta,
                        const float* dO, void* dO16, const int* offsets, const int* list,
                        float* dk, float* dv, float* part, int* err, cudaStream_t s,
                        bool dO16_ready = false);
bool dkdv_tc_eligible(const Dims& d, int mode);
// workspace of the compression branch's row shares (tensor-core dK/dV)
size_t dkdv_cmp_part_bytes(const Dims& d);
cudaError_t launch_dkdv_tc(const Dims& d, int mode, const void* q, const void* keys,
                           const void* vals, const float* lse, const float* delta,
                           const float* dO, void* dO16, const int* offsets, const int* list,
                           float* dk, float* dv, float* part, int* err, cudaStream_t s,
                           bool dO16_ready = false);

// Parametric (one linear layer) compression, bf16, D = 64: kc = sum_i k rows
// j d + i times W[i], same for vc (k_cmp_mlp.cu).  The backward overwrites
// dwk / dwv and adds the raw rows' gradient into dk / dv; ws holds
// cmp_mlp_bwd_ws_bytes(d) bytes, 256-byte aligned.
bool cmp_mlp_eligible(const Dims& d);
size_t cmp_mlp_fwd_ws_bytes(const Dims& d);  // 256-byte aligned, may be 0
size_t cmp_mlp_bwd_ws_bytes(const Dims& d);
cudaError_t launch_cmp_mlp_fwd(const Dims& d, const void* k, const void* v, const void* wk,
                               const void* wv, void* kc, void* vc, void* ws, int* err,
                               cudaStream_t s);
cudaError_t launch_cmp_mlp_bwd(const Dims& d, const void* k, const void* v, const void* wk,
                               const void* wv, const float* dkc, const float* dvc, float* dk,
                               float* dv, float* dwk, float* dwv, void* ws, int* err,
                               cudaStream_t s);

cudaError_t launch_pool_bwd(const Dims& d, const float* dkc, const float* dvc, float* dk,
                            float* dv, cudaStream_t s);

// ---- decode split into HBM-streaming kernels (k_decode.cu) ----
bool decode_split_eligible(const Dims& d);
size_t decode_split_ws_bytes(const Dims& d);
cudaError_t launch_decode_split(const Dims& d, const void* q, const void* kcache,
                                const void* vcache, const void* kc, const void* vc,
                                const float* gates, void* out, int32_t* idx_out, void* ws,
                                int* err, cudaStream_t s);

}  // namespace nsa
