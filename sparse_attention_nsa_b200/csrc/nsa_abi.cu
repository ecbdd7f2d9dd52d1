// nsa_abi.cu -- the extern "C" entry points of libnsa (declared in nsa.h).
//
// This layer validates arguments, derives sizes, carves the caller's
// workspace, and enqueues kernels on the caller's stream.  It allocates no
// device memory and never synchronises except in nsa_last_device_error.
#include <algorithm>
#include <initializer_list>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "nsa.h"

using nsa::Dims;

// The device error word: kernels record the first failing check here.
__device__ int g_nsa_error_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {};

// Device address of the error word on the current device (looked up once
// per device, with that device current).
int* err_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_nsa_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = (int*)p;
  }
  return g_err_ptr[dev];
}

bool aligned16(const void* p) { return p && (((uintptr_t)p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

nsa_status fill_dims(const nsa_params* p, Dims* d) {
  if (!p) return NSA_ERR_INVALID_ARG;
  if (p->B < 1 || p->T < 1 || p->Tq < 1 || p->Tq > p->T || p->Hq < 1 || p->Hkv < 1 ||
      p->D < 1 || p->cmp_block < 1 || p->cmp_stride < 1 || p->sel_block < 1 ||
      p->topk < 2 || p->window < 1)
    return NSA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return NSA_ERR_INVALID_ARG;
  if (p->dtype != NSA_F32 && p->dtype != NSA_BF16) return NSA_ERR_INVALID_ARG;
  if (p->branch_mask < 1 || p->branch_mask > NSA_BRANCH_ALL) return NSA_ERR_INVALID_ARG;
  // a positive finite scale: the kernels take each row's max before scaling
  if (!(p->scale > 0.f) || p->scale == INFINITY) return NSA_ERR_INVALID_ARG;
  // valid NSA geometry, but outside what this build runs
  if (p->D != 64) return NSA_ERR_UNSUPPORTED;
  const int G = p->Hq / p->Hkv;
  if (G > 32 || (G & (G - 1)) != 0) return NSA_ERR_UNSUPPORTED;
  if (p->Hkv > 64 || p->topk > 64) return NSA_ERR_UNSUPPORTED;
  const int l = p->sel_block;
  const long long Nb = ((long long)p->T + l - 1) / l;  // T + l - 1 may pass INT_MAX
  const int Nc = p->T < p->cmp_block ? 0 : (p->T - p->cmp_block) / p->cmp_stride + 1;
  if (Nb > 1024 || Nc > 1024) return NSA_ERR_UNSUPPORTED;
  // key / value rows (b T + t) are addressed by signed 32-bit tensor-map
  // coordinates
  if ((long long)p->B * p->T >= (1LL << 31)) return NSA_ERR_UNSUPPORTED;
  d->B = p->B;
  d->T = p->T;
  d->Tq = p->Tq;
  d->Hq = p->Hq;
  d->Hkv = p->Hkv;
  d->D = p->D;
  d->G = G;
  d->l = l;
  d->lc = p->cmp_block;
  d->dc = p->cmp_stride;
  d->Nc = Nc;
  d->Nb = (int)Nb;
  d->topk = p->topk;
  d->window = p->window;
  d->scale = p->scale;
  d->dtype = p->dtype;
  d->branch_mask = p->branch_mask;
  d->q_off = p->T - p->Tq;
  return NSA_OK;
}

size_t esize(const Dims& d) { return d.dtype == NSA_BF16 ? 2 : 4; }

// Workspace layout of nsa_forward / nsa_decode: every intermediate the
// caller did not supply, each 256-byte aligned, in this order.
struct Carve {
  size_t off[11];
  size_t total;
};

enum { W_KC, W_VC, W_OCMP, W_LSECMP, W_SCORE, W_IDX, W_OSEL, W_LSESEL, W_OSWA, W_LSESWA, W_SELBM };

// The selection branch runs block-major (reverse map, per-slot partials,
// merge) when a query tile's union of blocks would be mostly unselected:
// the query-tiled kernel's work grows with Nb / topk, the block-major
// kernel's does not (measured on B200: equal at Nb = 8 topk, 1.6x faster at
// Nb = 32 topk).
bool use_sel_bm(const Dims& d) {
  return (d.branch_mask & NSA_BRANCH_SEL) && d.Tq >= 64 && d.Nb >= 8 * d.topk &&
         nsa::sel_bm_eligible(d);
}

void tensor_bytes(const Dims& d, size_t out[11]) {
  const size_t es = esize(d);
  const size_t kcb = (size_t)d.B * d.Nc * d.Hkv * 64 * es;
  const size_t ob = (size_t)d.B * d.Tq * d.Hq * 64 * es;
  const size_t lb = (size_t)d.B * d.Tq * d.Hq * 4;
  out[W_KC] = kcb;
  out[W_VC] = kcb;
  out[W_OCMP] = ob;
  out[W_LSECMP] = lb;
  out[W_SCORE] = (size_t)d.B * d.Tq * d.Hkv * d.Nc * 4;
  out[W_IDX] = (size_t)d.B * d.Tq * d.Hkv * d.topk * 4;
  out[W_OSEL] = ob;
  out[W_LSESEL] = lb;
  out[W_OSWA] = ob;
  out[W_LSESWA] = lb;
  out[W_SELBM] = use_sel_bm(d) ? nsa::sel_bm_ws_bytes(d) : 0;
}

Carve carve(const Dims& d, const nsa_saved* sv) {
  size_t bytes[11];
  tensor_bytes(d, bytes);
  const void* given[11] = {};
  if (sv) {
    given[W_KC] = sv->kc;
    given[W_VC] = sv->vc;
    given[W_OCMP] = sv->o_cmp;
    given[W_LSECMP] = sv->lse_cmp;
    given[W_SCORE] = sv->score;
    given[W_IDX] = sv->idx;
    given[W_OSEL] = sv->o_sel;
    given[W_LSESEL] = sv->lse_sel;
    given[W_OSWA] = sv->o_swa;
    given[W_LSESWA] = sv->lse_swa;
  }
  Carve c{};
  size_t at = 0;
  for (int i = 0; i < 11; ++i) {
    c.off[i] = at;
    if (!given[i]) at += align256(bytes[i]);
  }
  c.total = at;
  return c;
}

#define NSA_TRY_CUDA(expr)                           \
  do {                                               \
    if ((expr) != cudaSuccess) return NSA_ERR_CUDA;  \
  } while (0)

}  // namespace

extern "C" {

const char* nsa_status_string(nsa_status s) {
  switch (s) {
    case NSA_OK: return "NSA_OK";
    case NSA_ERR_INVALID_ARG: return "NSA_ERR_INVALID_ARG";
    case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED";
    case NSA_ERR_CUDA: return "NSA_ERR_CUDA";
    case NSA_ERR_TIMEOUT: return "NSA_ERR_TIMEOUT";
    case NSA_ERR_DEVICE_CHECK: return "NSA_ERR_DEVICE_CHECK";
    case NSA_ERR_WORKSPACE: return "NSA_ERR_WORKSPACE";
    case NSA_ERR_SCRATCH_TOO_SMALL: return "NSA_ERR_SCRATCH_TOO_SMALL";
  }
  return "NSA_ERR_UNKNOWN";
}

nsa_status nsa_check_params(const nsa_params* p) {
  Dims d;
  return fill_dims(p, &d);
}

nsa_status nsa_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = carve(d, nullptr).total;
  if (nsa::decode_split_eligible(d)) *bytes = std::max(*bytes, nsa::decode_split_ws_bytes(d));
  return NSA_OK;
}

nsa_status nsa_last_device_error(void* stream) {
  int* ew = err_word();
  if (!ew) return NSA_ERR_CUDA;
  NSA_TRY_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int v = 0;
  NSA_TRY_CUDA(cudaMemcpy(&v, ew, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    const int zero = 0;
    NSA_TRY_CUDA(cudaMemcpy(ew, &zero, sizeof(int), cudaMemcpyHostToDevice));
  }
  if (v == nsa::kDevTimeout) return NSA_ERR_TIMEOUT;
  if (v != 0) return NSA_ERR_DEVICE_CHECK;
  return NSA_OK;
}

nsa_status nsa_compress(const nsa_params* p, const void* k, const void* v, void* kc,
                        void* vc, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(k) || !aligned16(v)) return NSA_ERR_INVALID_ARG;
  if (d.Nc > 0 && (!aligned16(kc) || !aligned16(vc))) return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_compress(d, k, v, kc, vc, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_cmp_attn_scores(const nsa_params* p, const void* q, const void* kc,
                               const void* vc, void* o_cmp, float* lse_cmp,
                               float* score, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || (d.Nc > 0 && (!aligned16(kc) || !aligned16(vc))))
    return NSA_ERR_INVALID_ARG;
  if (d.Nc > 0 && !aligned16(score)) return NSA_ERR_INVALID_ARG;
  if (o_cmp && !aligned16(o_cmp)) return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_cmp_scores(d, q, kc, vc, o_cmp, lse_cmp, score, err_word(),
                                      (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_select_topk(const nsa_params* p, const float* score, int32_t* idx,
                           void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if ((d.Nc > 0 && !aligned16(score)) || !aligned16(idx)) return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_topk(d, score, idx, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_sel_attn_fwd(const nsa_params* p, const void* q, const void* k,
                            const void* v, const int32_t* idx, void* o_sel,
                            float* lse_sel, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) ||
      !aligned16(o_sel))
    return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_sel_fwd(d, q, k, v, idx, o_sel, lse_sel, err_word(),
                                   (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_set_kernel_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return NSA_ERR_INVALID_ARG;
  nsa::set_sel_bm_events((cudaEvent_t)start, (cudaEvent_t)stop);
  return NSA_OK;
}

nsa_status nsa_sel_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  if (!nsa::sel_bm_eligible(d)) return NSA_ERR_UNSUPPORTED;
  *bytes = nsa::sel_bm_ws_bytes(d);
  return NSA_OK;
}

nsa_status nsa_sel_attn_fwd_ws(const nsa_params* p, const void* q, const void* k,
                               const void* v, const int32_t* idx, void* o_sel, float* lse_sel,
                               void* workspace, size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) ||
      (o_sel && !aligned16(o_sel)))
    return NSA_ERR_INVALID_ARG;
  if (!nsa::sel_bm_eligible(d)) return NSA_ERR_UNSUPPORTED;
  const size_t need = nsa::sel_bm_ws_bytes(d);
  if (!workspace || workspace_bytes < need || (((uintptr_t)workspace) & 255u) != 0)
    return NSA_ERR_WORKSPACE;
  NSA_TRY_CUDA(nsa::launch_sel_bm(d, q, k, v, idx, o_sel, lse_sel, err_word(), nullptr,
                                  workspace, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_swa_fwd(const nsa_params* p, const void* q, const void* k, const void* v,
                       void* o_swa, float* lse_swa, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_swa))
    return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_swa_fwd(d, q, k, v, o_swa, lse_swa, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_gate_combine(const nsa_params* p, const float* gates, const void* o_cmp,
                            const void* o_sel, const void* o_swa, void* out,
                            void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(gates) || !aligned16(out)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_CMP) && !aligned16(o_cmp)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_SEL) && !aligned16(o_sel)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_SWA) && !aligned16(o_swa)) return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_combine(d, gates, o_cmp, o_sel, o_swa, out,
                                   (cudaStream_t)stream));
  return NSA_OK;
}

// Library-owned side stream per device, at the device's highest stream
// priority, for the dependent chain compression -> top-k -> reverse map of a
// forward while the window branch runs on the caller's stream: the block
// scheduler gives the chain's blocks the SMs first as they free up, and the
// window's fill the rest (launched the other way round, the window's blocks
// took every SM before the chain could start).  Created on first use (with
// that device current) and kept until exit.
struct SideStream {
  cudaStream_t s2 = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static std::mutex g_side_mu;  // also held across each fork ... join enqueue
static SideStream g_side[64];

static SideStream* side_stream_locked() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev];
  if (!ss.s2) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
    if (cudaStreamCreateWithPriority(&ss.s2, cudaStreamNonBlocking, greatest) != cudaSuccess)
      return nullptr;
    if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
  }
  return &ss;
}

// Shared body of nsa_forward and nsa_decode.  kc_given means the compressed
// tensors in sv->kc / sv->vc are inputs (decode) and compression is skipped.
static nsa_status run_forward(const Dims& d, const void* q, const void* k, const void* v,
                              bool kc_given, const float* gates, void* out,
                              const nsa_saved* sv, void* ws, size_t ws_bytes,
                              cudaStream_t s) {
  const Carve c = carve(d, sv);
  if (c.total > 0 && (!ws || ws_bytes < c.total || (((uintptr_t)ws) & 255u) != 0))
    return NSA_ERR_WORKSPACE;
  char* w = (char*)ws;
  auto pick = [&](void* given, int slot) -> void* {
    return given ? given : (void*)(w + c.off[slot]);
  };
  const nsa_saved z{};
  const nsa_saved& S = sv ? *sv : z;
  void* kc = kc_given ? S.kc : pick(S.kc, W_KC);
  void* vc = kc_given ? S.vc : pick(S.vc, W_VC);
  void* o_cmp = pick(S.o_cmp, W_OCMP);
  float* lse_cmp = (float*)pick(S.lse_cmp, W_LSECMP);
  float* score = (float*)pick(S.score, W_SCORE);
  int32_t* idx = (int32_t*)pick(S.idx, W_IDX);
  void* o_sel = pick(S.o_sel, W_OSEL);
  float* lse_sel = (float*)pick(S.lse_sel, W_LSESEL);
  void* o_swa = pick(S.o_swa, W_OSWA);
  float* lse_swa = (float*)pick(S.lse_swa, W_LSESWA);
  const bool cmp = d.branch_mask & NSA_BRANCH_CMP;
  const bool sel = d.branch_mask & NSA_BRANCH_SEL;
  const bool swa = d.branch_mask & NSA_BRANCH_SWA;
  const bool bm = use_sel_bm(d);
  if (sel && swa && nsa::swa_combine_fusable(d)) {
    // The window branch does not depend on compression, top-k or selection:
    // those run as a high-priority chain on the side stream while the window
    // runs here, and the selection kernel, last on this stream, applies the
    // gates in its epilogue.
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream* ss = side_stream_locked();
    if (ss) {
      if (cudaEventRecord(ss->fork, s) != cudaSuccess ||
          cudaStreamWaitEvent(ss->s2, ss->fork, 0) != cudaSuccess)
        return NSA_ERR_CUDA;
      cudaError_t em = cudaSuccess;
      if (!kc_given) em = nsa::launch_compress(d, k, v, kc, vc, ss->s2);
      if (em == cudaSuccess)
        em = nsa::launch_cmp_scores(d, q, kc, vc, cmp ? o_cmp : nullptr, cmp ? lse_cmp : nullptr,
                                    score, err_word(), ss->s2);
      // with the block-major kernel, the top-k also counts the reverse map's
      // entries (the map then has no count pass of its own)
      int* rc = bm ? nsa::sel_bm_rev_counts(d, w + c.off[W_SELBM]) : nullptr;
      if (em == cudaSuccess) em = nsa::launch_topk(d, score, idx, ss->s2, rc);
      if (em == cudaSuccess && bm)
        em = nsa::launch_sel_bm_prep(d, idx, err_word(), w + c.off[W_SELBM], ss->s2, true);
      // the join is enqueued whatever happens, so no side-stream work can
      // outlive this call's ordering on the caller's stream
      const cudaError_t ej = cudaEventRecord(ss->join, ss->s2);
      const cudaError_t ew = nsa::launch_swa_fwd(d, q, k, v, o_swa, S.lse_swa, s);
      const cudaError_t ewait = cudaStreamWaitEvent(s, ss->join, 0);
      if (ew != cudaSuccess || ej != cudaSuccess || em != cudaSuccess || ewait != cudaSuccess)
        return NSA_ERR_CUDA;
      if (bm) {
        const nsa::EpilogueFuse fz{gates,
                                   {cmp ? o_cmp : nullptr, o_swa},
                                   {0, 2},
                                   1,
                                   out};
        NSA_TRY_CUDA(nsa::launch_sel_bm_run(d, q, k, v, idx, S.o_sel, S.lse_sel, err_word(), &fz,
                                            w + c.off[W_SELBM], s));
        return NSA_OK;
      }
      NSA_TRY_CUDA(nsa::launch_sel_fwd_combine(d, q, k, v, idx, S.o_sel, S.lse_sel, err_word(),
                                               gates, o_cmp, o_swa, out, s));
      return NSA_OK;
    }
  }
  if (cmp || sel) {
    if (!kc_given) NSA_TRY_CUDA(nsa::launch_compress(d, k, v, kc, vc, s));
    NSA_TRY_CUDA(nsa::launch_cmp_scores(d, q, kc, vc, cmp ? o_cmp : nullptr,
                                        cmp ? lse_cmp : nullptr, score, err_word(), s));
  }
  if (sel) {
    NSA_TRY_CUDA(nsa::launch_topk(d, score, idx, s));
    if (!swa && bm) {
      // no window branch: the merge runs last and applies the gates
      const nsa::EpilogueFuse fz{gates, {cmp ? o_cmp : nullptr, nullptr}, {0, 2}, 1, out};
      NSA_TRY_CUDA(nsa::launch_sel_bm(d, q, k, v, idx, S.o_sel, S.lse_sel, err_word(), &fz,
                                      w + c.off[W_SELBM], s));
      return NSA_OK;
    }
    if (!swa && nsa::swa_combine_fusable(d)) {
      // no window branch: the selection kernel runs last and applies the gates
      NSA_TRY_CUDA(nsa::launch_sel_fwd_combine(d, q, k, v, idx, S.o_sel, S.lse_sel, err_word(),
                                               gates, o_cmp, nullptr, out, s));
      return NSA_OK;
    }
    if (bm)
      NSA_TRY_CUDA(nsa::launch_sel_bm(d, q, k, v, idx, o_sel, lse_sel, err_word(), nullptr,
                                      w + c.off[W_SELBM], s));
    else
      NSA_TRY_CUDA(nsa::launch_sel_fwd(d, q, k, v, idx, o_sel, lse_sel, err_word(), s));
  }
  if (swa && nsa::swa_combine_fusable(d)) {
    // the window branch runs last and writes `out` itself; its own output
    // and lse are stored only when the caller asked for them
    NSA_TRY_CUDA(nsa::launch_swa_fwd_combine(d, q, k, v, S.o_swa, S.lse_swa, gates, o_cmp, o_sel,
                                             out, s));
    return NSA_OK;
  }
  if (swa) NSA_TRY_CUDA(nsa::launch_swa_fwd(d, q, k, v, o_swa, lse_swa, s));
  NSA_TRY_CUDA(nsa::launch_combine(d, gates, o_cmp, o_sel, o_swa, out, s));
  return NSA_OK;
}

nsa_status nsa_forward(const nsa_params* p, const void* q, const void* k, const void* v,
                       const float* gates, void* out, const nsa_saved* saved,
                       void* workspace, size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) ||
      !aligned16(out))
    return NSA_ERR_INVALID_ARG;
  if (saved) {
    const void* ptrs[10] = {saved->kc, saved->vc, saved->o_cmp, saved->lse_cmp,
                            saved->score, saved->idx, saved->o_sel, saved->lse_sel,
                            saved->o_swa, saved->lse_swa};
    for (const void* ptr : ptrs)
      if (ptr && (((uintptr_t)ptr) & 15u)) return NSA_ERR_INVALID_ARG;
  }
  return run_forward(d, q, k, v, false, gates, out, saved, workspace, workspace_bytes,
                     (cudaStream_t)stream);
}

}  // extern "C"

namespace {
// device copies of nsa_forward_host's inputs and output, then the forward's
// own workspace, each 256-byte aligned
struct HostCarve {
  size_t q, k, v, gates, out, fwd, total, qb, kb, gb;
};
HostCarve host_carve(const Dims& d, size_t fwd_bytes) {
  HostCarve c{};
  const size_t es = d.dtype == 1 ? 2 : 4;
  c.qb = (size_t)d.B * d.Tq * d.Hq * d.D * es;   // q and out
  c.kb = (size_t)d.B * d.T * d.Hkv * d.D * es;   // k and v
  c.gb = (size_t)d.B * d.Tq * d.Hq * 3 * sizeof(float);
  size_t at = 0;
  auto take = [&](size_t b) {
    const size_t o = at;
    at += align256(b);
    return o;
  };
  c.q = take(c.qb);
  c.k = take(c.kb);
  c.v = take(c.kb);
  c.gates = take(c.gb);
  c.out = take(c.qb);
  c.fwd = take(fwd_bytes);
  c.total = at;
  return c;
}
}  // namespace

extern "C" {

nsa_status nsa_forward_host_workspace_size(const nsa_params* p, size_t* bytes) {
  if (!bytes) return NSA_ERR_INVALID_ARG;
  size_t fwd = 0;
  nsa_status st = nsa_workspace_size(p, &fwd);
  if (st != NSA_OK) return st;
  Dims d{};
  if ((st = fill_dims(p, &d)) != NSA_OK) return st;
  *bytes = host_carve(d, fwd).total;
  return NSA_OK;
}

nsa_status nsa_forward_host(const nsa_params* p, const void* q, const void* k, const void* v,
                            const float* gates, void* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!q || !k || !v || !gates || !out) return NSA_ERR_INVALID_ARG;
  size_t fwd = 0;
  if ((st = nsa_workspace_size(p, &fwd)) != NSA_OK) return st;
  const HostCarve c = host_carve(d, fwd);
  if (!workspace || workspace_bytes < c.total || (((uintptr_t)workspace) & 255u) != 0)
    return NSA_ERR_WORKSPACE;
  char* w = (char*)workspace;
  const cudaStream_t s = (cudaStream_t)stream;
  // one copy per tensor, in order on the caller's stream
  NSA_TRY_CUDA(cudaMemcpyAsync(w + c.q, q, c.qb, cudaMemcpyHostToDevice, s));
  NSA_TRY_CUDA(cudaMemcpyAsync(w + c.k, k, c.kb, cudaMemcpyHostToDevice, s));
  NSA_TRY_CUDA(cudaMemcpyAsync(w + c.v, v, c.kb, cudaMemcpyHostToDevice, s));
  NSA_TRY_CUDA(cudaMemcpyAsync(w + c.gates, gates, c.gb, cudaMemcpyHostToDevice, s));
  st = run_forward(d, w + c.q, w + c.k, w + c.v, false, (const float*)(w + c.gates), w + c.out,
                   nullptr, w + c.fwd, workspace_bytes - c.fwd, s);
  if (st != NSA_OK) return st;
  NSA_TRY_CUDA(cudaMemcpyAsync(out, w + c.out, c.qb, cudaMemcpyDeviceToHost, s));
  return NSA_OK;
}

nsa_status nsa_decode(const nsa_params* p, const void* q, const void* k_cache,
                      const void* v_cache, const void* kc_cache, const void* vc_cache,
                      const float* gates, void* out, int32_t* idx_out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (d.Tq != 1) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(gates) ||
      !aligned16(out))
    return NSA_ERR_INVALID_ARG;
  if (d.Nc > 0 && (!aligned16(kc_cache) || !aligned16(vc_cache))) return NSA_ERR_INVALID_ARG;
  if (idx_out && (((uintptr_t)idx_out) & 15u)) return NSA_ERR_INVALID_ARG;
  if (nsa::decode_split_eligible(d)) {
    const size_t need = nsa::decode_split_ws_bytes(d);
    if (!workspace || workspace_bytes < need || (((uintptr_t)workspace) & 255u) != 0)
      return NSA_ERR_WORKSPACE;
    NSA_TRY_CUDA(nsa::launch_decode_split(d, q, k_cache, v_cache, kc_cache, vc_cache, gates, out,
                                          idx_out, workspace, err_word(), (cudaStream_t)stream));
    return NSA_OK;
  }
  nsa_saved sv{};
  sv.idx = idx_out;
  sv.kc = (void*)kc_cache;  // inputs here; NULL only when Nc == 0 (never read)
  sv.vc = (void*)vc_cache;
  return run_forward(d, q, k_cache, v_cache, true, gates, out, &sv, workspace,
                     workspace_bytes, (cudaStream_t)stream);
}

}  // extern "C"

namespace nsa {
// Workspace bytes nsa_decode carves when the compressed caches are inputs,
// with or without a caller-provided idx_out (used by the no-alloc variant).
nsa_status decode_scratch_bytes(const nsa_params* p, bool idx_given, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  if (decode_split_eligible(d)) {
    *bytes = decode_split_ws_bytes(d);
    return NSA_OK;
  }
  nsa_saved sv{};
  sv.kc = (void*)1;  // marks the slot as supplied; never dereferenced
  sv.vc = (void*)1;
  if (idx_given) sv.idx = (int32_t*)1;
  *bytes = carve(d, &sv).total;
  return NSA_OK;
}
}  // namespace nsa

// ============================================================================
// Backward entry points
// ============================================================================
namespace {

// Backward workspace layout, each part 256-byte aligned:
//   delta [B*Tq*Hq] f32 | dO_cmp, dO_sel, dO_swa [B*Tq*Hq*64] f32 |
//   dkc, dvc [B*Nc*Hkv*64] f32 | reverse-map chunk positions
//   [B*Hkv*ceil(Tq/256)*Nb] i32 | offsets [B*Hkv*(Nb+1)] i32 |
//   list [B*Hkv*Tq*topk] i32 | compression dK/dV row shares (tensor-core path) |
//   dO split into fp16 hi, lo [2*B*Tq*Hq*64] (tensor-core dK/dV path) |
//   the whole backward's per-branch fp16 pairs, written by the gate backward
//   [3][2*B*Tq*Hq*64] (tensor-core dK/dV path)
struct BwdCarve {
  size_t delta, dO[3], dkc, dvc, counts, offsets, list, part, dO16, dO16b[3], total;
};

BwdCarve bwd_carve(const Dims& d) {
  BwdCarve c{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t o = at;
    at += align256(bytes);
    return o;
  };
  const size_t rows = (size_t)d.B * d.Tq * d.Hq;
  c.delta = take(rows * 4);
  for (int i = 0; i < 3; ++i) c.dO[i] = take(rows * 64 * 4);
  c.dkc = take((size_t)d.B * d.Nc * d.Hkv * 64 * 4);
  c.dvc = take((size_t)d.B * d.Nc * d.Hkv * 64 * 4);
  c.counts = take(nsa::revmap_chunk_ints(d) * 4);
  c.offsets = take((size_t)d.B * d.Hkv * (d.Nb + 1) * 4);
  c.list = take((size_t)d.B * d.Hkv * d.Tq * d.topk * 4);
  c.part = take(nsa::dkdv_tc_eligible(d, 2) ? nsa::dkdv_cmp_part_bytes(d) : 0);
  c.dO16 = take(nsa::dkdv_tc_eligible(d, 0) ? 2 * rows * 64 * 2 : 0);
  for (int i = 0; i < 3; ++i)  // branch i: compression (mode 2), selection (0), window (1)
    c.dO16b[i] = take(nsa::dkdv_tc_eligible(d, i == 0 ? 2 : i - 1) ? 2 * rows * 64 * 2 : 0);
  c.total = at;
  return c;
}

bool ws_ok(const void* ws, size_t bytes, size_t need) {
  return ws && bytes >= need && (((uintptr_t)ws) & 255u) == 0;
}

nsa_status sel_bwd_body(const Dims& d, const void* q, const void* k, const void* v,
                        const int32_t* idx, const void* o_sel, const float* lse_sel,
                        const float* dO_sel, float* dq, float* dk, float* dv, char* w,
                        const BwdCarve& c, cudaStream_t s, void* pre16 = nullptr) {
  float* delta = (float*)(w + c.delta);
  int* counts = (int*)(w + c.counts);
  int* offsets = (int*)(w + c.offsets);
  int* list = (int*)(w + c.list);
  NSA_TRY_CUDA(nsa::launch_dq(d, 0, q, k, v, idx, o_sel, lse_sel, dO_sel, dq, delta, err_word(), s));
  NSA_TRY_CUDA(nsa::launch_revmap(d, idx, counts, offsets, list, s));
  NSA_TRY_CUDA(nsa::launch_dkdv(d, 0, q, k, v, lse_sel, delta, dO_sel, pre16 ? pre16 : w + c.dO16,
                                offsets, list, dk, dv, nullptr, err_word(), s, pre16 != nullptr));
  return NSA_OK;
}

nsa_status swa_bwd_body(const Dims& d, const void* q, const void* k, const void* v,
                        const void* o_swa, const float* lse_swa, const float* dO_swa,
                        float* dq, float* dk, float* dv, char* w, const BwdCarve& c,
                        cudaStream_t s, void* pre16 = nullptr) {
  float* delta = (float*)(w + c.delta);
  NSA_TRY_CUDA(nsa::launch_dq(d, 1, q, k, v, nullptr, o_swa, lse_swa, dO_swa, dq, delta, nullptr, s));
  NSA_TRY_CUDA(nsa::launch_dkdv(d, 1, q, k, v, lse_swa, delta, dO_swa, pre16 ? pre16 : w + c.dO16,
                                nullptr, nullptr, dk, dv, nullptr, err_word(), s,
                                pre16 != nullptr));
  return NSA_OK;
}

// The parametric compressor of nsa_backward_mlp: its inputs, its weights'
// gradients and its own workspace.
struct MlpGrad {
  const void *k, *v, *wk, *wv;
  float *dwk, *dwv;
  void* ws;
};

nsa_status cmp_bwd_body(const Dims& d, const void* q, const void* kc, const void* vc,
                        const void* o_cmp, const float* lse_cmp, const float* dO_cmp,
                        float* dq, float* dk, float* dv, char* w, const BwdCarve& c,
                        cudaStream_t s, const MlpGrad* mlp = nullptr, void* pre16 = nullptr) {
  float* delta = (float*)(w + c.delta);
  float* dkc = (float*)(w + c.dkc);
  float* dvc = (float*)(w + c.dvc);
  if (d.Nc == 0) {  // nothing visible anywhere: no gradient
    if (mlp)
      NSA_TRY_CUDA(nsa::launch_cmp_mlp_bwd(d, mlp->k, mlp->v, mlp->wk, mlp->wv, dkc, dvc, dk, dv,
                                           mlp->dwk, mlp->dwv, mlp->ws, err_word(), s));
    return NSA_OK;
  }
  const size_t nkc = (size_t)d.B * d.Nc * d.Hkv * 64 * 4;
  NSA_TRY_CUDA(cudaMemsetAsync(dkc, 0, nkc, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dvc, 0, nkc, s));
  NSA_TRY_CUDA(nsa::launch_dq(d, 2, q, kc, vc, nullptr, o_cmp, lse_cmp, dO_cmp, dq, delta, nullptr, s));
  NSA_TRY_CUDA(nsa::launch_dkdv(d, 2, q, kc, vc, lse_cmp, delta, dO_cmp, pre16 ? pre16 : w + c.dO16,
                                nullptr, nullptr, dkc, dvc, (float*)(w + c.part), err_word(), s,
                                pre16 != nullptr));
  if (mlp)
    NSA_TRY_CUDA(nsa::launch_cmp_mlp_bwd(d, mlp->k, mlp->v, mlp->wk, mlp->wv, dkc, dvc, dk, dv,
                                         mlp->dwk, mlp->dwv, mlp->ws, err_word(), s));
  else
    NSA_TRY_CUDA(nsa::launch_pool_bwd(d, dkc, dvc, dk, dv, s));
  return NSA_OK;
}

}  // namespace

extern "C" {

nsa_status nsa_backward_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = bwd_carve(d).total;
  return NSA_OK;
}

nsa_status nsa_gate_combine_bwd(const nsa_params* p, const float* gates, const void* dout,
                                const void* o_cmp, const void* o_sel, const void* o_swa,
                                float* dgates, float* dO_cmp, float* dO_sel, float* dO_swa,
                                void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(gates) || !aligned16(dout) || !aligned16(dgates)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_CMP) && !aligned16(o_cmp)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_SEL) && !aligned16(o_sel)) return NSA_ERR_INVALID_ARG;
  if ((d.branch_mask & NSA_BRANCH_SWA) && !aligned16(o_swa)) return NSA_ERR_INVALID_ARG;
  for (const void* ptr : {(const void*)dO_cmp, (const void*)dO_sel, (const void*)dO_swa})
    if (ptr && (((uintptr_t)ptr) & 15u)) return NSA_ERR_INVALID_ARG;
  NSA_TRY_CUDA(nsa::launch_gate_bwd(d, gates, dout, o_cmp, o_sel, o_swa, dgates, dO_cmp, dO_sel,
                                    dO_swa, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_sel_attn_bwd(const nsa_params* p, const void* q, const void* k, const void* v,
                            const int32_t* idx, const void* o_sel, const float* lse_sel,
                            const float* dO_sel, float* dq, float* dk, float* dv, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  for (const void* ptr : {q, k, v, (const void*)idx, o_sel, (const void*)lse_sel,
                          (const void*)dO_sel, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  const BwdCarve c = bwd_carve(d);
  if (!ws_ok(workspace, workspace_bytes, c.total)) return NSA_ERR_WORKSPACE;
  return sel_bwd_body(d, q, k, v, idx, o_sel, lse_sel, dO_sel, dq, dk, dv, (char*)workspace, c,
                      (cudaStream_t)stream);
}

nsa_status nsa_sel_attn_bwd_atomic(const nsa_params* p, const void* q, const void* k,
                                   const void* v, const int32_t* idx, const void* o_sel,
                                   const float* lse_sel, const float* dO_sel, float* dq,
                                   float* dk, float* dv, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  for (const void* ptr : {q, k, v, (const void*)idx, o_sel, (const void*)lse_sel,
                          (const void*)dO_sel, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  if (!nsa::dq_tc_eligible(d, 0)) return NSA_ERR_UNSUPPORTED;
  const BwdCarve c = bwd_carve(d);
  if (!ws_ok(workspace, workspace_bytes, c.total)) return NSA_ERR_WORKSPACE;
  float* delta = (float*)((char*)workspace + c.delta);
  NSA_TRY_CUDA(nsa::launch_sel_bwd_atomic(d, q, k, v, idx, o_sel, lse_sel, dO_sel, dq, delta, dk,
                                          dv, err_word(), (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_swa_bwd(const nsa_params* p, const void* q, const void* k, const void* v,
                       const void* o_swa, const float* lse_swa, const float* dO_swa, float* dq,
                       float* dk, float* dv, void* workspace, size_t workspace_bytes,
                       void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  for (const void* ptr : {q, k, v, o_swa, (const void*)lse_swa, (const void*)dO_swa,
                          (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  const BwdCarve c = bwd_carve(d);
  if (!ws_ok(workspace, workspace_bytes, c.total)) return NSA_ERR_WORKSPACE;
  return swa_bwd_body(d, q, k, v, o_swa, lse_swa, dO_swa, dq, dk, dv, (char*)workspace, c,
                      (cudaStream_t)stream);
}

nsa_status nsa_cmp_bwd(const nsa_params* p, const void* q, const void* kc, const void* vc,
                       const void* o_cmp, const float* lse_cmp, const float* dO_cmp, float* dq,
                       float* dk, float* dv, void* workspace, size_t workspace_bytes,
                       void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  for (const void* ptr : {q, o_cmp, (const void*)lse_cmp, (const void*)dO_cmp, (const void*)dq,
                          (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  if (d.Nc > 0 && (!aligned16(kc) || !aligned16(vc))) return NSA_ERR_INVALID_ARG;
  const BwdCarve c = bwd_carve(d);
  if (!ws_ok(workspace, workspace_bytes, c.total)) return NSA_ERR_WORKSPACE;
  return cmp_bwd_body(d, q, kc, vc, o_cmp, lse_cmp, dO_cmp, dq, dk, dv, (char*)workspace, c,
                      (cudaStream_t)stream);
}

}  // extern "C"

namespace {

nsa_status backward_body(const Dims& d, const void* q, const void* k, const void* v,
                         const float* gates, const void* dout, const nsa_saved* sv, float* dq,
                         float* dk, float* dv, float* dgates, void* workspace,
                         size_t workspace_bytes, cudaStream_t s, MlpGrad* mlp) {
  nsa_status st = NSA_OK;
  if (!sv) return NSA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)gates, dout, (const void*)dq, (const void*)dk,
                          (const void*)dv, (const void*)dgates})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  const bool cmp = d.branch_mask & NSA_BRANCH_CMP;
  const bool sel = d.branch_mask & NSA_BRANCH_SEL;
  const bool swa = d.branch_mask & NSA_BRANCH_SWA;
  if (cmp && (!aligned16(sv->o_cmp) || !aligned16(sv->lse_cmp) ||
              (d.Nc > 0 && (!aligned16(sv->kc) || !aligned16(sv->vc)))))
    return NSA_ERR_INVALID_ARG;
  if (sel && (!aligned16(sv->idx) || !aligned16(sv->o_sel) || !aligned16(sv->lse_sel)))
    return NSA_ERR_INVALID_ARG;
  if (swa && (!aligned16(sv->o_swa) || !aligned16(sv->lse_swa))) return NSA_ERR_INVALID_ARG;
  const BwdCarve c = bwd_carve(d);
  const size_t need = c.total + (mlp ? nsa::cmp_mlp_bwd_ws_bytes(d) : 0);
  if (!ws_ok(workspace, workspace_bytes, need)) return NSA_ERR_WORKSPACE;
  char* w = (char*)workspace;
  if (mlp) mlp->ws = w + c.total;
  float* dO[3] = {(float*)(w + c.dO[0]), (float*)(w + c.dO[1]), (float*)(w + c.dO[2])};
  // the gate backward also writes each tensor-core branch's dO as the fp16
  // pair its dK/dV kernel reads, so those kernels skip their own split
  const bool on[3] = {cmp && d.Nc > 0, sel, swa};
  void* pre16[3];
  for (int i = 0; i < 3; ++i)
    pre16[i] = on[i] && nsa::dkdv_tc_eligible(d, i == 0 ? 2 : i - 1) ? w + c.dO16b[i] : nullptr;
  NSA_TRY_CUDA(nsa::launch_gate_bwd(d, gates, dout, sv->o_cmp, sv->o_sel, sv->o_swa, dgates,
                                    cmp ? dO[0] : nullptr, sel ? dO[1] : nullptr,
                                    swa ? dO[2] : nullptr, s, pre16, err_word()));
  NSA_TRY_CUDA(cudaMemsetAsync(dq, 0, (size_t)d.B * d.Tq * d.Hq * 64 * 4, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dk, 0, (size_t)d.B * d.T * d.Hkv * 64 * 4, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dv, 0, (size_t)d.B * d.T * d.Hkv * 64 * 4, s));
  if (cmp) {
    st = cmp_bwd_body(d, q, sv->kc, sv->vc, sv->o_cmp, sv->lse_cmp, dO[0], dq, dk, dv, w, c, s,
                      mlp, pre16[0]);
    if (st != NSA_OK) return st;
  } else if (mlp) {
    // compressed keys reach only the selection scores, and top-k passes no gradient
    const size_t wbytes = (size_t)d.lc * 64 * 64 * sizeof(float);
    NSA_TRY_CUDA(cudaMemsetAsync(mlp->dwk, 0, wbytes, s));
    NSA_TRY_CUDA(cudaMemsetAsync(mlp->dwv, 0, wbytes, s));
  }
  if (sel) {
    st = sel_bwd_body(d, q, k, v, sv->idx, sv->o_sel, sv->lse_sel, dO[1], dq, dk, dv, w, c, s,
                      pre16[1]);
    if (st != NSA_OK) return st;
  }
  if (swa) {
    st = swa_bwd_body(d, q, k, v, sv->o_swa, sv->lse_swa, dO[2], dq, dk, dv, w, c, s, pre16[2]);
    if (st != NSA_OK) return st;
  }
  return NSA_OK;
}

// d, the parametric compressor's pointers: bf16, D = 64, 16-byte aligned
nsa_status mlp_args_ok(const Dims& d, std::initializer_list<const void*> ptrs) {
  if (!nsa::cmp_mlp_eligible(d)) return NSA_ERR_UNSUPPORTED;
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  return NSA_OK;
}

}  // namespace

extern "C" {

nsa_status nsa_backward(const nsa_params* p, const void* q, const void* k, const void* v,
                        const float* gates, const void* dout, const nsa_saved* sv, float* dq,
                        float* dk, float* dv, float* dgates, void* workspace,
                        size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  return backward_body(d, q, k, v, gates, dout, sv, dq, dk, dv, dgates, workspace,
                       workspace_bytes, (cudaStream_t)stream, nullptr);
}

// ---- parametric compression ----------------------------------------------------

nsa_status nsa_compress_mlp_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = nsa::cmp_mlp_fwd_ws_bytes(d);
  return NSA_OK;
}

nsa_status nsa_compress_mlp(const nsa_params* p, const void* k, const void* v, const void* wk,
                            const void* wv, void* kc, void* vc, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  st = mlp_args_ok(d, {k, v, wk, wv});
  if (st != NSA_OK) return st;
  if (d.Nc > 0 && (!aligned16(kc) || !aligned16(vc))) return NSA_ERR_INVALID_ARG;
  const size_t need = nsa::cmp_mlp_fwd_ws_bytes(d);
  if (need > 0 && !ws_ok(workspace, workspace_bytes, need)) return NSA_ERR_WORKSPACE;
  NSA_TRY_CUDA(nsa::launch_cmp_mlp_fwd(d, k, v, wk, wv, kc, vc, workspace, err_word(),
                                       (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_compress_mlp_bwd_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = nsa::cmp_mlp_bwd_ws_bytes(d);
  return NSA_OK;
}

nsa_status nsa_compress_mlp_bwd(const nsa_params* p, const void* k, const void* v,
                                const void* wk, const void* wv, const float* dkc,
                                const float* dvc, float* dk, float* dv, float* dwk, float* dwv,
                                void* workspace, size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  st = mlp_args_ok(d, {k, v, wk, wv, dk, dv, dwk, dwv});
  if (st != NSA_OK) return st;
  if (d.Nc > 0 && (!aligned16(dkc) || !aligned16(dvc))) return NSA_ERR_INVALID_ARG;
  if (!ws_ok(workspace, workspace_bytes, nsa::cmp_mlp_bwd_ws_bytes(d))) return NSA_ERR_WORKSPACE;
  NSA_TRY_CUDA(nsa::launch_cmp_mlp_bwd(d, k, v, wk, wv, dkc, dvc, dk, dv, dwk, dwv, workspace,
                                       err_word(), (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_forward_mlp(const nsa_params* p, const void* q, const void* k, const void* v,
                           const void* wk, const void* wv, const float* gates, void* out,
                           const nsa_saved* saved, void* workspace, size_t workspace_bytes,
                           void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  st = mlp_args_ok(d, {q, k, v, wk, wv, gates, out});
  if (st != NSA_OK) return st;
  nsa_saved sv = saved ? *saved : nsa_saved{};
  const void* ptrs[10] = {sv.kc, sv.vc, sv.o_cmp, sv.lse_cmp, sv.score,
                          sv.idx, sv.o_sel, sv.lse_sel, sv.o_swa, sv.lse_swa};
  for (const void* ptr : ptrs)
    if (ptr && (((uintptr_t)ptr) & 15u)) return NSA_ERR_INVALID_ARG;
  const Carve c = carve(d, saved);
  const size_t need = c.total + nsa::cmp_mlp_fwd_ws_bytes(d);
  if (need > 0 && !ws_ok(workspace, workspace_bytes, need)) return NSA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)workspace;
  // kc / vc take the first two slots, the compressor's partial sums the end;
  // the rest of the forward carves what lies between
  if (!sv.kc) sv.kc = w + c.off[W_KC];
  if (!sv.vc) sv.vc = w + c.off[W_VC];
  const bool need_kc = d.branch_mask & (NSA_BRANCH_CMP | NSA_BRANCH_SEL);
  if (need_kc)
    NSA_TRY_CUDA(nsa::launch_cmp_mlp_fwd(d, k, v, wk, wv, sv.kc, sv.vc, w + c.total, err_word(), s));
  const size_t used = c.off[W_OCMP];
  return run_forward(d, q, k, v, true, gates, out, &sv, used ? w + used : workspace,
                     c.total - used, s);
}

nsa_status nsa_forward_mlp_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = carve(d, nullptr).total + nsa::cmp_mlp_fwd_ws_bytes(d);
  return NSA_OK;
}

nsa_status nsa_backward_mlp_workspace_size(const nsa_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  *bytes = bwd_carve(d).total + nsa::cmp_mlp_bwd_ws_bytes(d);
  return NSA_OK;
}

nsa_status nsa_backward_mlp(const nsa_params* p, const void* q, const void* k, const void* v,
                            const void* wk, const void* wv, const float* gates, const void* dout,
                            const nsa_saved* sv, float* dq, float* dk, float* dv, float* dwk,
                            float* dwv, float* dgates, void* workspace, size_t workspace_bytes,
                            void* stream) {
  Dims d;
  nsa_status st = fill_dims(p, &d);
  if (st != NSA_OK) return st;
  st = mlp_args_ok(d, {wk, wv, dwk, dwv});
  if (st != NSA_OK) return st;
  MlpGrad mlp{k, v, wk, wv, dwk, dwv, nullptr};
  return backward_body(d, q, k, v, gates, dout, sv, dq, dk, dv, dgates, workspace,
                       workspace_bytes, (cudaStream_t)stream, &mlp);
}

}  // extern "C"

// ============================================================================
// MoBA block attention on the selection kernels
// ============================================================================
namespace {

// Dims of the selection attention that runs MoBA: 64-key selection blocks,
// top-k = k L / 64; compression (pooling) over MoBA blocks of L tokens.
nsa_status fill_moba_dims(const nsa_moba_params* p, Dims* d) {
  if (!p) return NSA_ERR_INVALID_ARG;
  if (p->block < 1 || p->topk < 1) return NSA_ERR_INVALID_ARG;
  nsa_params q{};
  q.B = p->B;
  q.T = p->T;
  q.Tq = p->Tq;
  q.Hq = p->Hq;
  q.Hkv = p->Hkv;
  q.D = p->D;
  q.cmp_block = p->block;
  q.cmp_stride = p->block;
  q.sel_block = 64;
  q.topk = 2;  // validated below
  q.window = 1;
  q.scale = p->scale;
  q.dtype = p->dtype;
  q.branch_mask = NSA_BRANCH_SEL;
  nsa_status st = fill_dims(&q, d);
  if (st != NSA_OK) return st;
  if (p->block % 64 != 0 || p->T / p->block > 128 ||
      (long long)p->topk * (p->block / 64) > 64)  // k <= 64 also bounds the MoBA index rows
    return NSA_ERR_UNSUPPORTED;
  d->topk = p->topk * (p->block / 64);
  if (d->topk < 2) return NSA_ERR_UNSUPPORTED;  // the selection kernels take >= 2 blocks
  return NSA_OK;
}

struct MobaCarve {
  size_t kc, vc, idx64, idxm, selbm, total;
};

MobaCarve moba_carve(const Dims& d, int n) {
  MobaCarve c{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t o = at;
    at += align256(bytes);
    return o;
  };
  const size_t rows = (size_t)d.B * d.Tq * d.Hkv;
  c.kc = take((size_t)d.B * d.Nc * d.Hkv * 64 * esize(d));
  c.vc = take((size_t)d.B * d.Nc * d.Hkv * 64 * esize(d));
  c.idx64 = take(rows * d.topk * 4);
  c.idxm = take(rows * (size_t)n * 4);
  c.selbm = take(use_sel_bm(d) ? nsa::sel_bm_ws_bytes(d) : 0);
  c.total = at;
  return c;
}

}  // namespace

extern "C" {

nsa_status nsa_moba_workspace_size(const nsa_moba_params* p, size_t* bytes) {
  Dims d;
  nsa_status st = fill_moba_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!bytes) return NSA_ERR_INVALID_ARG;
  const size_t rows = (size_t)d.B * d.Tq * d.Hkv;
  *bytes = std::max(moba_carve(d, p->topk).total,
                    bwd_carve(d).total + align256(rows * d.topk * 4));
  return NSA_OK;
}

nsa_status nsa_moba_forward(const nsa_moba_params* p, const void* q, const void* k, const void* v,
                            void* out, float* lse, int32_t* idx, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_moba_dims(p, &d);
  if (st != NSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (idx && !aligned16(idx)))
    return NSA_ERR_INVALID_ARG;
  const MobaCarve c = moba_carve(d, p->topk);
  if (!ws_ok(workspace, workspace_bytes, c.total)) return NSA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)workspace;
  int32_t* idx64 = (int32_t*)(w + c.idx64);
  if (d.Nc > 0) NSA_TRY_CUDA(nsa::launch_compress(d, k, v, w + c.kc, w + c.vc, s));
  NSA_TRY_CUDA(nsa::launch_moba_select(d, q, w + c.kc, idx ? idx : (int32_t*)(w + c.idxm), idx64,
                                       p->block, p->topk, s));
  if (use_sel_bm(d))
    NSA_TRY_CUDA(nsa::launch_sel_bm(d, q, k, v, idx64, out, lse, err_word(), nullptr,
                                    w + c.selbm, s));
  else
    NSA_TRY_CUDA(nsa::launch_sel_fwd(d, q, k, v, idx64, out, lse, err_word(), s));
  return NSA_OK;
}

nsa_status nsa_moba_backward(const nsa_moba_params* p, const void* q, const void* k,
                             const void* v, const int32_t* idx, const void* out, const float* lse,
                             const float* dout, float* dq, float* dk, float* dv, void* workspace,
                             size_t workspace_bytes, void* stream) {
  Dims d;
  nsa_status st = fill_moba_dims(p, &d);
  if (st != NSA_OK) return st;
  for (const void* ptr : {q, k, v, (const void*)idx, out, (const void*)lse, (const void*)dout,
                          (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return NSA_ERR_INVALID_ARG;
  // the selection backward's workspace, then the expanded indices after it
  const BwdCarve c = bwd_carve(d);
  const size_t rows = (size_t)d.B * d.Tq * d.Hkv;
  const size_t need = c.total + align256(rows * d.topk * 4);
  if (!ws_ok(workspace, workspace_bytes, need)) return NSA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)workspace;
  int32_t* idx64 = (int32_t*)(w + c.total);
  NSA_TRY_CUDA(nsa::launch_moba_expand(d, idx, idx64, p->block, p->topk, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dq, 0, (size_t)d.B * d.Tq * d.Hq * 64 * 4, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dk, 0, (size_t)d.B * d.T * d.Hkv * 64 * 4, s));
  NSA_TRY_CUDA(cudaMemsetAsync(dv, 0, (size_t)d.B * d.T * d.Hkv * 64 * 4, s));
  return sel_bwd_body(d, q, k, v, idx64, out, lse, dout, dq, dk, dv, w, c, s);
}

}  // extern "C"
