/*
 * nsa.h -- C ABI of libnsa, a B200 (sm_100a) implementation of Native
 * Sparse Attention (NSA) with mean-pooled compression.
 *
 * The method: "DeepSeek's Native Sparse Attention" (bycloud newsletter #44,
 * section "How Does Native Sparse Attention Work?") describes three
 * attention branches per query -- COMPRESSION (attend to one summary
 * key/value per block of tokens), SELECTION (score the blocks, keep the most
 * important ones in raw form and attend to them) and SLIDING WINDOW (attend
 * to the most recent tokens) -- whose outputs are merged by learned gates.
 * "Sparsity is Cool: Reverse-Engineering MoBA and NSA" (sections TL;DR,
 * Method, Key claims) fixes the variant built here: mean-pooling instead of
 * an MLP for compression, block 64, top-k 16, window 512, GQA/MQA KV
 * sharing with one selection per KV group, the first block always selected,
 * and branch pruning at inference.
 *
 * ------------------------------------------------------------------------
 * Conventions shared by every entry point
 * ------------------------------------------------------------------------
 * Pointers.  Every tensor argument is a DEVICE pointer owned by the caller,
 *   contiguous in the layout stated, 16-byte aligned.  The library keeps no
 *   reference after the call returns and allocates no device memory:
 *   scratch space comes from a caller-provided workspace.
 * Stream.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every entry point only enqueues work on that stream and
 *   returns without synchronising, except nsa_last_device_error.
 * Shapes.  B batch, T keys per sequence, Tq queries per sequence (the
 *   queries are the LAST Tq positions of the T-key sequence: query i sits at
 *   position T - Tq + i; prefill has Tq = T, decode Tq = 1), Hq query heads,
 *   Hkv key/value heads, G = Hq / Hkv query heads per KV group (query head h
 *   reads KV head h / G), D head dim (64).  l' = selection block size,
 *   Nb = ceil(T / l') selection blocks; compressed blocks of l tokens every
 *   d tokens (block j covers tokens [j d, j d + l)), Nc = (T - l) / d + 1
 *   of them (complete blocks only; 0 if T < l).
 * Layouts (row-major):
 *   q, o_*, out          [B, Tq, Hq, D]   dtype
 *   k, v                 [B, T, Hkv, D]   dtype
 *   kc, vc               [B, Nc, Hkv, D]  dtype
 *   gates                [B, Tq, Hq, 3]   float32, branch order (cmp, sel, swa)
 *   lse_*                [B, Tq, Hq]      float32, natural-log sum-exp
 *   score                [B, Tq, Hkv, Nc] float32
 *   idx                  [B, Tq, Hkv, topk] int32, ascending, -1 padded
 *   dtype is float32 (NSA_F32) or bfloat16 (NSA_BF16) for the whole call.
 * Errors.  Arguments are validated before anything is enqueued; a bad
 *   argument returns NSA_ERR_INVALID_ARG and a valid but unimplemented
 *   geometry NSA_ERR_UNSUPPORTED, with nothing launched.  A failed launch
 *   returns NSA_ERR_CUDA.  Device-side bounded waits and checks never trap:
 *   they record a code read back by nsa_last_device_error.  When that
 *   returns anything but NSA_OK, the outputs of every call enqueued since
 *   the previous check are undefined (a kernel that gave up on a wait
 *   leaves its part of the result unwritten).
 */
#ifndef NSA_H_
#define NSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape or parameter        */
  NSA_ERR_UNSUPPORTED = 2,  /* valid NSA geometry this build does not run  */
  NSA_ERR_CUDA = 3,         /* a CUDA call or launch failed                */
  NSA_ERR_TIMEOUT = 4,      /* a bounded device-side wait expired          */
  NSA_ERR_DEVICE_CHECK = 5, /* a device-side consistency check failed      */
  NSA_ERR_WORKSPACE = 6,    /* workspace missing or smaller than required  */
  NSA_ERR_SCRATCH_TOO_SMALL = 7 /* problem needs more than the fixed scratch
                                   of nsa_decode_noalloc                    */
} nsa_status;

typedef enum { NSA_F32 = 0, NSA_BF16 = 1 } nsa_dtype;

enum {
  NSA_BRANCH_CMP = 1, /* compression branch  */
  NSA_BRANCH_SEL = 2, /* selection branch    */
  NSA_BRANCH_SWA = 4, /* sliding window      */
  NSA_BRANCH_ALL = 7
};

/* Problem description.  The block geometry follows the pages' problem
 * statement: compression block size l and stride d, selection block size l',
 * top-k n, window w ("Sparsity is Cool", Method, uses l = d = l' = 64).
 * Any l, d, l' >= 1 run, up to 1024 selection blocks and 1024 compressed
 * blocks per sequence and B T < 2^31 key rows (NSA_ERR_UNSUPPORTED beyond);
 * the bf16 tensor-core selection, window and backward kernels take l' = 64,
 * other l' the CUDA-core kernels. */
typedef struct {
  int B, T, Tq, Hq, Hkv, D;
  int cmp_block;   /* l  : tokens per compressed block              */
  int cmp_stride;  /* d  : stride between compressed blocks          */
  int sel_block;   /* l' : tokens per selection block               */
  int topk;        /* n  : selected blocks per (query, KV group), >= 2 */
  int window;      /* w  : sliding-window length in keys, >= 1      */
  float scale;     /* softmax scale, finite and > 0, normally 1/sqrt(D) */
  int dtype;       /* nsa_dtype of q/k/v/kc/vc/o_*                   */
  int branch_mask; /* NSA_BRANCH_* bits of the branches to combine   */
} nsa_params;

/* Optional intermediate tensors of nsa_forward.  A non-NULL pointer makes
 * nsa_forward write that tensor there (layouts above); a NULL pointer puts
 * it in the workspace.  nsa_sel_attn_bwd needs idx, o_sel and lse_sel. */
typedef struct {
  void* kc;
  void* vc;
  void* o_cmp;
  float* lse_cmp;
  float* score;
  int32_t* idx;
  void* o_sel;
  float* lse_sel;
  void* o_swa;
  float* lse_swa;
} nsa_saved;

/* Human-readable name of a status code (static string, never NULL). */
const char* nsa_status_string(nsa_status s);

/* Validate a parameter block without launching anything.  Returns NSA_OK,
 * NSA_ERR_INVALID_ARG or NSA_ERR_UNSUPPORTED. */
nsa_status nsa_check_params(const nsa_params* p);

/* Bytes of workspace nsa_forward / nsa_decode need for parameters p (with
 * every nsa_saved pointer NULL; passing buffers never increases it). */
nsa_status nsa_workspace_size(const nsa_params* p, size_t* bytes);

/* Synchronise `stream`, then read and clear the library's device error
 * word: NSA_OK, NSA_ERR_TIMEOUT or NSA_ERR_DEVICE_CHECK (NSA_ERR_CUDA if
 * the synchronisation itself failed). */
nsa_status nsa_last_device_error(void* stream);

/* ---- compression: mean-pool blocks of l tokens every d tokens ------------
 * kc[b, j, g, :] = (1/l) * sum_{i<l} k[b, j*d + i, g, :], same for vc.
 * Passage: "Sparsity is Cool", Method and Key claims (mean-pooling replaces
 * NSA's MLP); "DeepSeek's Native Sparse Attention", COMPRESSION.
 * k, v [B, T, Hkv, D] -> kc, vc [B, Nc, Hkv, D].  The sum is exact (fp64)
 * and rounded once to dtype (round-to-nearest-even).  Tq is ignored. */
nsa_status nsa_compress(const nsa_params* p, const void* k, const void* v,
                        void* kc, void* vc, void* stream);

/* ---- compression branch and block importance ----------------------------
 * For query position t: compressed block j is visible iff its last token
 * j*d + l - 1 <= t.  P[t,h,:] = softmax over visible j of scale*q.kc_j;
 * o_cmp = sum_j P v c_j (0 and lse = -inf when nothing is visible);
 * score[t,g,j] = sum over the G heads h of group g of P[t,h,j] (0 for
 * invisible j).  Passage: "DeepSeek's Native Sparse Attention", COMPRESSION
 * and SELECTION (importance reuses the compression attention scores).
 * o_cmp and lse_cmp may be NULL (scores only: the branch-pruned case of
 * "Sparsity is Cool", Key claims). */
nsa_status nsa_cmp_attn_scores(const nsa_params* p, const void* q,
                               const void* kc, const void* vc, void* o_cmp,
                               float* lse_cmp, float* score, void* stream);

/* ---- top-k block selection per (query, KV group) ------------------------
 * cur = t / l'.  If cur + 1 <= topk, idx = 0..cur then -1 padding.  Else
 * blocks 0 and cur are forced and the topk - 2 highest-scoring blocks of
 * 1..cur-1 are added (equal scores: lower block index first); idx is
 * ascending.  The score of selection block j (tokens [j l', (j+1) l')) is
 * the sum, in ascending order, of score[.., i] over the compressed blocks i
 * whose tokens [i d, i d + l) overlap it (the pages give no rule for
 * mapping compressed blocks onto selection blocks of another geometry; this
 * is the plainest one, and with l = d = l' it is score[.., j] itself).
 * Passage: "DeepSeek's Native Sparse Attention", SELECTION; "Sparsity is
 * Cool", Method (block 64 / top-k 16) and Key claims (always include the
 * first block).  score [B,Tq,Hkv,Nc] -> idx [B,Tq,Hkv,topk]. */
nsa_status nsa_select_topk(const nsa_params* p, const float* score,
                           int32_t* idx, void* stream);

/* ---- selection branch ----------------------------------------------------
 * o_sel[t,h] = softmax-weighted sum of v over the keys s <= t that lie in
 * the blocks idx[t, h/G, :] (entries < 0 ignored); lse_sel its log-sum-exp.
 * Passage: "DeepSeek's Native Sparse Attention", SELECTION and the kernel
 * paragraph (queries sharing the same blocks are grouped: one selection per
 * KV group, all G heads read the same blocks).  Block indices must be
 * ascending, distinct and causal (<= t / l'); the kernel checks this and
 * records NSA_ERR_DEVICE_CHECK instead of reading out of bounds. */
nsa_status nsa_sel_attn_fwd(const nsa_params* p, const void* q, const void* k,
                            const void* v, const int32_t* idx, void* o_sel,
                            float* lse_sel, void* stream);

/* The same selection branch, block-major, with a caller workspace of at
 * least nsa_sel_workspace_size(p) bytes (256-byte aligned).  The queries
 * that chose each block are gathered from a reverse map (block -> queries),
 * each (query, head, block) pair gets its own softmax over the block's keys,
 * and each row's partials are merged exactly with their log-sum-exps (the
 * split-softmax identity); results match nsa_sel_attn_fwd up to rounding.
 * nsa_forward takes this path itself when Tq >= 64 and Nb >= 8 topk (the
 * query-tiled kernel's union of blocks grows with Nb / topk).  Passage: as for
 * nsa_sel_attn_fwd, plus the kernel paragraph (each block is loaded once for
 * all the queries that selected it).  o_sel may be NULL (not
 * stored), as may lse_sel.  Index errors are recorded as in nsa_sel_attn_fwd;
 * the per-block partial outputs are held in fp16, and a value beyond its
 * range (|v| > 65504) is recorded as NSA_ERR_DEVICE_CHECK.
 * Returns NSA_ERR_UNSUPPORTED for shapes the block-major kernels do not
 * cover (fp32, block size != 64, D != 64, 128 % G != 0). */
nsa_status nsa_sel_workspace_size(const nsa_params* p, size_t* bytes);

/* Profiling aid: record the CUDA events `start` and `stop` (cudaEvent_t,
 * owned by the caller) on the launching stream immediately before and after
 * the block-major selection kernel of every later call that runs it, so a
 * caller can time that kernel alone with cudaEventElapsedTime.  Both NULL
 * turns it off (the default); one NULL is NSA_ERR_INVALID_ARG.
 * Process-wide; not for concurrent use from several threads. */
nsa_status nsa_set_kernel_events(void* start, void* stop);
nsa_status nsa_sel_attn_fwd_ws(const nsa_params* p, const void* q, const void* k,
                               const void* v, const int32_t* idx, void* o_sel,
                               float* lse_sel, void* workspace, size_t workspace_bytes,
                               void* stream);

/* ---- sliding-window branch -----------------------------------------------
 * o_swa[t,h] attends to keys max(0, t-w+1) <= s <= t.
 * Passage: "DeepSeek's Native Sparse Attention", SLIDING WINDOW;
 * "Sparsity is Cool", Method (window 512). */
nsa_status nsa_swa_fwd(const nsa_params* p, const void* q, const void* k,
                       const void* v, void* o_swa, float* lse_swa,
                       void* stream);

/* ---- gated combination ---------------------------------------------------
 * out = g_cmp*o_cmp + g_sel*o_sel + g_swa*o_swa over the branches enabled
 * in branch_mask (a disabled branch's pointer may be NULL).  Gates are
 * post-sigmoid values.  Passage: "DeepSeek's Native Sparse Attention"
 * (outputs merged by gates from a small network); "Sparsity is Cool",
 * TL;DR and Key claims (unused branches pruned at inference). */
nsa_status nsa_gate_combine(const nsa_params* p, const float* gates,
                            const void* o_cmp, const void* o_sel,
                            const void* o_swa, void* out, void* stream);

/* ---- whole forward ---------------------------------------------------------
 * compress -> compression branch + scores -> top-k -> selection branch ->
 * window branch -> gated combination, in one call.  With NSA_BRANCH_CMP
 * off, the scores are still computed (selection needs them) but the
 * compression output is not.  With NSA_BRANCH_SEL off the selection path
 * (scores, top-k, selection) is skipped entirely, and so is the compression
 * branch if it is off too.  `saved` may be NULL.  workspace must hold at
 * least nsa_workspace_size(p) bytes (256-byte aligned).
 * Passage: "DeepSeek's Native Sparse Attention", How Does Native Sparse
 * Attention Work? (three key/value sets per query, three attention outputs
 * merged by gates); "Sparsity is Cool", Method (mean-pool compression,
 * block 64, top-k 16, window 512) and Key claims (later layers pruned to
 * fewer branches at inference: the branch mask).
 * With selection and window both enabled, the steps up to the reverse map
 * run on a library-owned stream of the current device (highest stream
 * priority, created on first use) while the window runs on `stream`; the
 * call forks from and joins back into `stream` with events, so to the
 * caller everything is ordered on `stream` as usual (graph capture
 * included).  Concurrent calls serialise their enqueueing on a lock. */
nsa_status nsa_forward(const nsa_params* p, const void* q, const void* k,
                       const void* v, const float* gates, void* out,
                       const nsa_saved* saved, void* workspace,
                       size_t workspace_bytes, void* stream);

/* ---- whole forward from host memory ------------------------------------------
 * nsa_forward for a caller whose q, k, v, gates and out live in host memory
 * (same layouts): on `stream`, one host-to-device copy per input into the
 * workspace, the forward, one device-to-host copy of out.  The call returns
 * once everything is enqueued; out is valid after the stream has been
 * synchronised, and the host buffers must stay untouched until then.  Page-
 * locked host memory makes the copies asynchronous (pageable memory works,
 * with copies staged by the driver).  workspace is device memory of at least
 * nsa_forward_host_workspace_size(p) bytes, 256-byte aligned: the device
 * copies of the five tensors, then nsa_forward's own workspace.  Errors as
 * nsa_forward, plus NSA_ERR_INVALID_ARG for a NULL host pointer and
 * NSA_ERR_CUDA if a copy cannot be enqueued. */
nsa_status nsa_forward_host_workspace_size(const nsa_params* p, size_t* bytes);
nsa_status nsa_forward_host(const nsa_params* p, const void* q, const void* k,
                            const void* v, const float* gates, void* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ---- decode ----------------------------------------------------------------
 * One query per sequence at position T-1 (p->Tq must be 1) against caches
 * k_cache/v_cache [B, T, Hkv, D] that already hold that position, and the
 * compressed caches kc_cache/vc_cache [B, Nc, Hkv, D] (nsa_compress of the
 * caches).  q [B, 1, Hq, D], gates [B, 1, Hq, 3], out [B, 1, Hq, D];
 * idx_out [B, 1, Hkv, topk] may be NULL (it is written only when the
 * selection branch is enabled).  Same arithmetic as nsa_forward for that
 * one position.  For bf16, block 64, at most 16 query heads per KV group
 * and at most 512 compressed blocks, decode runs as three kernels that
 * stream the caches across all SMs (compression + scores + top-k per
 * sequence; one small CTA per selected or window block; a merge); other
 * shapes reuse the prefill kernels.  Passage: as nsa_forward, for the one
 * query a generation step adds ("DeepSeek's Native Sparse Attention",
 * kernel paragraph: the same block-grouped reads serve training and
 * inference; "Sparsity is Cool", TL;DR and Key claims: branch pruning at
 * inference).  idx_out is an addition of this ABI: the decode's block
 * selection, returned so a caller can inspect or reuse it. */
nsa_status nsa_decode(const nsa_params* p, const void* q, const void* k_cache,
                      const void* v_cache, const void* kc_cache,
                      const void* vc_cache, const float* gates, void* out,
                      int32_t* idx_out, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ========================================================================
 * Backward.  Gradients are float32 and ACCUMULATED (+=) by the branch calls
 * so that branches can be summed; nsa_backward overwrites its outputs.
 *   dO_* (branch upstream gradients)  [B, Tq, Hq, D]  float32
 *   dq                                 [B, Tq, Hq, D]  float32
 *   dk, dv                             [B, T, Hkv, D]  float32
 *   dgates                             [B, Tq, Hq, 3]  float32
 * No gradient flows through the discrete top-k: the selection (idx) of the
 * forward is an input.  Every gradient element is produced by one thread
 * in a fixed order (no atomics on gradients), so results are deterministic.
 * ======================================================================== */

/* Bytes of workspace nsa_backward needs (the branch backward calls need no
 * more than this). */
nsa_status nsa_backward_workspace_size(const nsa_params* p, size_t* bytes);

/* ---- gated combination backward --------------------------------------------
 * dgates[.., i] = dout . o_i for enabled branches (0 otherwise) and
 * dO_i = gate_i * dout (any dO_i may be NULL).  Passage: "DeepSeek's Native
 * Sparse Attention" (gated merge of the three outputs).  dout, o_* dtype. */
nsa_status nsa_gate_combine_bwd(const nsa_params* p, const float* gates,
                                const void* dout, const void* o_cmp,
                                const void* o_sel, const void* o_swa,
                                float* dgates, float* dO_cmp, float* dO_sel,
                                float* dO_swa, void* stream);

/* ---- selection backward, two passes ----------------------------------------
 * "Sparsity is Cool", Method and Key claims: a query-stationary pass computes
 * dQ over each query's selected blocks; a reverse block->query map is
 * rebuilt from idx (counting sort, queries in ascending order, no atomics on
 * data); a key-stationary pass then computes dK/dV of each block over the
 * queries that selected it.  o_sel, lse_sel are the forward's outputs.
 * workspace: at least nsa_backward_workspace_size(p) bytes, 256-aligned. */
nsa_status nsa_sel_attn_bwd(const nsa_params* p, const void* q, const void* k,
                            const void* v, const int32_t* idx, const void* o_sel,
                            const float* lse_sel, const float* dO_sel, float* dq,
                            float* dk, float* dv, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---- selection backward, single pass with atomics ----------------------------
 * The alternative "Sparsity is Cool", Method and Key claims, compare the
 * two-pass kernel against: one query-stationary pass computes dQ over each
 * query's selected blocks and, in the same kernel, each block's dK / dV
 * contribution from the query tile, added to dk / dv with atomics
 * (contention where many queries share a key: the pages report the two-pass
 * form faster).  Same arguments and results as nsa_sel_attn_bwd (dq, dk, dv
 * accumulated, +=), except that dk / dv depend on the order in which the
 * atomics land (equal to the two-pass results up to fp32 rounding, not bit
 * for bit).  bf16, 64-key blocks only (NSA_ERR_UNSUPPORTED otherwise);
 * workspace: nsa_backward_workspace_size(p) bytes, 256-byte aligned. */
nsa_status nsa_sel_attn_bwd_atomic(const nsa_params* p, const void* q, const void* k,
                                   const void* v, const int32_t* idx, const void* o_sel,
                                   const float* lse_sel, const float* dO_sel, float* dq,
                                   float* dk, float* dv, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ---- sliding-window backward (same two-pass shape; the reverse map of key
 * s is the query range [s, s + w - 1]).  Passage: "DeepSeek's Native Sparse
 * Attention", SLIDING WINDOW. */
nsa_status nsa_swa_bwd(const nsa_params* p, const void* q, const void* k,
                       const void* v, const void* o_swa, const float* lse_swa,
                       const float* dO_swa, float* dq, float* dk, float* dv,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ---- compression-branch backward: gradients reach kc/vc and, through the
 * mean pool, each raw row of a block (d kc_j / d k_t = 1/l).  dk, dv are
 * the RAW key/value gradients [B, T, Hkv, D].  Passage: "Sparsity is Cool",
 * Key claims (the compression scores receive direct gradient through the
 * gated combination; mean-pooling as the compressor). */
nsa_status nsa_cmp_bwd(const nsa_params* p, const void* q, const void* kc,
                       const void* vc, const void* o_cmp, const float* lse_cmp,
                       const float* dO_cmp, float* dq, float* dk, float* dv,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ---- whole backward ------------------------------------------------------------
 * Gradient of out = nsa_forward(q, k, v, gates) for upstream dout, with the
 * forward's saved tensors (kc, vc, o_cmp, lse_cmp for the compression branch;
 * idx, o_sel, lse_sel for selection; o_swa, lse_swa for the window; entries
 * of disabled branches may be NULL).  Overwrites dq, dk, dv, dgates.
 * Passage: "Sparsity is Cool", Method (the selection backward in two
 * passes, query-stationary dQ then key-stationary dK/dV over the reverse
 * block->query map) and Key claims (the compression branch's scores get
 * direct gradient through the gated combination; no gradient through the
 * discrete top-k); "DeepSeek's Native Sparse Attention", How Does Native
 * Sparse Attention Work? (the gated merge whose gradient gives dgates). */
nsa_status nsa_backward(const nsa_params* p, const void* q, const void* k,
                        const void* v, const float* gates, const void* dout,
                        const nsa_saved* saved, float* dq, float* dk, float* dv,
                        float* dgates, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ========================================================================
 * Parametric compression: NSA's own compressor.
 * "DeepSeek's Native Sparse Attention", COMPRESSION (a small learned layer
 * turns each block of keys / values into one compressed key / value; blocks
 * of length l every d tokens) and "Sparsity is Cool", Method and Key claims
 * (the study replaces it with mean-pooling).  The pages give no shape for
 * the layer: this is the plainest reading, one linear map over the block's
 * l rows flattened in token order, shared by every sequence, block and KV
 * group:
 *   kc[b, j, g, n] = sum_{i<l} sum_{e<D} k[b, j*d + i, g, e] * wk[i*D + e, n]
 * and vc likewise with wv.  wk, wv: [l*D, D] row-major, the dtype of k
 * (bf16 only here; NSA_ERR_UNSUPPORTED otherwise).  Mean-pooling is the
 * special case wk[i*D + e, n] = (e == n) / l.  The products accumulate in
 * fp32 on the tensor cores; kc, vc are stored as bf16.  The whole-path
 * entries below run NSA with this compressor in place of the mean pool.
 * ======================================================================== */

/* kc, vc [B, Nc, Hkv, D] from k, v [B, T, Hkv, D] and the weights.
 * workspace: nsa_compress_mlp_workspace_size(p) bytes, 256-byte aligned
 * (fp32 partial sums when the blocks alone would leave SMs idle; it may be
 * 0, and then workspace may be NULL). */
nsa_status nsa_compress_mlp_workspace_size(const nsa_params* p, size_t* bytes);
nsa_status nsa_compress_mlp(const nsa_params* p, const void* k, const void* v,
                            const void* wk, const void* wv, void* kc, void* vc,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Gradient of nsa_compress_mlp for upstream dkc, dvc (fp32 [B, Nc, Hkv, D]):
 *   dwk[i*D + e, n] = sum over (b, j, g) of k[b, j*d + i, g, e] dkc[b, j, g, n]
 * (overwritten; dwv likewise, both fp32 [l*D, D]) and the raw rows'
 *   dk[b, j*d + i, g, e] += sum_n wk[i*D + e, n] dkc[b, j, g, n]
 * summed, in block order, over every block j holding the row (dk, dv fp32
 * [B, T, Hkv, D], ADDED to).  dkc, dvc enter the tensor cores as a bf16
 * pair (value and remainder), so they are carried to about 16 bits.
 * workspace: nsa_compress_mlp_bwd_workspace_size(p) bytes, 256-byte aligned. */
nsa_status nsa_compress_mlp_bwd_workspace_size(const nsa_params* p, size_t* bytes);
nsa_status nsa_compress_mlp_bwd(const nsa_params* p, const void* k, const void* v,
                                const void* wk, const void* wv, const float* dkc,
                                const float* dvc, float* dk, float* dv, float* dwk,
                                float* dwv, void* workspace, size_t workspace_bytes,
                                void* stream);

/* nsa_forward with kc, vc from nsa_compress_mlp.  Same arguments and saved
 * tensors as nsa_forward; workspace: nsa_forward_mlp_workspace_size(p)
 * bytes, 256-byte aligned (nsa_forward's plus the compressor's). */
nsa_status nsa_forward_mlp_workspace_size(const nsa_params* p, size_t* bytes);
nsa_status nsa_forward_mlp(const nsa_params* p, const void* q, const void* k,
                           const void* v, const void* wk, const void* wv,
                           const float* gates, void* out, const nsa_saved* saved,
                           void* workspace, size_t workspace_bytes, void* stream);

/* nsa_backward for nsa_forward_mlp: also overwrites dwk, dwv (fp32 [l*D, D];
 * zero when the compression branch is off, as top-k passes no gradient) and
 * adds the compressor's share to dk, dv.  saved must hold the kc, vc that
 * nsa_forward_mlp wrote.  workspace: nsa_backward_mlp_workspace_size(p)
 * bytes, 256-byte aligned. */
nsa_status nsa_backward_mlp_workspace_size(const nsa_params* p, size_t* bytes);
nsa_status nsa_backward_mlp(const nsa_params* p, const void* q, const void* k,
                            const void* v, const void* wk, const void* wv,
                            const float* gates, const void* dout,
                            const nsa_saved* saved, float* dq, float* dk, float* dv,
                            float* dwk, float* dwv, float* dgates, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ========================================================================
 * MoBA block attention on the same selection kernels.
 * "Sparsity is Cool: Reverse-Engineering MoBA and NSA", Method (MoBA with
 * block 512 and top-k 3) and Key claims (dense below about 1.5k tokens);
 * "DeepSeek's Native Sparse Attention" newsletter, MoBA section (the
 * context in blocks, a top-k gate sending each query to its most relevant
 * past blocks, causal protection).  Per (query at t, KV group g):
 *   cur = t / L.  With cur + 1 <= k all blocks 0..cur are read.  Otherwise
 *   the gate of each complete past block j < cur is the sum over the
 *   group's query heads h of q_h . mean(k of block j); the k - 1 best gates
 *   (equal gates: lower block) and the query's own block are read.  The
 *   pages do not say how the gate is formed or shared under GQA: this is the
 *   plainest reading (the block's mean-pooled key, one selection per KV
 *   group as in NSA's selection).
 * out[t, h] = softmax attention of q_h over the keys s <= t of the chosen
 * blocks (no gates, no other branch); lse its log-sum-exp.
 * ======================================================================== */
typedef struct {
  int B, T, Tq, Hq, Hkv, D; /* as in nsa_params (D = 64)                      */
  int block;                /* L: tokens per MoBA block, a multiple of 64     */
  int topk;                 /* k: blocks per (query, KV group), own included  */
  float scale;              /* softmax scale, finite and > 0                  */
  int dtype;                /* nsa_dtype of q, k, v, out                      */
} nsa_moba_params;

/* Workspace bytes of nsa_moba_forward and nsa_moba_backward.  Limits: T / L
 * <= 128 MoBA blocks, k L / 64 <= 64, T <= 65536 (else NSA_ERR_UNSUPPORTED). */
nsa_status nsa_moba_workspace_size(const nsa_moba_params* p, size_t* bytes);

/* q [B, Tq, Hq, D], k, v [B, T, Hkv, D] -> out [B, Tq, Hq, D] (dtype),
 * lse [B, Tq, Hq] f32 (may be NULL), idx [B, Tq, Hkv, k] int32 (the chosen
 * MoBA blocks, ascending, -1 padded; may be NULL).  The blocks are read as
 * 64-key selection blocks by the selection attention kernels. */
nsa_status nsa_moba_forward(const nsa_moba_params* p, const void* q, const void* k,
                            const void* v, void* out, float* lse, int32_t* idx,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Gradients (float32, overwritten) of out for upstream dout [B, Tq, Hq, D]
 * (float32), the forward's idx, out and lse held fixed (no gradient through
 * the discrete gate): the two-pass selection backward on the chosen blocks. */
nsa_status nsa_moba_backward(const nsa_moba_params* p, const void* q, const void* k,
                             const void* v, const int32_t* idx, const void* out,
                             const float* lse, const float* dout, float* dq, float* dk,
                             float* dv, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ---- decode without any allocation by the caller ---------------------------
 * No counterpart in the paper: this is a deployment variant of nsa_decode.
 * Some callers cannot allocate device memory -- for example a plugin that
 * its host framework hands only input and output buffers, or a runtime that
 * serves from a fixed memory pool with no allocation hook -- so they cannot
 * provide nsa_decode's workspace.  This entry point takes the same
 * arguments as nsa_decode minus the workspace and runs the same kernels,
 * with the scratch taken from a fixed array inside the library's device
 * memory (nsa_decode_noalloc_max_scratch() bytes, 16 MiB, held on every GPU
 * that loads the library until the process exits).  It allocates nothing.
 * A problem whose scratch would not fit returns NSA_ERR_SCRATCH_TOO_SMALL
 * before anything is launched (B=64 sequences, 16 heads on one KV head,
 * 32768-token caches, top-k 16, window 512 need about 11 MiB).  Every call
 * looks up the array's device address in the current context (the caller's
 * device must be current); the first lookup on a device may load the
 * library's device code, so make the first call before any stream capture.
 * All calls on a device share the array and it keeps the previous call's
 * contents (a call reads only scratch it has written itself, so nothing
 * needs clearing); calls that overlap on the GPU race on it, so order them
 * on one stream.  As for every entry point, out and idx_out are undefined
 * if nsa_last_device_error() then reports an error. */
nsa_status nsa_decode_noalloc(const nsa_params* p, const void* q,
                              const void* k_cache, const void* v_cache,
                              const void* kc_cache, const void* vc_cache,
                              const float* gates, void* out, int32_t* idx_out,
                              void* stream);

/* Size in bytes of nsa_decode_noalloc's fixed scratch array. */
size_t nsa_decode_noalloc_max_scratch(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H_ */
