/*
 * stem.h: C ABI of the B200 (sm_100a) library for Stem block-sparse causal prefill.
 *
 * The method: "Stem: Rethinking Causal Information Flow in Sparse Attention"
 * (arXiv 2603.06274). Passages are cited by page and section:
 *   [es] gist.science/es, "Resumen tecnico"        [it] gist.science/it, "Sommario tecnico"
 *   [nl] gist.science/nl, "Technische samenvatting" [fr] gist.science/fr, "Resume technique"
 *   [zh] shd-paper.top index page (English abstract, "key design" paragraph)
 *
 * Problem ([es] 1, [it] 1, [nl] Probleemstelling, [zh] abstract): causal prefill
 * attention over Q, K, V in which each query block attends only to a kept set of
 * key blocks. The pages leave the budget schedule and the pooling open; this
 * library fixes them as parameters:
 *   nb = ceil(S / block), query block i in [0, nb);
 *   rho(i) = rho_min + (1 - rho_min) * exp(-i / tau);
 *   k(i)   = min(i+1, max(k_min, ceil(rho(i) * (i+1)))), raised to 2 for i >= 1, k(0) = 1;
 *   pooled qbar_i, kbar_j = mean of the block's rows; n_j = mean of the block's V-row L2 norms;
 *   m_ij   = softmax_{j<=i}(qbar_i . kbar_j / sqrt(D)) * n_j;
 *   kept(i) = {0, i} plus the k(i)-2 best j in [1, i-1] by (m_ij descending, j ascending);
 *   out[r] = softmax attention of query token r over every token of kept(i), token-causal
 *            inside block i, logits scaled by 1/sqrt(D).
 * The pages' own parameterisations are selectable per call (stem_method_t below): the linear
 * budget k(i) = ceil(k_start * (1 - (1 - mu) * i/(nb-1))) ([es] 2.A, [it] 2.A, [nl] TPD,
 * [fr] 2.A), the additive metric s_ij + beta * max(0, log n_j^2) ([es] 2.B, [it] 2.B, [nl] OAM,
 * [fr] 2.B) and the largest V-row norm as n_j ([nl] Implementatie step 1).
 *
 * Conventions shared by every call:
 *   - Tensors are contiguous [B, H, S, D] (row-major, D fastest). Q and out have Hq heads, K and
 *     V have Hkv heads; query head h reads key/value head h / (Hq / Hkv).
 *   - dtype: STEM_BF16 (bfloat16) or STEM_F32 (float32); out has the input dtype.
 *   - Device pointers must be 16-byte aligned (int32 arrays: 4-byte aligned). All buffers are
 *     owned by the caller; the library never frees or retains them past the call.
 *   - CSR layout of the kept blocks: row (b, h, i) occupies
 *       sel_idx[(b*Hq + h)*cap + off(i) .. + k(i)), ascending block indices,
 *     with off(i) = k(0) + ... + k(i-1) and cap = off(nb) (stem_sel_capacity); sel_cnt[b,h,i] = k(i).
 *   - Supported shapes: D in {64, 128}; block in {64, 128}; Hq % Hkv == 0; any S >= 0, with
 *     nb = ceil(S / block) <= STEM_MAX_NB. When S is not a multiple of block the last block
 *     holds the S - (nb-1)*block remaining tokens: it is pooled over those rows only, and
 *     out rows past S are never written. B == 0 or S == 0 is an empty problem: success,
 *     nothing launched.
 *   - Device calls are asynchronous on the given stream: a 0 return means the work was enqueued.
 *     Faults surface at the caller's next synchronisation. The library never prints or aborts.
 *   - Arguments are validated before anything is enqueued; on a negative return nothing was
 *     launched and no buffer was written.
 *   - Host state: the budget plan of each distinct (nb, schedule parameters, k_min) is built on
 *     first use and kept in pinned host memory for the life of the process (3*nb + 1 int32 per
 *     plan, shared by all threads under a lock). Plans are never freed, since a copy enqueued
 *     from one may still be in flight; a caller with many distinct sequence lengths holds one
 *     plan per length.
 */
#ifndef STEM_H
#define STEM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define STEM_OK 0
#define STEM_ERR_ARG (-1)         /* bad argument: null/misaligned pointer, bad shape or parameter */
#define STEM_ERR_WORKSPACE (-2)   /* workspace missing or smaller than stem_workspace_size() */
#define STEM_ERR_CUDA (-3)        /* a CUDA call failed (launch error, no device, no sm_100a) */
#define STEM_ERR_TIMEOUT (-4)     /* a device-side wait exceeded its bound (reported via status) */
#define STEM_ERR_UNSUPPORTED (-5) /* valid request beyond this build's limits (e.g. nb > STEM_MAX_NB) */

/* Element types. */
#define STEM_BF16 0
#define STEM_F32 1

/* Budget schedules, metrics and V summaries of stem_method_t. */
#define STEM_SCHED_EXP 0       /* rho(i) = rho_min + (1 - rho_min) exp(-i / tau) (the default) */
#define STEM_SCHED_LINEAR 1    /* k_start at block 0 down to mu * k_start at block nb-1 */
#define STEM_METRIC_PRODUCT 0  /* m_ij = softmax_j(s_ij) * n_j (the default) */
#define STEM_METRIC_ADDITIVE 1 /* M_ij = s_ij + beta * max(0, log n_j^2) */
#define STEM_VSUM_MEAN 0       /* n_j = mean of the block's V-row L2 norms (the default) */
#define STEM_VSUM_MAX 1        /* n_j = largest V-row L2 norm of the block */
#define STEM_SHARE_HEAD 0      /* one selection per query head (the default) */
#define STEM_SHARE_GROUP 1     /* one selection per kv-head group, shared by its query heads */
#define STEM_SCORE_POOLED 0    /* block scores from mean-pooled Q and K (the default) */
#define STEM_SCORE_ANTIDIAG 1  /* block probabilities by anti-diagonal sampling */

/*
 * Method parameters: budget schedule, block metric and V summary.
 *   STEM_SCHED_EXP:     k(i) = min(i+1, max(k_min, ceil(rho(i) * (i+1)))), rho as above;
 *                       rho_min in (0, 1], tau > 0 and finite.
 *   STEM_SCHED_LINEAR:  k(i) = min(i+1, max(k_min, ceil(k_start * (1 - (1 - mu) * t)))),
 *                       t = i / (nb - 1) (0 when nb == 1), in double precision from the float
 *                       parameters; k_start > 0 and finite (blocks), mu in (0, 1].
 *   Both: k(0) = 1 and k(i) >= 2 for i >= 1 (sink and diagonal); k_min >= 1.
 *   STEM_METRIC_PRODUCT:  rank by s_ij + ln n_j (= log m_ij + const).
 *   STEM_METRIC_ADDITIVE: rank by s_ij + beta * e_j, e_j = 2 ln n_j, clamped at 0 when clamp is
 *                         1; beta >= 0 and finite (beta == 0: e_j is not evaluated, so
 *                         n_j = 0 is allowed); clamp in {0, 1}.
 *   vsum: STEM_VSUM_MEAN or STEM_VSUM_MAX (pooling of ||V row|| into n_j).
 *   share: STEM_SHARE_HEAD, or STEM_SHARE_GROUP: the G = Hq/Hkv query heads of a kv-head group
 *          keep one list, chosen by the metric summed over them (product: n_j * sum_h p_hij,
 *          ranked in log space; additive: sum_h s_hij + G * beta * e_j) and written to each
 *          head's CSR row. The pages are silent on GQA; this is an alternative reading. With
 *          share = GROUP and G > 1, nb beyond 1024 returns STEM_ERR_UNSUPPORTED.
 *   score: STEM_SCORE_POOLED (s_ij from the pooled Q and K above), or STEM_SCORE_ANTIDIAG: the
 *          block probability p_ij comes from anti-diagonal sampling ([fr] 2.C step 1: block
 *          metrics "with anti-diagonal sampling"; the pages give no formula, this is the
 *          reading used). Tokens form groups of `stride` consecutive tokens; query group u and
 *          key group w are scored by the mean of the anti-diagonal samples of their
 *          stride x stride logit sub-tile,
 *            a_uw = (1/stride) sum_t Q[u*stride+t] . K[w*stride+stride-1-t] / sqrt(D),
 *          each query group takes a softmax over w <= u, and p_ij is the mass the query groups
 *          of block i put on the key groups of block j, averaged over those query groups.
 *          ln p_ij then takes the place of s_ij - logsumexp_j s_ij in the metric (product:
 *          rank by ln p_ij + ln n_j; additive: ln p_ij + beta * e_j; group share: the summed
 *          metric as above). Requires bfloat16 inputs (else STEM_ERR_UNSUPPORTED), a power-of-two
 *          stride with block % stride == 0, block / stride <= 32 and S % stride == 0 (else
 *          STEM_ERR_ARG). The sampled products run on the tensor cores (bf16 in, fp32
 *          accumulation); it costs about 1/stride of a dense causal Q K^T.
 * Fields the chosen schedule and metric do not use are ignored. Zero-initialise the struct
 * (score 0 = pooled) before setting fields.
 */
typedef struct stem_method {
  int32_t schedule;
  float rho_min;
  float tau;
  float k_start;
  float mu;
  int32_t k_min;
  int32_t metric;
  float beta;
  int32_t clamp;
  int32_t vsum;
  int32_t share;
  int32_t score;
  int32_t stride; /* STEM_SCORE_ANTIDIAG only */
} stem_method_t;

/* Largest number of blocks per sequence (the selection kernel keeps one score row per
 * query block in shared memory). */
#define STEM_MAX_NB 4096

/*
 * Full argument set of one prefill. Sizes are element counts.
 *   q   [B,Hq,S,D], k, v [B,Hkv,S,D]      inputs (device, or host for stem_prefill_host)
 *   out [B,Hq,S,D]                         output, same dtype as the inputs
 *   sel_idx [B,Hq,cap] int32, sel_cnt [B,Hq,nb] int32   kept blocks (CSR, see above)
 *   workspace / workspace_bytes            device scratch of at least stem_workspace_size() bytes,
 *                                          256-byte aligned; ignored by stem_prefill_host
 *   status                                 optional device int32: set to 0 when the call is
 *                                          enqueued, to a negative STEM_ERR_* by a kernel that
 *                                          fails a bounded device-side wait; NULL to skip
 *   events                                 optional: 4 cudaEvent_t (as void*) recorded on the
 *                                          stream before pooling, before selection, before
 *                                          attention and after attention (per-stage timing);
 *                                          NULL to skip
 *   method                                 optional method parameters (stem_method_t)
 */
typedef struct stem_args {
  const void* q;
  const void* k;
  const void* v;
  int32_t B, Hq, Hkv, S, D, block;
  float rho_min; /* in (0, 1] */
  float tau;     /* decay length in blocks, > 0 and finite */
  int32_t k_min; /* >= 1 */
  int32_t dtype; /* STEM_BF16 or STEM_F32 */
  void* out;
  int32_t* sel_idx;
  int32_t* sel_cnt;
  void* workspace;
  size_t workspace_bytes;
  int32_t* status;
  void* const* events;
  /* optional: NULL keeps the exponential schedule of rho_min, tau and k_min above, the product
   * metric and mean-pooled V norms; otherwise it sets every method parameter and rho_min, tau
   * and k_min above are ignored */
  const stem_method_t* method;
} stem_args_t;

/*
 * The whole hot path ([es] 2 "Implementacion" steps 1-3, [it] 2.C, [nl] Implementatie,
 * [fr] 2.C): block pooling, budget, metric and selection, block-sparse attention.
 * bfloat16 device tensors, the default stream, and a workspace the library allocates on first
 * use and keeps per device (grow-only, freed at process exit). Returns STEM_OK or STEM_ERR_*.
 */
int stem_prefill(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int S,
                 int D, int block, float rho_min, float tau, int k_min, void* out,
                 int32_t* sel_idx, int32_t* sel_cnt);

/* Same as stem_prefill with every argument explicit: dtype, caller workspace, status word, and
 * the CUDA stream (a cudaStream_t passed as void*; NULL = legacy default stream). */
int stem_prefill_ex(const stem_args_t* a, void* stream);

/* stem_prefill_ex for HOST buffers (q, k, v, out, sel_idx, sel_cnt in host memory; pinned
 * memory gives the fastest copies). Copies inputs to the device, runs the path on an internal
 * stream and workspace, copies out, sel_idx and sel_cnt back, and returns after they have
 * arrived. a->workspace and a->status are ignored. */
int stem_prefill_host(const stem_args_t* a);

/*
 * Token Position-Decay budget ([es] 2.A, [it] 2.A, [nl] TPD, [fr] 2.A; exponential decay:
 * [zh] key design). Host only. Writes k_out[nb] = k(i) and off_out[nb+1] = prefix sums into
 * host arrays (either may be NULL). Returns 0, or STEM_ERR_ARG for nb < 0, rho_min outside (0, 1],
 * tau <= 0 or not finite, k_min < 1, or a total that overflows int32.
 */
int stem_budget(int nb, float rho_min, float tau, int k_min, int32_t* k_out, int32_t* off_out);

/* cap = sum_i k(i): the per-(b, h) stride of sel_idx. Host only. Negative STEM_ERR_ARG on bad
 * parameters. */
int64_t stem_sel_capacity(int nb, float rho_min, float tau, int k_min);

/* Bytes of device workspace stem_prefill_ex needs for this shape (pooled summaries, the budget
 * plan and the status word). 0 for an invalid or empty shape. Host only. */
size_t stem_workspace_size(int B, int Hq, int Hkv, int S, int D, int block);

/* Static description of a return code. Never NULL. */
const char* stem_strerror(int code);

/* ---------------------------------------------------------------------------------------
 * Stage entry points: the same kernels the full path launches, one at a time. They exist so
 * each stage can be checked on its own; the device layout of every intermediate is fixed here.
 * --------------------------------------------------------------------------------------- */

/*
 * Block downsampling ([es] 2 "Implementacion" step 1, [it] 2.C step 1, [nl] Implementatie
 * step 1, [fr] 2.C step 1), mean pooling. Writes (device, float32):
 *   qbar [B,Hq,nb,D]  = mean of the block's Q rows,
 *   kbar [B,Hkv,nb,D] = mean of the block's K rows,
 *   vnorm [B,Hkv,nb]  = mean over the block's rows of ||V row||_2.
 * Accumulation is float32 in a fixed tree order (deterministic).
 */
int stem_pool(const void* q, const void* k, const void* v, int dtype, int B, int Hq, int Hkv,
              int S, int D, int block, float* qbar, float* kbar, float* vnorm, void* stream);

/*
 * Output-Aware Metric and variable-k selection ([es] 2.B and 2 "Implementacion" step 3,
 * [it] 2.B, [nl] OAM, [fr] 2.B; sink retention: [es] 1, [zh] abstract). From pooled summaries
 * (device float32, layouts of stem_pool) writes the CSR kept-block lists sel_idx / sel_cnt.
 * Ranking uses log m_ij + const = s_ij + ln n_j with s_ij from a float32 dot product, compared
 * in double; ties go to the lower block index.
 * m_out: optional (NULL to skip) float32 [B,Hq,nb*(nb+1)/2], row i at offset i*(i+1)/2, the
 * metric m_ij for j <= i (softmax over j <= i in float32).
 * workspace: as for stem_prefill_ex. Given stem_workspace_size bytes, the scores s_ij of the
 * lower triangle are written to the workspace region after the plan (a chunk of heads at a
 * time) and the rows are selected from there by a second kernel; given only the plan region
 * (smaller workspaces down to that size are accepted), one fused kernel computes the same
 * scores in shared memory. Both select identically.
 */
int stem_select(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                int Hkv, int nb, int D, float rho_min, float tau, int k_min, int32_t* sel_idx,
                int32_t* sel_cnt, float* m_out, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * Exact attention over the kept blocks ([es] 2 "Implementacion" step 3, [it] 2.C step 3,
 * [nl] Implementatie step 3, [fr] 2.C step 3). Reads any valid CSR with the budget's layout
 * (sel_cnt[b,h,i] must equal k(i); each row ascending, in [0, i], containing i). bfloat16 runs
 * on the tensor cores with float32 accumulation and float32 online softmax; float32 runs on the
 * CUDA cores in float32.
 */
int stem_sparse_attn(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                     int Hkv, int S, int D, int block, float rho_min, float tau, int k_min,
                     const int32_t* sel_idx, const int32_t* sel_cnt, void* out, void* workspace,
                     size_t workspace_bytes, int32_t* status, void* stream);

/*
 * Method-parameterised forms of the calls above: the same behaviour, with the schedule, metric
 * and V summary taken from m (see stem_method_t) instead of (rho_min, tau, k_min). m must not
 * be NULL; an invalid field returns STEM_ERR_ARG. stem_pool_m reads only m->vsum.
 */
int stem_budget_m(int nb, const stem_method_t* m, int32_t* k_out, int32_t* off_out);
int64_t stem_sel_capacity_m(int nb, const stem_method_t* m);
int stem_pool_m(const void* q, const void* k, const void* v, int dtype, int B, int Hq, int Hkv,
                int S, int D, int block, const stem_method_t* m, float* qbar, float* kbar,
                float* vnorm, void* stream);
/* m_out holds the metric of the chosen form: m_ij (product) or M_ij (additive), float32. */
int stem_select_m(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                  int Hkv, int nb, int D, const stem_method_t* m, int32_t* sel_idx,
                  int32_t* sel_cnt, float* m_out, void* workspace, size_t workspace_bytes,
                  void* stream);
int stem_sparse_attn_m(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                       int Hkv, int S, int D, int block, const stem_method_t* m,
                       const int32_t* sel_idx, const int32_t* sel_cnt, void* out,
                       void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/* Workspace bytes stem_prefill_ex needs for this shape and method. With STEM_SCORE_ANTIDIAG it
 * also holds the block probabilities (4 * B * Hq * nb * (nb+1) / 2 bytes) and the estimator's
 * partials, per head 4 * (R*nb*(nb+1)/2 + c*n - 32*c*(c-1)/2 + 256*t*parts) bytes with
 * n = S/stride groups, R = block/stride, c = ceil(n/32), t = ceil(n/128) and
 * parts = ceil(ceil(n/256)/4) (about 690 MB at S = 131072, block 128, stride 16, B*Hq = 32).
 * 0 for an invalid or empty request. Host only. */
size_t stem_workspace_size_m(int B, int Hq, int Hkv, int S, int D, int block,
                             const stem_method_t* m);

/*
 * Block probabilities by anti-diagonal sampling (score STEM_SCORE_ANTIDIAG of stem_method_t;
 * [fr] 2.C step 1). Reads bfloat16 q [B,Hq,S,D] and k [B,Hkv,S,D] (device, 16-byte aligned)
 * and writes p (device float32 [B,Hq,nb*(nb+1)/2], row i at offset i*(i+1)/2, p_ij for j <= i;
 * each row sums to 1 up to rounding). m->stride must satisfy the stem_method_t rules (m->score
 * is not read). workspace: stem_workspace_size_m bytes for a method with this stride; status
 * as in stem_args_t.
 */
int stem_antidiag_m(const void* q, const void* k, int dtype, int B, int Hq, int Hkv, int S, int D,
                    int block, const stem_method_t* m, float* p, void* workspace,
                    size_t workspace_bytes, int32_t* status, void* stream);

/*
 * Variable-k selection from block probabilities p (layout of stem_antidiag_m) and the V
 * magnitudes vnorm [B,Hkv,nb] (layout of stem_pool_m): the metric of m (product, additive,
 * per head or group-shared, see stem_method_t score) ranked in double, ties to the lower block
 * index. m_out as in stem_select_m: m_ij = p_ij * n_j (product) or M_ij = ln p_ij + beta * e_j
 * (additive), the group's summed metric under group share. workspace: as for stem_select_m.
 */
int stem_select_p_m(const float* p, const float* vnorm, int B, int Hq, int Hkv, int nb,
                    const stem_method_t* m, int32_t* sel_idx, int32_t* sel_cnt, float* m_out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Variable-length batches. nseq sequences of lengths S_s = cu_seqlens[s+1] - cu_seqlens[s]
 * (cu_seqlens: host int32[nseq+1], cu_seqlens[0] = 0, non-decreasing), packed back to back, each
 * as a contiguous [H, S_s, D] slab: sequence s's Q (and out) starts at element Hq*D*cu[s], its K
 * and V at element Hkv*D*cu[s]. Every sequence is its own problem (its own nb_s = ceil(S_s/block),
 * budget, selection and attention); an empty sequence contributes nothing. The CSR of sequence s
 * is [Hq, cap_s] at sel_idx + Hq * (cap_0 + ... + cap_{s-1}), its counts [Hq, nb_s] at
 * sel_cnt + Hq * (nb_0 + ... + nb_{s-1}), cap_s = stem_sel_capacity_m(nb_s, method).
 * --------------------------------------------------------------------------------------- */
typedef struct stem_varlen_args {
  const void* q;
  const void* k;
  const void* v;
  int32_t nseq;
  const int32_t* cu_seqlens; /* host */
  int32_t Hq, Hkv, D, block;
  int32_t dtype;
  const stem_method_t* method; /* required */
  void* out;
  int32_t* sel_idx;
  int32_t* sel_cnt;
  void* workspace;             /* stem_varlen_workspace_size bytes, 256-byte aligned */
  size_t workspace_bytes;
  int32_t* status;             /* optional, as in stem_args_t: one word for the whole call */
} stem_varlen_args_t;

/* Runs the sequences one after another on the stream (the workspace is reused between them). */
int stem_prefill_varlen(const stem_varlen_args_t* a, void* stream);
/* Workspace bytes for these sequences (the largest sequence's), 0 on invalid input. Host only. */
size_t stem_varlen_workspace_size(int nseq, const int32_t* cu_seqlens, int Hq, int Hkv, int D,
                                  int block);
/* The same for a method (needed with STEM_SCORE_ANTIDIAG, whose workspace is larger). */
size_t stem_varlen_workspace_size_m(int nseq, const int32_t* cu_seqlens, int Hq, int Hkv, int D,
                                    int block, const stem_method_t* m);
/* Total CSR entries per query head: sum over the sequences of cap_s; negative STEM_ERR_* on
 * invalid input. Host only. */
int64_t stem_varlen_sel_capacity(int nseq, const int32_t* cu_seqlens, int block,
                                 const stem_method_t* m);

/*
 * stem_select_static: stem_select for callers that cannot allocate device memory. The paper
 * has no counterpart; this is an interface addition.
 *
 * Some callers cannot call cudaMalloc or hand this library a workspace (a host application
 * that owns every device allocation through its own budgeted allocator, a plugin that may not
 * allocate behind that allocator's back). This entry point allocates nothing: the selection
 * kernel's scratch, the budget plan (3*nb+1 int32), lives in a 64 KiB file-scope device array
 * that every GPU loading the library holds until the process exits. Inputs and outputs are
 * those of stem_select (no m_out). nb beyond STEM_MAX_NB returns STEM_ERR_UNSUPPORTED.
 * The first call on a device looks the array up (with that device current), and so does the
 * first call after the device's context changed (a cudaDeviceReset loads the library's device
 * code anew); make such a call before any stream capture. The plan goes to the array as the
 * launch parameters of a small kernel (no host-to-device copy, so no host buffer that a later
 * call could rewrite). All calls share the device array: calls whose kernels overlap on the GPU
 * race, so issue them in stream order. Same errors as stem_select, except that there is no
 * workspace.
 */
int stem_select_static(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                       int Hkv, int nb, int D, float rho_min, float tau, int k_min,
                       int32_t* sel_idx, int32_t* sel_cnt, void* stream);

/*
 * stem_test_withhold_q: TEST ONLY. With on != 0, later launches of the bfloat16 block-128
 * attention kernel (stem_prefill*, stem_sparse_attn*) skip each CTA's first Q tile, and later
 * launches of the anti-diagonal estimator (score STEM_SCORE_ANTIDIAG, stem_antidiag_m) skip each
 * CTA's first stage of copies, so the kernel's bounded wait for them expires (after about 2 s):
 * the kernel then records STEM_ERR_TIMEOUT in the status word, every role leaves its loop, issued
 * copies and products are drained, TMEM is freed and the kernel returns, leaving the CUDA
 * context usable. It exists to exercise that path; the outputs of such a call are undefined.
 * Process-wide; returns the previous setting (0 or 1). The paper has no counterpart.
 */
int stem_test_withhold_q(int on);

#ifdef __cplusplus
}
#endif

#endif /* STEM_H */
