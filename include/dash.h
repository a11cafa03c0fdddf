/*
 * dash.h -- C ABI of the DashAttention forward path on NVIDIA B200 (sm_100a).
 *
 * The method ("DashAttention: Differentiable and Adaptive Sparse Hierarchical
 * Attention"; gist.science technical summary, sections "Fase 0/1/2" and
 * "阶段0/1/2"; aiexpert.news article, interface paragraph) has three stages:
 *   stage 0  dash_summarize  learned-query local SDPA summary of each chunk of
 *                            B keys, cached once the chunk is complete;
 *   stage 1  dash_route      alpha-entmax(gamma * z_bar) routing of every query
 *                            over the summaries of the complete chunks before
 *                            its own, averaged over the query heads of a GQA
 *                            group, written as weights w and a bit-packed mask;
 *   stage 2  dash_attn_fwd   prior-induced sparse softmax: p_ij proportional to
 *                            g_ij exp(q_i.k_j / sqrt(d)), g = w_b^sigma on the
 *                            active routed chunks, 1 on the query's own chunk
 *                            (causal), 0 elsewhere; flash-style over the mask.
 *   decode   dash_decode     stages 1 and 2 for one new query per sequence
 *                            against a cached KV and summary cache.
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers to row-major contiguous buffers
 *     owned by the caller.  The library never allocates, frees or
 *     synchronises (except dash_get_error, which says so).  Work is enqueued on
 *     `stream` (a cudaStream_t; NULL = the legacy default stream) and runs
 *     asynchronously.
 *   - Element type of Q/K/V/Kbar/O/q/o is given by dash_problem.dtype
 *     (DASH_F32 = float, DASH_BF16 = bfloat16).  qbar, w and lse are float.
 *   - Every device pointer must be non-NULL (unless marked nullable) and
 *     16-byte aligned.
 *   - Return value: a dash_status.  Invalid arguments are rejected before any
 *     work is enqueued.  Nothing aborts, exits or prints.
 *
 * Shapes (b = batch, Hq/Hkv = query/KV heads, G = Hq/Hkv, N = seq_len,
 * d = head_dim, B = chunk, n_c = ceil(N / B), n_w = ceil(n_c / 32)):
 *   Q     [b, Hq,  N, d]          K, V [b, Hkv, N, d]
 *   qbar  [Hkv, d] float          Kbar [b, Hkv, floor(N / B), d]  (dtype of K)
 *   w     [b, Hkv, N, n_c] float  mask [b, Hkv, N, n_w] uint32:
 *                                 bit (c % 32) of word (c / 32) <=> chunk c active
 *   O     [b, Hq,  N, d]          lse  [b, Hq, N] float (natural log)
 * Query head h uses KV head h / G.
 */
#ifndef DASH_H_
#define DASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DASH_OK = 0,
  DASH_ERR_INVALID_ARG = 1,   /* NULL/misaligned pointer, bad size, bad scalar */
  DASH_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype/shape combo) */
  DASH_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
  DASH_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
  DASH_ERR_WORKSPACE = 5      /* workspace missing or smaller than required */
} dash_status;

typedef enum { DASH_F32 = 0, DASH_BF16 = 1 } dash_dtype;

typedef struct {
  int32_t batch;        /* b >= 1 */
  int32_t n_q_heads;    /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads;   /* Hkv >= 1 */
  int32_t seq_len;      /* prefill: N (multiple of chunk); decode: cache length L >= 1 */
  int32_t head_dim;     /* d in {64, 128} */
  int32_t chunk;        /* B in {64, 128} */
  float alpha;          /* entmax alpha, 1 < alpha <= 2 */
  float gamma;          /* routing logit scale, finite and > 0 */
  float sigma;          /* prior strength, finite and >= 0 */
  int32_t dtype;        /* dash_dtype */
  int32_t estimate_diagonal;  /* 0 or 1; see dash_route */
} dash_problem;

/* Human-readable name of a status code (static string, never NULL). */
const char* dash_status_str(int status);

/* ABI version of this library: (major << 16) | minor. */
int dash_version(void);

/*
 * Stage 0 -- chunk summary (gist.science summary, "Fase 0: Lokale Chunk
 * Samenvatting"): for chunks c in [chunk_begin, chunk_end),
 *   a_t = softmax_t(qbar[h] . K[b, h, cB + t] / sqrt(d)),  t < B,
 *   Kbar[b, h, c] = sum_t a_t K[b, h, cB + t]      (fp32 accumulation,
 *                                                  stored in the dtype of K).
 * qbar = 0 gives mean pooling.  Only rows [chunk_begin, chunk_end) of Kbar
 * are written, so a decoder can append one finished chunk at a time.
 * Requires 0 <= chunk_begin <= chunk_end <= floor(seq_len / chunk).
 */
int dash_summarize(const dash_problem* p, const void* K, const float* qbar,
                   int chunk_begin, int chunk_end, void* Kbar, void* stream);

/*
 * Summary-cache append for incremental decoding (gist.science summary, Fase 0
 * "Efficiëntie": a chunk's summary is fixed once the chunk is complete and is
 * cached).  p->seq_len is the caches' capacity L_max; cache_lens (device
 * int32 [b], 4-byte aligned) the sequences' current lengths.  Every sequence
 * bi whose length L_b is a multiple of B has just completed chunk
 * c = L_b / B - 1: Kbar[bi, :, c] is written, with the same arithmetic (and so
 * the same bits) as dash_summarize over that chunk.  Other sequences' rows are
 * not touched.
 *   K: the key cache [b, Hkv, L_max, d], or with page_table (device int32
 *   [b, max_pages], 4-byte aligned, max_pages >= ceil(L_max / B)) the page
 *   pool [n_pages, Hkv, B, d] of dash_decode_paged.  qbar [Hkv, d] fp32;
 *   Kbar [b, Hkv, floor(L_max / B), d], dtype of K.
 * Errors: NULL/misaligned pointers, bad problem, max_pages or n_pages ->
 * DASH_ERR_INVALID_ARG.  Lengths and page ids are read on the device: a
 * sequence whose length or page id is out of range is skipped and the next
 * dash_get_error returns DASH_ERR_INVALID_ARG.
 */
int dash_summarize_append(const dash_problem* p, const int32_t* cache_lens,
                          const int32_t* page_table, int max_pages, int n_pages, const void* K,
                          const float* qbar, void* Kbar, void* stream);

/*
 * Stage 1 -- entmax chunk routing (gist.science summary, "Fase 1: Entmax
 * Chunk Routering"; aiexpert.news, threshold paragraph).  For every query
 * position i, c_i = floor(i / B), and eligible chunks c < c_i:
 *   z[h, c] = Q[b, h, i] . Kbar[b, h / G, c]
 *   p[h]    = alpha-entmax(gamma z[h])
 *           = [(alpha - 1) gamma z[h, c] - tau_h]_+ ^ (1 / (alpha - 1)), sum = 1
 *   w[b, g, i, c] = mean of p over the G query heads of KV head g
 *   mask bit      = (w > 0), i.e. the union of the member supports.
 * Entries for c >= c_i are written as 0.  Requires n_c <= 2048.
 *
 * p->estimate_diagonal = 1 (aiexpert.news, interface paragraph: a flag for a
 * diagonal correction of the alpha-entmax normalisation; gist.science
 * summary, Fase 2 "Diagonaal Afhandeling": the chunk on the diagonal has no
 * summary yet): the query's own chunk c_i joins the entmax as one more
 * candidate, z[h, c_i] = Q[b, h, i] . Khat_i, where Khat_i is stage 0's
 * learned-query summary of the keys K[b, g, c_i B .. i] (the part of the
 * chunk the query sees), computed here in fp32 and not stored.  Its group
 * mean goes to w[b, g, i, c_i] (so the routed chunks share 1 - w[.., c_i]);
 * mask bit c_i stays clear: stage 2 attends to the query's own chunk with
 * weight 1 whatever w[.., c_i] is.  Rows of the first chunk get
 * w[.., 0] = 1.  K [b, Hkv, N, d] (dtype of Q) and qbar [Hkv, d] fp32 are
 * then required (16-byte aligned); with estimate_diagonal = 0 they are
 * ignored and may be NULL.
 */
int dash_route(const dash_problem* p, const void* Q, const void* Kbar, const void* K,
               const float* qbar, float* w, uint32_t* mask, void* stream);

/*
 * Stage 1 with its weights in compact form: for each row, only the routed
 * chunks, in increasing chunk order (gist.science summary, Fase 2
 * "Implementatie": the attention kernel walks the active chunks of a
 * bit-packed mask and adds the routing bias).  Same routing as dash_route
 * (estimate_diagonal included; the query's own chunk is not a routed
 * chunk and is not listed); instead of the dense w it writes
 *   mask   [b, Hkv, N, n_w] uint32, as dash_route;
 *   weight [b, Hkv, N, n_c] float: entry k of a row is the weight of the
 *          chunk of the k-th set bit of the row's mask;
 *   count  [b, Hkv, N] int32 (nullable): the number of set bits of the row;
 *   index  [b, Hkv, N, n_c] int32 (nullable): entry k is that chunk.
 * Only the first count entries of a row of weight and index are written;
 * the rest of the row is left as it was.  A row's bytes written are thus
 * proportional to its support, not to n_c.  dash_attn_fwd_packed reads
 * (weight, mask).  Errors: as dash_route (count/index misaligned ->
 * DASH_ERR_INVALID_ARG).
 */
int dash_route_packed(const dash_problem* p, const void* Q, const void* Kbar, const void* K,
                      const float* qbar, uint32_t* mask, int32_t* count, int32_t* index,
                      float* weight, void* stream);

/*
 * Fixed-budget top-k routing on the same summaries: the baseline the pages
 * contrast with (gist.science summary, "Probleemstelling": NSA and
 * InfLLMv2 select the top-k KV blocks by coarse attention scores, then run
 * softmax attention on the selected tokens).  For every query position i and
 * KV head, over the eligible chunks c < floor(i / B): score_c = mean over the
 * G query heads of softmax_c(gamma q_h . Kbar_c); the k best chunks (equal
 * scores: lower chunk index first; all when fewer than k are eligible) get
 * the uniform weight 1 / (number selected) in w and their bit in mask, in
 * dash_route's layouts.  Feeding these to dash_attn_fwd with sigma = 0 gives
 * softmax attention on the selected chunks plus the diagonal chunk, with the
 * same stage-2 kernel.  A reference kernel on CUDA cores (one warp per row),
 * not a tuned router.
 * Errors: as dash_route; k < 1 -> DASH_ERR_INVALID_ARG; G > 16, more than
 * 2048 chunks or p->estimate_diagonal = 1 (there is no entmax normalisation
 * to correct) -> DASH_ERR_UNSUPPORTED.
 */
int dash_route_topk(const dash_problem* p, const void* Q, const void* Kbar, int k, float* w,
                    uint32_t* mask, void* stream);

/*
 * Stage 2 -- prior-induced block-sparse softmax attention (gist.science
 * summary, "Fase 2: Prior-Geinduceerde Spaarzame Softmax").  For query i of
 * head h (KV head g = h / G) and keys j <= i in chunk b(j):
 *   bias_ij = 0                           if b(j) == c_i   (diagonal branch)
 *           = sigma * ln w[b, g, i, b(j)] if b(j) < c_i and its mask bit is set
 *                                          (0 when sigma == 0)
 *           = -inf                        otherwise
 *   O[b, h, i] = sum_j softmax_j(q_i . k_j / sqrt(d) + bias_ij) v_j
 *   lse[b, h, i] = log sum_j exp(q_i . k_j / sqrt(d) + bias_ij)   (nullable)
 * Mask bits at or after c_i are ignored.  w and mask are inputs, so a caller
 * may pass its own (e.g. all ones for dense causal attention).
 * bf16 runs on tcgen05 tensor cores (requires G in {4, 8, 16}, 128 / G <= B);
 * f32 runs on CUDA cores.  workspace: dash_workspace_bytes(p, 0) bytes
 * (may be 0, then workspace may be NULL).
 */
int dash_attn_fwd(const dash_problem* p, const void* Q, const void* K, const void* V,
                  const float* w, const uint32_t* mask, void* O, float* lse,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 2 backward: gradients of dash_attn_fwd's O for the cotangent dO.
 * The pages state that the hierarchy is differentiable end to end
 * (gist.science summary, "Belangrijkste Bijdragen" item 1) but print no
 * gradients; these are the chain rule of stage 2's definition:
 * ds = p (dO.v - dO.O), dQ = ds K / sqrt(d), dK = ds^T Q / sqrt(d),
 * dV = p^T dO, and dw_c = sigma / w_c * (sum of ds over block c's keys and
 * the KV group's heads) on every active routed block (the diagonal chunk's
 * bias is 0, the mask is piecewise constant: neither has a gradient).
 *   Q, K, V, w, mask, O, lse: the forward call's inputs and outputs (lse
 *   required); dO [b, Hq, N, d] (dtype of Q).
 *   dQ [b, Hq, N, d], dK, dV [b, Hkv, N, d] fp32: written; dw
 *   [b, Hkv, N, n_c] fp32, nullable: written, 0 off the active routed blocks.
 *   workspace: dash_workspace_bytes(p, 2) bytes, 256-byte aligned (may be
 *   NULL when that is 0).
 * bf16 with d = 128 and G in {4, 8, 16} runs on tcgen05 tensor cores: a
 * query-major kernel (dQ, dw; it also writes each row's dO.O and each
 * 128-row tile's routed union to the workspace), then a key-major kernel
 * (dK, dV) over the tiles that attend to each 128 keys; when there are few
 * key blocks (short sequences) their tile lists are split and the splits'
 * partial dK | dV rows (in the workspace) are summed in split order.  Every
 * output element is written once, in a fixed order (no atomics).  Other shapes run
 * a reference kernel on CUDA cores that zeroes dK, dV on the stream and
 * accumulates them with atomics (summation order varies from run to run).
 * Errors: NULL or misaligned required pointers, a bad problem ->
 * DASH_ERR_INVALID_ARG; G > 16 -> DASH_ERR_UNSUPPORTED; a missing, short or
 * misaligned workspace -> DASH_ERR_WORKSPACE.
 */
int dash_attn_bwd(const dash_problem* p, const void* Q, const void* K, const void* V,
                  const float* w, const uint32_t* mask, const void* O, const float* lse,
                  const void* dO, float* dQ, float* dK, float* dV, float* dw, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Stage 1 backward: the gradient of dash_route's w for the cotangent dw,
 * through the GQA mean and alpha-entmax (Jacobian diag(s) - s s^T / sum(s),
 * s = p^(2 - alpha) on the support: Peters, Niculae & Martins 2019) and the
 * logits z = q . Kbar (the mask is piecewise constant: no gradient).
 *   Q, Kbar: the forward's inputs; dw [b, Hkv, N, n_c] fp32 (e.g. from
 *   dash_attn_bwd); dQ [b, Hq, N, d] fp32 and dKbar [b, Hkv, N / B, d] fp32 are
 *   ACCUMULATED into (dQ after dash_attn_bwd wrote it; dKbar zeroed by the
 *   caller; dKbar by atomics).
 * Reference kernel on CUDA cores (one warp per position and KV head, the
 * threshold recomputed by bisection).  Errors: as dash_route;
 * p->estimate_diagonal = 1 -> DASH_ERR_UNSUPPORTED (the gradient through the
 * diagonal candidate is not built).
 */
int dash_route_bwd(const dash_problem* p, const void* Q, const void* Kbar, const float* dw,
                   float* dQ, float* dKbar, void* stream);

/*
 * Stage 0 backward: the gradient of dash_summarize's Kbar for the cotangent
 * dKbar [b, Hkv, N / B, d] fp32 (e.g. from dash_route_bwd), through the
 * learned-query softmax of each chunk: dK [b, Hkv, N, d] fp32 and
 * dqbar [Hkv, d] fp32 are ACCUMULATED into (dK after dash_attn_bwd wrote it;
 * dqbar zeroed by the caller, added with atomics).  Reference kernel (one
 * warp per chunk).  Errors: NULL or misaligned pointers, a bad problem ->
 * DASH_ERR_INVALID_ARG.
 */
int dash_summarize_bwd(const dash_problem* p, const void* K, const float* qbar, const float* dKbar,
                       float* dK, float* dqbar, void* stream);

/*
 * dash_attn_fwd on the compact weights of dash_route_packed: `weight` holds,
 * per row, the weights of the row's routed chunks in increasing chunk order
 * (entry k belongs to the k-th set bit of the row's mask); the entries past
 * a row's count are never used.  Same output, errors and limits as
 * dash_attn_fwd.
 */
int dash_attn_fwd_packed(const dash_problem* p, const void* Q, const void* K, const void* V,
                         const float* weight, const uint32_t* mask, void* O, float* lse,
                         void* stream);

/*
 * Workspace bytes needed by dash_attn_fwd (which = 0), dash_decode and its
 * variants (1) or dash_attn_bwd (2); 0 for an invalid problem or `which`.
 */
size_t dash_workspace_bytes(const dash_problem* p, int which);

/*
 * Decode -- one new query per sequence at position L - 1 of an L-token cache
 * (L = p->seq_len) whose K/V already hold the new token (gist.science
 * summary, "Efficiëntie" bullet of Fase 0: summaries of complete chunks are
 * cached; "Belangrijkste Bijdragen" item 4: incremental decoding).
 *   q [b, Hq, d]; Kcache, Vcache [b, Hkv, L, d]; Kbar [b, Hkv, floor(L / B), d]
 *   (only the chunks before the query's own, c < floor((L - 1) / B), are read);
 *   o [b, Hq, d]; lse [b, Hq] (nullable); w [b, Hkv, n_c] (nullable);
 *   mask [b, Hkv, n_w] (nullable).
 * Equals row L - 1 of stage 1 + stage 2 on the same data.
 * qbar [Hkv, d] fp32: required with p->estimate_diagonal = 1 (the query's
 * own chunk c_q joins the entmax with stage 0's summary of the cache rows
 * c_q B .. L - 1, as in dash_route; its weight goes to w[.., c_q] and is not
 * a mask bit), else ignored and may be NULL.
 * workspace: dash_workspace_bytes(p, 1) bytes, 256-byte aligned.
 */
int dash_decode(const dash_problem* p, const void* q, const void* Kcache,
                const void* Vcache, const void* Kbar, const float* qbar, void* o,
                float* lse, float* w, uint32_t* mask, void* workspace,
                size_t workspace_bytes, void* stream);

/*
 * Decode for a batch of sequences with different cache lengths (each at its
 * own point of generation; the same incremental decoding as dash_decode,
 * one sequence at a time).  p->seq_len is the caches' capacity L_max:
 *   Kcache, Vcache [b, Hkv, L_max, d]; Kbar [b, Hkv, floor(L_max / B), d].
 * cache_lens: device int32 [b], 4-byte aligned; sequence bi holds L_b =
 * cache_lens[bi] tokens, 1 <= L_b <= L_max, and its query sits at position
 * L_b - 1: only cache rows < L_b and summary rows < floor((L_b - 1) / B) of
 * that sequence are read.  o, lse as in dash_decode; w [b, Hkv, n_c] and
 * mask [b, Hkv, n_w] with n_c = ceil(L_max / B), columns from
 * floor((L_b - 1) / B) on are 0 for sequence bi.  Equals dash_decode run on
 * each sequence alone with L = L_b.  Same workspace as dash_decode for the
 * problem with seq_len = L_max.
 * Errors: those of dash_decode; cache_lens NULL or misaligned ->
 * DASH_ERR_INVALID_ARG.  The lengths are read on the device only: a length
 * outside [1, L_max] is clamped into it (every access stays inside the
 * caches, that sequence's outputs are meaningless) and makes the next
 * dash_get_error return DASH_ERR_INVALID_ARG.
 */
int dash_decode_varlen(const dash_problem* p, const int32_t* cache_lens, const void* q,
                       const void* Kcache, const void* Vcache, const void* Kbar,
                       const float* qbar, void* o, float* lse, float* w, uint32_t* mask,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * dash_decode_varlen over paged K/V caches, the layout a serving engine keeps
 * its caches in.  One page holds one chunk: the B = p->chunk tokens of one
 * chunk for every KV head.
 *   Kpool, Vpool [n_pages, Hkv, B, d] (bf16); page_table: device int32
 *   [b, max_pages], 4-byte aligned, max_pages >= ceil(L_max / B): chunk c of
 *   sequence bi is pool page page_table[bi * max_pages + c] (entries for
 *   chunks at or past ceil(L_b / B) are never read; pages may be shared).
 *   cache_lens, Kbar (still one contiguous summary cache per sequence), qbar,
 *   q, o, lse, w, mask, workspace: as in dash_decode_varlen with
 *   L_max = p->seq_len.
 * Equals dash_decode_varlen on the caches the pages spell out.
 * Errors: those of dash_decode_varlen; page_table NULL or misaligned,
 * max_pages < ceil(L_max / B) or n_pages < 1 -> DASH_ERR_INVALID_ARG;
 * n_pages * Hkv * B >= 2^31 -> DASH_ERR_UNSUPPORTED.  Page ids are read on the
 * device: one outside [0, n_pages) is replaced by page 0 (every access stays
 * inside the pools, that sequence's outputs are meaningless) and makes the
 * next dash_get_error return DASH_ERR_INVALID_ARG.
 */
int dash_decode_paged(const dash_problem* p, const int32_t* cache_lens, const int32_t* page_table,
                      int max_pages, int n_pages, const void* q, const void* Kpool,
                      const void* Vpool, const void* Kbar, const float* qbar, void* o,
                      float* lse, float* w, uint32_t* mask, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * Decode without a caller-provided workspace.  The pages on DashAttention
 * have no counterpart to this call; it exists for callers that cannot
 * allocate device memory: an inference engine that hands every byte of the
 * GPU to its own pool, or a plugin interface that forbids allocation, cannot
 * supply the dash_workspace_bytes(p, 1) scratch that dash_decode needs.
 *
 * Same arguments, result and errors as dash_decode, minus the workspace and
 * qbar (p->estimate_diagonal = 1 returns DASH_ERR_UNSUPPORTED).
 * The scratch is a fixed 8 MiB array in device memory, reserved on every GPU
 * that loads this library until the process exits; no cudaMalloc/cudaFree or
 * other allocating routine is called.  Every problem dash_decode accepts
 * (at most 64 (sequence, KV head) pairs and 2048 chunks) needs at most
 * about 6 MB (the 8-sequence, 2-KV-head, 131072-token cache case about
 * 4.7 MB); a problem whose scratch exceeded 8 MiB would return
 * DASH_ERR_WORKSPACE.
 * Every call looks up the current device's address of the array (with that
 * device current), so a device reset between calls leaves nothing stale; the
 * first call on a device also loads the library's device code there, so make
 * that first call before any stream capture.
 * All calls on a device share the one array and it keeps the last call's
 * contents (nothing in it needs to start at zero), so calls that overlap on
 * the GPU -- concurrent streams, or threads using the same device -- race
 * and must be serialised by the caller.
 */
int dash_decode_noalloc(const dash_problem* p, const void* q, const void* Kcache,
                        const void* Vcache, const void* Kbar, void* o, float* lse, float* w,
                        uint32_t* mask, void* stream);

/*
 * Synchronises `stream`, then reports (and clears) the device-side error
 * word: DASH_ERR_TIMEOUT if a bounded wait gave up, DASH_ERR_INVALID_ARG if a
 * kernel found an argument it reads on the device out of range (a cache
 * length or a page id), DASH_ERR_UNSUPPORTED if a kernel met a size
 * limit it cannot handle (the host sizes launches so that this does not
 * happen), else DASH_OK; DASH_ERR_CUDA if the synchronisation itself failed.
 */
int dash_get_error(void* stream);

/*
 * Failure-path self-test (no counterpart in the pages): launches one kernel
 * whose bounded wait on an mbarrier that nothing completes runs out after
 * the limit every wait in this library has (2 s), records the timeout in the
 * device error word and returns.  The next dash_get_error reports
 * DASH_ERR_TIMEOUT and the CUDA context stays usable; nothing faults, traps
 * or hangs.  Returns DASH_ERR_CUDA if the launch fails, else DASH_OK.
 */
int dash_selftest_wait_timeout(void* stream);

/*
 * Accuracy self-test (no counterpart in the pages): y[i] = the attention
 * kernel's FMA-pipe evaluation of 2^x[i] (a Cody-Waite split x = n + f,
 * |f| <= 1/2, and a degree-3 polynomial for 2^f fitted for minimum maximum
 * relative error, 7.5e-5), which computes part of stage 2's softmax
 * exponentials.  Inputs below -125 are clamped to -125 (so -inf gives
 * about 2^-125, not 0).  x and y: device float [n], 4-byte aligned.
 * Returns DASH_ERR_INVALID_ARG for n < 0 or NULL pointers with n > 0,
 * DASH_ERR_CUDA if the launch fails, else DASH_OK.
 */
int dash_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * Test hook (no counterpart in the pages): the number of CTAs the
 * tensor-core dash_attn_bwd splits each key block's tile list over, for
 * every later call in this process (n = 1 .. 8), or the automatic choice
 * (n = 0: split only when there are fewer key blocks than about four waves
 * of SMs).  dash_workspace_bytes(p, 2) follows the setting.  Not thread-safe:
 * for tests that reach both the split and the unsplit path on small inputs.
 * Returns the previous setting, or -1 (nothing changed) for n outside 0 .. 8.
 */
int dash_selftest_bwd_split(int n);

#ifdef __cplusplus
}
#endif

#endif /* DASH_H_ */
