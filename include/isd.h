/*
 * isd.h -- C ABI of libisd.so, one Introspective Strided Decoding (ISD) step
 * on an NVIDIA B200 (sm_100a).
 *
 * The method comes from "Introspective Diffusion Language Models"
 * (arXiv 2604.11035).  Its project summary (hada.io pages) describes one
 * forward pass that verifies the previous stride and drafts the next one
 * ("Introspective Strided Decoding (ISD)"), new tokens proposed from q at
 * MASK positions and verified with p at clean positions, kept with
 * probability min(1, p(x)/q(x)) ("Inference & ISD"), strict causal
 * attention with a logit shift ("Méthodologie d'I-DLM"), and a paged KV
 * cache read by a paged-only attention kernel ("Serving (SGLang)").
 *
 * One step is three calls, in this order, on one stream:
 *   isd_attn_strided     strided-query causal GQA attention, paged KV
 *   isd_accept_resample  vocab softmax stats, ratio test, resample / bonus /
 *                        draft sampling
 *   isd_kv_commit        commit of the accepted prefix, rollback of the rest
 * or two, the last two fused: isd_accept_commit (the same results, with the
 * commit running beside the draws).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer is a DEVICE pointer into memory the caller owns and keeps
 *   alive until the enqueued work has finished.  The library never
 *   allocates, frees or synchronises; all work is enqueued on `stream`
 *   (0 = the legacy default stream) of the current device.
 * - Arrays are dense, row-major, in the layouts stated below, 16-byte
 *   aligned.
 * - Stride rows: sequence b holds K = 2N query rows at absolute positions
 *   L_b .. L_b + K - 1 (L_b = seq_len[b], its committed length).  Rows
 *   0 .. n_b - 1 hold the pending tokens (row 0 the stride's exact token,
 *   rows 1.. drafts under verification); rows n_b .. K - 1 are MASK rows.
 *   Row r's logits score position L_b + r + 1 (logit shift).
 * - Paged KV: page_size = 16 token slots; cache layout
 *   [num_pages][Hkv][16][d]; logical page i of sequence b is physical page
 *   page_table[b * page_table_stride + i].
 * - Return value: ISD_OK when the work was enqueued.  Invalid arguments are
 *   rejected on the host before anything is launched (ISD_ERR_INVALID_ARG,
 *   ISD_ERR_UNSUPPORTED, ISD_ERR_WORKSPACE).  A failed launch returns
 *   ISD_ERR_CUDA.  Conditions only the device can see (pool exhausted,
 *   page-table row full, malformed state, page id out of range, a bounded
 *   wait that ran out) are written as an ISD_ERR_* code to the caller's
 *   `status` word, and the affected work is skipped; no kernel traps and no
 *   kernel waits on another.
 * - The status word keeps the FIRST error written to it: kernels never
 *   clear it and never replace an error already there (atomic
 *   compare-and-swap from ISD_OK).  The caller zeroes it before use; one
 *   word may serve all three calls of a step, and after the step it holds
 *   the earliest failure.
 * - The calls are asynchronous and capture into CUDA graphs: they read no
 *   device memory on the host and launch a fixed set of kernels.
 */
#ifndef ISD_H_
#define ISD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ISD_ABI_VERSION 4
#define ISD_PAGE_SIZE 16

/* Return / status codes. */
enum {
  ISD_OK = 0,
  ISD_ERR_INVALID_ARG = 1,     /* null pointer, bad size, aliasing       */
  ISD_ERR_UNSUPPORTED = 2,     /* valid but outside the built kernels    */
  ISD_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed   */
  ISD_ERR_WORKSPACE = 4,       /* workspace missing or too small         */
  /* written by the device into *status */
  ISD_ERR_POOL_EXHAUSTED = 16, /* commit needs more pages than are free  */
  ISD_ERR_PAGE_TABLE_FULL = 17,/* a sequence outgrew its page-table row  */
  ISD_ERR_BAD_STATE = 18,      /* n_pending, token or q row out of range */
  ISD_ERR_BAD_PAGE = 19        /* page id outside [0, num_pages)         */
};

/* Element types. */
enum { ISD_BF16 = 0, ISD_F32 = 1 };

/* Uniform streams of the sampler (Philox counter word 3). */
enum { ISD_STREAM_ACCEPT = 0, ISD_STREAM_RESAMPLE = 1, ISD_STREAM_DRAFT = 2 };

/* ------------------------------------------------------------------------
 * isd_attn_strided -- strided-query causal GQA attention over a paged KV
 * cache (the "paged-only attention kernel" of the pages' serving stack).
 *
 * For sequence b, KV head h, stride row r and group member j (query head
 * hq = h * g + j, g = Hq / Hkv):
 *   keys   = cached positions [0, L_b) of head h, then k_new[b, 0..r, h]
 *   O[b, r, hq] = sum_t softmax(softmax_scale * q[b, r, hq] . key_t) value_t
 *   lse[b, r, hq] = log(sum_t exp(softmax_scale * q . key_t))   (natural)
 * Strict causal: row r never sees stride rows > r; no window, no bias; Q/K
 * arrive post-rotary.  Every row, including MASK and spare rows, is computed.
 *
 * Layouts: q, out [B][K][Hq][d]; k_new, v_new [B][K][Hkv][d];
 * k_cache, v_cache [num_pages][Hkv][16][d]; page_table int32
 * [B][page_table_stride]; seq_len int32 [B]; lse f32 [B][K][Hq] or NULL.
 * dtype ISD_BF16 (tcgen05 tensor cores: d = 128, K <= 16, K * g <= 128)
 * or ISD_F32 (exact-fp32 SIMT path; d a multiple of 32, at most 128).
 * `out` may not alias any input.
 * Workspace: isd_attn_workspace_bytes(args) bytes (split-KV partials);
 * its contents need no initialisation.  `status` (optional) receives
 * ISD_ERR_BAD_PAGE / ISD_ERR_PAGE_TABLE_FULL for malformed page tables;
 * pages out of range read as zeros.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t B, Hq, Hkv, d, K;
  int32_t num_pages, page_table_stride;
  int32_t dtype;
  float softmax_scale;
  int32_t num_ctas;            /* 0: one CTA per SM, or fewer for small
                                  problems (at most one per 40 units of
                                  the largest work the page table
                                  admits); else 1..1024 CTAs             */
  const void* q;
  const void* k_new;
  const void* v_new;
  const void* k_cache;
  const void* v_cache;
  const int32_t* page_table;
  const int32_t* seq_len;
  void* out;
  float* lse;                  /* optional                                */
  int32_t* status;             /* optional                                */
  void* workspace;
  size_t workspace_bytes;
} isd_attn_args;

size_t isd_attn_workspace_bytes(const isd_attn_args* a);
int isd_attn_strided(const isd_attn_args* a, void* stream);

/* ------------------------------------------------------------------------
 * isd_accept_resample -- vocab softmax of p and q, the min(1, p/q) ratio
 * test, and the residual / bonus / draft draws.
 *
 * Per sequence b with n = n_pending_in[b] (1 or N), L = seq_len[b]:
 *  1. Row statistics m = max_v l_v, s = sum_v exp(l_v - m) (fp32) of
 *     logits_cur rows 0 .. n + N - 2 (p rows 0..n-1, draft rows n..n+N-2).
 *  2. Drafts i = 1 .. n-1 in order: p_i(x) from row i-1 of logits_cur,
 *     q_i(x) = exp(l_x - ln Z) from row q_row_in[b][i] of logits_prev and
 *     its stored log-normaliser ln Z = q_stats_in[b][i][0] + [1];
 *     u_i = U(seed, b, step, L + i, ACCEPT);
 *     accept iff u_i < p_i(x)/q_i(x).  a_b = drafts accepted before the
 *     first rejection; n_commit[b] = 1 + a_b; commit_tokens[b][0..a_b] =
 *     pending_in[b][0..a_b] (the rest -1).
 *  3. Rejected at draft a+1: the exact token at L + a + 1 is drawn from
 *     normalise(max(0, p - q)) (p from row a, q of draft a+1; p if that
 *     mass is zero), stream RESAMPLE; next n = 1.
 *     All accepted: the exact token at L + n is drawn from p of row n-1
 *     (stream RESAMPLE), and drafts j = 1..N-1 at L + n + j from q of row
 *     n + j - 1 (stream DRAFT), whose log-normaliser goes to
 *     q_stats_out[b][j] and row index to q_row_out[b][j]; next n = N.
 *  A draw with uniform u from masses w returns the smallest index v whose
 *  running sum (ascending vocabulary order) exceeds u * sum(w).
 *  U(seed, b, step, pos, stream) = (x0 >> 8) * 2^-24 with x0 the first word
 *  of Philox4x32-10(key = (seed lo, seed hi), counter = (b, step, pos,
 *  stream)) (Salmon et al., SC'11).
 *
 * Argmax proposals (proposal = ISD_PROPOSAL_ARGMAX): the pages' serving
 *  option of proposing the most likely token at each MASK position
 *  (summary, "Serving (SGLang)").  Drafts are x = argmax q (the first
 *  maximal index) instead of draws, so the proposal is a point mass: a
 *  draft is accepted iff u < p(x), and at a rejection the replacement is
 *  drawn from p without x (max(0, p - delta_x)); stream DRAFT is unused.
 *  The pending drafts must have been proposed the same way.
 *
 * Sizes: N <= 16, V <= 262 144 (otherwise ISD_ERR_UNSUPPORTED).
 * Layouts: logits_cur, logits_prev [B][K][V] (dtype); pending_*, q_row_*
 * int32 [B][N]; n_pending_* int32 [B]; q_stats_* f32 [B][N][2]: the
 * natural-log normaliser ln sum_v exp(l_v) of each draft's q row as a float
 * pair hi + lo (hi the value rounded to fp32, lo the remainder; fp32 alone
 * would cost the residual of peaked rows its accuracy; entry 0 unused);
 * n_commit int32 [B]; commit_tokens int32 [B][N]; row_stats f32
 * [B][K][2] or NULL (m, s of the rows used, others untouched); ratio f32
 * [B][N] or NULL (p/q of each verified draft, others untouched).
 * The *_out state arrays must not alias the *_in ones.  A sequence whose
 * state is malformed gets ISD_ERR_BAD_STATE in *status (if given),
 * n_commit 0 and its state copied through unchanged.
 * Workspace: isd_accept_workspace_bytes(args) bytes; no initialisation.
 * vocab_stats (optional, 16-byte aligned): the figures isd_lm_head wrote for
 * the same logits_cur; the row statistics of step 1 are then merged from
 * them and logits_cur is read only where the ratio tests and draws need it.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t B, N, K, V;
  int32_t dtype;
  uint32_t step;
  uint64_t seed;
  const void* logits_cur;
  const void* logits_prev;
  const int32_t* seq_len;
  const int32_t* pending_in;
  const int32_t* n_pending_in;
  const int32_t* q_row_in;
  const float* q_stats_in;
  int32_t* pending_out;
  int32_t* n_pending_out;
  int32_t* q_row_out;
  float* q_stats_out;
  int32_t* n_commit;
  int32_t* commit_tokens;
  float* row_stats;            /* optional                                */
  float* ratio;                /* optional                                */
  int32_t* status;             /* optional                                */
  void* workspace;
  size_t workspace_bytes;
  const uint32_t* step_dev;    /* optional: read the step index from device
                                  memory instead of `step` (lets one
                                  captured CUDA graph serve every step)    */
  int32_t proposal;            /* ISD_PROPOSAL_SAMPLE or _ARGMAX          */
  const void* vocab_stats;     /* optional: the sub-chunk statistics of
                                  logits_cur written by isd_lm_head (M =
                                  B * K rows); when given, step 1 takes
                                  them instead of reading logits_cur      */
} isd_accept_args;

#define ISD_PROPOSAL_SAMPLE 0  /* drafts drawn from q (default)           */
#define ISD_PROPOSAL_ARGMAX 1  /* drafts x = argmax q                      */

size_t isd_accept_workspace_bytes(const isd_accept_args* a);
int isd_accept_resample(const isd_accept_args* a, void* stream);

/* ------------------------------------------------------------------------
 * isd_accept_resample_static -- the same step as isd_accept_resample, for
 * callers that cannot allocate device memory.  The paper's pages have no
 * counterpart to this entry point: it exists for integration only.
 *
 * Some callers have no way to provide the workspace: a host program that
 * links this C ABI directly and has no device allocator of its own (a
 * cudaMalloc per call would synchronise the device and fragment memory), or
 * a serving process whose framework has already reserved the device memory
 * pool.  This entry point takes its scratch from a buffer of
 * ISD_ACCEPT_STATIC_SCRATCH bytes compiled into the library; every GPU that
 * loads the library holds that buffer until the process exits.  It calls no
 * allocating routine.
 *
 * - `workspace` and `workspace_bytes` in *a are ignored; every other field
 *   means what it means for isd_accept_resample, with the same results.
 * - The arguments are checked exactly as isd_accept_resample checks them,
 *   in the same order; then problems whose isd_accept_workspace_bytes(a)
 *   exceeds ISD_ACCEPT_STATIC_SCRATCH are rejected with ISD_ERR_WORKSPACE
 *   before any launch (at N = 4 and V = 151 936 the limit admits 1 840
 *   sequences).
 * - The first call on each device looks up the buffer's device address
 *   (with that device current) and keeps it for the current CUDA context;
 *   make that first call before any stream capture begins.  A call from a
 *   different context on that device looks the address up again.
 * - All calls on a device share the one buffer, which keeps the previous
 *   call's contents (nothing needs clearing: each call writes every scratch
 *   word before reading it).  Calls whose work may overlap on the GPU, such
 *   as calls on two unordered streams, race on it: order them.
 * ---------------------------------------------------------------------- */
#define ISD_ACCEPT_STATIC_SCRATCH (16u << 20)
int isd_accept_resample_static(const isd_accept_args* a, void* stream);

/* ------------------------------------------------------------------------
 * isd_kv_commit -- copy the staged K/V of rows 0 .. n_commit[b]-1 to cache
 * positions L_b .. L_b + n_commit[b] - 1 and grow seq_len[b] by n_commit[b].
 * Rows >= n_commit[b] (rejected drafts, MASK rows) are never written: that
 * is the rollback.  When a committed position enters a new page, pages are
 * popped from the free stack (entries [0, *free_top) are free, the top is
 * free_stack[*free_top - 1]), sequence 0 first, and recorded in the page
 * table; no page is freed.  All-or-nothing: the whole commit is validated
 * before anything is written, and if the pool or a page-table row is too
 * small (ISD_ERR_POOL_EXHAUSTED, ISD_ERR_PAGE_TABLE_FULL), a length, count
 * or free-stack top is out of range (ISD_ERR_BAD_STATE), or a page id the
 * commit would write through or pop is outside [0, num_pages)
 * (ISD_ERR_BAD_PAGE), *status gets the code (the lowest in that order when
 * several hold) and no cache byte, page-table entry, length or top changes.
 *
 * Layouts: k_new, v_new [B][K][Hkv][d]; k_cache, v_cache
 * [num_pages][Hkv][16][d]; page_table int32 [B][page_table_stride];
 * seq_len, n_commit int32 [B] (0 <= n_commit <= K); free_stack int32
 * [num_pages]; free_top int32 [1]; status int32 [1] (required; written
 * only on error, see the conventions above).  B <= 32 768.
 * Workspace: isd_commit_workspace_bytes(args) bytes (a counter), zeroed by
 * the caller once before its first use; every call leaves it zeroed.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t B, K, Hkv, d;
  int32_t num_pages, page_table_stride;
  int32_t dtype;
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  int32_t* page_table;
  int32_t* seq_len;
  const int32_t* n_commit;
  const int32_t* free_stack;
  int32_t* free_top;
  int32_t* status;
  void* workspace;
  size_t workspace_bytes;
} isd_commit_args;

size_t isd_commit_workspace_bytes(const isd_commit_args* a);
int isd_kv_commit(const isd_commit_args* a, void* stream);

/* ------------------------------------------------------------------------
 * isd_accept_commit -- isd_accept_resample(a) followed by isd_kv_commit(c)
 * in one call, with the same outputs, state and status as those two calls
 * in that order.  The KV commit needs only the decisions (n_commit), not
 * the draws ("Serving (SGLang)": the commit of the accepted prefix), so
 * after the statistics and the ratio-test decisions the commit runs and the
 * residual / bonus / draft draws run beside it.  c must describe the same
 * sequences: c->B == a->B, c->K == a->K, c->n_commit == a->n_commit and
 * c->seq_len == a->seq_len, and the two workspaces must not overlap (else
 * ISD_ERR_INVALID_ARG); every other rule of the two calls applies unchanged
 * (both workspaces, both checks, checked before anything is launched).
 * ---------------------------------------------------------------------- */
int isd_accept_commit(const isd_accept_args* a, const isd_commit_args* c,
                      void* stream);

/* ------------------------------------------------------------------------
 * isd_lm_head -- the LM head that makes a step's logits, with the R-ISD
 * gated LoRA at MASK rows and the vocabulary statistics of every row.
 *
 * One forward pass gives every row of the stride its distribution over the
 * vocabulary, p at the clean rows and q at the MASK rows (summary,
 * "Inference & ISD"); a row's logits are its final hidden state times the
 * output embedding.  R-ISD adds a rank-r LoRA (r = 128 on the pages) that
 * acts only at MASK positions, so the clean rows stay the base model's
 * (summary, "Speedup Factor Explorer", R-ISD):
 *
 *   logits[m][v] = sum_d hidden[m][d] weight[v][d]
 *                + gate_m sum_j U[m][j] lora_b[v][j],
 *   U[m][j] = bf16(lora_scale * sum_d hidden[m][d] lora_a[j][d]),
 *
 * gate_m = 1 when row m is a MASK row (stride row m % rows_per_seq >=
 * n_pending[m / rows_per_seq]), else 0.  Sums are accumulated in fp32 on the
 * tensor cores and the logits are rounded to bf16 (nearest, ties to even).
 * A sequence whose n_pending lies outside [0, rows_per_seq] gets no LoRA and
 * ISD_ERR_BAD_STATE in *status.
 *
 * vocab_stats (optional): for every row m and vocabulary sub-chunk c of
 * 2048 entries (C = ceil(V / 2048), the last one ragged), computed from the
 * bf16 logits as stored: csum f64 [M][C] (sum of exp(l - max)), then cmax
 * f32 [M][C] (the max), then cidx int32 [M][C] (first index of the max in
 * the row), packed in that order from vocab_stats; isd_vocab_stats_bytes(M,
 * V) bytes.  isd_accept_resample takes them through its vocab_stats field.
 *
 * Layouts: hidden bf16 [M][D]; weight bf16 [V][D] (one row per vocabulary
 * entry); logits bf16 [M][V]; lora_a bf16 [r][D]; lora_b bf16 [V][r];
 * n_pending int32 [M / rows_per_seq].  Sizes: D a multiple of 64; V a
 * multiple of 8; r = 0 (no LoRA) or a multiple of 64 up to 256; M >= 1.
 * Every pointer 16-byte aligned.  Workspace: isd_lm_head_workspace_bytes
 * (args) bytes; no initialisation.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t M, D, V;
  int32_t dtype;               /* ISD_BF16                                */
  const void* hidden;
  const void* weight;
  void* logits;
  void* vocab_stats;           /* optional                                */
  int32_t lora_rank;           /* 0: no LoRA                              */
  int32_t rows_per_seq;        /* K of the stride (LoRA only)             */
  const void* lora_a;
  const void* lora_b;
  const int32_t* n_pending;    /* LoRA only                               */
  float lora_scale;
  int32_t* status;             /* optional                                */
  void* workspace;
  size_t workspace_bytes;
} isd_lm_head_args;

size_t isd_lm_head_workspace_bytes(const isd_lm_head_args* a);
size_t isd_vocab_stats_bytes(int32_t M, int32_t V);
int isd_lm_head(const isd_lm_head_args* a, void* stream);
/* The number of kernels isd_lm_head launches for these arguments on the
 * current device (the LoRA down-projection and its sum, the GEMM, a split-K
 * fix-up when the last wave is split, the statistics merge); 0 when the
 * arguments fail the size checks.  Host only, launches nothing. */
int isd_lm_head_launches(const isd_lm_head_args* a);

/* Utilities. */
int isd_abi_version(void);
const char* isd_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* ISD_H_ */
