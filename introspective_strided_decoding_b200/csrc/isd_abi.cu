// C ABI of libisd.so (declared in include/isd.h): host-side validation and
// dispatch.  Nothing here allocates, frees or synchronises.
#include <algorithm>
#include <cstdint>

#include "common.cuh"

namespace isd {
size_t accept_workspace_bytes(int B, int N, int K, int V);
int launch_accept(const isd_accept_args* a, cudaStream_t st,
                  const isd_commit_args* c);
size_t commit_workspace_bytes(int B);
int commit_max_batch();
int launch_commit(const isd_commit_args* a, cudaStream_t st, bool trigger);
size_t attn_workspace_bytes_impl(int B, int M, int D, int G);
size_t attn_tc_smem_bytes(int B, int M);
int launch_attn_bf16(const isd_attn_args* a, int G, cudaStream_t st);
int launch_attn_f32(const isd_attn_args* a, cudaStream_t st);
size_t lm_head_workspace_bytes(const isd_lm_head_args* a);
size_t vocab_stats_bytes(int M, int V);
int launch_lm_head(const isd_lm_head_args* a, cudaStream_t st);
int lm_head_launches(const isd_lm_head_args* a);
}  // namespace isd

namespace {

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return 0;
  return n;
}

// Persistent CTAs of the bf16 path: one per SM, fewer when even the most
// work the page table admits (B Hkv (stride + 1) units: pages plus the
// stride's own tail unit) would give a CTA under kMinUnitsPerCta units; a
// CTA's fixed costs and the merge of a (b, h) split over many CTAs then
// outweigh its share of the stream (measured at B = 1, L = 4096: 29.7 us on
// 48-64 CTAs, 37.9 us on 148).
constexpr long long kMinUnitsPerCta = 40;

int attn_ctas(const isd_attn_args* a) {
  if (a->num_ctas > 0) return a->num_ctas;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  const long long most = (long long)a->B * a->Hkv * (a->page_table_stride + 1);
  const long long want = (most + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
  return (int)std::max<long long>(1, std::min<long long>(sms, want));
}

// Shape checks shared by the workspace query and the call.
int attn_check(const isd_attn_args* a) {
  if (!a) return ISD_ERR_INVALID_ARG;
  if (a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->d <= 0 || a->K <= 0 ||
      a->num_pages <= 0 || a->page_table_stride <= 0 || a->num_ctas < 0 ||
      a->num_ctas > 1024)
    return ISD_ERR_INVALID_ARG;
  if (a->Hq % a->Hkv != 0) return ISD_ERR_INVALID_ARG;
  if (!(a->softmax_scale > 0.0f)) return ISD_ERR_INVALID_ARG;
  if (a->dtype == ISD_BF16) {
    const int M = a->K * (a->Hq / a->Hkv);
    if (a->K > ISD_PAGE_SIZE || M > 128) return ISD_ERR_UNSUPPORTED;
    // tcgen05 path: head dim 128, any row count up to 128 (rows padded to
    // a multiple of 32); the stage ring must fit next to Q, P and the unit
    // prefix.
    if (a->d != 128) return ISD_ERR_UNSUPPORTED;
    if (isd::attn_tc_smem_bytes(a->B, M) == (size_t)-1)
      return ISD_ERR_UNSUPPORTED;
  } else if (a->dtype == ISD_F32) {
    if (a->d % 32 != 0 || a->d > 128) return ISD_ERR_UNSUPPORTED;
  } else {
    return ISD_ERR_INVALID_ARG;
  }
  return ISD_OK;
}

}  // namespace

namespace isd {

int accept_check(const isd_accept_args* a) {
  if (!a) return ISD_ERR_INVALID_ARG;
  if (a->B <= 0 || a->N < 2 || a->V <= 0 || a->K != 2 * a->N)
    return ISD_ERR_INVALID_ARG;
  if (a->N > 16) return ISD_ERR_UNSUPPORTED;
  if (a->V > 128 * 2048) return ISD_ERR_UNSUPPORTED;  // <= 128 sub-chunks
  if (a->dtype != ISD_BF16 && a->dtype != ISD_F32) return ISD_ERR_INVALID_ARG;
  if (a->proposal != ISD_PROPOSAL_SAMPLE && a->proposal != ISD_PROPOSAL_ARGMAX)
    return ISD_ERR_INVALID_ARG;
  return ISD_OK;
}

// Every check of isd_accept_resample except the workspace's (shared with
// the allocation-free entry point, so both report the same errors first).
int accept_validate(const isd_accept_args* a) {
  const int rc = accept_check(a);
  if (rc != ISD_OK) return rc;
  if (!a->logits_cur || !a->logits_prev || !a->seq_len || !a->pending_in ||
      !a->n_pending_in || !a->q_row_in || !a->q_stats_in || !a->pending_out ||
      !a->n_pending_out || !a->q_row_out || !a->q_stats_out || !a->n_commit ||
      !a->commit_tokens)
    return ISD_ERR_INVALID_ARG;
  if ((const void*)a->pending_out == (const void*)a->pending_in ||
      (const void*)a->n_pending_out == (const void*)a->n_pending_in ||
      (const void*)a->q_row_out == (const void*)a->q_row_in ||
      (const void*)a->q_stats_out == (const void*)a->q_stats_in)
    return ISD_ERR_INVALID_ARG;
  if (!aligned16(a->logits_cur) || !aligned16(a->logits_prev) ||
      !aligned16(a->vocab_stats))
    return ISD_ERR_INVALID_ARG;
  return ISD_OK;
}

}  // namespace isd

extern "C" {

int isd_abi_version(void) { return ISD_ABI_VERSION; }

const char* isd_status_string(int code) {
  switch (code) {
    case ISD_OK: return "ok";
    case ISD_ERR_INVALID_ARG: return "invalid argument";
    case ISD_ERR_UNSUPPORTED: return "unsupported shape or type";
    case ISD_ERR_CUDA: return "CUDA error";
    case ISD_ERR_WORKSPACE: return "workspace missing or too small";
    case ISD_ERR_POOL_EXHAUSTED: return "KV page pool exhausted";
    case ISD_ERR_PAGE_TABLE_FULL: return "page-table row full";
    case ISD_ERR_BAD_STATE: return "malformed decoding state";
    case ISD_ERR_BAD_PAGE: return "page id out of range";
    default: return "unknown status";
  }
}

// ------------------------------------------------------------- attention
size_t isd_attn_workspace_bytes(const isd_attn_args* a) {
  if (attn_check(a) != ISD_OK) return 0;
  if (a->dtype == ISD_F32) return 0;
  const int G = attn_ctas(a);
  if (G <= 0) return 0;
  return isd::attn_workspace_bytes_impl(a->B, a->K * (a->Hq / a->Hkv), a->d, G);
}

int isd_attn_strided(const isd_attn_args* a, void* stream) {
  const int rc = attn_check(a);
  if (rc != ISD_OK) return rc;
  if (!a->q || !a->k_new || !a->v_new || !a->k_cache || !a->v_cache ||
      !a->page_table || !a->seq_len || !a->out)
    return ISD_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k_new) || !aligned16(a->v_new) ||
      !aligned16(a->k_cache) || !aligned16(a->v_cache) || !aligned16(a->out))
    return ISD_ERR_INVALID_ARG;
  if (a->out == a->q || a->out == a->k_new || a->out == a->v_new ||
      a->out == a->k_cache || a->out == a->v_cache)
    return ISD_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->dtype == ISD_F32) return isd::launch_attn_f32(a, st);
  const int G = attn_ctas(a);
  if (G <= 0) return ISD_ERR_CUDA;
  const size_t need =
      isd::attn_workspace_bytes_impl(a->B, a->K * (a->Hq / a->Hkv), a->d, G);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return ISD_ERR_WORKSPACE;
  return isd::launch_attn_bf16(a, G, st);
}

// ---------------------------------------------------------------- accept
size_t isd_accept_workspace_bytes(const isd_accept_args* a) {
  if (isd::accept_check(a) != ISD_OK) return 0;
  return isd::accept_workspace_bytes(a->B, a->N, a->K, a->V);
}

int isd_accept_resample(const isd_accept_args* a, void* stream) {
  const int rc = isd::accept_validate(a);
  if (rc != ISD_OK) return rc;
  const size_t need = isd::accept_workspace_bytes(a->B, a->N, a->K, a->V);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return ISD_ERR_WORKSPACE;
  return isd::launch_accept(a, static_cast<cudaStream_t>(stream), nullptr);
}

// ---------------------------------------------------------------- commit
static int commit_check(const isd_commit_args* a) {
  if (!a) return ISD_ERR_INVALID_ARG;
  if (a->B <= 0 || a->K <= 0 || a->Hkv <= 0 || a->d <= 0 ||
      a->num_pages <= 0 || a->page_table_stride <= 0)
    return ISD_ERR_INVALID_ARG;
  if (a->dtype != ISD_BF16 && a->dtype != ISD_F32) return ISD_ERR_INVALID_ARG;
  const int es = a->dtype == ISD_BF16 ? 2 : 4;
  if ((a->d * es) % 16 != 0) return ISD_ERR_UNSUPPORTED;
  if (a->B > isd::commit_max_batch()) return ISD_ERR_UNSUPPORTED;
  return ISD_OK;
}

size_t isd_commit_workspace_bytes(const isd_commit_args* a) {
  if (commit_check(a) != ISD_OK) return 0;
  return isd::commit_workspace_bytes(a->B);
}

static int commit_validate(const isd_commit_args* a) {
  const int rc = commit_check(a);
  if (rc != ISD_OK) return rc;
  if (!a->k_new || !a->v_new || !a->k_cache || !a->v_cache || !a->page_table ||
      !a->seq_len || !a->n_commit || !a->free_stack || !a->free_top ||
      !a->status)
    return ISD_ERR_INVALID_ARG;
  if (!aligned16(a->k_new) || !aligned16(a->v_new) || !aligned16(a->k_cache) ||
      !aligned16(a->v_cache))
    return ISD_ERR_INVALID_ARG;
  const size_t need = isd::commit_workspace_bytes(a->B);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return ISD_ERR_WORKSPACE;
  return ISD_OK;
}

int isd_kv_commit(const isd_commit_args* a, void* stream) {
  const int rc = commit_validate(a);
  if (rc != ISD_OK) return rc;
  return isd::launch_commit(a, static_cast<cudaStream_t>(stream), false);
}

// ------------------------------------------------------ accept + commit
int isd_accept_commit(const isd_accept_args* a, const isd_commit_args* c,
                      void* stream) {
  int rc = isd::accept_validate(a);
  if (rc != ISD_OK) return rc;
  const size_t need = isd::accept_workspace_bytes(a->B, a->N, a->K, a->V);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return ISD_ERR_WORKSPACE;
  rc = commit_validate(c);
  if (rc != ISD_OK) return rc;
  // The commit consumes this step's decisions on the same sequences.
  if (c->B != a->B || c->K != a->K || c->n_commit != a->n_commit ||
      c->seq_len != a->seq_len)
    return ISD_ERR_INVALID_ARG;
  // The two workspaces are in use at the same time: they must not overlap.
  const uintptr_t wa = reinterpret_cast<uintptr_t>(a->workspace);
  const uintptr_t wc = reinterpret_cast<uintptr_t>(c->workspace);
  const size_t need_c = isd::commit_workspace_bytes(c->B);
  if (wa < wc + need_c && wc < wa + need) return ISD_ERR_INVALID_ARG;
  return isd::launch_accept(a, static_cast<cudaStream_t>(stream), c);
}

// --------------------------------------------------------------- LM head
static int lm_head_check(const isd_lm_head_args* a) {
  if (!a) return ISD_ERR_INVALID_ARG;
  if (a->M <= 0 || a->D <= 0 || a->V <= 0 || a->lora_rank < 0)
    return ISD_ERR_INVALID_ARG;
  if (a->dtype != ISD_BF16) return ISD_ERR_UNSUPPORTED;
  if (a->D % 64 != 0 || a->V % 8 != 0) return ISD_ERR_UNSUPPORTED;
  if (a->lora_rank % 64 != 0 || a->lora_rank > 256) return ISD_ERR_UNSUPPORTED;
  if (a->lora_rank > 0) {
    if (a->rows_per_seq <= 0 || a->M % a->rows_per_seq != 0)
      return ISD_ERR_INVALID_ARG;
  }
  return ISD_OK;
}

size_t isd_lm_head_workspace_bytes(const isd_lm_head_args* a) {
  if (lm_head_check(a) != ISD_OK) return 0;
  return isd::lm_head_workspace_bytes(a);
}

int isd_lm_head_launches(const isd_lm_head_args* a) {
  if (lm_head_check(a) != ISD_OK) return 0;
  return isd::lm_head_launches(a);
}

size_t isd_vocab_stats_bytes(int32_t M, int32_t V) {
  if (M <= 0 || V <= 0) return 0;
  return isd::vocab_stats_bytes(M, V);
}

int isd_lm_head(const isd_lm_head_args* a, void* stream) {
  const int rc = lm_head_check(a);
  if (rc != ISD_OK) return rc;
  if (!a->hidden || !a->weight || !a->logits) return ISD_ERR_INVALID_ARG;
  if (a->lora_rank > 0 && (!a->lora_a || !a->lora_b || !a->n_pending))
    return ISD_ERR_INVALID_ARG;
  if (!aligned16(a->hidden) || !aligned16(a->weight) ||
      !aligned16(a->logits) || !aligned16(a->vocab_stats) ||
      !aligned16(a->lora_a) || !aligned16(a->lora_b))
    return ISD_ERR_INVALID_ARG;
  if (a->logits == a->hidden || a->logits == a->weight)
    return ISD_ERR_INVALID_ARG;
  const size_t need = isd::lm_head_workspace_bytes(a);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return ISD_ERR_WORKSPACE;
  return isd::launch_lm_head(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
