// isd_kv_commit kernels: commit of the accepted stride prefix into the
// paged KV cache, rollback of the rest.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io), "Serving (SGLang)": the engine keeps a paged KV cache.  Which
// rows are committed follows the stride schedule: the exact token and the
// accepted drafts (rows 0 .. n_commit-1); rejected drafts and MASK rows are
// never written, so rolling them back costs nothing.
//
// Two kernels on one stream:
//   plan  one CTA: per-sequence page demand, exclusive scan in sequence
//         order, pops from the free stack, page-table and length update;
//         all-or-nothing when the pool or a page-table row is too small
//   copy  grid (B, K): one CTA per committed row copies Hkv*d elements of
//         K and of V into the row's page slot with 16-byte stores
#include "common.cuh"

namespace isd {

struct CommitDev {
  int B, K, Hkv, d, P, stride, esize;
  const uint8_t* k_new;
  const uint8_t* v_new;
  uint8_t* k_cache;
  uint8_t* v_cache;
  int32_t* page_table;
  int32_t* seq_len;
  const int32_t* n_commit;
  const int32_t* free_stack;
  int32_t* free_top;
  int32_t* status;
  int32_t* old_len;  // workspace [B]
  int32_t* go;       // workspace [1]: 1 when the copy may proceed
  int32_t* offs;     // workspace [B]
};

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) commit_plan_kernel(CommitDev p) {
  __shared__ int sh[33];
  __shared__ int s_err;
  if (threadIdx.x == 0) s_err = ISD_OK;
  __syncthreads();
  auto need = [&](int b) -> int {
    const int L = p.seq_len[b], n = p.n_commit[b];
    if (L < 0 || n < 0 || n > p.K) { s_err = ISD_ERR_BAD_STATE; return 0; }
    const int old_pages = (L + kPage - 1) / kPage;
    const int new_pages = (L + n + kPage - 1) / kPage;
    if (new_pages > p.stride) { s_err = ISD_ERR_PAGE_TABLE_FULL; return 0; }
    return new_pages - old_pages;
  };
  const int total = block_exclusive_scan_int(p.B, need, p.offs, sh);
  __syncthreads();
  const int top = *p.free_top;
  int err = s_err;
  if (err == ISD_OK && total > top) err = ISD_ERR_POOL_EXHAUSTED;
  if (err != ISD_OK) {
    if (threadIdx.x == 0) { *p.status = err; *p.go = 0; }
    return;
  }
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int L = p.seq_len[b], n = p.n_commit[b];
    const int old_pages = (L + kPage - 1) / kPage;
    const int new_pages = (L + n + kPage - 1) / kPage;
    const int off = p.offs[b];
    for (int k = 0; k < new_pages - old_pages; ++k) {
      const int page = p.free_stack[top - 1 - (off + k)];
      if (page < 0 || page >= p.P) err = ISD_ERR_BAD_PAGE;
      p.page_table[(size_t)b * p.stride + old_pages + k] = page;
    }
    p.old_len[b] = L;
    p.seq_len[b] = L + n;
  }
  if (err != ISD_OK) atomicExch(&s_err, err);
  __syncthreads();
  if (threadIdx.x == 0) {
    *p.free_top = top - total;
    *p.status = s_err;
    *p.go = s_err == ISD_OK ? 1 : 0;
  }
}

__global__ void __launch_bounds__(256) commit_copy_kernel(CommitDev p) {
  const int b = blockIdx.x, r = blockIdx.y;
  if (*p.go == 0) return;
  if (r >= p.n_commit[b]) return;
  const int pos = p.old_len[b] + r;
  const int page = p.page_table[(size_t)b * p.stride + pos / kPage];
  if (page < 0 || page >= p.P) return;
  const int slot = pos % kPage;
  const size_t row_bytes = (size_t)p.d * p.esize;       // one head's row
  const int vec_per_head = (int)(row_bytes / 16);
  const int nvec = p.Hkv * vec_per_head;
  for (int i = threadIdx.x; i < 2 * nvec; i += blockDim.x) {
    const bool is_v = i >= nvec;
    const int j = is_v ? i - nvec : i;
    const int h = j / vec_per_head, c = j % vec_per_head;
    const uint8_t* src = (is_v ? p.v_new : p.k_new) +
                         (((size_t)b * p.K + r) * p.Hkv + h) * row_bytes + c * 16;
    uint8_t* dst = (is_v ? p.v_cache : p.k_cache) +
                   (((size_t)page * p.Hkv + h) * kPage + slot) * row_bytes + c * 16;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

size_t commit_workspace_bytes(int B) { return (size_t)(2 * B + 1) * 4 + 256; }

int launch_commit(const isd_commit_args* a, cudaStream_t st) {
  CommitDev p;
  p.B = a->B; p.K = a->K; p.Hkv = a->Hkv; p.d = a->d;
  p.P = a->num_pages; p.stride = a->page_table_stride;
  p.esize = a->dtype == ISD_BF16 ? 2 : 4;
  p.k_new = static_cast<const uint8_t*>(a->k_new);
  p.v_new = static_cast<const uint8_t*>(a->v_new);
  p.k_cache = static_cast<uint8_t*>(a->k_cache);
  p.v_cache = static_cast<uint8_t*>(a->v_cache);
  p.page_table = a->page_table; p.seq_len = a->seq_len;
  p.n_commit = a->n_commit; p.free_stack = a->free_stack;
  p.free_top = a->free_top; p.status = a->status;
  int32_t* ws = static_cast<int32_t*>(a->workspace);
  p.old_len = ws;
  p.offs = ws + a->B;
  p.go = ws + 2 * a->B;
  commit_plan_kernel<<<1, kPlanThreads, 0, st>>>(p);
  commit_copy_kernel<<<dim3(a->B, a->K), 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

}  // namespace isd
