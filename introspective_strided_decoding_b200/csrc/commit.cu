// isd_kv_commit: commit of the accepted stride prefix into the paged KV
// cache, rollback of the rest, in one kernel.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io), "Serving (SGLang)": the engine keeps a paged KV cache.  Which
// rows are committed follows the stride schedule: the exact token and the
// accepted drafts (rows 0 .. n_commit-1); rejected drafts and MASK rows are
// never written, so rolling them back costs nothing.
//
// One CTA per group of sequences (one each up to B = 1024).  Every CTA
//   1. scans the page demand of ALL sequences in sequence order (a few
//      hundred bytes from L2) and validates the whole commit: lengths and
//      counts, page-table rows, the pool size, every page id the commit
//      would write through or pop (the free-stack entries below the top are
//      read while the scan runs);
//   2. if anything is wrong, writes nothing (the verdict is the same in
//      every CTA, so the commit is all-or-nothing) and CTA 0 reports it;
//   3. otherwise records its sequences' new pages in the page table and
//      copies their committed K/V rows with 16-byte stores (the rows' pages
//      looked up once, eight loads a thread in flight before their stores);
//   4. counts itself done; the last CTA (a self-resetting counter in the
//      workspace) grows every seq_len and lowers the free-stack top, once
//      every CTA has read the old values.
#include "common.cuh"

namespace isd {

struct CommitDev {
  int B, K, Hkv, d, P, stride, esize, per;   // per: sequences per CTA
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
  unsigned int* done;   // workspace: CTAs finished; back to 0 after a call
  int trigger;          // let the next grid launch once this one has waited
};

constexpr int kCommitThreads = 256;
constexpr int kCommitMaxCtas = 1024;
constexpr int kCommitMaxPer = 32;            // so B <= 32 768
// When several conditions hold, the lowest rank is reported (the same
// choice on every run and in every CTA).
constexpr int kRankNone = INT_MAX, kRankBadState = 1, kRankTableFull = 2,
              kRankPool = 3, kRankBadPage = 4;

ISD_DEV int code_of_rank(int r) {
  return r == kRankBadState ? ISD_ERR_BAD_STATE
       : r == kRankTableFull ? ISD_ERR_PAGE_TABLE_FULL
       : r == kRankPool ? ISD_ERR_POOL_EXHAUSTED
                        : ISD_ERR_BAD_PAGE;
}

__global__ void __launch_bounds__(kCommitThreads) commit_kernel(CommitDev p) {
  __shared__ int sh[33];
  __shared__ int s_rank;
  __shared__ int s_last;
  __shared__ int s_off[kCommitMaxPer];   // first popped slot of own sequences
  __shared__ int s_fs[kCommitThreads];   // free_stack[top - 1 - k], k < 256
  __shared__ int s_pg[2];                // pages of the sequence's new rows
  const int c = blockIdx.x, G = gridDim.x, tid = threadIdx.x;
  if (tid == 0) s_rank = kRankNone;
  grid_dep_wait();
  if (p.trigger) grid_dep_trigger();
  __syncthreads();
  // The free-stack top and the first entries below it are read while the
  // page demand is being scanned (they do not depend on it).
  const int top = *p.free_top;
  const bool top_ok = top >= 0 && top <= p.P;
  if (tid == 0 && !top_ok) atomicMin(&s_rank, kRankBadState);
  s_fs[tid] = top_ok && tid < top ? p.free_stack[top - 1 - tid] : -1;
  // 1. Page demand of every sequence, scanned in sequence order.
  auto need = [&](int b) -> int {
    const int L = p.seq_len[b], n = p.n_commit[b];
    if (L < 0 || n < 0 || n > p.K) {
      atomicMin(&s_rank, kRankBadState);
      return 0;
    }
    const int old_pages = (L + kPage - 1) / kPage;
    const int new_pages = (L + n + kPage - 1) / kPage;
    if (new_pages > p.stride) {
      atomicMin(&s_rank, kRankTableFull);
      return 0;
    }
    // A partly filled last page receives rows: its id is written through.
    if (n > 0 && L % kPage != 0) {
      const int pg = p.page_table[(size_t)b * p.stride + L / kPage];
      if (pg < 0 || pg >= p.P) atomicMin(&s_rank, kRankBadPage);
    }
    return new_pages - old_pages;
  };
  const int total = block_exclusive_scan_int(
      p.B, need,
      [&](int b, int e) {
        if (b % G == c) s_off[b / G] = e;
      },
      sh);
  __syncthreads();
  int rank = s_rank;
  if (rank == kRankNone && total > top) rank = kRankPool;
  if (rank == kRankNone) {
    // 2. Every page to pop, free_stack[top - total .. top - 1], is an id.
    for (int k = tid; k < total; k += blockDim.x) {
      const int pg = k < kCommitThreads ? s_fs[k] : p.free_stack[top - 1 - k];
      if (pg < 0 || pg >= p.P) atomicMin(&s_rank, kRankBadPage);
    }
    __syncthreads();
    rank = s_rank;
  }
  if (rank != kRankNone) {
    if (c == 0 && tid == 0) report(p.status, code_of_rank(rank));
    return;   // nothing written; no CTA counts itself, the counter stays 0
  }
  // 3. This CTA's sequences: new pages, then the committed rows.
  auto popped = [&](int k) {
    return k < kCommitThreads ? s_fs[k] : p.free_stack[top - 1 - k];
  };
  const size_t row_bytes = (size_t)p.d * p.esize;   // one head's row
  const int vec_per_head = (int)(row_bytes / 16);
  const int nvec = p.Hkv * vec_per_head;            // per row, K or V
  for (int k = 0; k < p.per; ++k) {
    const int b = c + k * G;
    if (b >= p.B) break;
    const int L = p.seq_len[b], n = p.n_commit[b];
    if (n == 0) continue;
    const int old_pages = (L + kPage - 1) / kPage;
    const int grow = (L + n + kPage - 1) / kPage - old_pages;
    const int off = s_off[k];
    const int lp0 = L / kPage;                      // first page written
    // The (at most two) pages the rows land in, and the table entries.
    if (tid < 2 && lp0 + tid <= (L + n - 1) / kPage) {
      const int lp = lp0 + tid;
      s_pg[tid] = lp < old_pages ? p.page_table[(size_t)b * p.stride + lp]
                                 : popped(off + lp - old_pages);
    }
    if (tid < grow)
      p.page_table[(size_t)b * p.stride + old_pages + tid] = popped(off + tid);
    __syncthreads();
    // Eight 16-byte vectors a thread in flight before their stores.
    const int nv = n * 2 * nvec;
    for (int i0 = 0; i0 < nv; i0 += 8 * blockDim.x) {
      uint4 val[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x + tid;
        if (i < nv) {
          const int r = i / (2 * nvec);
          const int j2 = i - r * 2 * nvec;
          const bool is_v = j2 >= nvec;
          const int j = is_v ? j2 - nvec : j2;
          const int h = j / vec_per_head, cv = j - h * vec_per_head;
          const uint8_t* src = (is_v ? p.v_new : p.k_new) +
                               (((size_t)b * p.K + r) * p.Hkv + h) * row_bytes +
                               cv * 16;
          val[u] = __ldg(reinterpret_cast<const uint4*>(src));
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x + tid;
        if (i < nv) {
          const int r = i / (2 * nvec);
          const int j2 = i - r * 2 * nvec;
          const bool is_v = j2 >= nvec;
          const int j = is_v ? j2 - nvec : j2;
          const int h = j / vec_per_head, cv = j - h * vec_per_head;
          const int pos = L + r;
          const int page = s_pg[pos / kPage - lp0];
          uint8_t* dst = (is_v ? p.v_cache : p.k_cache) +
                         (((size_t)page * p.Hkv + h) * kPage + pos % kPage) *
                             row_bytes +
                         cv * 16;
          *reinterpret_cast<uint4*>(dst) = val[u];
        }
      }
    }
    __syncthreads();                                // s_pg is reused
  }
  // 4. The last CTA publishes the new lengths and the free-stack top.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicInc(p.done, (unsigned)(G - 1)) == (unsigned)(G - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int b = tid; b < p.B; b += blockDim.x) p.seq_len[b] += p.n_commit[b];
  if (tid == 0) *p.free_top = top - total;
}

size_t commit_workspace_bytes(int) { return 256; }

int commit_max_batch() { return kCommitMaxCtas * kCommitMaxPer; }

int launch_commit(const isd_commit_args* a, cudaStream_t st, bool trigger) {
  CommitDev p;
  p.B = a->B; p.K = a->K; p.Hkv = a->Hkv; p.d = a->d;
  p.P = a->num_pages; p.stride = a->page_table_stride;
  p.esize = a->dtype == ISD_BF16 ? 2 : 4;
  p.per = (a->B + kCommitMaxCtas - 1) / kCommitMaxCtas;
  if (p.per > kCommitMaxPer) return ISD_ERR_UNSUPPORTED;
  p.k_new = static_cast<const uint8_t*>(a->k_new);
  p.v_new = static_cast<const uint8_t*>(a->v_new);
  p.k_cache = static_cast<uint8_t*>(a->k_cache);
  p.v_cache = static_cast<uint8_t*>(a->v_cache);
  p.page_table = a->page_table; p.seq_len = a->seq_len;
  p.n_commit = a->n_commit; p.free_stack = a->free_stack;
  p.free_top = a->free_top; p.status = a->status;
  p.done = static_cast<unsigned int*>(a->workspace);
  p.trigger = trigger ? 1 : 0;
  const int G = (a->B + p.per - 1) / p.per;
  return launch_pdl(commit_kernel, dim3(G), dim3(kCommitThreads), 0, st, p) ==
                 cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

}  // namespace isd
