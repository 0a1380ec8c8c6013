// isd_attn_strided on the 5th-generation tensor cores (tcgen05 + TMEM), for
// bf16 with head dim 128 and up to 128 query rows per KV head.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io): strict causal attention with a logit shift ("Méthodologie"),
// a paged KV cache read by a paged-only attention kernel ("Serving
// (SGLang)").  Row r of sequence b attends to cached positions [0, L_b)
// and stride rows 0..r.
//
// Work split: the flat list of (sequence, KV head, page) units plus one
// tail unit per (sequence, head) is cut into equal contiguous ranges, one
// per persistent CTA.  Inside a CTA the units of each (b, h) segment are
// taken in blocks of up to kNB pages (16 * kNB keys).  Warp roles:
//
//   loaders (kLoadWarps)  each block's K pages through the TMA engine (one
//                         thread, 64-column boxes) and its V pages with
//                         16-byte cp.async from every loader thread, both
//                         into 128-byte-swizzled tiles with the pages
//                         stacked along the key axis; two copy engines run
//                         in parallel.  Also each segment's Q rows.  The
//                         stage barrier counts every loader thread's
//                         cp.async arrival plus the TMA transaction bytes
//   MMA warp              one thread issues S = Q K^T (M = 128 padded rows,
//                         N = keys of the block, 8 k-steps) into a double-
//                         buffered S in TMEM, and O += P V (one k-step per
//                         page) into O in TMEM; completion is committed to
//                         mbarriers.  QK of block i+1 is issued before PV of
//                         block i so the softmax of a block overlaps the
//                         tensor core.  It also allocates and frees TMEM.
//   softmax (4 warps)     one query row per thread: reads its S row from
//                         TMEM, masks the tail / partial page, keeps the
//                         running max and sum in registers, writes P (bf16)
//                         to shared memory; O is rescaled in TMEM only when
//                         a row's max grows by more than 2^8 (base 2), so
//                         most blocks need no correction.  At a segment's
//                         end it reads O, normalises and stores it (or a
//                         partial for the combine kernel when the (b, h)
//                         straddles CTAs).
//
// Shared operands use the tensor cores' canonical 128-byte-swizzle layouts:
// Q and K and P K-major (reduction dimension contiguous), V MN-major (head
// dimension contiguous).  Every mbarrier wait is bounded; after one timeout
// a thread records ISD_ERR_CUDA and stops waiting, so the kernel ends.
#include "common.cuh"

namespace isd {

// Shared with attn.cu: unit prefix, partial layout and combine kernel.
int launch_attn_combine(const isd_attn_args* a, int G, cudaStream_t st);

namespace tc {

constexpr int D = 128;
constexpr int kNB = 4;                       // pages per block
constexpr int kBlockKeys = 16 * kNB;         // 64
constexpr int kStagesTc = 4;
constexpr int kHalf = kBlockKeys * 128;      // one 64-column half, bytes
constexpr int kStageBytes = 4 * kHalf;       // K0 K1 V0 V1 = 32 KB
constexpr int kQHalf = 128 * 128;            // 128 rows x 128 B
constexpr int kQBytes = 2 * kQHalf;          // 32 KB
constexpr int kPBytes = 128 * 128;           // 128 rows x 64 keys bf16
constexpr int kSmWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarps = 11;
constexpr int kThreads = (kSmWarps + 1 + kLoadWarps) * 32;   // 512
constexpr int kLoadThreads = kLoadWarps * 32;
constexpr uint32_t kTmemCols = 256;          // O: 0..127, S: 128..255
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kWaitCycles = 400000000ull;   // ~0.2 s

struct Params {
  int B, Hq, Hkv, K, g, M, P, stride;
  float scale_log2;
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const __nv_bfloat16* kn;
  const __nv_bfloat16* vn;
  __nv_bfloat16* out;
  float* lse;
  const int32_t* page_table;
  const int32_t* seq_len;
  int32_t* status;
  float* part;
  int32_t* ws_int;
};

// ------------------------------------------------------------------ PTX
ISD_DEV uint64_t sdesc(uint32_t start, uint32_t lbo, uint32_t sbo) {
  // Shared-memory matrix descriptor (sm_100): start, leading / stride byte
  // offsets (16-byte units), descriptor version 1, 128-byte swizzle.
  return (uint64_t)((start >> 4) & 0x3FFFu) |
         ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (2ull << 61);
}
ISD_DEV uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  // kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B,
  // A K-major, B K-major (0) or MN-major (1), N >> 3, M >> 4.
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
ISD_DEV void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                  uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}
ISD_DEV void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(smem_u32(bar))
      : "memory");
}
ISD_DEV void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
ISD_DEV void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
ISD_DEV void proxy_fence() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// TMEM -> registers, 16 columns of this thread's lane.  The wait is tied
// to the destination registers ("+r"), so no use can be scheduled before
// the load has landed.
ISD_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,"
      "%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]),
                 "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]),
                 "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
ISD_DEV void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,"
      "%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
      "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])),
      "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
ISD_DEV void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Bounded wait; after the first timeout (`failed` set) waits are skipped.
ISD_DEV void wait_or_fail(uint64_t* bar, uint32_t parity, bool& failed,
                          int32_t* status) {
  if (failed) return;
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if ((uint64_t)(clock64() - t0) > kWaitCycles) {
      failed = true;
      if (status) *status = ISD_ERR_CUDA;
      return;
    }
  }
}

ISD_DEV int find_seq_tc(const int* prefix, int B, int u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Walks the blocks of a CTA's unit range in the order every role uses.
struct BlockWalk {
  const int* prefix;
  int B, Hkv, u1;
  int u;           // first unit of the current segment's remaining part
  int b, h, units, idx0, seg_end, seg_begin_u;
  bool complete;
  int k;           // offset of the next block inside the segment
  int nseg;

  ISD_DEV void open_segment() {
    b = find_seq_tc(prefix, B, u);
    units = (prefix[b + 1] - prefix[b]) / Hkv;
    const int rel = u - prefix[b];
    h = rel / units;
    idx0 = rel - h * units;
    const int bh_end = prefix[b] + (h + 1) * units;
    seg_end = min(u1, bh_end);
    nseg = seg_end - u;
    complete = idx0 == 0 && seg_end == bh_end;
    seg_begin_u = u;
    k = 0;
  }
  ISD_DEV void init(const int* pf, int B_, int Hkv_, int u0, int u1_) {
    prefix = pf; B = B_; Hkv = Hkv_; u1 = u1_; u = u0;
    if (u < u1) open_segment();
  }
  ISD_DEV bool done() const { return u >= u1; }
  // Current block: units idx0 + k .. idx0 + k + nu - 1 of segment (b, h).
  ISD_DEV int nu() const { return min(kNB, nseg - k); }
  ISD_DEV bool first() const { return k == 0; }
  ISD_DEV bool last() const { return k + kNB >= nseg; }
  ISD_DEV void next() {
    k += kNB;
    if (k >= nseg) {
      u = seg_end;
      if (u < u1) open_segment();
    }
  }
};

// R: replicas of the query rows in the 128-row tile (4 for up to 32 rows,
// 2 for up to 64, 1 for 128).  With R > 1 every TMEM lane quarter holds a
// copy of the rows, so all four softmax warps work on every block: warp w
// takes 4/R pages of it for its 32 rows, the warps sharing rows exchange
// row maxima, and P and O come out replicated, the output columns split
// between the replicas.
template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_kn, Params p) {
  constexpr int Mq = 128 / R;            // rows per replica (padded)
  constexpr int QPR = Mq / 32;           // lane quarters per replica
  constexpr int UPW = kNB / R;           // pages per softmax warp and block
  constexpr int OPW = D / R;             // output columns per softmax warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kv = base;                                  // stages
  uint8_t* qs = kv + kStagesTc * kStageBytes;          // Q tile
  uint8_t* ps = qs + kQBytes;                          // 2 P tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(ps + 2 * kPBytes);
  uint64_t* kv_full = bars;                            // [kStagesTc]
  uint64_t* kv_empty = kv_full + kStagesTc;            // [kStagesTc]
  uint64_t* s_full = kv_empty + kStagesTc;             // [2]
  uint64_t* s_free = s_full + 2;                       // [2]
  uint64_t* p_full = s_free + 2;                       // [2]
  uint64_t* p_empty = p_full + 2;                      // [2]
  uint64_t* q_full = p_empty + 2;
  uint64_t* q_empty = q_full + 1;
  uint64_t* o_done = q_empty + 1;
  uint64_t* o_free = o_done + 1;
  uint64_t* fin = o_free + 1;                          // all MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);
  __shared__ int scan_sh[33];
  __shared__ int s_bad;
  __shared__ float x_max[2][kSmWarps][32];   // row-max exchange, per S buffer
  __shared__ float x_sum[kSmWarps][32];      // row-sum exchange (epilogue)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, Hkv = p.Hkv, M = p.M;
  const int active_sm = kSmWarps;                      // all take part
  if (tid == 0) s_bad = 0;
  __syncthreads();
  const int T = block_exclusive_scan_int(
      B,
      [&](int b) {
        int L = p.seq_len[b];
        bool bad = false;
        if (L < 0) { bad = true; L = 0; }
        int n = (L + kPage - 1) / kPage;
        if (n > p.stride) { bad = true; n = p.stride; }
        if (bad) s_bad = 1;
        return Hkv * (n + 1);
      },
      prefix, scan_sh);
  if (tid == 0) prefix[B] = T;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = (int)(((long long)c * T) / G);
  const int u1 = (int)(((long long)(c + 1) * T) / G);
  if (tid == 0) {
    for (int s = 0; s < kStagesTc; ++s) {
      // Loader threads' cp.async arrivals (V) + one expect_tx arrival
      // covering the TMA bytes (K).
      mbar_init(&kv_full[s], kLoadThreads + 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], active_sm);
      mbar_init(&p_full[s], active_sm);
      mbar_init(&p_empty[s], 1);
    }
    mbar_init(q_full, kLoadThreads);
    mbar_init(q_empty, 1);
    mbar_init(o_done, 1);
    mbar_init(o_free, active_sm);
    mbar_init(fin, 1);
    fence_barrier_init();
  }
  // Padding rows of every replica (index within the replica >= M) stay
  // zero for the whole kernel.
  for (int i = tid; i < 128 * 16; i += blockDim.x) {
    const int row = i / 16, ch = i % 16;
    if (row % Mq < M) continue;
    *reinterpret_cast<uint4*>(qs + (ch >> 3) * kQHalf + row * 128 +
                              (((ch & 7) ^ (row & 7)) << 4)) =
        make_uint4(0, 0, 0, 0);
  }
  proxy_fence();
  if (warp == kMmaWarp) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::
            "r"(smem_u32(tmem_slot)),
        "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (c == 0) {
    for (int i = tid; i <= B; i += blockDim.x) p.ws_int[i] = prefix[i];
    if (tid == 0) {
      p.ws_int[B + 1] = G;
      if (s_bad && p.status) *p.status = ISD_ERR_PAGE_TABLE_FULL;
    }
  }
  const uint32_t kv_s = smem_u32(kv), q_s = smem_u32(qs), p_s = smem_u32(ps);
  bool failed = false;

  if (warp > kMmaWarp) {
    // ------------------------------------------------------------ loaders
    const int lt = tid - (kMmaWarp + 1) * 32;
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    int i = 0, nseg_done = 0;
    while (!w.done()) {
      if (w.first()) {
        // Q rows of (b, h): row m = r * g + j holds q[b][r][h*g + j][:].
        wait_or_fail(q_empty, (nseg_done & 1) ^ 1, failed, p.status);
        for (int q = lt; q < R * M * 16; q += kLoadThreads) {
          const int rep = q / (M * 16), rem = q - rep * M * 16;
          const int m = rem >> 4, ch = rem & 15;
          const int r = m / p.g, j = m - r * p.g;
          const int row = rep * Mq + m;
          const __nv_bfloat16* src =
              p.q + (((size_t)w.b * p.K + r) * p.Hq + w.h * p.g + j) * D + ch * 8;
          cp_async_16(q_s + (ch >> 3) * kQHalf + row * 128 +
                          (((ch & 7) ^ (row & 7)) << 4),
                      src, 16);
        }
        cp_async_arrive(q_full);
        ++nseg_done;
      }
      const int st = i % kStagesTc;
      wait_or_fail(&kv_empty[st], ((i / kStagesTc) & 1) ^ 1, failed, p.status);
      const int nu = w.nu();
      const uint32_t sb = kv_s + st * kStageBytes;
      uint8_t* sbp = kv + st * kStageBytes;
      const int Lb = p.seq_len[w.b];
      // K tiles through the TMA engine (one thread): two 64-column boxes per
      // page, landing in the block's 128-byte-swizzled K-major halves.
      // Rows past K of the tail lie outside the staging tensor and read as
      // zeros, as does a page id out of range.
      if (lt == 0) {
        mbar_arrive_expect_tx(&kv_full[st], nu * 2 * 2048);
        for (int k = 0; k < nu; ++k) {
          const int uidx = w.idx0 + w.k + k;
          if (uidx == w.units - 1) {
            for (int hb = 0; hb < 2; ++hb)
              tma_load_4d(sbp + hb * kHalf + k * 2048, &tm_kn, &kv_full[st],
                          hb * 64, w.h, 0, w.b);
          } else {
            int page = p.page_table[(size_t)w.b * p.stride + uidx];
            if (page < 0 || page >= p.P) {
              if (p.status) *p.status = ISD_ERR_BAD_PAGE;
              page = p.P;
            }
            for (int hb = 0; hb < 2; ++hb)
              tma_load_4d(sbp + hb * kHalf + k * 2048, &tm_kc, &kv_full[st],
                          hb * 64, 0, w.h, page);
          }
        }
      }
      // V tiles with cp.async from every loader thread.  Slots past L_b (a
      // partial last page) are zero-filled, never copied: they may hold any
      // bits, and 0 * NaN would reach O through P V.
      for (int q = lt; q < nu * 256; q += kLoadThreads) {
        const int k = q >> 8, ww = q & 255;
        const int row = ww >> 4, ch = ww & 15;
        const int uidx = w.idx0 + w.k + k;
        const int key = k * 16 + row;
        const uint32_t dst = sb + 2 * kHalf + (ch >> 3) * kHalf + key * 128 +
                             (((ch & 7) ^ (key & 7)) << 4);
        const __nv_bfloat16* src = p.vc;
        uint32_t bytes = 0;
        if (uidx == w.units - 1) {          // tail: the stride's own rows
          if (row < p.K) {
            src = p.vn + (((size_t)w.b * p.K + row) * Hkv + w.h) * D + ch * 8;
            bytes = 16;
          }
        } else if (row < Lb - uidx * kPage) {
          const int page = p.page_table[(size_t)w.b * p.stride + uidx];
          if (page >= 0 && page < p.P) {
            src = p.vc + (((size_t)page * Hkv + w.h) * kPage + row) * D + ch * 8;
            bytes = 16;
          }
        }
        cp_async_16(dst, src, bytes);
      }
      cp_async_arrive(&kv_full[st]);
      w.next();
      ++i;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    int i = 0, nseg = 0;
    int prev_nu = 0, prev_st = 0, prev_pb = 0;
    bool prev_first = false, have_prev = false;
    const uint32_t id_pv = idesc_bf16(128, D, 1);
    auto issue_pv = [&](int j_blk) {
      // O += P V for block j_blk (its P buffer, stage and page count).
      wait_or_fail(&p_full[prev_pb], (j_blk >> 1) & 1, failed, p.status);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pa = p_s + prev_pb * kPBytes;
        const uint32_t vb = kv_s + prev_st * kStageBytes + 2 * kHalf;
        for (int j = 0; j < prev_nu; ++j)
          umma(tmem, sdesc(pa + j * 32, 16, 1024),
               sdesc(vb + j * 2048, kHalf, 1024), id_pv,
               (prev_first && j == 0) ? 0u : 1u);
        umma_commit(&kv_empty[prev_st]);
        umma_commit(&p_empty[prev_pb]);
        umma_commit(o_done);
      }
      __syncwarp();
    };
    int seg_pv = 0;  // segments whose first PV has been issued
    while (!w.done()) {
      const int st = i % kStagesTc, sbuf = i & 1;
      if (w.first()) {
        wait_or_fail(q_full, nseg & 1, failed, p.status);
        ++nseg;
      }
      wait_or_fail(&kv_full[st], (i / kStagesTc) & 1, failed, p.status);
      wait_or_fail(&s_free[sbuf], ((i >> 1) & 1) ^ 1, failed, p.status);
      // Q and V arrived through cp.async (generic proxy); the tensor core
      // reads them through the async proxy.
      proxy_fence();
      tc_fence_after();
      const int nu = w.nu();
      if (lane == 0) {
        const uint32_t id_qk = idesc_bf16(128, 16 * nu, 0);
        const uint32_t kb = kv_s + st * kStageBytes;
        for (int kk = 0; kk < 8; ++kk)
          umma(tmem + 128 + sbuf * kBlockKeys,
               sdesc(q_s + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024),
               sdesc(kb + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024), id_qk,
               kk > 0 ? 1u : 0u);
        umma_commit(&s_full[sbuf]);
        if (w.last()) umma_commit(q_empty);
      }
      __syncwarp();
      if (have_prev) {
        if (prev_first && seg_pv > 0)
          wait_or_fail(o_free, (seg_pv - 1) & 1, failed, p.status);
        if (prev_first) ++seg_pv;
        issue_pv(i - 1);
      }
      have_prev = true;
      prev_nu = nu; prev_st = st; prev_pb = sbuf; prev_first = w.first();
      w.next();
      ++i;
    }
    if (have_prev) {
      if (prev_first && seg_pv > 0)
        wait_or_fail(o_free, (seg_pv - 1) & 1, failed, p.status);
      issue_pv(i - 1);
    }
    // Every MMA this CTA issued has completed before TMEM is released.
    if (lane == 0) umma_commit(fin);
    __syncwarp();
    bool fin_failed = false;
    wait_or_fail(fin, 0, fin_failed, p.status);
  } else if (warp < kSmWarps) {
    // ---------------------------------------------------------- softmax
    const int rep = warp / QPR;                        // replica of this warp
    const int rbase = (warp % QPR) * 32;
    const int row = rbase + lane;                      // query row m
    const bool real = row < M;
    const int rq = real ? row / p.g : 0, jq = real ? row - rq * p.g : 0;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float c2 = p.scale_log2;
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    int i = 0;
    float m_ref = -INFINITY, l = 0.0f;                 // l: this warp's pages
    while (!w.done()) {
      const int sbuf = i & 1;
      const bool first = w.first();
      if (first) { m_ref = -INFINITY; l = 0.0f; }
      const int nu = w.nu();
      const int L = p.seq_len[w.b];
      wait_or_fail(&s_full[sbuf], (i >> 1) & 1, failed, p.status);
      tc_fence_after();
      float s[UPW * 16];
#pragma unroll
      for (int k = 0; k < UPW; ++k) {
        const int ku = rep * UPW + k;                  // page within block
        if (ku < nu) {
          float v[16];
          tmem_ld16(tmem + lane_base + 128 + sbuf * kBlockKeys + ku * 16, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) s[k * 16 + e] = v[e];
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) s[k * 16 + e] = -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sbuf]);
      // Mask: keys past the valid slots of a partial page, and for the tail
      // unit stride rows after this row's own (causal inside the stride).
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < UPW; ++k) {
        const int ku = rep * UPW + k;
        if (ku < nu) {
          const int uidx = w.idx0 + w.k + ku;
          const bool tail = uidx == w.units - 1;
          const int valid = tail ? min(p.K, rq + 1)
                                 : min(kPage, L - uidx * kPage);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float& x = s[k * 16 + e];
            x = e < valid ? x : -INFINITY;
            mx = fmaxf(mx, x);
          }
        }
      }
      if (R > 1) {
        // Row max over the block: combine the R warps holding these rows.
        x_max[sbuf][warp][lane] = mx;
        asm volatile("bar.sync 1, %0;" ::"r"(kSmWarps * 32));
#pragma unroll
        for (int o = 0; o < R; ++o)
          mx = fmaxf(mx, x_max[sbuf][(warp % QPR) + o * QPR][lane]);
      }
      // Lazy rescale: move the reference max only when it grew by more
      // than 2^kRescaleLog2 (or on the segment's first block).  The warps
      // sharing rows take the same decision (same maxima).
      bool need = (mx - m_ref) * c2 > kRescaleLog2;
      if (first) need = false;
      if (__any_sync(0xffffffffu, need)) {
        // O must hold every earlier block's P V before it is scaled; each
        // warp scales the output columns it owns in its own lane quarter.
        wait_or_fail(o_done, (i - 1) & 1, failed, p.status);
        tc_fence_after();
        const float alpha = need ? ex2((m_ref - mx) * c2) : 1.0f;
#pragma unroll 1
        for (int c0 = rep * OPW; c0 < (rep + 1) * OPW; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + lane_base + c0, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] *= alpha;
          tmem_st16(tmem + lane_base + c0, v);
          tmem_st_wait();
        }
        l *= alpha;
        if (need) m_ref = mx;
      }
      if (first) m_ref = mx;
      // P = 2^((s - m_ref) c) in bf16 for this warp's pages, written into
      // every replica of these rows.
      wait_or_fail(&p_empty[sbuf], ((i >> 1) & 1) ^ 1, failed, p.status);
      const float off = m_ref * c2;
      float ls = 0.0f;
#pragma unroll
      for (int k = 0; k < UPW; ++k) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = ex2(fmaf(s[k * 16 + 2 * e], c2, -off));
          const float b2 = ex2(fmaf(s[k * 16 + 2 * e + 1], c2, -off));
          ls += a + b2;
          pk[e] = pack_bf16(a, b2);
        }
        const int ch0 = (rep * UPW + k) * 2;           // 16-byte chunk
#pragma unroll
        for (int o = 0; o < R; ++o) {
          const int trow = o * Mq + row;
          uint8_t* prow = ps + sbuf * kPBytes + trow * 128;
          *reinterpret_cast<uint4*>(prow + (((ch0 & 7) ^ (trow & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(
              prow + ((((ch0 + 1) & 7) ^ (trow & 7)) << 4)) =
              make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      l += ls;
      proxy_fence();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sbuf]);
      if (w.last()) {
        // Epilogue: O of this segment is complete once its last P V lands.
        float lt = l;
        if (R > 1) {
          x_sum[warp][lane] = l;
          asm volatile("bar.sync 1, %0;" ::"r"(kSmWarps * 32));
          lt = 0.0f;
#pragma unroll
          for (int o = 0; o < R; ++o) lt += x_sum[(warp % QPR) + o * QPR][lane];
          asm volatile("bar.sync 1, %0;" ::"r"(kSmWarps * 32));
        }
        wait_or_fail(o_done, i & 1, failed, p.status);
        tc_fence_after();
        const int slot = (w.seg_begin_u == u0) ? 0 : 1;
        float* part = p.part + ((size_t)(c * 2 + slot)) * M * (D + 2);
        const float inv = 1.0f / lt;
#pragma unroll 1
        for (int c0 = rep * OPW; c0 < (rep + 1) * OPW; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + lane_base + c0, v);
          if (real) {
            if (w.complete) {
              __nv_bfloat16* o = p.out +
                  (((size_t)w.b * p.K + rq) * p.Hq + w.h * p.g + jq) * D + c0;
              uint32_t pk[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                pk[e] = pack_bf16(v[2 * e] * inv, v[2 * e + 1] * inv);
              *reinterpret_cast<uint4*>(o) =
                  make_uint4(pk[0], pk[1], pk[2], pk[3]);
              *reinterpret_cast<uint4*>(o + 8) =
                  make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else {
#pragma unroll
              for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(part + (size_t)row * D + c0 + e) =
                    make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
          }
        }
        if (real && rep == 0) {
          if (w.complete) {
            if (p.lse)
              p.lse[((size_t)w.b * p.K + rq) * p.Hq + w.h * p.g + jq] =
                  (m_ref * c2 + log2f(lt)) * kLn2;
          } else {
            part[(size_t)M * D + row] = m_ref;
            part[(size_t)M * D + M + row] = lt;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
      w.next();
      ++i;
    }
  }
  // Everyone meets before TMEM is released.
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                     tmem),
                 "r"(kTmemCols));
  }
}

}  // namespace tc

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

static bool encode_tiled_4d(CUtensorMap* m, const void* base,
                            const uint64_t dims[4], const uint64_t strides[3],
                            const uint32_t box[4]) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
            gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_tc_smem_bytes(int B) {
  return 1024 + (size_t)tc::kStagesTc * tc::kStageBytes + tc::kQBytes +
         2 * tc::kPBytes + 32 * 8 + 16 + (size_t)(B + 1) * 4;
}

bool attn_tc_supported(const isd_attn_args* a) {
  const int M = a->K * (a->Hq / a->Hkv);
  return a->dtype == ISD_BF16 && a->d == 128 && M >= 1 && M <= 128 &&
         a->K <= kPage && attn_tc_smem_bytes(a->B) <= 227 * 1024;
}

int launch_attn_tc(const isd_attn_args* a, int G, cudaStream_t st) {
  tc::Params p;
  p.B = a->B; p.Hq = a->Hq; p.Hkv = a->Hkv; p.K = a->K;
  p.g = a->Hq / a->Hkv; p.M = a->K * p.g; p.P = a->num_pages;
  p.stride = a->page_table_stride;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.kc = static_cast<const __nv_bfloat16*>(a->k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(a->v_cache);
  p.kn = static_cast<const __nv_bfloat16*>(a->k_new);
  p.vn = static_cast<const __nv_bfloat16*>(a->v_new);
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.lse = a->lse; p.page_table = a->page_table; p.seq_len = a->seq_len;
  p.status = a->status;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  p.ws_int = reinterpret_cast<int32_t*>(ws);
  p.part = reinterpret_cast<float*>(
      ws + (((size_t)(a->B + 2) * 4 + 255) & ~size_t(255)));
  // K tensor maps: the cache [P][Hkv][16][128] and the stride's staged
  // rows [B][K][Hkv][128], 64-column boxes with the 128-byte swizzle.
  CUtensorMap tkc, tkn;
  const uint64_t dc[4] = {128, (uint64_t)kPage, (uint64_t)a->Hkv,
                          (uint64_t)a->num_pages};
  const uint64_t sc[3] = {256, (uint64_t)kPage * 256,
                          (uint64_t)a->Hkv * kPage * 256};
  const uint32_t bc[4] = {64, (uint32_t)kPage, 1, 1};
  const uint64_t dn[4] = {128, (uint64_t)a->Hkv, (uint64_t)a->K,
                          (uint64_t)a->B};
  const uint64_t sn[3] = {256, (uint64_t)a->Hkv * 256,
                          (uint64_t)a->K * a->Hkv * 256};
  const uint32_t bn[4] = {64, 1, (uint32_t)kPage, 1};
  if (!encode_tiled_4d(&tkc, a->k_cache, dc, sc, bc) ||
      !encode_tiled_4d(&tkn, a->k_new, dn, sn, bn))
    return ISD_ERR_CUDA;
  const size_t smem = attn_tc_smem_bytes(a->B);
  auto kern = p.M <= 32 ? tc::attn_tc_kernel<4>
                        : (p.M <= 64 ? tc::attn_tc_kernel<2>
                                     : tc::attn_tc_kernel<1>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  kern<<<G, tc::kThreads, smem, st>>>(tkc, tkn, p);
  if (cudaGetLastError() != cudaSuccess) return ISD_ERR_CUDA;
  return launch_attn_combine(a, G, st);
}

}  // namespace isd
