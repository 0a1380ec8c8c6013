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
// taken in blocks of up to kNB = 8 pages: 128 keys.
//
// Transposed products.  A decoding stride has few query rows per KV head
// (M = K * g, often 32) and many keys, so the keys take the MMA's 128-row
// side and the rows its N side (N = M rounded up to 32):
//   S^T[key][row]  = K Q^T        (A = K tile, B = Q, both K-major)
//   O^T[d][row]   += V^T P^T      (A = V tile read MN-major, B = P^T read
//                                  MN-major from a [key][row] tile)
// with S^T, O^T and the per-key partial row sums in TMEM.  No MMA row is
// padding, and each block costs 16 MMAs whatever M is.
//
// Warp roles (10 warps):
//   loaders (4 warps)   two warps copy K tiles, two copy V tiles, each pair
//                       in its own loop so a V slot in use never holds back
//                       a K copy; a warp covers 4 pages of every block and
//                       its lanes 0..7 issue the 8 TMA boxes (64-column
//                       halves, 128-byte swizzle) in one instruction.  A
//                       partial last page is loaded from valid - 16 rows
//                       up, so its slots past L_b read as zeros (from
//                       outside the tensor) and its keys take the last
//                       slots.  Page ids are read two blocks ahead.  Warp 0
//                       also loads each segment's Q rows by TMA.
//   QK MMA warp         one thread issues S^T of block i into a double-
//                       buffered S in TMEM and commits completion.  It
//                       also allocates and frees TMEM.
//   P V MMA warp        one thread issues O^T += V^T P^T of block i once
//                       its P is written (from 96 rows up also the row
//                       sums, a ones tile times the same P^T).  Two issuing
//                       warps: one thread issuing both kinds in order made
//                       each P V wait for the next K tile and capped the
//                       issue rate (measured: the two-warp split is 10%
//                       faster on the C=64 step).
//   softmax (4 warps)   thread t owns key t of the block (TMEM lane t): it
//                       masks its scores, writes P = 2^(s c - m_row c) in
//                       bf16 into P^T, and (up to 64 rows) adds P to its
//                       per-row partial sums (TMEM).  The reference max
//                       m_row moves only when some score of the block
//                       exceeds it by more than 2^8 (a vote over the 128
//                       threads); then the exact block max is reduced
//                       across the threads and O^T and the sums are
//                       rescaled.  At a segment's end the sums (reduced
//                       over the keys, or read from the ones product) give
//                       O^T / l, stored (or a partial for the combine
//                       kernel when the (b, h) straddles CTAs).
//
// Every mbarrier wait is bounded; after one timeout a thread records
// ISD_ERR_CUDA (unless an earlier error is already recorded) and stops
// waiting, so the kernel ends.
#include "tcgen05.cuh"

namespace isd {

// Shared with attn.cu: unit prefix, partial layout and combine kernel.
int launch_attn_combine(const isd_attn_args* a, int G, cudaStream_t st);
void attn_partial_ptrs(const isd_attn_args* a, int G, float** part_o,
                       float** part_ml);

namespace tc {

constexpr int kNB = 8;                       // pages per block
constexpr int kKeys = kNB * kPage;           // 128 keys = TMEM lanes
constexpr int kKH = kKeys * 128;             // one 64-column half of K or V
constexpr int kTile = 2 * kKH;               // a K or V tile: 32 KB
// Warp roles for NCH 32-row chunks: softmax warps (warpgroups of four;
// two for NCH >= 3, splitting the chunks between them), the QK and the P V
// MMA warps, then the loaders: two K and two V warps, or one of each
// (covering all 8 pages of a block) next to two softmax warpgroups, which
// keeps the CTA at 384 threads and 170 registers a thread.  Measured: at
// 128 rows (the softmax bounds the kernel) two warpgroups are 22% faster;
// at 64 rows the kernel is near the HBM bound and the single loader warps
// cost more (16% slower), so 64 rows keep one warpgroup.
constexpr int sm_warps_of(int nch) { return nch >= 3 ? 8 : 4; }
constexpr int load_warps_of(int nch) { return nch >= 3 ? 2 : 4; }
constexpr int threads_of(int nch) {
  return (sm_warps_of(nch) + 2 + load_warps_of(nch)) * 32;
}
constexpr int kBarBytes = 32 * 8;            // mbarriers (2 (SK + SV) + 17)
// Q and P^T tiles in shared memory for N = 32 * nch padded rows.  Two let
// the next (b, h) segment start (its Q load, its first softmax) while the
// previous one finishes; the largest row counts keep one where memory is
// short.
constexpr int nqb_of(int nch) { return nch == 4 ? 1 : 2; }
constexpr int npb_of(int nch) { return nch >= 3 ? 1 : 2; }
// __shared__ arrays of the kernel, rounded up.
// From three chunks up the row sums are accumulated by the tensor core: an
// M = 64 product of a tile of ones with the same P^T the P V product reads,
// so every row of it is the row sums (the softmax threads then neither load
// nor store per-key partial sums); up to two chunks keep the partials
// (measured at 64 rows: 6% slower with the extra product, 2.5% faster at
// 128 rows).
constexpr bool mma_rowsum_of(int nch) { return nch >= 3; }
constexpr int static_smem_of(int nch) {
  return (nch >= 3 ? 4096 : 3072) + (mma_rowsum_of(nch) ? 2048 : 0);
}
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  int B, Hq, Hkv, K, g, M, P, stride, sk, sv;
  float scale_log2;
  const __nv_bfloat16* q;
  const __nv_bfloat16* vc;
  __nv_bfloat16* out;
  float* lse;
  const int32_t* page_table;
  const int32_t* seq_len;
  int32_t* status;
  float* part_o;      // [G][2][M][128]: unnormalised O of split segments
  float* part_ml;     // [G][2][2][M]: raw row max, then row sum
  int lse_tma;        // lse [B][K][Hq] written by TMA (else plain stores)
  int ml_bulk;        // part_ml rows written by a bulk copy (else plain)
  int32_t* ws_int;
};

// Scales 32 TMEM columns of this thread's lane by f[0..31] (shared
// memory), 16 at a time.
ISD_DEV void tmem_scale32(uint32_t taddr, const float* f) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,"
        "%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
          "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
          "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15])
        : "r"(taddr + h * 16));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]),
                   "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]),
                   "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
#pragma unroll
    for (int e = 0; e < 16; ++e)
      r[e] = __float_as_uint(__uint_as_float(r[e]) * f[h * 16 + e]);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,"
        "%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr + h * 16),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
        "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
}


// Named barrier 1 + gi joins the four warps of softmax warpgroup gi;
// barrier 3 joins every softmax warp (`n` threads).
ISD_DEV void sm_sync(int gi) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + gi) : "memory");
}
ISD_DEV void sm_sync_all(int n) {
  asm volatile("bar.sync 3, %0;" ::"r"(n) : "memory");
}
// OR of `v` over the four warps of warpgroup gi (also a barrier among them).
ISD_DEV bool sm_any(int gi, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " bar.red.or.pred q, %2, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + gi)
      : "memory");
  return r != 0;
}

// v[c] of every lane combined over the warp; afterwards lane c holds the
// result for column c in v[0].  Recursive halving: at distance o each lane
// keeps the half of its columns selected by its bit o and trades the other
// half with lane ^ o (31 shuffles in all).
template <bool kMax>
ISD_DEV void warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float send = upper ? v[j] : v[j + o];
      const float keep = upper ? v[j + o] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
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

// What the segment epilogue needs besides the finished segment itself.
template <int NCH>
struct EpiIn {
  __nv_bfloat16* out;
  float* part_o;
  float* lse;
  float* part_ml;
  const CUtensorMap* tm_out;
  const CUtensorMap* tm_part;
  const CUtensorMap* tm_lse;
  float* small;              // staged lse, or the partial's max and sum
  int lse_tma, ml_bulk;
  uint32_t tmem_lane;        // TMEM base + this warp's lane quarter
  uint8_t* ps;               // P tiles (staging)
  uint64_t* p_empty;
  uint64_t* o_free;
  const float* m_raw;        // [NOB][N]
  float* x_red;              // [softmax warps][32]
  float* r_val;              // [warpgroups][32]
  int g, K, Hq, M, c;
  float c2;
};

// Stores the finished segment `code` (packed b, h, O buffer, complete,
// slot) whose last block is `blk`: reduces the per-key row sums over the
// 128 keys (each softmax warpgroup its own 32-row chunks), stages O / l
// (bf16) or the unnormalised O (fp32, 64 columns at a time) in the P tile
// of block blk, and writes it with TMA stores
// issued by thread 0; the lse or the partial's max and sum go directly.
// Runs on the four softmax warps.  Not inlined: its registers would
// otherwise add to those live across the block loop.  `stage_buf` is a
// P tile an earlier store may still be reading.  Returns `failed`.
template <int NCH>
__device__ __noinline__ bool store_segment(const EpiIn<NCH>& in, int blk, int code,
                                           int stage_buf, bool failed) {
  constexpr int N = 32 * NCH;
  constexpr int NPB = npb_of(NCH);
  constexpr int NOB = NCH <= 2 ? 2 : 1;
  constexpr int PB = NCH * kKeys * 64;
  constexpr uint32_t kO = 0, kL = NOB * N + 2 * N;
  constexpr int kSm = sm_warps_of(NCH), kGroups = kSm / 4;
  constexpr bool kMmaL = mma_rowsum_of(NCH);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kl = tid & 127, gi = tid >> 7, wq = warp & 3;
  const int ch_lo = gi * ((NCH + kGroups - 1) / kGroups);
  const int ch_hi = min(NCH, ch_lo + (NCH + kGroups - 1) / kGroups);
  float* r_val = in.r_val + gi * 32;
  const int b = code >> 12, h = (code >> 3) & 511, tb = (code >> 2) & 1;
  const bool complete = (code >> 1) & 1;
  const int slot = code & 1, M = in.M;
  auto stage_sync = [&]() {    // the earlier store has read its tile
    if (tid == 0) bulk_wait_read();
    sm_sync_all(kSm * 32);
  };
  // O^T of the segment is complete once the P V of its last block lands:
  // phase blk / NPB of p_empty[blk % NPB], at most one phase past the last
  // one these threads waited for there.
  wait_or_fail(&in.p_empty[blk % NPB], (blk / NPB) & 1, failed);
  tc_fence_after();
  if (stage_buf >= 0) stage_sync();
  const uint32_t eo = kO + tb * N, el = kL + tb * N;
  const float* em = in.m_raw + tb * N;
  uint8_t* stg = in.ps + (blk % NPB) * PB;          // N * 256 bytes
  float* pml = in.part_ml + ((size_t)(in.c * 2 + slot)) * 2 * M;
  const int prow = (in.c * 2 + slot) * M;           // first part_o row
#pragma unroll 1
  for (int hb = 0; hb < (complete ? 1 : 2); ++hb) {
    // A complete segment stores bf16 rows [M][128] in one pass; a partial
    // one fp32 rows, 64 columns per pass ([M][64] staged).
    if (hb == 1) stage_sync();
#pragma unroll 1
    for (int ch = ch_lo; ch < ch_hi; ++ch) {
      if constexpr (kMmaL) {
        // Row 0 of the ones product (TMEM lane 0) holds the row sums.
        if (wq == 0) {
          float v[32];
          tmem_ld32(in.tmem_lane + el + ch * 32, v);
          if (lane == 0) {
#pragma unroll
            for (int q = 0; q < 32; q += 4)
              *reinterpret_cast<float4*>(&r_val[q]) =
                  make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
          }
        }
      } else {
        float v[32];
        tmem_ld32(in.tmem_lane + el + ch * 32, v);
        warp_transpose_reduce<false>(v, lane);
        in.x_red[warp * 32 + lane] = v[0];
        sm_sync(gi);
        if (wq == 0) {
          const float* xr = in.x_red + gi * 128;
          r_val[lane] = (xr[lane] + xr[32 + lane]) + (xr[64 + lane] + xr[96 + lane]);
        }
      }
      sm_sync(gi);
      float o[32];
      tmem_ld32(in.tmem_lane + eo + ch * 32, o);   // lane = d = kl
      if (complete) {
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(&r_val[q]);
          const float inv[4] = {1.0f / l4.x, 1.0f / l4.y, 1.0f / l4.z,
                                1.0f / l4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = ch * 32 + q + u;
            if (col < M)
              *reinterpret_cast<__nv_bfloat16*>(stg + col * 256 + kl * 2) =
                  __float2bfloat16_rn(o[q + u] * inv[u]);
          }
        }
      } else if ((kl >> 6) == hb) {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int col = ch * 32 + q;
          if (col < M)
            *reinterpret_cast<float*>(stg + col * 256 + (kl & 63) * 4) = o[q];
        }
      }
      if (wq == 0 && hb == 0) {
        // lse, or the partial's max and sum: staged for a TMA / bulk store
        // when the layout allows one (plain stores stall behind the KV
        // stream), else written directly.
        const int col = ch * 32 + lane;
        if (col < M) {
          const float lt = r_val[lane], mr = em[col];
          if (complete) {
            if (in.lse) {
              const float v = (mr * in.c2 + log2f(lt)) * kLn2;
              if (in.lse_tma) {
                in.small[col] = v;
              } else {
                const int rq = col / in.g, jq = col - rq * in.g;
                in.lse[((size_t)b * in.K + rq) * in.Hq + h * in.g + jq] = v;
              }
            }
          } else if (in.ml_bulk) {
            in.small[col] = mr;
            in.small[M + col] = lt;
          } else {
            pml[col] = mr;
            pml[M + col] = lt;
          }
        }
      }
    }
    // Staged rows (every warpgroup's) -> global through the async proxy.
    proxy_fence();
    sm_sync_all(kSm * 32);
    if (tid == 0) {
      if (complete) {
        tma_store_4d(in.tm_out, stg, 0, h * in.g, 0, b);
        if (in.lse && in.lse_tma) tma_store_3d(in.tm_lse, in.small, h * in.g, 0, b);
      } else {
        tma_store_2d(in.tm_part, stg, hb * 64, prow);
        if (hb == 0 && in.ml_bulk) bulk_store(pml, in.small, 8 * M);
      }
      bulk_commit();
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&in.o_free[tb]);
  return failed;
}

// NCH: 32-column chunks of the padded query rows (N = 32 * NCH).
template <int NCH>
__global__ void __launch_bounds__(threads_of(NCH), 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc,
                   const __grid_constant__ CUtensorMap tm_kn,
                   const __grid_constant__ CUtensorMap tm_vn,
                   const __grid_constant__ CUtensorMap tm_out,
                   const __grid_constant__ CUtensorMap tm_part,
                   const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_lse, Params p) {
  constexpr int N = 32 * NCH;
  constexpr int kSm = sm_warps_of(NCH);    // softmax warps
  constexpr int kGroups = kSm / 4;         // their warpgroups
  constexpr int kMmaWarp = kSm;            // issues the QK products
  constexpr int kPvWarp = kSm + 1;         // issues the P V products
  constexpr int kLoadWarps = load_warps_of(NCH);
  constexpr int kPagesPerLoader = kNB / (kLoadWarps / 2);   // of a block
  constexpr int QH = N * 128;              // one 64-column half of Q
  // P tile [128 keys][N rows]: 32-row atoms of 128 keys x 64 B (64-byte
  // swizzle), atom a holding rows 32a..32a+31.
  constexpr int PA = kKeys * 64;           // one 32-row atom (8 KB)
  constexpr int PB = NCH * PA;             // one P buffer
  constexpr int NQB = nqb_of(NCH);         // Q tiles (shared memory)
  constexpr int NPB = npb_of(NCH);         // P tiles (shared memory)
  // O^T accumulators, row-sum partials (TMEM) and row maxima: with two, a
  // segment's epilogue is deferred until the next segment's first block
  // has been handed to the MMA warp, so the pipeline never waits on it.
  constexpr int NOB = NCH <= 2 ? 2 : 1;
  constexpr bool kDefer = NOB == 2;
  constexpr bool kLazyP = NCH >= 2;        // see the softmax loop
  constexpr bool kMmaL = mma_rowsum_of(NCH);
  constexpr int QB = 2 * QH;               // one Q tile
  // TMEM columns: O^T buffers, two S^T buffers, the row-sum buffers.
  constexpr uint32_t kO = 0, kS = NOB * N, kL = NOB * N + 2 * N;
  constexpr uint32_t kColsUsed = kL + NOB * N;
  constexpr uint32_t kCols = kColsUsed <= 128 ? 128 : (kColsUsed <= 256 ? 256 : 512);
  static_assert(kColsUsed <= 512, "TMEM columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // K and V rings: a K tile is consumed by the QK MMAs of its block and
  // freed right after them; a V tile waits for the block's softmax and its
  // P V, so the V ring is deeper.
  const int SK = p.sk, SV = p.sv;
  uint8_t* kr = base;                                  // SK K tiles
  uint8_t* vr = kr + SK * kTile;                       // SV V tiles
  uint8_t* qs = vr + SV * kTile;                       // Q tile [N][128]
  uint8_t* ps = qs + NQB * QB;                         // NPB P^T tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(ps + NPB * PB);
  uint64_t* k_full = bars;                             // [SK]
  uint64_t* k_empty = k_full + SK;                     // [SK]
  uint64_t* v_full = k_empty + SK;                     // [SV]
  uint64_t* v_empty = v_full + SV;                     // [SV]
  uint64_t* s_full = v_empty + SV;                     // [2]
  uint64_t* s_free = s_full + 2;                       // [2]
  uint64_t* p_full = s_free + 2;                       // [NPB]
  uint64_t* p_empty = p_full + 2;                      // [NPB]
  uint64_t* q_full = p_empty + 2;                      // [NQB]
  uint64_t* q_empty = q_full + 2;                      // [NQB]
  uint64_t* o_free = q_empty + 2;                      // [NOB]
  uint64_t* fin = o_free + 2;                          // all MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarBytes / 8);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);  // [B + 1]
  int* seqL = prefix + p.B + 1;                          // [B] clamped L_b
  __shared__ int scan_sh[33];
  __shared__ int s_bad;
  __shared__ __align__(16) float m_raw[NOB][N];  // reference max per row
  __shared__ __align__(16) float m_sc[N];     // the same times c (-inf kept)
  __shared__ float x_red[kSm][32];            // cross-warp reduction
  __shared__ __align__(16) float r_val[kGroups][32];  // per-row factors
  __shared__ __align__(128) float ep_small[2 * 128];  // staged lse / max, sum
  // bf16 ones: the A operand (64 x 16, K-major, no swizzle) of the row-sum
  // product; every address its descriptor reaches lies inside.
  __shared__ __align__(128) uint32_t ones_tile[512];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, Hkv = p.Hkv, M = p.M;
  if (tid == 0) {
    s_bad = 0;
    for (int s = 0; s < SK; ++s) {
      mbar_init(&k_full[s], kLoadWarps / 2);   // one arrival per K warp
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(&v_full[s], kLoadWarps / 2);   // one arrival per V warp
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], kSm);
      mbar_init(&p_full[s], kSm);
      mbar_init(&p_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);             // one expect_tx arrival (TMA)
      mbar_init(&q_empty[s], 1);
      mbar_init(&o_free[s], kSm);
    }
    mbar_init(fin, 2);                      // both MMA warps commit
    fence_barrier_init();
  }
  if constexpr (kMmaL)
    for (int i = tid; i < 512; i += blockDim.x) ones_tile[i] = 0x3F803F80u;
  // Padding rows of Q (M..N-1) stay zero for the whole kernel.
  for (int i = tid; i < NQB * N * 16; i += blockDim.x) {
    const int qb = i / (N * 16), row = (i >> 4) % N, ch = i & 15;
    if (row < M) continue;
    *reinterpret_cast<uint4*>(qs + qb * QB + (ch >> 3) * QH + row * 128 +
                              (((ch & 7) ^ (row & 7)) << 4)) =
        make_uint4(0, 0, 0, 0);
  }
  proxy_fence();
  // Everything above is independent of the kernel before this one.
  grid_dep_wait();
  __syncthreads();
  const int T = block_exclusive_scan_int(
      B,
      [&](int b) {
        int L = p.seq_len[b];
        bool bad = false;
        if (L < 0) { bad = true; L = 0; }
        int n = (L + kPage - 1) / kPage;
        if (n > p.stride) { bad = true; n = p.stride; L = n * kPage; }
        if (bad) s_bad = 1;
        seqL[b] = L;
        return Hkv * (n + 1);
      },
      [&](int b, int v) { prefix[b] = v; }, scan_sh);
  if (tid == 0) prefix[B] = T;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = split_point(prefix, B, T, Hkv, c, G);
  const int u1 = split_point(prefix, B, T, Hkv, c + 1, G);
  if (warp == kMmaWarp) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::
            "r"(smem_u32(tmem_slot)),
        "r"(kCols));
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
      p.ws_int[B + 2 + G] = T;
      if (s_bad) report(p.status, ISD_ERR_PAGE_TABLE_FULL);
    }
  }
  if (tid == 0) p.ws_int[B + 2 + c] = u0;   // range starts, for the combine
  const uint32_t kr_s = smem_u32(kr), vr_s = smem_u32(vr);
  const uint32_t q_s = smem_u32(qs), p_s = smem_u32(ps);
  bool failed = false;

  if (warp > kPvWarp) {
    // ------------------------------------------------------------ loaders
    // K tiles and V tiles are copied by separate warps, each in its own
    // loop, so a V slot still in use (its block's softmax and P V pending)
    // never holds back the next K copy.  With two warps of each kind, warp
    // lw handles pages 4 (lw & 1) .. 4 (lw & 1) + 3 of every block; with one,
    // all eight.  Lanes 0 .. 2 * pages - 1 issue their TMA boxes (page q =
    // lane / 2, 64-column half lane % 2) in one instruction: the TMA issue
    // rate, not only the bytes in flight, bounds the stream.  Each warp registers its TMA bytes, then arrives
    // once per block on k_full (K warps) or v_full (V warps).
    const int lt = tid - (kPvWarp + 1) * 32;
    const int lw = lt >> 5;
    const bool is_k = lw < kLoadWarps / 2;
    const int pg0 = (lw % (kLoadWarps / 2)) * kPagesPerLoader;   // first page
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    // Page ids of this warp's pages (-1: none or the tail), read two blocks
    // ahead: a global load waits microseconds behind the KV stream, and a
    // copy must not wait on one.
    auto page_id = [&](const BlockWalk& x, int k) {
      const int uidx = x.idx0 + x.k + k;
      return (k < x.nu() && uidx != x.units - 1)
                 ? __ldg(p.page_table + (size_t)x.b * p.stride + uidx)
                 : -1;
    };
    BlockWalk wa = w;                 // two blocks ahead of w
    int pa[kPagesPerLoader], pb[kPagesPerLoader];   // blocks i and i + 1
#pragma unroll
    for (int q = 0; q < kPagesPerLoader; ++q) pa[q] = pb[q] = -1;
    if (!wa.done()) {
#pragma unroll
      for (int q = 0; q < kPagesPerLoader; ++q) pa[q] = page_id(wa, pg0 + q);
      wa.next();
    }
    if (!wa.done()) {
#pragma unroll
      for (int q = 0; q < kPagesPerLoader; ++q) pb[q] = page_id(wa, pg0 + q);
      wa.next();
    }
    int i = 0, t = 0;    // block and segment of this CTA
    while (!w.done()) {
      const int Lb = seqL[w.b];
      if (w.first() && lt == 0) {
        // Q rows of (b, h) by TMA: row m = r * g + j holds q[b][r][h*g + j],
        // the box {64, g, K} of the [B][K][Hq][128] tensor, per 64 columns.
        const int qb = t % NQB;
        wait_or_fail(&q_empty[qb], ((t / NQB) & 1) ^ 1, failed);
        mbar_arrive_expect_tx(&q_full[qb], 2 * M * 128);
        for (int hb = 0; hb < 2; ++hb)
          tma_load_4d(qs + qb * QB + hb * QH, &tm_q, &q_full[qb], hb * 64,
                      w.h * p.g, 0, w.b);
      }
      if (w.first()) ++t;
      // This warp's pages of the block: page id (out of range: recorded,
      // then read as zeros from coordinate P, outside the cache tensors),
      // tail or cached, partial or full.
      bool use[kPagesPerLoader], tail[kPagesPerLoader], part[kPagesPerLoader];
      int page[kPagesPerLoader], valid[kPagesPerLoader];
#pragma unroll
      for (int q = 0; q < kPagesPerLoader; ++q) {
        const int k = pg0 + q;
        const int uidx = w.idx0 + w.k + k;
        use[q] = k < w.nu();
        tail[q] = use[q] && uidx == w.units - 1;
        int pg = pa[q];
        const bool bad = use[q] && !tail[q] && (pg < 0 || pg >= p.P);
        if (bad) {
          if (lane == 0) report(p.status, ISD_ERR_BAD_PAGE);
          pg = p.P;
        }
        page[q] = pg;
        valid[q] = Lb - uidx * kPage;          // >= 1 for a cached unit
        part[q] = use[q] && !tail[q] && !bad && valid[q] < kPage;
      }
      // This lane's box: page q = lane / 2 (lanes 0..7), half lane % 2.
      const int lq = (lane >> 1) & (kPagesPerLoader - 1), hb = lane & 1;
      bool l_use = false, l_tail = false;
      int l_page = 0, l_row = 0;
#pragma unroll
      for (int q = 0; q < kPagesPerLoader; ++q)
        if (q == lq) {
          l_use = use[q]; l_tail = tail[q]; l_page = page[q];
          // A partial page starts valid - 16 rows up: its slots past L_b
          // are read from outside the tensor, as zeros, and its keys land
          // in the last `valid` slots (K and V alike).
          l_row = part[q] ? valid[q] - kPage : 0;
        }
      l_use = l_use && lane < 2 * kPagesPerLoader;
      const uint32_t box_off = (pg0 + lq) * 2048 + hb * kKH;
      if (is_k) {
        // K tiles.  Rows past K of the tail lie outside the staging tensor
        // and read as zeros.
        const int ks = i % SK;
        int n_use = 0;
#pragma unroll
        for (int q = 0; q < kPagesPerLoader; ++q) n_use += use[q] ? 1 : 0;
        wait_or_fail(&k_empty[ks], ((i / SK) & 1) ^ 1, failed);
        if (lane == 0) mbar_expect_tx(&k_full[ks], (uint32_t)(n_use * 4096));
        __syncwarp();
        if (l_use) {
          uint8_t* kd = kr + ks * kTile + box_off;
          if (l_tail)
            tma_load_4d(kd, &tm_kn, &k_full[ks], hb * 64, w.h, 0, w.b);
          else
            tma_load_4d(kd, &tm_kc, &k_full[ks], hb * 64, l_row, w.h, l_page);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&k_full[ks]);
      } else {
        // V tiles, placed like the K tiles: the zeros a partial page reads
        // above its first key matter here (its slots past L_b may hold any
        // bits, and 0 * NaN would reach O through P V).
        const int vs = i % SV;
        int n_use = 0;
#pragma unroll
        for (int q = 0; q < kPagesPerLoader; ++q) n_use += use[q] ? 1 : 0;
        wait_or_fail(&v_empty[vs], ((i / SV) & 1) ^ 1, failed);
        if (lane == 0) mbar_expect_tx(&v_full[vs], (uint32_t)(n_use * 4096));
        __syncwarp();
        if (l_use) {
          uint8_t* vd = vr + vs * kTile + box_off;
          if (l_tail)
            tma_load_4d(vd, &tm_vn, &v_full[vs], hb * 64, w.h, 0, w.b);
          else
            tma_load_4d(vd, &tm_vc, &v_full[vs], hb * 64, l_row, w.h, l_page);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&v_full[vs]);
      }
      w.next();
#pragma unroll
      for (int q = 0; q < kPagesPerLoader; ++q) {
        pa[q] = pb[q];
        pb[q] = -1;
      }
      if (!wa.done()) {
#pragma unroll
        for (int q = 0; q < kPagesPerLoader; ++q) pb[q] = page_id(wa, pg0 + q);
        wa.next();
      }
      ++i;
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- QK MMA
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    int i = 0, t = -1;   // block and segment of this CTA
    const uint32_t id_qk = idesc_bf16(128, N, 0, 0);
    while (!w.done()) {
      const int ks = i % SK, sbuf = i & 1;
      if (w.first()) {
        ++t;
        wait_or_fail(&q_full[t % NQB], (t / NQB) & 1, failed);
      }
      const int qb = t % NQB;
      wait_or_fail(&k_full[ks], (i / SK) & 1, failed);
      wait_or_fail(&s_free[sbuf], ((i >> 1) & 1) ^ 1, failed);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t kb = kr_s + ks * kTile;
        for (int kk = 0; kk < 8; ++kk)
          umma(tmem + kS + sbuf * N,
               sdesc(kb + (kk >> 2) * kKH + (kk & 3) * 32, 16, 1024),
               sdesc(q_s + qb * QB + (kk >> 2) * QH + (kk & 3) * 32, 16, 1024),
               id_qk, kk > 0 ? 1u : 0u);
        umma_commit(&s_full[sbuf]);
        umma_commit(&k_empty[ks]);
        if (w.last()) umma_commit(&q_empty[qb]);
      }
      __syncwarp();
      w.next();
      ++i;
    }
    if (lane == 0) umma_commit(fin);
    __syncwarp();
    bool fin_failed = false;
    wait_or_fail(fin, 0, fin_failed);
    failed = failed || fin_failed;
  } else if (warp == kPvWarp) {
    // ---------------------------------------------------------- P V MMA
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    int i = 0, t = -1;
    const uint32_t id_pv = idesc_bf16(128, N, 1, 1);
    const uint32_t id_l = idesc_bf16(64, N, 0, 1);
    const uint64_t ones_d = sdesc(smem_u32(ones_tile), 128, 256, 0);
    while (!w.done()) {
      const bool first = w.first();
      if (first) ++t;
      const int pb = i % NPB, vs = i % SV;
      // The first P V of segment t overwrites O^T buffer t % NOB: the
      // epilogue of segment t - NOB must have read it.
      if (first && t >= NOB)
        wait_or_fail(&o_free[t % NOB], ((t / NOB) & 1) ^ 1, failed);
      wait_or_fail(&p_full[pb], (i / NPB) & 1, failed);
      wait_or_fail(&v_full[vs], (i / SV) & 1, failed);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pa = p_s + pb * PB;
        const uint32_t vb = vr_s + vs * kTile;
        const int nu = w.nu();
        for (int j = 0; j < nu; ++j)
          umma(tmem + kO + (t % NOB) * N, sdesc(vb + j * 2048, kKH, 1024),
               sdesc(pa + j * 1024, PA, 512, 4), id_pv,
               (first && j == 0) ? 0u : 1u);
        if constexpr (kMmaL)
          for (int j = 0; j < nu; ++j)
            umma(tmem + kL + (t % NOB) * N, ones_d,
                 sdesc(pa + j * 1024, PA, 512, 4), id_l,
                 (first && j == 0) ? 0u : 1u);
        umma_commit(&v_empty[vs]);
        umma_commit(&p_empty[pb]);
      }
      __syncwarp();
      w.next();
      ++i;
    }
    if (lane == 0) umma_commit(fin);
    __syncwarp();
    bool fin_failed = false;
    wait_or_fail(fin, 0, fin_failed);
    failed = failed || fin_failed;
  } else {
    // ---------------------------------------------------------- softmax
    // Warpgroup gi (threads 128 gi ..) owns 32-row chunks ch_lo .. ch_hi - 1;
    // thread kl of a warpgroup owns key kl of the block (TMEM lane kl).
    const int kl = tid & 127, gi = tid >> 7;
    const int ch_lo = gi * ((NCH + kGroups - 1) / kGroups);
    const int ch_hi = min(NCH, ch_lo + (NCH + kGroups - 1) / kGroups);
    const int kp = kl >> 4, rr = kl & 15;     // its page and slot
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float c2 = p.scale_log2;
    BlockWalk w;
    w.init(prefix, B, Hkv, u0, u1);
    // A finished segment whose O^T and row sums still have to be stored.
    // Packed into two words (the pending state lives across the block loop):
    // blk, then b << 12 | h << 3 | (t % NOB) << 2 | complete << 1 | slot.
    struct Pending {
      int blk, code;
      ISD_DEV int b() const { return code >> 12; }
      ISD_DEV int h() const { return (code >> 3) & 511; }
      ISD_DEV int tb() const { return (code >> 2) & 1; }
      ISD_DEV bool complete() const { return (code >> 1) & 1; }
      ISD_DEV int slot() const { return code & 1; }
    };
    Pending ep{-1, 0};
    // The epilogue stages each segment's output in the P tile of its last
    // block (free once that block's P V has landed) and writes it with TMA
    // stores issued by one thread: per-thread global stores queue behind
    // the KV stream and stall the softmax warps for microseconds.
    int stage_buf = -1;          // P tile a TMA store may still be reading
    auto stage_sync = [&]() {    // wait for that read (every softmax warp)
      if (tid == 0) bulk_wait_read();
      sm_sync_all(kSm * 32);
      stage_buf = -1;
    };
    const EpiIn<NCH> ein{p.out, p.part_o, p.lse, p.part_ml, &tm_out,
                         &tm_part, &tm_lse, ep_small, p.lse_tma, p.ml_bulk,
                         tmem + lane_base, ps, p_empty, o_free, &m_raw[0][0],
                         &x_red[0][0], &r_val[0][0], p.g, p.K, p.Hq, M, c, c2};
    auto epilogue = [&](const Pending& e) {
      failed = store_segment<NCH>(ein, e.blk, e.code, stage_buf, failed);
      stage_buf = e.blk % NPB;
    };
    int i = 0, t = -1, L = 0;    // block and segment of this CTA
    while (!w.done()) {
      const int sbuf = i & 1;
      const bool first = w.first();
      if (first) {
        L = seqL[w.b];
        ++t;
      }
      const uint32_t o_col = kO + (t % NOB) * N;   // this segment's O^T
      const uint32_t l_col = kL + (t % NOB) * N;   // and row sums
      float* m_row = m_raw[t % NOB];
      // Which rows may see this thread's key: every row for a cached slot
      // inside the prefix; rows at stride position >= rr for stride row rr
      // of the tail (columns col >= rr * g); none past the block's end.
      const int uidx = w.idx0 + w.k + kp;
      const bool in_blk = kp < w.nu();
      const bool tail = in_blk && uidx == w.units - 1;
      // A cached page holding v < 16 keys keeps them in its last v slots.
      const bool key_all = in_blk && !tail && rr >= kPage - (L - uidx * kPage);
      const int col_min =
          (tail && rr < p.K) ? rr * p.g : (key_all ? 0 : (1 << 30));
      wait_or_fail(&s_full[sbuf], (i >> 1) & 1, failed);
      tc_fence_after();
      const int pbi = i % NPB;
      // The P tile is free once the P V that read it last has completed
      // (and a TMA store staged in it has read it).  From two chunks up
      // (kLazyP) this is waited for only just before the first P store, so
      // that the first chunk's S load and exponentials overlap that P V;
      // every softmax thread reaches the wait at the same point (its first
      // chunk), as stage_sync's barrier requires.  With one chunk the S
      // buffer is released right after its load instead (measured: the
      // later release costs 4% at B = 1, where the block loop is a latency
      // chain, while at 64 rows the overlap gains 6%).
      auto ensure_p = [&]() {
        wait_or_fail(&p_empty[pbi], ((i / NPB) & 1) ^ 1, failed);
        if (stage_buf == pbi) stage_sync();   // a TMA store still reads it
      };
      if constexpr (!kLazyP) ensure_p();
      bool o_ready = false;
      uint8_t* pt = ps + pbi * PB;
      uint8_t* prow = pt + kl * 64;               // this key's row of P
      const int psw = (kl >> 1) & 3;              // its 64-byte swizzle
#pragma unroll 1
      for (int ch = ch_lo; ch < ch_hi; ++ch) {
        float s[32];
        auto load_s = [&]() {
          tmem_ld32(tmem + lane_base + kS + sbuf * N + ch * 32, s);
          if (col_min != 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              s[e] = (ch * 32 + e >= col_min) ? s[e] : -INFINITY;
          }
        };
        auto free_s = [&]() {    // the block's S has been read (last chunk)
          if (ch == ch_hi - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sbuf]);
          }
        };
        load_s();
        // P = 2^(s c - m c) against the current references (masked scores
        // give 0), written as this key's 32 values of the chunk and added
        // to its row sums.  Returns the largest exponent s c - m c.
        float l[32];
        auto p_pass = [&]() {
          float xmax = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 ma = *reinterpret_cast<const float4*>(&m_sc[ch * 32 + q * 8]);
            const float4 mb = *reinterpret_cast<const float4*>(&m_sc[ch * 32 + q * 8 + 4]);
            const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e = q * 8 + 2 * u;
              const float x0 = fmaf(s[e], c2, -mm[2 * u]);
              const float x1 = fmaf(s[e + 1], c2, -mm[2 * u + 1]);
              xmax = fmaxf(xmax, fmaxf(x0, x1));
              const float p0 = ex2(x0), p1 = ex2(x1);
              if constexpr (!kMmaL) {
                l[e] += p0;
                l[e + 1] += p1;
              }
              pk[u] = pack_bf16(p0, p1);
            }
            *reinterpret_cast<uint4*>(prow + ch * PA + ((q ^ psw) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          return xmax;
        };
        auto load_l = [&]() {
          if (first) {
#pragma unroll
            for (int e = 0; e < 32; ++e) l[e] = 0.0f;
          } else {
            tmem_ld32(tmem + lane_base + l_col + ch * 32, l);
          }
        };
        // Exact block max per row, then move the references (and rescale
        // O^T and the row sums).
        auto move_refs = [&]() {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = s[e];
          warp_transpose_reduce<true>(v, lane);
          x_red[warp][lane] = v[0];
          sm_sync(gi);
          float* rv = r_val[gi];
          if ((warp & 3) == 0) {
            const int col = ch * 32 + lane;
            const int w0 = 4 * gi;
            const float bm =
                fmaxf(fmaxf(x_red[w0][lane], x_red[w0 + 1][lane]),
                      fmaxf(x_red[w0 + 2][lane], x_red[w0 + 3][lane]));
            const float m_old = first ? -INFINITY : m_row[col];
            const float m_new = fmaxf(m_old, bm);
            rv[lane] = m_old == -INFINITY ? 0.0f : ex2((m_old - m_new) * c2);
            m_row[col] = m_new;
            // Finite stand-in for a row with no key yet, so that masked
            // scores still give 0 and an unmasked one votes.
            m_sc[col] = fmaxf(m_new * c2, -3.0e38f);
          }
          sm_sync(gi);
          if (!first) {
            // O^T must hold every earlier block's P V before it is scaled.
            // P V of block j completes phase j / NPB of p_empty[j % NPB],
            // a barrier this thread waits on every NPB blocks, so a parity
            // wait names that phase unambiguously.
            if (!o_ready) {
              wait_or_fail(&p_empty[(i - 1) % NPB], ((i - 1) / NPB) & 1, failed);
              tc_fence_after();
              o_ready = true;
            }
            tmem_scale32(tmem + lane_base + o_col + ch * 32, rv);
            tmem_scale32(tmem + lane_base + l_col + ch * 32, rv);
          }
        };
        if constexpr (!kLazyP) {
          // Optimistic pass; the vote asks whether any exponent exceeded 8
          // (then the references move and the pass is redone).  The first
          // block of a segment has no references yet.
          free_s();
          bool need = first;
          if (!first) {
            load_l();
            need = p_pass() > kRescaleLog2;
          }
          if (sm_any(gi, need)) {
            move_refs();
            load_l();
            p_pass();
          }
          tmem_st32(tmem + lane_base + l_col + ch * 32, l);
          continue;
        }
        // Optimistic pass against the current references, its exponentials
        // computed in place of the scores (phase A); the vote asks whether
        // any exponent exceeded 8 (then the references move, the scores are
        // read again and the pass is redone).  The first block of a segment
        // has no references yet.
        bool need = first;
        if (!first) {
          if constexpr (!kMmaL) load_l();
          float xmax = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 ma = *reinterpret_cast<const float4*>(&m_sc[ch * 32 + q * 8]);
            const float4 mb = *reinterpret_cast<const float4*>(&m_sc[ch * 32 + q * 8 + 4]);
            const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float x = fmaf(s[q * 8 + u], c2, -mm[u]);
              xmax = fmaxf(xmax, x);
              s[q * 8 + u] = ex2(x);
            }
          }
          need = xmax > kRescaleLog2;
        }
        need = sm_any(gi, need);
        if (ch == ch_lo) ensure_p();
        if (!(need && !first)) free_s();
        if (!need) {
          // Phase B: the row sums and the bf16 P of the chunk.
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e = q * 8 + 2 * u;
              if constexpr (!kMmaL) {
                l[e] += s[e];
                l[e + 1] += s[e + 1];
              }
              pk[u] = pack_bf16(s[e], s[e + 1]);
            }
            *reinterpret_cast<uint4*>(prow + ch * PA + ((q ^ psw) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
          if (!first) {
            load_s();    // phase A replaced the scores
            free_s();
          }
          move_refs();
          if constexpr (!kMmaL) load_l();
          p_pass();
        }
        if constexpr (!kMmaL) tmem_st32(tmem + lane_base + l_col + ch * 32, l);
      }
      proxy_fence();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pbi]);
      if (kDefer) {
        if (ep.blk >= 0) epilogue(ep);
        ep.blk = -1;
      }
      if (w.last()) {
        const Pending cur{i, (w.b << 12) | (w.h << 3) | ((t % NOB) << 2) |
                                 ((w.complete ? 1 : 0) << 1) |
                                 (w.seg_begin_u == u0 ? 0 : 1)};
        if (kDefer) ep = cur; else epilogue(cur);
      }
      w.next();
      ++i;
    }
    if (kDefer && ep.blk >= 0) epilogue(ep);
    if (tid == 0) bulk_wait_all();
  }
  if (failed) report(p.status, ISD_ERR_CUDA);   // a bounded wait ran out
  // Everyone meets before TMEM is released.
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                     tmem),
                 "r"(kCols));
  }
}

}  // namespace tc

static bool encode_tiled_4d(CUtensorMap* m, const void* base,
                            const uint64_t dims[4], const uint64_t strides[3],
                            const uint32_t box[4]) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims,
                      strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

constexpr size_t kSmemLimit = 227 * 1024;

// Dynamic shared memory of the kernel for N = 32 * nch rows, a K ring of
// `sk` and a V ring of `sv` tiles.
static size_t tc_smem(int B, int nch, int sk, int sv) {
  const size_t N = 32 * (size_t)nch;
  return 1024 + (size_t)(sk + sv) * tc::kTile +
         (size_t)tc::nqb_of(nch) * 2 * N * 128 +
         (size_t)tc::npb_of(nch) * 2 * N * 128 + tc::kBarBytes + 16 +
         (size_t)(2 * B + 1) * 4;
}

// K and V ring depths, the first of these that fits next to Q, P and the
// unit prefix (the deeper a ring, the more bytes each SM keeps in flight;
// a K tile is held for its QK products, a V tile until its block's
// softmax and P V are done).
struct Stages {
  int sk, sv;
};
constexpr Stages kStagePrefs[] = {{2, 4}, {2, 3}, {2, 2}};

static Stages tc_stages(int B, int M) {
  const int nch = (M + 31) / 32;
  for (const Stages& st : kStagePrefs)
    if (tc_smem(B, nch, st.sk, st.sv) + tc::static_smem_of(nch) <= kSmemLimit)
      return st;
  return Stages{0, 0};
}

size_t attn_tc_smem_bytes(int B, int M) {
  const Stages st = tc_stages(B, M);
  return st.sk ? tc_smem(B, (M + 31) / 32, st.sk, st.sv) : (size_t)-1;
}

bool attn_tc_supported(const isd_attn_args* a) {
  const int M = a->K * (a->Hq / a->Hkv);
  return a->dtype == ISD_BF16 && a->d == 128 && M >= 1 && M <= 128 &&
         a->K <= kPage && tc_stages(a->B, M).sk > 0;
}

int launch_attn_tc(const isd_attn_args* a, int G, cudaStream_t st) {
  tc::Params p;
  p.B = a->B; p.Hq = a->Hq; p.Hkv = a->Hkv; p.K = a->K;
  p.g = a->Hq / a->Hkv; p.M = a->K * p.g; p.P = a->num_pages;
  p.stride = a->page_table_stride;
  const Stages stg = tc_stages(a->B, p.M);
  if (stg.sk == 0) return ISD_ERR_UNSUPPORTED;
  p.sk = stg.sk;
  p.sv = stg.sv;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.vc = static_cast<const __nv_bfloat16*>(a->v_cache);
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.lse = a->lse; p.page_table = a->page_table; p.seq_len = a->seq_len;
  p.status = a->status;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  p.ws_int = reinterpret_cast<int32_t*>(ws);
  attn_partial_ptrs(a, G, &p.part_o, &p.part_ml);
  float* part_o = p.part_o;
  // K and V tensor maps: the caches [P][Hkv][16][128] and the stride's
  // staged rows [B][K][Hkv][128], 64-column boxes with the 128-byte swizzle.
  CUtensorMap tkc, tvc, tkn, tvn;
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
      !encode_tiled_4d(&tvc, a->v_cache, dc, sc, bc) ||
      !encode_tiled_4d(&tkn, a->k_new, dn, sn, bn) ||
      !encode_tiled_4d(&tvn, a->v_new, dn, sn, bn))
    return ISD_ERR_CUDA;
  // Store maps: out [B][K][Hq][128] bf16, one (b, h) block of g heads by K
  // stride rows per box; part_o [G * 2 * M][128] fp32, 64-column boxes of
  // M rows.  No swizzle (rows are staged plainly).
  CUtensorMap tout, tpart;
  const uint64_t dq[4] = {128, (uint64_t)a->Hq, (uint64_t)a->K,
                          (uint64_t)a->B};
  const uint64_t sq[3] = {256, (uint64_t)a->Hq * 256,
                          (uint64_t)a->K * a->Hq * 256};
  const uint32_t bq[4] = {128, (uint32_t)p.g, (uint32_t)a->K, 1};
  const uint64_t dp[2] = {128, (uint64_t)G * 2 * p.M};
  const uint64_t sp[1] = {512};
  const uint32_t bp[2] = {64, (uint32_t)p.M};
  if (!encode_tiled(&tout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a->out, dq, sq,
                    bq, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tiled(&tpart, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, part_o, dp, sp,
                    bp, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ISD_ERR_CUDA;
  // Q [B][K][Hq][128] bf16: a (b, h) tile is the box {64, g, K, 1}, landing
  // as rows m = r * g + j of 128 bytes in the 128-byte swizzle.
  CUtensorMap tq;
  const uint32_t bqq[4] = {64, (uint32_t)p.g, (uint32_t)a->K, 1};
  if (!encode_tiled(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a->q, dq, sq, bqq,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return ISD_ERR_CUDA;
  // lse [B][K][Hq] fp32 by TMA when rows of g values are whole 16-byte
  // units; part_ml rows (2M floats) by a bulk copy when M is even.
  p.lse_tma = a->lse != nullptr &&
              (reinterpret_cast<uintptr_t>(a->lse) & 15) == 0 &&
              p.g % 4 == 0 && a->Hq % 4 == 0;
  p.ml_bulk = p.M % 2 == 0;
  CUtensorMap tlse = tpart;   // any valid map when lse is not stored by TMA
  if (p.lse_tma) {
    const uint64_t dl[3] = {(uint64_t)a->Hq, (uint64_t)a->K, (uint64_t)a->B};
    const uint64_t sl[2] = {(uint64_t)a->Hq * 4, (uint64_t)a->K * a->Hq * 4};
    const uint32_t bl[3] = {(uint32_t)p.g, (uint32_t)a->K, 1};
    if (!encode_tiled(&tlse, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a->lse, dl, sl,
                      bl, CU_TENSOR_MAP_SWIZZLE_NONE))
      return ISD_ERR_CUDA;
  }
  const int nch = (p.M + 31) / 32;
  const size_t smem = tc_smem(a->B, nch, p.sk, p.sv);
  auto kern = nch == 1 ? tc::attn_tc_kernel<1>
            : nch == 2 ? tc::attn_tc_kernel<2>
            : nch == 3 ? tc::attn_tc_kernel<3>
                       : tc::attn_tc_kernel<4>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  if (launch_pdl(kern, dim3(G), dim3(tc::threads_of(nch)), smem, st, tkc, tvc, tkn,
                 tvn, tout, tpart, tq, tlse, p) != cudaSuccess)
    return ISD_ERR_CUDA;
  return launch_attn_combine(a, G, st);
}

}  // namespace isd
