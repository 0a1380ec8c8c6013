// isd_lm_head: the LM head that produces a step's logits, on the 5th-
// generation tensor cores, with the vocabulary statistics the accept step
// consumes computed in the GEMM's epilogue and the R-ISD gated LoRA at MASK
// rows.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io).  One forward pass gives p at the clean rows and q at the MASK
// rows ("Inference & ISD"); the logits of a row are its final hidden state
// times the output embedding.  R-ISD adds a rank-128 LoRA that acts only at
// MASK positions, so p stays the base model's ("Speedup Factor Explorer",
// R-ISD): for a MASK row m
//   logits[m] = h_m W^T + scale (h_m A^T) B^T,
// computed as one contraction over the concatenated K axis
//   [h_m | U_m] . [W | B]^T,  U_m = gate_m * scale * (h_m A^T)  (bf16),
// with gate_m = 1 at MASK rows and 0 at clean rows, so the clean rows'
// extra K steps multiply zeros.
//
// GEMM layout.  Rows (hidden states) take the MMA's M side and TMEM lanes,
// vocabulary entries its N side (a tile of 256), so each epilogue thread
// owns one row and reduces its row's statistics in registers.  A CTA keeps
// RT = 2 accumulators of 128 rows that share the weight tile (256 rows x
// 256 entries: 128 B of weight and hidden state loaded per 128 FLOPs
// instead of per 85 for a single accumulator, which keeps the L2-to-SM
// stream well under the L2's bandwidth); with 128 rows or fewer RT = 1 and
// the two TMEM buffers let the epilogue of one tile overlap the next.
//
// Warp roles (10 warps): warp 0 issues the TMA loads of the stage ring (one
// 64-wide K slice of the hidden rows and of the weight tile per stage),
// warp 1 allocates TMEM and one thread issues the tcgen05 MMAs, warps 2..9
// (RT = 2; warps 2..5 for RT = 1) drain the accumulators: round to bf16,
// stage 32 rows x 64 entries in shared memory (128-byte swizzle) and store
// them by TMA, and fold the rounded values into the row's (max, sum of
// exp(l - max), first index of the max) of the tile.  A second kernel merges
// the per-tile figures into the 2048-entry sub-chunk figures the accept
// step reads.
//
// Every mbarrier wait is bounded; after one timeout a thread records
// ISD_ERR_CUDA (unless an earlier error is recorded) and stops waiting.
#include "tcgen05.cuh"

namespace isd {
namespace lm {

using namespace tc;

constexpr int kBK = 64;                  // K elements per stage (128 bytes)
constexpr int kAccRows = 128;            // MMA M
constexpr int kEpiWarp0 = 2;
constexpr int kThreads = 10 * 32;
constexpr int kStoreCols = 64;           // entries per TMA store box
constexpr int kStoreBuf = 32 * 128;      // one warp's 32 rows x 128 bytes
constexpr int kSubChunk = 2048;          // accept step's sub-chunk width
constexpr size_t kSmemLimit = 227 * 1024;

struct Params {
  int M, V, tn, RTn, VT, kD, kR, ksplit, kps, tiles, stages, mode;
  // mode 0: logits (+ per-tile statistics when pmax is set)
  float* pmax;         // [VT][M]
  double* psum;        // [VT][M]
  int32_t* pidx;       // [VT][M]
  // mode 1: fp32 partial products [ksplit][M][tn] of the LoRA down-projection
  float* part;
  // mode 0 split-K tail: tiles [body, tiles) are cut into tsplit K ranges of
  // tkps steps, worker w < (tiles - body) * tsplit taking range w % tsplit
  // of tile body + w / tsplit and writing its fp32 accumulator to
  // tail[w][tile rows][tn]; a fix-up kernel sums them.
  int body, tsplit, tkps;
  float* tail;
  int32_t* status;
};

ISD_DEV float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
ISD_DEV float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Running statistics of one row over the 64-entry pieces of a tile: the max
// m of the rounded values, the sum s of exp(l - m) and the first index i of
// the max.
struct RowRun {
  float m = -INFINITY;
  double s = 0.0;
  int i = 0;
};

// Rounds a row's 64 accumulator values to bf16: w holds the packed pairs
// (what the logits store), v the rounded values as floats.
ISD_DEV void round_piece(float (&v)[64], uint32_t (&w)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
    v[2 * e] = bf_lo(w[e]);
    v[2 * e + 1] = bf_hi(w[e]);
  }
}

// Folds the rounded values of entries col0 .. col0 + 63 (those below V)
// into the row's running statistics.  The piece is reduced on its own
// (max, first index of the max, 64-term fp32 sum of exp(l - max)) and then
// merged in fp64.
ISD_DEV void fold_piece(const float (&v)[64], int col0, int V, RowRun& rr) {
  const int nv = V - col0;
  float pm = -INFINITY;
  float ps = 0.0f;
  int pi = 0;
  if (nv >= 64) {
#pragma unroll
    for (int e = 0; e < 64; ++e) pm = fmaxf(pm, v[e]);
    if (pm > rr.m) {
#pragma unroll
      for (int e = 63; e >= 0; --e)
        if (v[e] == pm) pi = col0 + e;
    }
#pragma unroll
    for (int e = 0; e < 64; ++e) ps += ex2((v[e] - pm) * kLog2e);
  } else {
#pragma unroll
    for (int e = 0; e < 64; ++e)
      if (e < nv) pm = fmaxf(pm, v[e]);
#pragma unroll
    for (int e = 63; e >= 0; --e)
      if (e < nv && v[e] == pm) pi = col0 + e;
#pragma unroll
    for (int e = 0; e < 64; ++e)
      if (e < nv) ps += ex2((v[e] - pm) * kLog2e);
  }
  if (pm > rr.m) {
    rr.s = (rr.m == -INFINITY ? 0.0 : rr.s * exp((double)rr.m - (double)pm)) +
           (double)ps;
    rr.m = pm;
    rr.i = pi;
  } else {
    rr.s += (double)ps * exp((double)pm - (double)rr.m);
  }
}

// Stages one warp's 32 rows x 64 entries (128-byte swizzle) and stores them
// by TMA at (col0, row0); the previous store from this buffer must have
// read it first.
ISD_DEV void stage_store(const uint32_t (&w)[32], uint8_t* sb,
                         const CUtensorMap* tm, int col0, int row0, int lane,
                         bool failed, bool& stored) {
  if (lane == 0 && stored) bulk_wait_read();
  __syncwarp();
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    *reinterpret_cast<uint4*>(sb + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
        make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
  proxy_fence();
  __syncwarp();
  if (lane == 0 && !failed) {
    tma_store_2d(tm, sb, col0, row0);
    bulk_commit();
    stored = true;
  }
  __syncwarp();
}

// Tile t -> (row tile, vocabulary tile, first and end K step).  `slot` >= 0
// marks a split-K piece of a tail tile (its partial buffer).
struct Tile {
  int rt, vt, k0, k1, slot;
};
ISD_DEV Tile tile_of(const Params& p, int t) {
  Tile x;
  x.slot = -1;
  x.rt = t % p.RTn;
  if (p.mode == 0) {
    x.vt = t / p.RTn;
    x.k0 = 0;
    x.k1 = p.kD + p.kR;
  } else {
    x.vt = 0;
    const int s = t / p.RTn;
    x.k0 = s * p.kps;
    x.k1 = min(p.kD, x.k0 + p.kps);
  }
  return x;
}

// The work of worker w of W (a CTA, or a CTA pair): whole tiles w, w + W, ...
// below p.body, then at most one split-K piece of a tail tile.
ISD_DEV int n_items(const Params& p, int w, int W) {
  const int whole = w < p.body ? (p.body - w + W - 1) / W : 0;
  const int tail = (p.tiles - p.body) * p.tsplit;
  return whole + (w < tail ? 1 : 0);
}
ISD_DEV Tile item(const Params& p, int w, int W, int it) {
  const int whole = w < p.body ? (p.body - w + W - 1) / W : 0;
  if (it < whole) return tile_of(p, w + it * W);
  Tile x = tile_of(p, p.body + w / p.tsplit);
  const int Kt = p.kD + p.kR;
  x.k0 = (w % p.tsplit) * p.tkps;
  x.k1 = min(Kt, x.k0 + p.tkps);
  x.slot = w;
  return x;
}

template <int RT, int NB>
__global__ void __launch_bounds__(kThreads, 1)
    lm_gemm_kernel(const __grid_constant__ CUtensorMap tm_h,
                   const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_out, Params p) {
  // NB accumulator buffers of RT accumulators of tn columns each.
  constexpr int kEpiWarps = 4 * RT;
  constexpr int ABytes = RT * kAccRows * 128;   // hidden rows of a stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  const int stage_bytes = ABytes + p.tn * 128;
  uint8_t* ring = base;
  uint8_t* stg = ring + (size_t)S * stage_bytes;          // store staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + kEpiWarps * kStoreBuf);
  uint64_t* full = bars;                  // [S]
  uint64_t* empty = full + S;             // [S]
  uint64_t* acc_full = empty + S;         // [NB]
  uint64_t* acc_empty = acc_full + NB;    // [NB]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + NB);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::
            "r"(smem_u32(tmem_slot)),
        "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The operands may come from the kernel before this one.
  grid_dep_wait();
  const int G = gridDim.x, c = blockIdx.x;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    int s = 0;
    uint32_t ph = 0;
    for (int it = 0, ni = n_items(p, c, G); it < ni; ++it) {
      const Tile x = item(p, c, G, it);
      for (int k = x.k0; k < x.k1; ++k) {
        wait_or_fail(&empty[s], ph ^ 1, failed);
        if (lane == 0 && !failed) {
          uint8_t* a = ring + (size_t)s * stage_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          if (k < p.kD) {
            tma_load_2d(a, &tm_h, &full[s], k * kBK, x.rt * RT * kAccRows);
            tma_load_2d(a + ABytes, &tm_w, &full[s], k * kBK, x.vt * p.tn);
          } else {
            tma_load_2d(a, &tm_u, &full[s], (k - p.kD) * kBK,
                        x.rt * RT * kAccRows);
            tma_load_2d(a + ABytes, &tm_b, &full[s], (k - p.kD) * kBK,
                        x.vt * p.tn);
          }
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMAs
    const uint32_t id = idesc_bf16(kAccRows, p.tn, 0, 0);
    int s = 0;
    uint32_t ph = 0, acc_ph = 0;   // bit b: phase of accumulator buffer b
    int n = 0;
    for (int ni = n_items(p, c, G); n < ni; ++n) {
      const Tile x = item(p, c, G, n);
      const int buf = NB == 2 ? (n & 1) : 0;
      wait_or_fail(&acc_empty[buf], ((acc_ph >> buf) & 1) ^ 1, failed);
      acc_ph ^= 1u << buf;
      tc_fence_after();
      for (int k = x.k0; k < x.k1; ++k) {
        wait_or_fail(&full[s], ph, failed);
        tc_fence_after();
        if (lane == 0 && !failed) {
          const uint32_t a = smem_u32(ring + (size_t)s * stage_bytes);
          const uint32_t b = a + ABytes;
#pragma unroll
          for (int r = 0; r < RT; ++r)
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma(tmem + (uint32_t)((buf * RT + r) * p.tn),
                   sdesc(a + r * kAccRows * 128 + kk * 32, 16, 1024),
                   sdesc(b + kk * 32, 16, 1024), id,
                   (k > x.k0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1; }
      }
      if (lane == 0 && !failed) umma_commit(&acc_full[buf]);
      __syncwarp();
    }
  } else if (warp - kEpiWarp0 < kEpiWarps) {
    // --------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;
    const int q = warp & 3;                  // TMEM lane quarter of the warp
    const int r = ew >> 2;                   // accumulator of the warp
    uint8_t* sb = stg + ew * kStoreBuf;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t acc_ph = 0;
    int n = 0;
    bool stored = false;
    for (int ni = n_items(p, c, G); n < ni; ++n) {
      const Tile x = item(p, c, G, n);
      const int buf = NB == 2 ? (n & 1) : 0;
      wait_or_fail(&acc_full[buf], (acc_ph >> buf) & 1, failed);
      acc_ph ^= 1u << buf;
      tc_fence_after();
      const int row0 = (x.rt * RT + r) * kAccRows + q * 32;   // warp's rows
      const int row = row0 + lane;
      const uint32_t tacc = tmem + lane_off + (uint32_t)((buf * RT + r) * p.tn);
      RowRun rr;
      for (int j = 0; j < p.tn / kStoreCols; ++j) {
        float v[64];
        {
          float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
          float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
          tmem_ld32(tacc + j * kStoreCols, v0);
          tmem_ld32(tacc + j * kStoreCols + 32, v1);
        }
        if (p.mode == 1 || x.slot >= 0) {
          // fp32 partials, plain stores: the LoRA down-projection's K
          // ranges, or a split-K piece of a tail tile.
          if (row < p.M && !failed) {
            float* base = x.slot >= 0
                ? p.tail + ((size_t)x.slot * RT * kAccRows + r * kAccRows +
                            q * 32 + lane) * p.tn
                : p.part + ((size_t)(x.k0 / p.kps) * p.M + row) * p.tn;
            float4* dst = reinterpret_cast<float4*>(base + j * kStoreCols);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2],
                                   v[4 * e + 3]);
          }
          continue;
        }
        uint32_t w[32];
        const int col0 = x.vt * p.tn + j * kStoreCols;
        round_piece(v, w);
        if (p.pmax && col0 < p.V) fold_piece(v, col0, p.V, rr);
        if (col0 < p.V && row0 < p.M)
          stage_store(w, sb, &tm_out, col0, row0, lane, failed, stored);
      }
      // This tile's TMEM reads are complete: hand the buffer back.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (p.mode == 0 && x.slot < 0 && p.pmax && row < p.M) {
        const size_t o = (size_t)x.vt * p.M + row;
        p.pmax[o] = rr.m;
        p.psum[o] = rr.s;
        p.pidx[o] = rr.i;
      }
    }
    if (lane == 0 && stored) bulk_wait_all();
  }
  if (failed) report(p.status, ISD_ERR_CUDA);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                     tmem),
                 "r"(512));
  }
}


// ---------------------------------------------------------------------------
// The same contraction on CTA pairs (more than 128 rows).  A cluster of two
// CTAs computes a 256-row x 256-entry tile with cta_group::2 MMAs: each CTA
// loads its 128 hidden rows and its half (128 entries) of the weight tile,
// the even CTA issues M = 256, N = 256 MMAs that read both CTAs' shared
// memory, and each CTA's TMEM receives its 128 rows x 256 entries.  Per SM
// that is the two-accumulator tile's traffic (64 bytes per 128 FLOPs) with
// half of its TMEM, so two accumulator buffers fit and the epilogue of one
// tile overlaps the MMAs of the next.
//
// Barriers: the even CTA's full[s] takes one expect-tx arrival (the even
// CTA's, for both CTAs' bytes) and both CTAs' TMA bytes; empty[s] and acc_full[b] of both CTAs are
// signalled by the even CTA's commits (multicast); the even CTA's
// acc_empty[b] counts the epilogue warps of both CTAs.  Before leaving,
// each CTA's loader waits until every stage it filled has been released
// (so no commit is still on its way to this CTA), and the pair meets.
constexpr int kPairThreads = 10 * 32;
constexpr int kPairEpiWarps = 8;           // two per TMEM lane quarter
constexpr int kPairRows = 256;             // rows of a pair tile
constexpr int kPairTn = 256;               // vocabulary entries of a tile
constexpr int kPairHalf = 128 * 128;       // 128 rows x 64 K (bf16) = 16 KB
constexpr int kPairAtoms = 2;              // 64-wide K slices per stage

__global__ void __launch_bounds__(kPairThreads, 1)
    lm_pair_kernel(const __grid_constant__ CUtensorMap tm_h,
                   const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_out, Params p) {
  // A stage: kPairAtoms slices of this CTA's hidden rows, then as many of
  // its weight rows.
  constexpr int kStage = 2 * kPairAtoms * kPairHalf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* ring = base;
  uint8_t* stg = ring + (size_t)S * kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + kPairEpiWarps * kStoreBuf);
  uint64_t* full = bars;                  // [S] (the even CTA's are used)
  uint64_t* empty = full + S;             // [S]
  uint64_t* acc_full = empty + S;         // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2] (the even CTA's are used)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();   // 0: issues the MMAs
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kPairEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile(
        "tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::
            "r"(smem_u32(tmem_slot)),
        "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();        // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    int s = 0;
    uint32_t ph = 0;
    for (int it = 0, ni = n_items(p, pair, npairs); it < ni; ++it) {
      const Tile x = item(p, pair, npairs, it);
      const int hrow = x.rt * kPairRows + (int)rank * 128;
      const int wrow = x.vt * kPairTn + (int)rank * 128;
      for (int k = x.k0; k < x.k1; k += kPairAtoms) {
        const int na = min(kPairAtoms, x.k1 - k);
        wait_or_fail(&empty[s], ph ^ 1, failed);
        if (lane == 0 && !failed) {
          uint8_t* a = ring + (size_t)s * kStage;
          const uint32_t fb = cluster_addr(&full[s], 0);
          // The even CTA arms its barrier for both CTAs' bytes; the odd
          // CTA's copies count against it too (possibly first: the
          // transaction count may go below zero until the arming).
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 4 * na * kPairHalf);
          for (int j = 0; j < na; ++j) {
            const int ka = k + j;
            uint8_t* aj = a + j * kPairHalf;
            uint8_t* bj = a + (kPairAtoms + j) * kPairHalf;
            if (ka < p.kD) {
              tma_load_2d_pair(aj, &tm_h, fb, ka * kBK, hrow);
              tma_load_2d_pair(bj, &tm_w, fb, ka * kBK, wrow);
            } else {
              tma_load_2d_pair(aj, &tm_u, fb, (ka - p.kD) * kBK, hrow);
              tma_load_2d_pair(bj, &tm_b, fb, (ka - p.kD) * kBK, wrow);
            }
          }
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1; }
      }
    }
    // Every stage this CTA filled has been released by the pair's MMAs.
    for (int i = 0; i < S; ++i) {
      wait_or_fail(&empty[s], ph ^ 1, failed);
      if (++s == S) { s = 0; ph ^= 1; }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMAs (even CTA)
    if (rank == 0) {
      const uint32_t id = idesc_bf16(kPairRows, kPairTn, 0, 0);
      int s = 0;
      uint32_t ph = 0, acc_ph = 0;
      int n = 0;
      for (int ni = n_items(p, pair, npairs); n < ni; ++n) {
        const Tile x = item(p, pair, npairs, n);
        const int buf = n & 1;
        wait_or_fail_cluster(&acc_empty[buf], ((acc_ph >> buf) & 1) ^ 1,
                             failed);
        acc_ph ^= 1u << buf;
        tc_fence_after();
        for (int k = x.k0; k < x.k1; k += kPairAtoms) {
          const int na = min(kPairAtoms, x.k1 - k);
          wait_or_fail_cluster(&full[s], ph, failed);
          tc_fence_after();
          if (lane == 0 && !failed) {
            const uint32_t a = smem_u32(ring + (size_t)s * kStage);
            for (int j = 0; j < na; ++j)
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                umma_pair(tmem + (uint32_t)(buf * kPairTn),
                          sdesc(a + j * kPairHalf + kk * 32, 16, 1024),
                          sdesc(a + (kPairAtoms + j) * kPairHalf + kk * 32, 16,
                                1024),
                          id, (k > x.k0 || j > 0 || kk > 0) ? 1u : 0u);
            umma_pair_commit(&empty[s], 0x3);
          }
          __syncwarp();
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (lane == 0 && !failed) umma_pair_commit(&acc_full[buf], 0x3);
        __syncwarp();
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Warp (q, h): TMEM lane quarter q (rows 32q..32q+31 of this CTA's
    // 128), entries 128h..128h+127 of the tile.
    const int ew = warp - kEpiWarp0;
    const int q = warp & 3;
    const int h = ew >> 2;
    uint8_t* sb = stg + ew * kStoreBuf;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t acc_ph = 0;
    int n = 0;
    bool stored = false;
    for (int ni = n_items(p, pair, npairs); n < ni; ++n) {
      const Tile x = item(p, pair, npairs, n);
      const int buf = n & 1;
      wait_or_fail(&acc_full[buf], (acc_ph >> buf) & 1, failed);
      acc_ph ^= 1u << buf;
      tc_fence_after();
      const int row0 = x.rt * kPairRows + (int)rank * 128 + q * 32;
      const int row = row0 + lane;
      const uint32_t tacc =
          tmem + lane_off + (uint32_t)(buf * kPairTn + h * 128);
      RowRun rr;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        float v[64];
        {
          float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
          float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
          tmem_ld32(tacc + j * kStoreCols, v0);
          tmem_ld32(tacc + j * kStoreCols + 32, v1);
        }
        if (x.slot >= 0) {
          // A split-K piece of a tail tile: fp32 partial of this CTA's
          // rows, summed by the fix-up kernel.
          if (!failed) {
            float4* dst = reinterpret_cast<float4*>(
                p.tail + ((size_t)x.slot * kPairRows + rank * 128 + q * 32 +
                          lane) * kPairTn + h * 128 + j * kStoreCols);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2],
                                   v[4 * e + 3]);
          }
          continue;
        }
        uint32_t w[32];
        const int col0 = x.vt * kPairTn + h * 128 + j * kStoreCols;
        round_piece(v, w);
        if (p.pmax && col0 < p.V) fold_piece(v, col0, p.V, rr);
        if (col0 < p.V && row0 < p.M)
          stage_store(w, sb, &tm_out, col0, row0, lane, failed, stored);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(cluster_addr(&acc_empty[buf], 0));
      if (x.slot < 0 && p.pmax && row < p.M) {
        // One record per 128-entry half tile.
        const size_t o = (size_t)(x.vt * 2 + h) * p.M + row;
        p.pmax[o] = rr.m;
        p.psum[o] = rr.s;
        p.pidx[o] = rr.i;
      }
    }
    if (lane == 0 && stored) bulk_wait_all();
  }
  if (failed) report(p.status, ISD_ERR_CUDA);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(
                     tmem),
                 "r"(512));
  }
}

// U[m][j] = bf16(gate_m * scale * sum over splits of part[s][m][j]), splits
// summed in order.  gate_m = 1 when row m is a MASK row (its stride row
// m % K is at or past n_pending of its sequence), else 0; a sequence with
// n_pending outside [0, K] is reported and gets no LoRA.
struct ReduceParams {
  int M, r, ksplit, K;
  float scale;
  const float* part;
  const int32_t* n_pending;
  __nv_bfloat16* u;
  int32_t* status;
};

__global__ void __launch_bounds__(256) lora_reduce_kernel(ReduceParams p) {
  grid_dep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.M * p.r) return;
  const int m = i / p.r;
  const int n = p.n_pending[m / p.K];
  const bool ok = n >= 0 && n <= p.K;
  if (!ok && i % p.r == 0 && (m % p.K) == 0) report(p.status, ISD_ERR_BAD_STATE);
  float g = ok && (m % p.K) >= n ? p.scale : 0.0f;
  float acc = 0.0f;
  for (int s = 0; s < p.ksplit; ++s) acc += p.part[(size_t)s * p.M * p.r + i];
  p.u[i] = __float2bfloat16_rn(g * acc);
}

// The tail tiles from their split-K pieces: one warp per (tail tile, row,
// record) sums the pieces in order, rounds to bf16, stores the logits and
// writes the record's statistics (max, sum of exp(l - max) over the rounded
// values, first index of the max).
struct FixupParams {
  int M, V, tn, RTn, body, ntail, tsplit, trows, rec_w;
  const float* tail;      // [ntail * tsplit][trows][tn]
  __nv_bfloat16* logits;  // [M][V]
  float* pmax;            // records [*][M] (or null)
  double* psum;
  int32_t* pidx;
};

__global__ void __launch_bounds__(256) lm_tail_fixup_kernel(FixupParams p) {
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int nrec = p.tn / p.rec_w;
  const int per_tile = p.trows * nrec;
  const int jt = gw / per_tile;                  // tail tile
  if (jt >= p.ntail) return;                     // warp-uniform
  const int rem = gw - jt * per_tile;
  const int local = rem / nrec, h = rem - local * nrec;
  const int t = p.body + jt;
  const int rt = t % p.RTn, vt = t / p.RTn;
  const int row = rt * p.trows + local;
  if (row >= p.M) return;                        // warp-uniform
  const int cpl = p.rec_w / 32;                  // 8 or 4 columns a lane
  const int c0 = h * p.rec_w + lane * cpl;       // within the tile
  const int col = vt * p.tn + c0;
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
  // The pieces in order, eight loads in flight at a time.
  const size_t pstride = (size_t)p.trows * p.tn;
  const float* src0 = p.tail + ((size_t)jt * p.tsplit * p.trows + local) * p.tn + c0;
  for (int i0 = 0; i0 < p.tsplit; i0 += 8) {
    float4 lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool ok = i0 + i < p.tsplit;
      const float* src = src0 + (size_t)(ok ? i0 + i : i0) * pstride;
      lo[i] = ok ? __ldcg(reinterpret_cast<const float4*>(src))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
      hi[i] = ok && cpl == 8 ? __ldcg(reinterpret_cast<const float4*>(src + 4))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[0] += lo[i].x; acc[1] += lo[i].y; acc[2] += lo[i].z; acc[3] += lo[i].w;
      acc[4] += hi[i].x; acc[5] += hi[i].y; acc[6] += hi[i].z; acc[7] += hi[i].w;
    }
  }
  // cpl columns starting at a multiple of cpl, V a multiple of 8: a lane's
  // columns are all inside the vocabulary or all past it.
  const bool valid = col < p.V;
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = pack_bf16(acc[2 * k], acc[2 * k + 1]);
  float v[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = bf_lo(w[k]);
    v[2 * k + 1] = bf_hi(w[k]);
  }
  if (valid) {
    __nv_bfloat16* dst = p.logits + (size_t)row * p.V + col;
    if (cpl == 8)
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    else
      *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  }
  if (!p.pmax) return;
  float m = -INFINITY;
  int idx = INT_MAX;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (valid && k < cpl && v[k] > m) { m = v[k]; idx = col + k; }
  const float wm = warp_max(m);
  int first = m == wm ? idx : INT_MAX;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1)
    first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
  float ls = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (valid && k < cpl) ls += ex2((v[k] - wm) * kLog2e);
  double sum = (double)ls;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) {
    const size_t o = (size_t)(vt * nrec + h) * p.M + row;
    p.pmax[o] = wm;
    p.psum[o] = sum;
    p.pidx[o] = first;
  }
}

// Sub-chunk figures from the per-tile ones: for (row, sub-chunk c) the
// tiles of c in ascending order give the max, the sum of exp(l - max)
// (fp64) and the first index of the max.
struct MergeParams {
  int M, V, VT, C, per;     // per: tiles per sub-chunk
  const float* pmax;
  const double* psum;
  const int32_t* pidx;
  double* csum;             // [M][C]
  float* cmax;
  int32_t* cidx;
};

__global__ void __launch_bounds__(256) lm_stats_merge_kernel(MergeParams p) {
  constexpr int kPer = 16;      // records per sub-chunk at most
  grid_dep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.M * p.C) return;
  const int row = i % p.M, c = i / p.M;
  const int v0 = c * p.per;
  // Every record of the sub-chunk is loaded up front (one round trip).
  float pm[kPer];
  double ps[kPer];
  int pi[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const bool ok = k < p.per && v0 + k < p.VT;
    const size_t o = (size_t)(ok ? v0 + k : v0) * p.M + row;
    pm[k] = ok ? __ldcg(p.pmax + o) : -INFINITY;
    ps[k] = ok ? __ldcg(p.psum + o) : 0.0;
    pi[k] = ok ? __ldcg(p.pidx + o) : 0;
  }
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kPer; ++k) m = fmaxf(m, pm[k]);
  double s = 0.0;
  int idx = -1;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    if (pm[k] != -INFINITY) s += ps[k] * exp((double)pm[k] - (double)m);
    if (idx < 0 && pm[k] == m) idx = pi[k];
  }
  const size_t o = (size_t)row * p.C + c;
  p.csum[o] = s;
  p.cmax[o] = m;
  p.cidx[o] = idx;
}

}  // namespace lm

// ---------------------------------------------------------------------------
// Host side.

namespace {

int sms_now() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return 0;
  return n;
}

struct LmLayout {
  size_t pmax, psum, pidx, part, u, tail, total;
};

constexpr int kLoraSplit = 16;

// Tile shape for M rows.  Up to 128 rows: one CTA per tile, RT = 1
// accumulator of 128 rows x tn entries, two TMEM buffers.  More rows: CTA
// pairs with 256-row x 256-entry tiles.  Statistics records cover rec_w
// entries each (a tile, or the half tile of a pair's epilogue warp).
struct Shape {
  int RT, tn, rec_w;
  bool pair;
  int nrec(int V) const {
    return pair ? 2 * ((V + tn - 1) / tn) : (V + tn - 1) / tn;
  }
};
Shape lm_shape(int M) {
  return M > lm::kAccRows ? Shape{2, lm::kPairTn, 128, true}
                          : Shape{1, 256, 256, false};
}

// Workers (CTAs, or CTA pairs) and the rows of one tile.
int lm_workers(const Shape& sh) {
  const int sms = sms_now();
  return sh.pair ? sms / 2 : sms;
}
int tile_rows(const Shape& sh) {
  return sh.pair ? lm::kPairRows : sh.RT * lm::kAccRows;
}

// Split-K tail.  The last wave of `tiles` tiles on W workers leaves
// tiles % W of them (all of them when tiles < W) to a few workers while the
// rest idle for a whole tile; instead each of those tail tiles is cut into
// tsplit K ranges (about W / tail of them, at most 16, none empty), one per
// worker, and a fix-up kernel sums the fp32 pieces.  Used when each tail
// tile gets at least two pieces.
struct TailPlan {
  int workers, body, tsplit, tkps;
};
TailPlan tail_plan(int tiles, int W, int Kt) {
  TailPlan t{std::min(tiles, W), tiles, 1, 0};
  if (W <= 0) return TailPlan{tiles, tiles, 1, 0};
  const int ntail = tiles >= W ? tiles % W : tiles;
  if (ntail == 0 || W / ntail < 2) return t;
  // At most 16 pieces a tile: the fix-up sums them per row.
  const int want = std::min(std::min(W / ntail, Kt), 16);
  t.tkps = (Kt + want - 1) / want;
  t.tsplit = (Kt + t.tkps - 1) / t.tkps;
  if (t.tsplit < 2) return TailPlan{std::min(tiles, W), tiles, 1, 0};
  t.workers = W;
  t.body = tiles - ntail;
  return t;
}

LmLayout lm_layout(const isd_lm_head_args* a) {
  LmLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t VT = (size_t)lm_shape(a->M).nrec(a->V);
  if (a->vocab_stats) {
    l.pmax = take(VT * a->M * 4);
    l.psum = take(VT * a->M * 8);
    l.pidx = take(VT * a->M * 4);
  }
  if (a->lora_rank > 0) {
    l.part = take((size_t)kLoraSplit * a->M * a->lora_rank * 4);
    l.u = take((size_t)a->M * a->lora_rank * 2);
  }
  // Split-K tail pieces: at most one per worker, a tile of fp32 each.
  const Shape sh = lm_shape(a->M);
  l.tail = take((size_t)std::max(lm_workers(sh), 1) * tile_rows(sh) * sh.tn * 4);
  l.total = std::max<size_t>(off, 256);
  return l;
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
               uint32_t box_inner, uint32_t box_outer) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {inner * 2};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims,
                      strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int stages_for(int RT, int tn) {
  const size_t stage = (size_t)RT * lm::kAccRows * 128 + (size_t)tn * 128;
  const size_t fixed = 1024 + (size_t)4 * RT * lm::kStoreBuf + 256;
  const size_t s = (lm::kSmemLimit - fixed) / stage;
  return (int)std::min<size_t>(s, 8);
}

size_t smem_for(int RT, int tn, int S) {
  return 1024 + (size_t)S * ((size_t)RT * lm::kAccRows * 128 + (size_t)tn * 128) +
         (size_t)4 * RT * lm::kStoreBuf + 256;
}

// Two accumulator buffers (the epilogue of one tile overlaps the MMAs of
// the next) whenever they fit in the 512 TMEM columns.
template <int RT, int NB>
int launch_gemm_t(const CUtensorMap& th, const CUtensorMap& tw,
                  const CUtensorMap& tu, const CUtensorMap& tb,
                  const CUtensorMap& tout, lm::Params p, int workers,
                  cudaStream_t st) {
  p.stages = stages_for(RT, p.tn);
  if (p.stages < 2) return ISD_ERR_UNSUPPORTED;
  const size_t smem = smem_for(RT, p.tn, p.stages);
  auto kern = lm::lm_gemm_kernel<RT, NB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  const int sms = sms_now();
  if (sms <= 0) return ISD_ERR_CUDA;
  const int G = std::min(workers, sms);
  return launch_pdl(kern, dim3(G), dim3(lm::kThreads), smem, st, th, tw, tu,
                    tb, tout, p) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

int launch_pair(const CUtensorMap& th, const CUtensorMap& tw,
                const CUtensorMap& tu, const CUtensorMap& tb,
                const CUtensorMap& tout, lm::Params p, int workers,
                cudaStream_t st) {
  const size_t fixed = 1024 + (size_t)lm::kPairEpiWarps * lm::kStoreBuf + 256;
  const size_t stage = (size_t)2 * lm::kPairAtoms * lm::kPairHalf;
  p.stages = (int)std::min<size_t>((lm::kSmemLimit - fixed) / stage, 8);
  const size_t smem = fixed + (size_t)p.stages * stage;
  if (cudaFuncSetAttribute(lm::lm_pair_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  const int sms = sms_now();
  if (sms < 2) return ISD_ERR_CUDA;
  const int pairs = std::min(workers, sms / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(lm::kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, lm::lm_pair_kernel, th, tw, tu, tb, tout,
                            p) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

int launch_gemm(int RT, const CUtensorMap& th, const CUtensorMap& tw,
                const CUtensorMap& tu, const CUtensorMap& tb,
                const CUtensorMap& tout, const lm::Params& p, int workers,
                cudaStream_t st) {
  const bool two = 2 * RT * p.tn <= 512;
  if (RT == 2)
    return two ? launch_gemm_t<2, 2>(th, tw, tu, tb, tout, p, workers, st)
               : launch_gemm_t<2, 1>(th, tw, tu, tb, tout, p, workers, st);
  return two ? launch_gemm_t<1, 2>(th, tw, tu, tb, tout, p, workers, st)
             : launch_gemm_t<1, 1>(th, tw, tu, tb, tout, p, workers, st);
}

}  // namespace

size_t lm_head_workspace_bytes(const isd_lm_head_args* a) {
  return lm_layout(a).total;
}

size_t vocab_stats_bytes(int M, int V) {
  const size_t C = (size_t)(V + lm::kSubChunk - 1) / lm::kSubChunk;
  return std::max<size_t>(((size_t)M * C * 16 + 255) & ~size_t(255), 256);
}

// Tiles of the main GEMM and its split-K tail plan (below 64 rows the
// weight stream bounds the kernel and a lighter last wave gains nothing:
// measured at M = 8, 2.5% slower with the tail; M = 64 .. 256: 4.5-7%
// faster).
int lm_tiles(const isd_lm_head_args* a, const Shape& sh) {
  const int rows = tile_rows(sh);
  return ((a->M + rows - 1) / rows) * ((a->V + sh.tn - 1) / sh.tn);
}
TailPlan lm_plan(const isd_lm_head_args* a, const Shape& sh, int tiles) {
  const int Kt = a->D / lm::kBK + a->lora_rank / lm::kBK;
  return a->M >= 64 ? tail_plan(tiles, lm_workers(sh), Kt)
                    : tail_plan(tiles, 0, Kt);
}

int lm_head_launches(const isd_lm_head_args* a) {
  const Shape sh = lm_shape(a->M);
  const int tiles = lm_tiles(a, sh);
  const TailPlan tp = lm_plan(a, sh, tiles);
  return (a->lora_rank > 0 ? 2 : 0) + 1 + (tp.body < tiles ? 1 : 0) +
         (a->vocab_stats ? 1 : 0);
}

int launch_lm_head(const isd_lm_head_args* a, cudaStream_t st) {
  const int M = a->M, D = a->D, V = a->V, r = a->lora_rank;
  const Shape sh = lm_shape(M);
  const int RT = sh.RT, tn = sh.tn;
  const int rows_box = RT * lm::kAccRows;          // single-CTA tiles
  const int hbox = sh.pair ? 128 : rows_box;       // rows a CTA loads
  const int wbox = sh.pair ? tn / 2 : tn;          // entries a CTA loads
  const LmLayout l = lm_layout(a);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  CUtensorMap th, tw, tout, tu, tb;
  if (!encode_2d(&th, a->hidden, D, M, lm::kBK, hbox) ||
      !encode_2d(&tw, a->weight, D, V, lm::kBK, wbox) ||
      !encode_2d(&tout, a->logits, V, M, lm::kStoreCols, 32))
    return ISD_ERR_CUDA;
  tu = th;
  tb = tw;
  if (r > 0) {
    // 1. U = gate * scale * (H A^T): split-K partials on single-CTA tiles
    // (RT accumulators, r entries), then the ordered sum.
    CUtensorMap th1, ta;
    if (!encode_2d(&th1, a->hidden, D, M, lm::kBK, rows_box) ||
        !encode_2d(&ta, a->lora_a, D, r, lm::kBK, r))
      return ISD_ERR_CUDA;
    lm::Params q{};
    q.M = M; q.V = r; q.tn = r; q.RTn = (M + rows_box - 1) / rows_box;
    q.VT = 1; q.kD = D / lm::kBK; q.kR = 0;
    q.ksplit = std::min(kLoraSplit, q.kD);
    q.kps = (q.kD + q.ksplit - 1) / q.ksplit;
    q.ksplit = (q.kD + q.kps - 1) / q.kps;
    q.tiles = q.RTn * q.ksplit; q.mode = 1;
    q.body = q.tiles; q.tsplit = 1; q.tkps = 0;
    q.part = reinterpret_cast<float*>(ws + l.part);
    q.status = a->status;
    int rc = launch_gemm(RT, th1, ta, th1, ta, tout, q, q.tiles, st);
    if (rc != ISD_OK) return rc;
    __nv_bfloat16* u = reinterpret_cast<__nv_bfloat16*>(ws + l.u);
    lm::ReduceParams rp;
    rp.M = M; rp.r = r; rp.ksplit = q.ksplit; rp.K = a->rows_per_seq;
    rp.scale = a->lora_scale; rp.part = q.part; rp.n_pending = a->n_pending;
    rp.u = u; rp.status = a->status;
    const int blocks = (M * r + 255) / 256;
    if (launch_pdl(lm::lora_reduce_kernel, dim3(blocks), dim3(256), 0, st, rp) !=
        cudaSuccess)
      return ISD_ERR_CUDA;
    if (!encode_2d(&tu, u, r, M, lm::kBK, hbox) ||
        !encode_2d(&tb, a->lora_b, r, V, lm::kBK, wbox))
      return ISD_ERR_CUDA;
  }
  // 2. logits = [H | U] [W | B]^T with per-tile statistics.
  lm::Params p{};
  p.M = M; p.V = V; p.tn = tn;
  p.RTn = (M + tile_rows(sh) - 1) / tile_rows(sh);
  p.VT = (V + tn - 1) / tn; p.kD = D / lm::kBK; p.kR = r / lm::kBK;
  p.ksplit = 1; p.kps = 0; p.tiles = lm_tiles(a, sh); p.mode = 0;
  p.status = a->status;
  if (a->vocab_stats) {
    p.pmax = reinterpret_cast<float*>(ws + l.pmax);
    p.psum = reinterpret_cast<double*>(ws + l.psum);
    p.pidx = reinterpret_cast<int32_t*>(ws + l.pidx);
  }
  const TailPlan tp = lm_plan(a, sh, p.tiles);
  p.body = tp.body; p.tsplit = tp.tsplit; p.tkps = tp.tkps;
  p.tail = reinterpret_cast<float*>(ws + l.tail);
  int rc = sh.pair ? launch_pair(th, tw, tu, tb, tout, p, tp.workers, st)
                   : launch_gemm(RT, th, tw, tu, tb, tout, p, tp.workers, st);
  if (rc != ISD_OK) return rc;
  if (tp.body < p.tiles) {
    // 3. The tail tiles from their split-K pieces.
    lm::FixupParams fp;
    fp.M = M; fp.V = V; fp.tn = tn; fp.RTn = p.RTn; fp.body = tp.body;
    fp.ntail = p.tiles - tp.body;
    fp.tsplit = tp.tsplit; fp.trows = tile_rows(sh); fp.rec_w = sh.rec_w;
    fp.tail = p.tail;
    fp.logits = static_cast<__nv_bfloat16*>(a->logits);
    fp.pmax = p.pmax; fp.psum = p.psum; fp.pidx = p.pidx;
    const int warps = (p.tiles - tp.body) * fp.trows * (tn / sh.rec_w);
    if (launch_pdl(lm::lm_tail_fixup_kernel, dim3((warps + 7) / 8), dim3(256),
                   0, st, fp) != cudaSuccess)
      return ISD_ERR_CUDA;
  }
  if (!a->vocab_stats) return ISD_OK;
  // 4. Per-record figures -> sub-chunk figures in the accept step's layout.
  lm::MergeParams mp;
  mp.M = M; mp.V = V; mp.VT = sh.nrec(V);
  mp.C = (V + lm::kSubChunk - 1) / lm::kSubChunk;
  mp.per = lm::kSubChunk / sh.rec_w;
  mp.pmax = p.pmax; mp.psum = p.psum; mp.pidx = p.pidx;
  uint8_t* vs = static_cast<uint8_t*>(a->vocab_stats);
  mp.csum = reinterpret_cast<double*>(vs);
  mp.cmax = reinterpret_cast<float*>(vs + (size_t)M * mp.C * 8);
  mp.cidx = reinterpret_cast<int32_t*>(vs + (size_t)M * mp.C * 12);
  const int blocks = (M * mp.C + 255) / 256;
  return launch_pdl(lm::lm_stats_merge_kernel, dim3(blocks), dim3(256), 0, st,
                    mp) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

}  // namespace isd
