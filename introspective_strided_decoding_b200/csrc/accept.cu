// isd_accept_resample kernels: vocab softmax statistics, the min(1, p/q)
// ratio test, the residual / bonus / draft inverse-CDF draws.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io), "Inference & ISD": q proposes at MASK positions, p verifies at
// clean positions, x kept with probability min(1, p(x)/q(x)).  The residual
// normalise(max(0, p - q)) at the first rejection and the bonus draw when
// every draft passes are the standard speculative-sampling completion of
// that rule; the row layout is the stride schedule stated in isd.h.
//
// The vocabulary is cut into sub-chunks of 2048 elements, one warp's work
// (64 elements a lane).  Three kernels, one stream, no inter-CTA waiting:
//   stats  persistent warps stream the used rows sub-chunk by sub-chunk,
//          each warp an equal contiguous range of them, with 16-byte copies
//          kept in flight ahead of the reduction, and store each
//          sub-chunk's max, first index of the max and sum of
//          exp(l - max).                               [HBM and MUFU bound]
//   decide one CTA per sequence merges the sub-chunk figures into row
//          statistics, takes the ratio-test decision, writes its outputs
//          and leaves a record (decision, row max and sum of every row).
//   draw   grid (sequence, part) reads the record.  Rejected sequences:
//          part y sums max(0, p - q) over sub-chunks 4y .. 4y+3 (two warps
//          each) and the part that finishes last (atomic count, no
//          waiting) draws the replacement; accepted sequences: part t draws
//          token t (the bonus, then the drafts); other parts leave at once.
//          A draw picks the sub-chunk from a warp scan of the sub-chunk
//          masses, then scans its 2048 elements with eight warps of 256,
//          all in ascending vocabulary order.               [latency bound]
// isd_accept_commit launches the KV commit between decide and draw: the
// commit needs only the decisions, so the draws run beside it (the draw
// kernel then starts without its grid-dependency wait and one of its CTAs
// waits at its end; see the draw kernel).
// Element masses are fp32 (MUFU exp2 of exactly formed differences); every
// sum that places a sampling boundary or normalises a probability is
// accumulated in fp64 in a fixed order, so draws agree with an fp64
// reference except within a few 1e-8 of a boundary, and every run is
// bitwise reproducible.
#include <algorithm>

#include "common.cuh"

namespace isd {

constexpr int kSub = 2048;                 // vocabulary elements per sub-chunk
constexpr int kSubPerLane = 4;             // sub-chunks a lane owns in a row scan
constexpr int kMaxSub = 32 * kSubPerLane;  // V <= 262 144 (host check)
constexpr int kMaxRows = 32;               // K <= 32 (host check: N <= 16)
constexpr int kStatsWarps = 16;            // stats CTA: 512 threads
// The register-staged statistics kernel (two sub-chunks of 8 elements a
// lane held at once): 256 threads, so its registers are not capped at 128.
constexpr int kRegStatsWarps = 8;
constexpr int kDrawWarps = 8;              // draw CTA: 256 threads
constexpr int kResidPerCta = 4;            // residual sub-chunks per draw CTA
constexpr int kWarpElems = kSub / kDrawWarps;   // a draw warp's share: 256
// Warps per residual sub-chunk and the 8-element groups each lane sums.
constexpr int kResidWarps = kDrawWarps / kResidPerCta;
constexpr int kResidGroups = kSub / kResidWarps / 256;
static_assert(kDrawWarps % kResidPerCta == 0 && kResidGroups >= 1,
              "whole warps per residual sub-chunk");
static_assert(kWarpElems == 32 * 8, "a draw lane scans 8 elements");

template <typename T>
struct AcceptDev {
  int B, N, K, V, C, RU;
  int SR;              // rows per sequence in the sub-chunk arrays
  uint32_t step;
  const uint32_t* step_dev;  // when set, the step index is read from here
  uint64_t seed;
  const T* lc;
  const T* lp;
  const int32_t* seq_len;
  const int32_t* pending_in;
  const int32_t* n_in;
  const int32_t* q_row_in;
  const float* q_stats_in;
  int32_t* pending_out;
  int32_t* n_out;
  int32_t* q_row_out;
  float* q_stats_out;
  int32_t* n_commit;
  int32_t* commit_tokens;
  float* row_stats_out;
  float* ratio_out;
  int32_t* status;
  // workspace
  double* csum;        // [B][SR][C] sub-chunk sum of exp(l - sub-chunk max)
  float* cmax;         // [B][SR][C] sub-chunk max
  int32_t* cidx;       // [B][SR][C] first index of the sub-chunk max
  double* resid;       // [B][C] residual sub-chunk mass
  int32_t* count;      // [B] residual parts finished (zeroed by decide)
  int32_t* dec;        // [B][4] decision: flags (1 valid, 2 rejected), a, n, L
  float* rm;           // [B][RU] row max of every row (decide kernel)
  double* rs;          // [B][RU] row sum of every row
  int argmax;          // drafts are argmax q (point-mass proposals)
  int draw_nowait;     // draw launched behind the commit: no wait
};

// Eight consecutive elements kept in their storage format until use
// (bf16: one 16-byte word, half the registers of eight floats);
// out-of-range elements hold -inf.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  ISD_DEV float at(int e) const {
    const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
    return (e & 1) ? __uint_as_float(w & 0xFFFF0000u) : __uint_as_float(w << 16);
  }
};
template <> struct Raw8<float> {
  float v[8];
  ISD_DEV float at(int e) const { return v[e]; }
};

// Elements [idx, idx + 8) of a row of `hi` elements.  kVec: the row is
// 16-byte aligned and holds whole 16-byte units, so one vector load serves
// when idx + 8 <= hi; otherwise element loads, -inf past the end.
template <bool kVec>
ISD_DEV Raw8<__nv_bfloat16> load_raw8(const __nv_bfloat16* row, int idx,
                                      int hi) {
  Raw8<__nv_bfloat16> r;
  if (kVec && idx + 8 <= hi) {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.u.x), "=r"(r.u.y), "=r"(r.u.z), "=r"(r.u.w)
                 : "l"(row + idx));
  } else {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(row);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = idx + 2 * i < hi ? h[idx + 2 * i] : 0xFF80u;
      const uint32_t up = idx + 2 * i + 1 < hi ? h[idx + 2 * i + 1] : 0xFF80u;
      w[i] = lo | (up << 16);
    }
    r.u = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return r;
}
template <bool kVec>
ISD_DEV Raw8<float> load_raw8(const float* row, int idx, int hi) {
  Raw8<float> r;
  if (kVec && idx + 8 <= hi) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + idx));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + idx) + 1);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      r.v[e] = idx + e < hi ? row[idx + e] : -INFINITY;
  }
  return r;
}

ISD_DEV double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
ISD_DEV int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
ISD_DEV int warp_max_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Inclusive scan over the lanes in a fixed order; `excl` is exactly the
// previous lane's inclusive value (0 for lane 0).
ISD_DEV double warp_scan_f64(double v, double& excl) {
  const int lane = threadIdx.x & 31;
  double x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  excl = __shfl_up_sync(0xffffffffu, x, 1);
  if (lane == 0) excl = 0.0;
  return x;
}

template <typename T>
ISD_DEV uint32_t step_of(const AcceptDev<T>& p) {
  return p.step_dev ? *p.step_dev : p.step;
}

template <typename T>
ISD_DEV bool state_ok(const AcceptDev<T>& p, int b) {
  const int n = p.n_in[b];
  return (n == 1 || n == p.N) && p.seq_len[b] >= 0;
}

// ---------------------------------------------------------------------------
// Statistics, register-staged (fp32 logits, rows whose byte length is not
// a multiple of 16, batches too large for the shared-memory kernel's
// tables).  Items are the sub-chunks of the used rows, numbered row index
// first: it = (j * B + b) * C + c.  Global warp w takes items w, w + W,
// w + 2W, ... that are in use (a strided walk: the shared-memory kernel
// below gives each warp an equal contiguous range instead, which balances
// better when rows go unused); lane l holds elements
// lo + (k*32 + l)*8 + e (k, e < 8) of the sub-chunk, -inf past the row end,
// and lane 0 stores the max, the sum of exp(l - max) (8 terms in fp32, then
// fp64) and, for argmax proposals, the first index of the max (exact
// compares of the same values).
template <typename T, bool kVec>
ISD_DEV void load_sub(const AcceptDev<T>& p, int b, int j, int c,
                      Raw8<T> (&v)[8]) {
  const int lane = threadIdx.x & 31;
  const T* row = p.lc + ((size_t)b * p.K + j) * p.V;
  const int lo = c * kSub;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    v[k] = load_raw8<kVec>(row, lo + (k * 32 + lane) * 8, p.V);
}

template <typename T>
ISD_DEV void reduce_sub(const AcceptDev<T>& p, int b, int j, int c,
                        const Raw8<T> (&v)[8]) {
  const int lane = threadIdx.x & 31;
  float mk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    mk[k] = fmaxf(fmaxf(fmaxf(v[k].at(0), v[k].at(1)), fmaxf(v[k].at(2), v[k].at(3))),
                  fmaxf(fmaxf(v[k].at(4), v[k].at(5)), fmaxf(v[k].at(6), v[k].at(7))));
  }
  float m = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])),
                  fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7])));
  m = warp_max(m);
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float t = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) t += ex2((v[k].at(e) - m) * kLog2e);
    s += (double)t;
  }
  s = warp_sum_f64(s);
  const size_t o = ((size_t)b * p.SR + j) * p.C + c;
  if (p.argmax) {
    const int lo = c * kSub;
    int first = INT_MAX;
#pragma unroll
    for (int k = 7; k >= 0; --k)
#pragma unroll
      for (int e = 7; e >= 0; --e)
        if (v[k].at(e) == m) first = lo + (k * 32 + lane) * 8 + e;
    first = warp_min_int(first);
    if (lane == 0) p.cidx[o] = first;
  }
  if (lane == 0) {
    p.cmax[o] = m;
    p.csum[o] = s;
  }
}

// bf16 rows: the maximum over packed element pairs (a selection, so the
// same value as the unpacked compares) and the exponent arguments and sums
// in paired fp32 arithmetic: (l - m) * log2(e) is formed exactly as in the
// unpacked path, each sub-chunk group of 8 is summed as two interleaved
// halves of 4 in fp32, then in fp64.
ISD_DEV uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
ISD_DEV uint32_t word_of(const uint4& u, int i) {
  return i == 0 ? u.x : i == 1 ? u.y : i == 2 ? u.z : u.w;
}

template <>
ISD_DEV void reduce_sub<__nv_bfloat16>(
    const AcceptDev<__nv_bfloat16>& p, int b, int j, int c,
    const Raw8<__nv_bfloat16> (&v)[8]) {
  const int lane = threadIdx.x & 31;
  uint32_t mk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mk[k] = max_bf16x2(max_bf16x2(v[k].u.x, v[k].u.y),
                       max_bf16x2(v[k].u.z, v[k].u.w));
#pragma unroll
  for (int h = 4; h >= 1; h >>= 1)
#pragma unroll
    for (int k = 0; k < h; ++k) mk[k] = max_bf16x2(mk[k], mk[k + h]);
  float m = fmaxf(__uint_as_float(mk[0] << 16),
                  __uint_as_float(mk[0] & 0xFFFF0000u));
  m = warp_max(m);
  const float2 neg_m = make_float2(-m, -m);
  const float2 l2e = make_float2(kLog2e, kLog2e);
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t wd = word_of(v[k].u, i);
      const float2 x = make_float2(__uint_as_float(wd << 16),
                                   __uint_as_float(wd & 0xFFFF0000u));
      const float2 d = __fmul2_rn(__fadd2_rn(x, neg_m), l2e);
      const float2 e = make_float2(ex2(d.x), ex2(d.y));
      acc = i == 0 ? e : __fadd2_rn(acc, e);
    }
    s += (double)(acc.x + acc.y);
  }
  s = warp_sum_f64(s);
  const size_t o = ((size_t)b * p.SR + j) * p.C + c;
  if (p.argmax) {
    const int lo = c * kSub;
    int first = INT_MAX;
#pragma unroll
    for (int k = 7; k >= 0; --k)
#pragma unroll
      for (int e = 7; e >= 0; --e)
        if (v[k].at(e) == m) first = lo + (k * 32 + lane) * 8 + e;
    first = warp_min_int(first);
    if (lane == 0) p.cidx[o] = first;
  }
  if (lane == 0) {
    p.cmax[o] = m;
    p.csum[o] = s;
  }
}

// Walks one warp's items it, it + W, it + 2W, ... without divisions:
// W = (dj * B + db) * C + dc is split once, and (j, b, c) advance by
// (dj, db, dc) with carries.  `used` gives each sequence's rows in use
// (0 for a malformed state).
struct ItemWalk {
  int B, C, RU, dj, db, dc;
  int j, b, c;
  ISD_DEV void init(long long it, long long W, int B_, int C_, int RU_) {
    B = B_; C = C_; RU = RU_;
    c = (int)(it % C);
    const long long jb = it / C;
    b = (int)(jb % B);
    j = (int)(jb / B);
    dc = (int)(W % C);
    const long long q = W / C;
    db = (int)(q % B);
    dj = (int)(q / B);
  }
  ISD_DEV void step() {
    c += dc;
    int carry = c >= C;
    c -= carry ? C : 0;
    b += db + carry;
    carry = b >= B;
    b -= carry ? B : 0;
    j += dj + carry;
  }
  // Moves to the next item in use (at or after the current); false when
  // the items are exhausted.
  template <typename U>
  ISD_DEV bool next_used(const U& used) {
    for (; j < RU; step())
      if (j < used(b)) return true;
    return false;
  }
};

template <typename T, bool kVec>
__global__ void __launch_bounds__(kRegStatsWarps * 32)
    accept_stats_kernel(AcceptDev<T> p) {
  grid_dep_wait();
  auto used = [&](int b) {
    return state_ok(p, b) ? p.n_in[b] + p.N - 1 : 0;
  };
  ItemWalk w;
  w.init(blockIdx.x * kRegStatsWarps + (threadIdx.x >> 5),
         (long long)gridDim.x * kRegStatsWarps, p.B, p.C, p.RU);
  bool have = w.next_used(used);
  Raw8<T> cur[8];
  if (have) load_sub<T, kVec>(p, w.b, w.j, w.c, cur);
  while (have) {
    const int cb = w.b, cj = w.j, cc = w.c;
    w.step();
    have = w.next_used(used);
    Raw8<T> nxt[8];
    if (have) load_sub<T, kVec>(p, w.b, w.j, w.c, nxt);   // in flight ...
    reduce_sub(p, cb, cj, cc, cur);                      // ... during this
#pragma unroll
    for (int k = 0; k < 8; ++k) cur[k] = nxt[k];
  }
}

// A warp's share of the used sub-chunks for the shared-memory kernel:
// items are numbered in memory order (sequence, row, sub-chunk) over the
// rows in use only, and global warp g of G takes the contiguous range
// [g T / G, (g + 1) T / G) of the T items, so shares differ by at most one
// item (a strided walk that skips unused rows leaves some warps a quarter
// more work than the mean).  pre[b] is the number of rows in use before
// sequence b, pre[B] the total.
struct RangeWalk {
  int b, j, c, left, C;
  const int* pre;
  ISD_DEV void init(const int* pre_, int B, int C_, long long g,
                    long long G) {
    pre = pre_;
    C = C_;
    const long long T = (long long)pre[B] * C;
    const long long s = g * T / G;
    left = (int)((g + 1) * T / G - s);
    const int r = (int)(s / C);
    c = (int)(s % C);
    int lo = 0, hi = B;   // the last b with pre[b] <= r
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= r) lo = mid; else hi = mid;
    }
    b = lo;
    j = r - pre[lo];
  }
  // Moves to the next item of the range; the walker stays put once the
  // range is done, so it never looks past the last row in use.
  ISD_DEV void step() {
    if (--left <= 0) return;
    if (++c < C) return;
    c = 0;
    ++j;
    while (j >= pre[b + 1] - pre[b]) {
      ++b;
      j = 0;
    }
  }
};

// The same arithmetic for 16-byte aligned bf16 rows, staged through shared
// memory: each warp owns kStatsStages sub-chunk slots and keeps
// kStatsStages - 1 sub-chunks in flight with cp.async (16 bytes a lane, 8
// per sub-chunk) while it reduces the oldest.  Lane l copies and later
// reads back exactly its own elements, so a thread's own
// cp.async.wait_group is the only synchronisation.  A chunk past the row
// end is not copied; its elements read as -inf.
constexpr int kStatsStages = 3;
constexpr int kStatsSmem = kStatsWarps * kStatsStages * kSub * 2;   // 192 KB

ISD_DEV void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int kPending>
ISD_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Dynamic shared memory of the kernel below: the slots, then the per-
// sequence rows in use and their exclusive prefix.
static inline size_t stats_async_smem(int B) {
  return (size_t)kStatsSmem + (size_t)(2 * B + 1) * 4;
}

__global__ void __launch_bounds__(kStatsWarps * 32, 1)
    accept_stats_async_kernel(AcceptDev<__nv_bfloat16> p) {
  constexpr int S = kStatsStages;
  extern __shared__ __align__(16) unsigned char stats_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __nv_bfloat16* slots =
      reinterpret_cast<__nv_bfloat16*>(stats_smem) + (size_t)warp * S * kSub;
  grid_dep_wait();
  // Rows in use per sequence (0: malformed state), then their prefix.
  int* s_pre = reinterpret_cast<int*>(stats_smem + kStatsSmem);
  int* s_used = s_pre + p.B + 1;
  for (int i = threadIdx.x; i < p.B; i += blockDim.x)
    s_used[i] = state_ok(p, i) ? p.n_in[i] + p.N - 1 : 0;
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) s_pre[0] = 0;
    for (int base = 0; base < p.B; base += 32) {
      int x = base + lane < p.B ? s_used[base + lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (base + lane < p.B) s_pre[base + lane + 1] = carry + x;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  __syncthreads();
  RangeWalk w;
  w.init(s_pre, p.B, p.C, (long long)blockIdx.x * kStatsWarps + warp,
         (long long)gridDim.x * kStatsWarps);
  bool have = w.left > 0;
  // Copies this lane's 8 chunks of the walker's item into slot s.
  auto issue = [&](int s) {
    const __nv_bfloat16* row = p.lc + ((size_t)w.b * p.K + w.j) * p.V;
    const int lo = w.c * kSub;
    const uint32_t dst = smem_u32(slots + (size_t)s * kSub);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e0 = (k * 32 + lane) * 8;
      if (lo + e0 < p.V)   // whole 16-byte chunks: V is a multiple of 8
        cp_async_16(dst + e0 * 2, row + lo + e0, 16u);
    }
  };
  int qb[S], qj[S], qc[S];     // the item in each slot (qb < 0: none)
#pragma unroll
  for (int s = 0; s < S; ++s) qb[s] = -1;
  auto take = [&](int s) {     // the walker's item into slot s, then on
    if (have) {
      qb[s] = w.b; qj[s] = w.j; qc[s] = w.c;
      issue(s);
      w.step();
      have = w.left > 0;
    } else {
      qb[s] = -1;
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < S - 1; ++s) take(s);
  for (bool more = true; more;) {
#pragma unroll
    for (int u = 0; u < S; ++u) {
      // Refill the slot consumed in the previous round, then reduce slot u.
      take((u + S - 1) % S);
      cp_async_wait<S - 1>();
      if (qb[u] < 0) {
        more = false;
        break;
      }
      const int lo = qc[u] * kSub;
      const int n_el = min(kSub, p.V - lo);
      const __nv_bfloat16* src = slots + (size_t)u * kSub;
      Raw8<__nv_bfloat16> v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e0 = (k * 32 + lane) * 8;
        if (e0 < n_el)
          v[k].u = *reinterpret_cast<const uint4*>(src + e0);
        else
          v[k].u = make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u,
                              0xFF80FF80u);   // -inf
      }
      reduce_sub(p, qb[u], qj[u], qc[u], v);
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Residual element weight max(0, p - q), shared by the sub-chunk sums and
// the in-sub-chunk scan so both see the same per-element values.
// With argmax drafts q is a point mass at the rejected draft x, so the
// residual is p without x.
//
// Where p and q are close (peaked rows that agree on their top token) the
// plain difference of two rounded masses cancels: its absolute error, a few
// 1e-7 of q, can exceed the 1e-6 tie band of a small residual total.  Only
// elements of large mass can do that (the error scales with the mass), so
// for q > 2^-10 the weight is re-formed from delta = ln p - ln q =
// (l_p - l_q) - C, with l_p - l_q exact and C = (m_p + ln s_p) - ln Z_q in
// fp64 (a float pair): 0 for delta <= 0, q * expm1(delta) for
// 0 < delta <= 1 (relative error a few ulp whatever the cancellation), and
// the plain difference above 1 (p > e q: no cancellation).  That path is
// rare and kept out of line, so the unrolled element loops stay compact.
struct ResidRows {
  float mp, inv_sp;       // p row: max and 1 / sum
  float zq_hi, zq_lo;     // q row: log-normaliser ln Z_q as a float pair
  float c_hi, c_lo;       // C as a float pair
  int x;                  // rejected draft (argmax proposals), else -1
};
constexpr float kResidExactMass = 1.0f / 1024.0f;

__device__ __noinline__ float resid_exact(float qv, float lpv, float lqv,
                                          float c_hi, float c_lo, float w) {
  const float delta = ((lpv - lqv) - c_hi) - c_lo;
  if (!(delta > 0.0f)) return 0.0f;
  return delta <= 1.0f ? qv * expm1f(delta) : w;
}

ISD_DEV float resid_w(const ResidRows& r, float lpv, float lqv, int v) {
  const float pv = ex2((lpv - r.mp) * kLog2e) * r.inv_sp;
  if (r.x >= 0) return v == r.x ? 0.0f : pv;
  const float qv = ex2(((lqv - r.zq_hi) - r.zq_lo) * kLog2e);
  float w = pv - qv;
  if (qv > kResidExactMass) w = resid_exact(qv, lpv, lqv, r.c_hi, r.c_lo, w);
  return fmaxf(0.0f, w);
}

// The rows of a rejection at draft a + 1: p from row a of logits_cur (its
// max and sum `mp`, `sp`), q from the stored row of that draft (`x`, `qr`,
// `zhi` + `zlo`: the draft's token, q row and log-normaliser).
template <typename T>
ISD_DEV ResidRows resid_rows(const AcceptDev<T>& p, int b, int a, float mp,
                             double sp, int x, int qr, float zhi, float zlo,
                             const T*& prow, const T*& qrow) {
  const int K = p.K;
  prow = p.lc + ((size_t)b * K + a) * p.V;
  ResidRows r;
  r.mp = mp;
  r.inv_sp = (float)(1.0 / sp);
  if (p.argmax) {
    qrow = prow;                       // not read
    r.zq_hi = r.zq_lo = r.c_hi = r.c_lo = 0.0f;
    r.x = x;
  } else {
    qrow = p.lp + ((size_t)b * K + qr) * p.V;
    r.zq_hi = zhi;
    r.zq_lo = zlo;
    const double c = ((double)mp + log(sp)) - ((double)r.zq_hi + (double)r.zq_lo);
    r.c_hi = (float)c;
    r.c_lo = (float)(c - (double)r.c_hi);
    r.x = -1;
  }
  return r;
}

// Row statistics from the sub-chunk figures, by one warp: m = max of the
// sub-chunk maxima, s = sum_c csum_c * exp(cmax_c - m) (fp64, fixed order).
template <typename T>
ISD_DEV void merge_row(const AcceptDev<T>& p, int b, int r, float& m_out,
                       double& s_out) {
  const int lane = threadIdx.x & 31;
  const size_t o = ((size_t)b * p.SR + r) * p.C;
  float cm[kSubPerLane];
  double cs[kSubPerLane];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kSubPerLane; ++i) {
    const int c = lane * kSubPerLane + i;
    cm[i] = c < p.C ? p.cmax[o + c] : -INFINITY;
    cs[i] = c < p.C ? p.csum[o + c] : 0.0;
    m = fmaxf(m, cm[i]);
  }
  m = warp_max(m);
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < kSubPerLane; ++i) {
    const int c = lane * kSubPerLane + i;
    s += c < p.C ? cs[i] * exp((double)(cm[i] - m)) : 0.0;
  }
  m_out = m;
  s_out = warp_sum_f64(s);
}

// ---------------------------------------------------------------------------
// Decide: one CTA per sequence merges the sub-chunk figures of every row
// into row statistics (warps 1..7), takes the ratio-test decision (warp 0)
// and writes the decision's outputs, plus a record for the draw kernel:
// dec[b] = (flags: 1 valid, 2 rejected; a; n; the sequence length L it
// read) and the row max / sum of every row.  The draw kernel reads L from
// the record, not from seq_len, so a commit may grow seq_len meanwhile.
struct DecideShared {
  float m[kMaxRows];           // row max
  double s[kMaxRows];          // row sum
};

template <typename T>
__global__ void __launch_bounds__(kDrawWarps * 32)
    accept_decide_kernel(AcceptDev<T> p) {
  __shared__ DecideShared sh;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, K = p.K;
  grid_dep_wait();
  // ---- 0. The sequence's state and its drafts' logits (warp 0).
  int n = 0, L = 0, tok = 0, qr = 0;
  float zhi = 0.0f, zlo = 0.0f, lx = 0.0f, lqx = 0.0f;
  bool ok = false;
  if (warp == 0) {
    n = p.n_in[b];
    L = p.seq_len[b];
    tok = lane < N ? p.pending_in[b * N + lane] : 0;
    qr = lane < N ? p.q_row_in[b * N + lane] : 0;
    if (!p.argmax && lane < N) {
      zhi = p.q_stats_in[(b * N + lane) * 2];
      zlo = p.q_stats_in[(b * N + lane) * 2 + 1];
    }
    ok = (n == 1 || n == N) && L >= 0;
    if (ok && lane < n) ok = tok >= 0 && tok < p.V;
    if (ok && lane >= 1 && lane < n) ok = qr >= 0 && qr < K;
    ok = __all_sync(0xffffffffu, ok);
    if (ok && lane >= 1 && lane < n) {
      lx = to_f(p.lc[((size_t)b * K + lane - 1) * p.V + tok]);
      if (!p.argmax) lqx = to_f(p.lp[((size_t)b * K + qr) * p.V + tok]);
    }
  }
  if (threadIdx.x == 0) p.count[b] = 0;   // the draw kernel's residual parts
  // ---- 1. Row statistics of every row (warps 1..).
  if (warp > 0) {
    for (int r = warp - 1; r < p.RU; r += kDrawWarps - 1) {
      float m;
      double s;
      merge_row(p, b, r, m, s);
      if (lane == 0) {
        sh.m[r] = m;
        sh.s[r] = s;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < p.RU) {
    p.rm[(size_t)b * p.RU + threadIdx.x] = sh.m[threadIdx.x];
    p.rs[(size_t)b * p.RU + threadIdx.x] = sh.s[threadIdx.x];
  }
  if (warp != 0) return;
  if (!ok) {
    // Malformed state: reported once, passed through, nothing committed.
    if (lane == 0) {
      report(p.status, ISD_ERR_BAD_STATE);
      p.n_commit[b] = 0;
      p.n_out[b] = n;
      *reinterpret_cast<int4*>(p.dec + 4 * b) = make_int4(0, 0, n, L);
    }
    if (lane < N) {
      const int i = b * N + lane;
      p.commit_tokens[i] = -1;
      p.pending_out[i] = p.pending_in[i];
      p.q_row_out[i] = p.q_row_in[i];
      p.q_stats_out[2 * i] = p.q_stats_in[2 * i];
      p.q_stats_out[2 * i + 1] = p.q_stats_in[2 * i + 1];
    }
    return;
  }
  // ---- 2. Ratio tests of drafts 1 .. n-1 (lane i verifies draft i with
  //         row i-1); l - m is exact in fp32; p, q, the ratio fp64.
  const int rows_used = n + N - 1;
  const bool verifies = lane >= 1 && lane < n;
  bool acc = true;
  double r = 0.0;
  if (verifies) {
    const double px = exp((double)(lx - sh.m[lane - 1])) / sh.s[lane - 1];
    double qx = 1.0;      // argmax drafts: the proposal is a point mass
    if (!p.argmax) qx = exp(((double)lqx - (double)zhi) - (double)zlo);
    r = qx > 0.0 ? px / qx : INFINITY;
    const float u = uniform(p.seed, (uint32_t)b, step_of(p),
                            (uint32_t)(L + lane), ISD_STREAM_ACCEPT);
    acc = (double)u < r;
  }
  const uint32_t mask = __ballot_sync(0xffffffffu, acc);
  const uint32_t drafts = ((n >= 32) ? 0xffffffffu : ((1u << n) - 1u)) & ~1u;
  const uint32_t rej = drafts & ~mask;
  const bool rejected = rej != 0u;
  const int a = rejected ? (__ffs(rej) - 2) : (n - 1);
  // The decision's outputs.
  if (verifies && p.ratio_out) p.ratio_out[b * N + lane] = (float)r;
  if (lane < N) {
    p.commit_tokens[b * N + lane] = lane <= a ? tok : -1;
    // Next drafts' q rows and the log-normaliser log sum_v exp(l_v) of
    // each (lane j: row n + j - 1), stored as a float pair hi + lo.
    const bool has = !rejected && lane >= 1;
    const int src = n + lane - 1;
    p.q_row_out[b * N + lane] = has ? src : -1;
    const double lz = has ? (double)sh.m[src] + log(sh.s[src]) : 0.0;
    const float lz_hi = (float)lz;
    p.q_stats_out[(b * N + lane) * 2] = lz_hi;
    p.q_stats_out[(b * N + lane) * 2 + 1] = (float)(lz - (double)lz_hi);
    // After a rejection only the replacement is pending.
    if (rejected && lane >= 1) p.pending_out[b * N + lane] = -1;
  }
  if (p.row_stats_out && lane < rows_used) {
    p.row_stats_out[(b * K + lane) * 2] = sh.m[lane];
    p.row_stats_out[(b * K + lane) * 2 + 1] = (float)sh.s[lane];
  }
  if (lane == 0) {
    p.n_commit[b] = a + 1;
    p.n_out[b] = rejected ? 1 : N;
    *reinterpret_cast<int4*>(p.dec + 4 * b) =
        make_int4(rejected ? 3 : 1, a, n, L);
  }
}

// What a CTA of the draw kernel shares between its warps.
struct DrawShared {
  float m[kMaxRows];           // row max (from the decide record)
  double s[kMaxRows];          // row sum
  int tok[kMaxRows];           // pending tokens (drafts)
  int qr[kMaxRows];            // their q rows
  float zq[kMaxRows][2];       // their q log-normalisers (hi, lo)
  double tot[kDrawWarps];      // per-warp totals of an element scan
  int lastp[kDrawWarps];       // per-warp last positive element
  double rem;                  // target left inside the chosen sub-chunk
  int chosen;                  // chosen sub-chunk
  int found;                   // warp holding the target (-1: none)
  int ok, n, rejected, a, last, mode, L;
};

// One inverse-CDF draw by the whole CTA: the smallest index whose running
// mass (ascending order) exceeds u * total.  Sub-chunk masses: the
// residual's from `resid` (mode 0, written by this kernel; if their total
// is zero, p == q up to rounding, the draw falls back to p of row `row`),
// or those of row `row` of logits_cur (mode 1, row max m_row):
// csum_c * exp(cmax_c - m_row).
template <typename T, bool kVec>
ISD_DEV int cta_draw(const AcceptDev<T>& p, DrawShared& sh, int b, int mode,
                     int row, float m_row, const ResidRows& rr,
                     const T* prow, const T* qrow, float u) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, C = p.C;
  // 1. The sub-chunk (warp 0): lane l owns sub-chunks 4l .. 4l+3.
  if (warp == 0) {
    double mc[kSubPerLane];
    double own = 0.0;
    double excl = 0.0, incl = 0.0, total = 0.0;
    if (mode == 0) {
#pragma unroll
      for (int i = 0; i < kSubPerLane; ++i) {
        const int c = lane * kSubPerLane + i;
        mc[i] = c < C ? __ldcg(&p.resid[(size_t)b * C + c]) : 0.0;
        own += mc[i];
      }
      incl = warp_scan_f64(own, excl);
      total = __shfl_sync(0xffffffffu, incl, 31);
      // Zero residual mass: draw from p of row `row` instead.
      if (!(total > 0.0)) mode = 1;
    }
    if (mode == 1) {
      const size_t o = ((size_t)b * p.SR + row) * C;
      own = 0.0;
#pragma unroll
      for (int i = 0; i < kSubPerLane; ++i) {
        const int c = lane * kSubPerLane + i;
        mc[i] = c < C ? p.csum[o + c] * exp((double)(p.cmax[o + c] - m_row)) : 0.0;
        own += mc[i];
      }
      incl = warp_scan_f64(own, excl);
      total = __shfl_sync(0xffffffffu, incl, 31);
    }
    const double target = (double)u * total;
    const uint32_t hit = __ballot_sync(0xffffffffu, incl > target);
    const uint32_t pos = __ballot_sync(0xffffffffu, own > 0.0);
    // Rounding can leave the target past every running sum: then the last
    // sub-chunk with positive mass, scanned to its last positive entry.
    const int hl = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
    if (lane == hl) {
      double run = excl;
      int chosen = -1, lastpos = lane * kSubPerLane;
      double rem = INFINITY;
#pragma unroll
      for (int i = 0; i < kSubPerLane; ++i) {
        const int c = lane * kSubPerLane + i;
        if (c >= C) break;
        if (mc[i] > 0.0) lastpos = c;
        const double before = run;
        run += mc[i];
        if (hit && chosen < 0 && run > target) {
          chosen = c;
          rem = target - before;
        }
      }
      sh.chosen = chosen < 0 ? lastpos : chosen;
      sh.rem = rem;
      sh.mode = mode;
    }
  }
  __syncthreads();
  mode = sh.mode;
  // 2. Inside the sub-chunk: warp w scans elements lo + 256w .. +255, lane
  //    l elements lo + 256w + 8l .. +7, so warp order and lane order keep
  //    the scan ascending.  The warps' totals are taken in order from the
  //    target, which is what one warp scanning all eight parts would do.
  const int lo = sh.chosen * kSub, hi = min(p.V, lo + kSub);
  const int base = lo + warp * kWarpElems + lane * 8;
  const bool with_q = mode == 0 && rr.x < 0;
  const Raw8<T> cp = load_raw8<kVec>(prow, base, hi);
  Raw8<T> cq{};
  if (with_q) cq = load_raw8<kVec>(qrow, base, hi);
  float wv[8];
  double lt = 0.0;
  int lastr = -1;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    wv[e] = mode == 0 ? resid_w(rr, cp.at(e), with_q ? cq.at(e) : 0.0f, base + e)
                      : ex2((cp.at(e) - m_row) * kLog2e);
    lt += (double)wv[e];
    if (wv[e] > 0.0f) lastr = base + e;
  }
  double ex;
  const double inc = warp_scan_f64(lt, ex);
  const int lastw = warp_max_int(lastr);
  if (lane == 31) {
    sh.tot[warp] = inc;
    sh.lastp[warp] = lastw;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double rem = sh.rem;
    int f = -1;
    for (int w = 0; w < kDrawWarps; ++w) {
      if (rem < sh.tot[w]) {
        f = w;
        break;
      }
      rem -= sh.tot[w];
    }
    sh.found = f;
    sh.rem = rem;
  }
  __syncthreads();
  int tok = -1;
  if (sh.found < 0) {
    // Rounding left the target past every running sum: the last positive
    // entry of the sub-chunk.
    int lp = -1;
    for (int w = 0; w < kDrawWarps; ++w) lp = max(lp, sh.lastp[w]);
    tok = lp >= 0 ? lp : lo;
  } else if (warp == sh.found) {
    const double rem = sh.rem;
    const int hl2 = __ffs(__ballot_sync(0xffffffffu, inc > rem)) - 1;
    if (lane == hl2) {
      double run = ex;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        run += (double)wv[e];
        if (tok < 0 && run > rem) tok = base + e;
      }
      if (tok < 0) tok = lastr;  // rounding: this lane's last positive
    }
    tok = __shfl_sync(0xffffffffu, tok, hl2 < 0 ? 0 : hl2);
    if (hl2 < 0) tok = sh.lastp[warp] >= 0 ? sh.lastp[warp] : lo;
  }
  return tok;   // valid on every thread when found < 0, else on warp `found`
}

// The draw kernel, grid (sequence, part), after the decide kernel: it reads
// the decision record, then rejected sequences sum the residual over their
// parts' sub-chunks and the part that finishes last draws the replacement;
// accepted sequences draw token y in part y (the bonus, then the drafts).
// Parts with nothing to do leave as soon as the record is read.
template <typename T, bool kVec>
ISD_DEV void draw_body(const AcceptDev<T>& p, DrawShared& sh) {
  const int b = blockIdx.x, y = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, K = p.K;
  // Behind the commit (isd_accept_commit) the draws do not wait before
  // their work: the commit triggered this grid after its own wait, so the
  // decide kernel and everything before it have finished, and the two
  // kernels touch disjoint memory (the kernel waits at its end instead).
  if (!p.draw_nowait) grid_dep_wait();
  // ---- 0. The sequence's inputs and the decision record.
  if (warp == 0) {
    if (lane < N) {
      sh.tok[lane] = p.pending_in[b * N + lane];
      sh.qr[lane] = p.q_row_in[b * N + lane];
      sh.zq[lane][0] = p.argmax ? 0.0f : p.q_stats_in[(b * N + lane) * 2];
      sh.zq[lane][1] = p.argmax ? 0.0f : p.q_stats_in[(b * N + lane) * 2 + 1];
    }
  }
  if (threadIdx.x < p.RU) {
    sh.m[threadIdx.x] = __ldcg(&p.rm[(size_t)b * p.RU + threadIdx.x]);
    sh.s[threadIdx.x] = __ldcg(&p.rs[(size_t)b * p.RU + threadIdx.x]);
  }
  if (threadIdx.x == 32) {
    const int4 d = __ldcg(reinterpret_cast<const int4*>(p.dec + 4 * b));
    sh.ok = d.x & 1;
    sh.rejected = (d.x >> 1) & 1;
    sh.a = d.y;
    sh.n = d.z;
    sh.L = d.w;
  }
  __syncthreads();
  if (!sh.ok) return;             // malformed: handled by the decide kernel
  const int n = sh.n, L = sh.L;
  if (n == 1 && y >= N) return;   // no drafts: nothing to reject
  const bool rejected = sh.rejected;
  const int a = sh.a;
  if (rejected) {
    // ---- 2a. Residual sub-chunk sums: part y takes sub-chunks
    //          kResidPerCta y .. + kResidPerCta - 1, kResidWarps warps each,
    //          in fixed order.
    const int nparts = (p.C + kResidPerCta - 1) / kResidPerCta;
    if (y >= nparts) return;
    const T* prow;
    const T* qrow;
    const ResidRows rr =
        resid_rows(p, b, a, sh.m[a], sh.s[a], sh.tok[a + 1], sh.qr[a + 1],
                   sh.zq[a + 1][0], sh.zq[a + 1][1], prow, qrow);
    const int c = y * kResidPerCta + warp / kResidWarps;
    const int part = warp % kResidWarps;
    double s = 0.0;
    if (c < p.C) {
      const int lo = c * kSub + part * (kSub / kResidWarps);
      const int hi = min(p.V, c * kSub + kSub);
      Raw8<T> vp[kResidGroups], vq[kResidGroups];
#pragma unroll
      for (int k = 0; k < kResidGroups; ++k) {
        vp[k] = load_raw8<kVec>(prow, lo + (k * 32 + lane) * 8, hi);
        if (rr.x < 0) vq[k] = load_raw8<kVec>(qrow, lo + (k * 32 + lane) * 8, hi);
      }
#pragma unroll
      for (int k = 0; k < kResidGroups; ++k) {
        const int idx = lo + (k * 32 + lane) * 8;
        float t = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          t += resid_w(rr, vp[k].at(e), rr.x < 0 ? vq[k].at(e) : 0.0f, idx + e);
        s += (double)t;
      }
      s = warp_sum_f64(s);
    }
    if (lane == 0) sh.tot[warp] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int i = 0; i < kResidPerCta; ++i) {
        const int ci = y * kResidPerCta + i;
        if (ci >= p.C) continue;
        double r = 0.0;
        for (int k = 0; k < kResidWarps; ++k) r += sh.tot[kResidWarps * i + k];
        p.resid[(size_t)b * p.C + ci] = r;
      }
      __threadfence();
      sh.last = atomicAdd(&p.count[b], 1) == nparts - 1;
    }
    __syncthreads();
    if (!sh.last) return;
    // Last part of this sequence: every resid[b][*] is written.
    __threadfence();
    const float u = uniform(p.seed, (uint32_t)b, step_of(p),
                            (uint32_t)(L + a + 1), ISD_STREAM_RESAMPLE);
    const int t = cta_draw<T, kVec>(p, sh, b, 0, a, sh.m[a], rr, prow, qrow, u);
    if (sh.found < 0 ? threadIdx.x == 0 : (warp == sh.found && lane == 0))
      p.pending_out[b * N] = t;
    return;
  }
  // ---- 2b. All drafts accepted: part y draws token y (0: the bonus from p
  //          of row n-1; y >= 1: the draft at L + n + y from q of row
  //          n + y - 1).
  if (y >= N) return;
  const int row = n + y - 1;
  if (p.argmax && y >= 1) {
    // Argmax draft: the first sub-chunk whose max is the row max holds the
    // first maximal index (exact compares of the same values).
    if (warp == 0) {
      const size_t o = ((size_t)b * p.SR + row) * p.C;
      const float m = sh.m[row];
      int first = INT_MAX;
#pragma unroll
      for (int i = kSubPerLane - 1; i >= 0; --i) {
        const int ci = lane * kSubPerLane + i;
        if (ci < p.C && p.cmax[o + ci] == m) first = ci;
      }
      first = warp_min_int(first);
      if (lane == 0) p.pending_out[b * N + y] = first < p.C ? p.cidx[o + first] : -1;
    }
    return;
  }
  const float u = uniform(p.seed, (uint32_t)b, step_of(p), (uint32_t)(L + n + y),
                          y == 0 ? ISD_STREAM_RESAMPLE : ISD_STREAM_DRAFT);
  const ResidRows none{};
  const T* prow = p.lc + ((size_t)b * K + row) * p.V;
  const int t = cta_draw<T, kVec>(p, sh, b, 1, row, sh.m[row], none, prow,
                                  prow, u);
  if (sh.found < 0 ? threadIdx.x == 0 : (warp == sh.found && lane == 0))
    p.pending_out[b * N + y] = t;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kDrawWarps * 32)
    accept_draw_kernel(AcceptDev<T> p) {
  __shared__ DrawShared sh;
  draw_body<T, kVec>(p, sh);
  // Behind the commit one CTA waits, after its work, for the commit grid
  // to complete: the draw grid then completes only after the commit, so a
  // later kernel's wait on the draw grid covers the commit's writes too.
  // One is enough (a grid is complete when its last CTA exits); every CTA
  // waiting held the early-leaving parts' slots (measured: +5 us at C=64).
  if (p.draw_nowait && blockIdx.x == 0 && blockIdx.y == 0) grid_dep_wait();
}

// ---------------------------------------------------------------------------
// Host-side launcher (called from the C ABI after validation).

int launch_commit(const isd_commit_args* a, cudaStream_t st, bool trigger);

struct AcceptLayout {
  size_t csum, cmax, cidx, resid, count, dec, rm, rs, total;
};

static AcceptLayout accept_layout(int B, int N, int K, int V) {
  const size_t C = (V + kSub - 1) / kSub;
  const size_t RU = 2 * N - 1;
  (void)K;
  AcceptLayout l;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) & ~size_t(255);
    return at;
  };
  l.csum = take((size_t)B * RU * C * 8);
  l.cmax = take((size_t)B * RU * C * 4);
  l.cidx = take((size_t)B * RU * C * 4);
  l.resid = take((size_t)B * C * 8);
  l.count = take((size_t)B * 4);
  l.dec = take((size_t)B * 16);
  l.rm = take((size_t)B * RU * 4);
  l.rs = take((size_t)B * RU * 8);
  l.total = off;
  return l;
}

static int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return 0;
  return n;
}

// The register-staged statistics kernel: as many 256-thread CTAs as fit
// on every SM at once (the warps loop over the items), fewer for small
// problems.
template <typename T, bool kVec>
static int launch_reg_stats(const AcceptDev<T>& p, int sms, cudaStream_t st) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &per_sm, accept_stats_kernel<T, kVec>, kRegStatsWarps * 32, 0) !=
          cudaSuccess ||
      per_sm < 1)
    return ISD_ERR_CUDA;
  const long long items = (long long)p.B * p.RU * p.C;
  const long long ctas = (items + kRegStatsWarps - 1) / kRegStatsWarps;
  const int grid = (int)std::max<long long>(
      1, std::min<long long>((long long)per_sm * sms, ctas));
  return launch_pdl(accept_stats_kernel<T, kVec>, dim3(grid),
                    dim3(kRegStatsWarps * 32), 0, st, p) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

template <typename T, bool kVec>
static int launch_stats(const AcceptDev<T>& p, int sms, cudaStream_t st) {
  return launch_reg_stats<T, kVec>(p, sms, st);
}

// Aligned bf16 rows: the shared-memory pipeline, one 512-thread CTA per SM.
template <>
int launch_stats<__nv_bfloat16, true>(const AcceptDev<__nv_bfloat16>& p,
                                      int sms, cudaStream_t st) {
  // Slots, then the rows-in-use tables; too many sequences for the tables
  // take the register kernel.
  const size_t smem = stats_async_smem(p.B);
  if (smem > 227 * 1024) return launch_reg_stats<__nv_bfloat16, true>(p, sms, st);
  auto kern = accept_stats_async_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  const long long items = (long long)p.B * p.RU * p.C;
  const long long ctas = (items + kStatsWarps - 1) / kStatsWarps;
  const int grid = (int)std::max<long long>(1, std::min<long long>(sms, ctas));
  return launch_pdl(kern, dim3(grid), dim3(kStatsWarps * 32), smem, st,
                    p) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

template <typename T, bool kVec>
static int launch_accept_kernels(const AcceptDev<T>& p, int sms,
                                 cudaStream_t st, bool have_stats,
                                 const isd_commit_args* commit) {
  // With the sub-chunk figures from the LM head there is no statistics
  // kernel.
  if (!have_stats) {
    const int rc = launch_stats<T, kVec>(p, sms, st);
    if (rc != ISD_OK) return rc;
  }
  if (launch_pdl(accept_decide_kernel<T>, dim3(p.B), dim3(kDrawWarps * 32), 0,
                 st, p) != cudaSuccess)
    return ISD_ERR_CUDA;
  AcceptDev<T> q = p;
  if (commit) {
    // The commit of this step's decisions, then the draws beside it.
    const int rc = launch_commit(commit, st, true);
    if (rc != ISD_OK) return rc;
    q.draw_nowait = 1;
  }
  const int parts = std::max((p.C + kResidPerCta - 1) / kResidPerCta, p.N);
  if (launch_pdl(accept_draw_kernel<T, kVec>, dim3(p.B, parts),
                 dim3(kDrawWarps * 32), 0, st, q) != cudaSuccess)
    return ISD_ERR_CUDA;
  return ISD_OK;
}

template <typename T>
static int launch_accept_t(const isd_accept_args* a, cudaStream_t st,
                           const isd_commit_args* commit) {
  AcceptDev<T> p;
  p.B = a->B; p.N = a->N; p.K = a->K; p.V = a->V;
  p.C = (a->V + kSub - 1) / kSub;
  p.RU = 2 * a->N - 1;
  if (p.C > kMaxSub || p.K > kMaxRows) return ISD_ERR_UNSUPPORTED;
  p.step = a->step; p.step_dev = a->step_dev; p.seed = a->seed;
  p.lc = static_cast<const T*>(a->logits_cur);
  p.lp = static_cast<const T*>(a->logits_prev);
  p.seq_len = a->seq_len; p.pending_in = a->pending_in; p.n_in = a->n_pending_in;
  p.q_row_in = a->q_row_in; p.q_stats_in = a->q_stats_in;
  p.pending_out = a->pending_out; p.n_out = a->n_pending_out;
  p.q_row_out = a->q_row_out; p.q_stats_out = a->q_stats_out;
  p.n_commit = a->n_commit; p.commit_tokens = a->commit_tokens;
  p.row_stats_out = a->row_stats; p.ratio_out = a->ratio; p.status = a->status;
  const AcceptLayout l = accept_layout(a->B, a->N, a->K, a->V);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  p.csum = reinterpret_cast<double*>(ws + l.csum);
  p.cmax = reinterpret_cast<float*>(ws + l.cmax);
  p.cidx = reinterpret_cast<int32_t*>(ws + l.cidx);
  p.resid = reinterpret_cast<double*>(ws + l.resid);
  p.count = reinterpret_cast<int32_t*>(ws + l.count);
  p.dec = reinterpret_cast<int32_t*>(ws + l.dec);
  p.rm = reinterpret_cast<float*>(ws + l.rm);
  p.rs = reinterpret_cast<double*>(ws + l.rs);
  p.SR = p.RU;
  const bool have_stats = a->vocab_stats != nullptr;
  if (have_stats) {
    // isd_lm_head's layout: csum, cmax, cidx, each [B * K][C].
    const uint8_t* vs = static_cast<const uint8_t*>(a->vocab_stats);
    const size_t rows = (size_t)a->B * a->K;
    p.csum = const_cast<double*>(reinterpret_cast<const double*>(vs));
    p.cmax = const_cast<float*>(
        reinterpret_cast<const float*>(vs + rows * p.C * 8));
    p.cidx = const_cast<int32_t*>(
        reinterpret_cast<const int32_t*>(vs + rows * p.C * 12));
    p.SR = a->K;
  }
  p.argmax = a->proposal == ISD_PROPOSAL_ARGMAX;
  p.draw_nowait = 0;
  const int sms = num_sms();
  if (sms <= 0) return ISD_ERR_CUDA;
  // Vector loads need 16-byte aligned rows (logits_cur itself is checked
  // on the host) of whole 16-byte units.
  if (((size_t)a->V * sizeof(T)) % 16 == 0)
    return launch_accept_kernels<T, true>(p, sms, st, have_stats, commit);
  return launch_accept_kernels<T, false>(p, sms, st, have_stats, commit);
}

size_t accept_workspace_bytes(int B, int N, int K, int V) {
  return accept_layout(B, N, K, V).total;
}

// `commit`: null, or the KV commit of this step's decisions, launched
// between the decide and draw kernels (isd_accept_commit).
int launch_accept(const isd_accept_args* a, cudaStream_t st,
                  const isd_commit_args* commit) {
  if (a->dtype == ISD_BF16)
    return launch_accept_t<__nv_bfloat16>(a, st, commit);
  return launch_accept_t<float>(a, st, commit);
}

}  // namespace isd
