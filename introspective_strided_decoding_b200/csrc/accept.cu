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
// (64 elements a lane), so no step needs a block-wide barrier.  Three
// kernels, one stream, no inter-CTA waiting:
//   stats   one CTA per SM.  Six producer lanes stream the used rows into
//           a 12-slot shared-memory ring in 16 KB bulk asynchronous copies
//           (TMA engine, completion counted on mbarriers); six groups of
//           four consumer warps take the copies in turn, each warp reducing
//           one sub-chunk to its max, the first index of that max and the
//           sum of exp(l - max), in two passes over shared memory.
//           Rows whose byte length is not a multiple of 16 cannot be bulk
//           copied and go through a plain-load variant with the same
//           element order and arithmetic.                         [HBM bound]
//   decide  one CTA per sequence: warp j merges row j's sub-chunk figures
//           into the row's (m, s); warp 0 runs the ratio tests, ballots
//           the first rejection and writes the next state
//   draw    rejected sequences: one warp per sub-chunk sums max(0, p - q),
//           and the warp that finishes last (atomic count, no waiting)
//           draws the replacement; accepted sequences: warp t draws token
//           t (the bonus, then the drafts).  A draw scans the sub-chunk
//           masses to pick a sub-chunk, then that sub-chunk's elements,
//           both in ascending vocabulary order.
// Element masses are fp32 (MUFU exp2 of exactly formed differences); every
// sum that places a sampling boundary or normalises a probability is
// accumulated in fp64 in a fixed order, so draws agree with an fp64
// reference except within a few 1e-8 of a boundary, and every run is
// bitwise reproducible.
#include <algorithm>

#include "common.cuh"

namespace isd {

constexpr int kSub = 2048;          // vocabulary elements per sub-chunk
constexpr int kSubPerLane = 4;      // sub-chunks a lane owns in a row scan
constexpr int kMaxSub = 32 * kSubPerLane;  // V <= 262 144 (host check)
// Stats CTA: a ring of kSlots bulk copies of kCopyBytes (16 KB: 4 bf16 or
// 2 f32 sub-chunks of a row), filled by kIssuers producer lanes and read by
// kGroups groups of kGroupWarps consumer warps, warp i of a group taking
// sub-chunk i of each copy.  kSlots is a multiple of kGroups, so every use
// of a slot goes to the same group, in order: a warp never waits on a slot
// whose previous use (another group's) is still pending, which a parity
// wait could not tell from the use before that.
constexpr int kCopyBytes = 16 * 1024;
constexpr int kSlots = 12;
constexpr int kGroups = 6;
constexpr int kGroupWarps = 4;
constexpr int kConsumers = kGroups * kGroupWarps;
constexpr int kIssuers = 6;
constexpr uint32_t kIssuerMask = (1u << kIssuers) - 1u;
constexpr int kStatsThreads = (kConsumers + 1) * 32;  // + producer warp
static_assert(kStatsThreads <= 1024, "one CTA holds at most 1024 threads");
static_assert(kSlots % kGroups == 0 && kIssuers <= kSlots, "slot ownership");
static_assert(kCopyBytes / (kSub * 2) <= kGroupWarps &&
                  kCopyBytes % (kSub * 4) == 0,
              "a copy holds whole sub-chunks, at most one per group warp");
constexpr int kStatsSmem = kSlots * (kCopyBytes + 2 * 8 + 4);
constexpr int kDrawWarps = 8;
constexpr uint64_t kAcceptWait = 400000000ull;  // clock cycles, ~0.2 s

template <typename T>
struct AcceptDev {
  int B, N, K, V, C, RU;
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
  double* csum;        // [B][RU][C] sub-chunk sum of exp(l - sub-chunk max)
  float* cmax;         // [B][RU][C] sub-chunk max
  int32_t* cidx;       // [B][RU][C] first index of the sub-chunk max
  double* rsum;        // [B][K] row normaliser s
  float* rmax;         // [B][K] row max m
  double* resid;       // [B][C] residual sub-chunk mass
  int32_t* decision;   // [B][4]: valid, rejected, a, n
  int32_t* count;      // [B] residual sub-chunks finished
  int argmax;          // drafts are argmax q (point-mass proposals)
};

// Loads elements [idx, idx+8) of a row; out-of-range ones read as -inf.
template <typename T, bool kVec>
ISD_DEV void load_row8(const T* row, int idx, int hi, float (&v)[8]) {
  if (kVec && idx + 8 <= hi) {
    load8_stream(row + idx, v);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      v[k] = (idx + k < hi) ? to_f(row[idx + k]) : -INFINITY;
  }
}

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
  load_row8<float, kVec>(row, idx, hi, r.v);
  return r;
}

// 8 consecutive elements from shared memory (16-byte aligned).
ISD_DEV void lds8(const __nv_bfloat16* s, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(s);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
ISD_DEV void lds8(const float* s, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(s);
  const float4 b = *(reinterpret_cast<const float4*>(s) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
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

// Bounded mbarrier wait: false once ~0.2 s have passed without the phase.
ISD_DEV bool wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if ((uint64_t)(clock64() - t0) > kAcceptWait) return false;
  return true;
}

// Bulk asynchronous copy global -> shared (TMA engine), completion counted
// in bytes on `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.
ISD_DEV void bulk_load(void* dst, const void* src, uint32_t bytes,
                       uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
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
// Sub-chunk figures.  Lane l holds elements lo + (k*32 + l)*8 + e (k, e < 8)
// of the sub-chunk, -inf past the row end.  Lane 0 stores the max, the sum
// of exp(l - max) (8 terms in fp32, then fp64) and the first index of the
// max (exact compares of the same values).
template <typename T>
ISD_DEV void finish_sub(const AcceptDev<T>& p, size_t o, int lo,
                        const float (&v)[8][8]) {
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < 8; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, v[k][e]);
  m = warp_max(m);
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float t = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) t += ex2((v[k][e] - m) * kLog2e);
    s += (double)t;
  }
  s = warp_sum_f64(s);
  if (p.argmax) {
    int first = INT_MAX;
#pragma unroll
    for (int k = 7; k >= 0; --k)
#pragma unroll
      for (int e = 7; e >= 0; --e)
        if (v[k][e] == m) first = lo + (k * 32 + lane) * 8 + e;
    first = warp_min_int(first);
    if (lane == 0) p.cidx[o] = first;
  }
  if (lane == 0) {
    p.cmax[o] = m;
    p.csum[o] = s;
  }
}

// Copies are numbered it = (b * RU + j) * CC + cc (chunk cc of row j of
// sequence b, CC chunks of S sub-chunks per row); sub-chunk c = cc * S + i
// lands in slot `it`'s i-th kSub elements and its figures at
// (b * RU + j) * C + c.
template <typename T>
__global__ void __launch_bounds__(kStatsThreads, 1)
    accept_stats_kernel(AcceptDev<T> p) {
  constexpr int S = kCopyBytes / (kSub * (int)sizeof(T));  // sub-chunks/copy
  constexpr int kSlotElems = kCopyBytes / (int)sizeof(T);
  extern __shared__ __align__(128) unsigned char smem[];
  T* ring = reinterpret_cast<T*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kSlots * kCopyBytes);
  uint64_t* empty = full + kSlots;
  int* item = reinterpret_cast<int*>(empty + kSlots);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CC = (p.C + S - 1) / S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGroupWarps);
    }
    fence_barrier_init();
  }
  grid_dep_wait();
  __syncthreads();

  if (warp == kConsumers) {
    // Producers: lanes 0..kIssuers-1 look at kIssuers candidate copies at a
    // time (this CTA's are blockIdx.x + k * gridDim.x) and each lane whose
    // copy is of a row in use issues it.  Production q goes to slot
    // q % kSlots and to consumer group q % kGroups; after the copies comes
    // one end marker per group.
    if (lane >= kIssuers) return;
    const int total = p.B * p.RU * CC;
    bool failed = false;
    int q0 = 0;
    for (int first = blockIdx.x; first < total;
         first += kIssuers * gridDim.x) {
      const int it = first + lane * gridDim.x;
      int b = 0, j = 0, cc = 0;
      bool use = it < total;
      if (use) {
        cc = it % CC;
        const int bj = it / CC;
        j = bj % p.RU;
        b = bj / p.RU;
        use = state_ok(p, b) && j < p.n_in[b] + p.N - 1;
      }
      const uint32_t vote = __ballot_sync(kIssuerMask, use);
      const int q = q0 + __popc(vote & ((1u << lane) - 1u));
      q0 += __popc(vote);
      if (use) {
        const int s = q % kSlots;
        if (q >= kSlots && !wait_bounded(&empty[s], ((q / kSlots) - 1) & 1)) {
          failed = true;
        } else {
          const int lo = cc * S * kSub;
          const uint32_t bytes =
              (uint32_t)(min(S * kSub, p.V - lo) * (int)sizeof(T));
          item[s] = it;
          mbar_arrive_expect_tx(&full[s], bytes);
          bulk_load(ring + (size_t)s * kSlotElems,
                    p.lc + ((size_t)b * p.K + j) * p.V + lo, bytes, &full[s]);
        }
      }
      if (__any_sync(kIssuerMask, failed)) {
        failed = true;
        break;
      }
    }
    // End markers, one per consumer group, kIssuers at a time.
    for (int m = 0; m < kGroups && !failed; m += kIssuers) {
      const int q = q0 + lane, s = q % kSlots;
      if (m + lane < kGroups) {
        if (q >= kSlots && !wait_bounded(&empty[s], ((q / kSlots) - 1) & 1)) {
          failed = true;
        } else {
          item[s] = -1;
          mbar_arrive(&full[s]);
        }
      }
      failed = __any_sync(kIssuerMask, failed);
      if (!failed) q0 += min(kIssuers, kGroups - m);
    }
    if (lane == 0) {
      if (failed) report(p.status, ISD_ERR_CUDA);
      // Copies still in flight land before the CTA's shared memory goes
      // away (after a failure a slot may never fill: the wait is bounded).
      for (int k = max(0, q0 - kSlots); k < q0; ++k)
        if (!wait_bounded(&full[k % kSlots], (k / kSlots) & 1)) break;
    }
    return;
  }

  const int g = warp / kGroupWarps, i = warp % kGroupWarps;
  for (int t = 0;; ++t) {
    const int q = g + t * kGroups, s = q % kSlots;
    if (!wait_bounded(&full[s], (q / kSlots) & 1)) {
      if (lane == 0) report(p.status, ISD_ERR_CUDA);
      break;
    }
    const int it = item[s];
    const int c = it < 0 ? p.C : (it % CC) * S + i;
    if (i >= S || c >= p.C) {  // end marker, or no sub-chunk for this warp
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (it < 0) break;
      continue;
    }
    const int lo = c * kSub, n_el = min(kSub, p.V - lo);
    const T* src = ring + (size_t)s * kSlotElems + i * kSub;
    // Lane l reads elements (k*32 + l)*8 + e (k, e < 8) of the sub-chunk,
    // -inf past the row end; the slot is read once per pass, nothing kept.
    auto group = [&](int k, float (&v)[8]) {
      const int e0 = (k * 32 + lane) * 8;
      if (e0 + 8 <= n_el) {
        lds8(src + e0, v);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          v[e] = e0 + e < n_el ? to_f(src[e0 + e]) : -INFINITY;
      }
    };
    float mk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      group(k, v);
      mk[k] = fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])),
                    fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7])));
    }
    float m = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])),
                    fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7])));
    m = warp_max(m);
    double sum = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      group(k, v);
      float t8 = 0.0f;  // 8 terms in fp32, then fp64 across groups
#pragma unroll
      for (int e = 0; e < 8; ++e) t8 += ex2((v[e] - m) * kLog2e);
      sum += (double)t8;
    }
    int first = INT_MAX;
    if (p.argmax) {  // first index of the max (exact compares)
#pragma unroll
      for (int k = 7; k >= 0; --k) {
        float v[8];
        group(k, v);
#pragma unroll
        for (int e = 7; e >= 0; --e)
          if (v[e] == m) first = lo + (k * 32 + lane) * 8 + e;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp no longer reads it
    sum = warp_sum_f64(sum);
    const size_t o = (size_t)(it / CC) * p.C + c;
    if (p.argmax) {
      first = warp_min_int(first);
      if (lane == 0) p.cidx[o] = first;
    }
    if (lane == 0) {
      p.cmax[o] = m;
      p.csum[o] = sum;
    }
  }
}

// Same items, element order and arithmetic, read with plain loads.
template <typename T>
__global__ void __launch_bounds__(256) accept_stats_plain_kernel(AcceptDev<T> p) {
  const int lane = threadIdx.x & 31;
  grid_dep_wait();
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int total = p.B * p.RU * p.C;
  for (int it = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       it < total; it += warps) {
    const int c = it % p.C, bj = it / p.C, j = bj % p.RU, b = bj / p.RU;
    if (!state_ok(p, b) || j >= p.n_in[b] + p.N - 1) continue;
    const T* row = p.lc + ((size_t)b * p.K + j) * p.V;
    const int lo = c * kSub, hi = min(p.V, lo + kSub);
    float v[8][8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      load_row8<T, false>(row, lo + (k * 32 + lane) * 8, hi, v[k]);
    finish_sub(p, (size_t)it, lo, v);
  }
}

// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(1024) accept_decide_kernel(AcceptDev<T> p) {
  __shared__ float s_m[32];
  __shared__ double s_s[32];
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, K = p.K;
  grid_dep_wait();
  const int n = p.n_in[b];
  const int L = p.seq_len[b];
  const int tok = lane < N ? p.pending_in[b * N + lane] : 0;
  bool ok = (n == 1 || n == N) && L >= 0;
  if (ok && lane < n) ok = tok >= 0 && tok < p.V;
  int qr = 0;
  if (ok && lane >= 1 && lane < n) {
    qr = p.q_row_in[b * N + lane];
    ok = qr >= 0 && qr < K;
  }
  ok = __all_sync(0xffffffffu, ok);  // every warp reaches the same verdict
  int32_t* dec = p.decision + b * 4;
  if (!ok) {
    if (warp != 0) return;
    if (lane == 0) {
      report(p.status, ISD_ERR_BAD_STATE);
      p.n_commit[b] = 0;
      p.n_out[b] = n;
      p.count[b] = 0;
      dec[0] = 0; dec[1] = 0; dec[2] = -1; dec[3] = n;
    }
    if (lane < N) {
      p.commit_tokens[b * N + lane] = -1;
      p.pending_out[b * N + lane] = p.pending_in[b * N + lane];
      p.q_row_out[b * N + lane] = p.q_row_in[b * N + lane];
      p.q_stats_out[(b * N + lane) * 2] = p.q_stats_in[(b * N + lane) * 2];
      p.q_stats_out[(b * N + lane) * 2 + 1] =
          p.q_stats_in[(b * N + lane) * 2 + 1];
    }
    return;
  }
  // Warp 0 fetches the logits at the drafts first, so that their latency
  // overlaps the merge.
  const bool verifies = warp == 0 && lane >= 1 && lane < n;
  float lx = 0.0f, lqx = 0.0f, zhi = 0.0f, zlo = 0.0f;
  if (verifies) {
    lx = to_f(p.lc[((size_t)b * K + lane - 1) * p.V + tok]);
    if (!p.argmax) {
      zhi = p.q_stats_in[(b * N + lane) * 2];
      zlo = p.q_stats_in[(b * N + lane) * 2 + 1];
      lqx = to_f(p.lp[((size_t)b * K + qr) * p.V + tok]);
    }
  }
  // Row statistics: warp j merges the sub-chunks of row j.
  const int rows_used = n + N - 1;
  if (warp < rows_used) {
    const size_t o = ((size_t)b * p.RU + warp) * p.C;
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
    for (int i = 0; i < kSubPerLane; ++i)
      if (lane * kSubPerLane + i < p.C) s += cs[i] * exp((double)(cm[i] - m));
    s = warp_sum_f64(s);
    if (lane == 0) {
      s_m[warp] = m;
      s_s[warp] = s;
      p.rmax[b * K + warp] = m;
      p.rsum[b * K + warp] = s;
      if (p.row_stats_out) {
        p.row_stats_out[(b * K + warp) * 2] = m;
        p.row_stats_out[(b * K + warp) * 2 + 1] = (float)s;
      }
    }
  }
  __syncthreads();
  if (warp != 0) return;
  // Ratio test of drafts 1..n-1: lane i verifies draft i with row i-1.
  // l - m is exact in fp32 (both are logits); p, q and the ratio in fp64.
  bool acc = true;
  if (verifies) {
    const double px = exp((double)(lx - s_m[lane - 1])) / s_s[lane - 1];
    double qx = 1.0;      // argmax drafts: the proposal is a point mass
    if (!p.argmax) qx = exp(((double)lqx - (double)zhi) - (double)zlo);
    const double r = qx > 0.0 ? px / qx : INFINITY;
    const float u = uniform(p.seed, (uint32_t)b, step_of(p),
                            (uint32_t)(L + lane), ISD_STREAM_ACCEPT);
    acc = (double)u < r;
    if (p.ratio_out) p.ratio_out[b * N + lane] = (float)r;
  }
  const uint32_t mask = __ballot_sync(0xffffffffu, acc);
  const uint32_t drafts = ((n >= 32) ? 0xffffffffu : ((1u << n) - 1u)) & ~1u;
  const uint32_t rej = drafts & ~mask;
  const bool rejected = rej != 0u;
  const int a = rejected ? (__ffs(rej) - 2) : (n - 1);
  if (lane < N) {
    p.commit_tokens[b * N + lane] = lane <= a ? tok : -1;
    // Next drafts' q rows and the log-normaliser log sum_v exp(l_v) of
    // each (lane j: row n + j - 1), stored as a float pair hi + lo.
    const bool has = !rejected && lane >= 1;
    const int src = n + lane - 1;
    p.q_row_out[b * N + lane] = has ? src : -1;
    const double lz = has ? (double)s_m[src] + log(s_s[src]) : 0.0;
    const float lz_hi = (float)lz;
    p.q_stats_out[(b * N + lane) * 2] = lz_hi;
    p.q_stats_out[(b * N + lane) * 2 + 1] = (float)(lz - (double)lz_hi);
    // After a rejection only the replacement is pending.
    if (rejected && lane >= 1) p.pending_out[b * N + lane] = -1;
  }
  if (lane == 0) {
    p.n_commit[b] = a + 1;
    p.n_out[b] = rejected ? 1 : N;
    p.count[b] = 0;
    dec[0] = 1; dec[1] = rejected ? 1 : 0; dec[2] = a; dec[3] = n;
  }
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

template <typename T>
ISD_DEV ResidRows resid_rows(const AcceptDev<T>& p, int b, int a,
                             const T*& prow, const T*& qrow) {
  const int N = p.N, K = p.K;
  prow = p.lc + ((size_t)b * K + a) * p.V;
  ResidRows r;
  r.mp = p.rmax[b * K + a];
  const double sp = p.rsum[b * K + a];
  r.inv_sp = (float)(1.0 / sp);
  if (p.argmax) {
    qrow = prow;                       // not read
    r.zq_hi = r.zq_lo = r.c_hi = r.c_lo = 0.0f;
    r.x = p.pending_in[b * N + a + 1];
  } else {
    const int qr = p.q_row_in[b * N + a + 1];
    qrow = p.lp + ((size_t)b * K + qr) * p.V;
    r.zq_hi = p.q_stats_in[(b * N + a + 1) * 2];
    r.zq_lo = p.q_stats_in[(b * N + a + 1) * 2 + 1];
    const double c = ((double)r.mp + log(sp)) - ((double)r.zq_hi + (double)r.zq_lo);
    r.c_hi = (float)c;
    r.c_lo = (float)(c - (double)r.c_hi);
    r.x = -1;
  }
  return r;
}

// One inverse-CDF draw by a warp: the smallest index whose running mass
// (ascending order) exceeds u * total.  mode 0: the residual of sequence b
// (rr, prow, qrow; sub-chunk masses from `resid`, written in this kernel);
// mode 1: row `row` of logits_cur with its statistics.  Returns the token
// on every lane.
template <typename T, bool kVec>
ISD_DEV int warp_draw(const AcceptDev<T>& p, int b, int mode, int row,
                      const ResidRows& rr, const T* prow, const T* qrow,
                      float u) {
  const int lane = threadIdx.x & 31, C = p.C;
  const float m_row = mode ? p.rmax[b * p.K + row] : 0.0f;
  const size_t o = ((size_t)b * p.RU + row) * C;
  // 1. The sub-chunk: lane l owns sub-chunks 4l .. 4l+3.
  double mc[kSubPerLane];
  double own = 0.0;
#pragma unroll
  for (int i = 0; i < kSubPerLane; ++i) {
    const int c = lane * kSubPerLane + i;
    mc[i] = 0.0;
    if (c < C)
      mc[i] = mode == 0 ? __ldcg(&p.resid[(size_t)b * C + c])
                        : p.csum[o + c] * exp((double)(p.cmax[o + c] - m_row));
    own += mc[i];
  }
  double excl;
  const double incl = warp_scan_f64(own, excl);
  const double target = (double)u * __shfl_sync(0xffffffffu, incl, 31);
  const uint32_t hit = __ballot_sync(0xffffffffu, incl > target);
  const uint32_t pos = __ballot_sync(0xffffffffu, own > 0.0);
  // Rounding can leave the target past every running sum: then the last
  // sub-chunk with positive mass, scanned to its last positive entry.
  const int hl = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
  int chosen = -1;
  double rem = INFINITY;
  if (lane == hl) {
    double run = excl;
    int lastpos = lane * kSubPerLane;
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
    if (chosen < 0) chosen = lastpos;
  }
  chosen = __shfl_sync(0xffffffffu, chosen, hl);
  rem = __shfl_sync(0xffffffffu, rem, hl);
  // 2. Inside the sub-chunk, four rounds of 512 elements: in round r lane l
  //    owns elements lo + 512r + 16l .. +15, so the scan stays ascending.
  //    Round r + 1 is loaded while round r is scanned.
  const int lo = chosen * kSub, hi = min(p.V, lo + kSub);
  const bool with_q = mode == 0 && rr.x < 0;
  Raw8<T> cp[2], cq[2], np[2], nq[2];
  auto load_round = [&](int r, Raw8<T> (&rp)[2], Raw8<T> (&rq)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int idx = lo + r * 512 + lane * 16 + h * 8;
      rp[h] = load_raw8<kVec>(prow, idx, hi);
      if (with_q) rq[h] = load_raw8<kVec>(qrow, idx, hi);
    }
  };
  load_round(0, cp, cq);
  int tok = -1, lastp = -1;
  bool found = false;
#pragma unroll 1
  for (int r = 0; r < 4 && !found; ++r) {
    if (r < 3) load_round(r + 1, np, nq);
    const int base = lo + r * 512 + lane * 16;
    // Element weights are recomputed for the walk (the same operations, so
    // the same values) rather than kept.
    auto weight = [&](int h, int e) {
      return mode == 0
                 ? resid_w(rr, cp[h].at(e), with_q ? cq[h].at(e) : 0.0f,
                           base + h * 8 + e)
                 : ex2((cp[h].at(e) - m_row) * kLog2e);
    };
    double lt = 0.0;
    int lastr = -1;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float w = weight(h, e);
        lt += (double)w;
        if (w > 0.0f) lastr = base + h * 8 + e;
      }
    if (lastr >= 0) lastp = lastr;
    double ex;
    const double inc = warp_scan_f64(lt, ex);
    const double tot = __shfl_sync(0xffffffffu, inc, 31);
    if (rem < tot) {  // the same verdict on every lane
      const int hl2 = __ffs(__ballot_sync(0xffffffffu, inc > rem)) - 1;
      if (lane == hl2) {
        double run = ex;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            run += (double)weight(h, e);
            if (tok < 0 && run > rem) tok = base + h * 8 + e;
          }
        if (tok < 0) tok = lastr;  // rounding: this lane's last positive
      }
      tok = __shfl_sync(0xffffffffu, tok, hl2);
      found = true;
    }
    rem -= tot;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cp[h] = np[h];
      cq[h] = nq[h];
    }
  }
  // Rounding left the target past every running sum: the last positive
  // entry of the sub-chunk.
  if (tok < 0) {
    const int lp = warp_max_int(lastp);
    tok = lp >= 0 ? lp : lo;
  }
  return tok;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kDrawWarps * 32,
                                  sizeof(T) == 2 && kVec ? 2 : 1)
    accept_draw_kernel(AcceptDev<T> p) {
  // blockIdx.x is the sequence, so that the first block of every sequence
  // (its draws, or its first residual sub-chunks) is scheduled first.
  const int b = blockIdx.x, lane = threadIdx.x & 31;
  const int wi = blockIdx.y * kDrawWarps + (threadIdx.x >> 5);
  grid_dep_wait();
  const int32_t* dec = p.decision + b * 4;
  if (dec[0] == 0) return;  // malformed state: decide copied it through
  const bool rejected = dec[1] != 0;
  const int a = dec[2], n = dec[3];
  const int N = p.N, K = p.K;
  const int L = p.seq_len[b];
  // What this warp draws, if anything: mode 0 the residual, 1 a row of p/q.
  int mode, row, slot;
  float u;
  ResidRows rr{};
  const T* prow = nullptr;
  const T* qrow = nullptr;
  if (rejected) {
    if (wi >= p.C) return;
    rr = resid_rows(p, b, a, prow, qrow);
    const int lo = wi * kSub, hi = min(p.V, lo + kSub);
    // Argmax drafts read no q row (the q row pointer is p's, never used).
    const T* qsrc = rr.x < 0 ? qrow : prow;
    Raw8<T> vp[8], vq[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      vp[k] = load_raw8<kVec>(prow, lo + (k * 32 + lane) * 8, hi);
    if (rr.x < 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        vq[k] = load_raw8<kVec>(qsrc, lo + (k * 32 + lane) * 8, hi);
    }
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int idx = lo + (k * 32 + lane) * 8;
      float t = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        t += resid_w(rr, vp[k].at(e), rr.x < 0 ? vq[k].at(e) : 0.0f, idx + e);
      s += (double)t;
    }
    s = warp_sum_f64(s);
    int last = 0;
    if (lane == 0) {
      p.resid[(size_t)b * p.C + wi] = s;
      __threadfence();
      last = atomicAdd(&p.count[b], 1) == p.C - 1;
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    // Last sub-chunk of this sequence: every resid[b][*] is written.
    __threadfence();
    double W = 0.0;
#pragma unroll
    for (int i = 0; i < kSubPerLane; ++i) {
      const int c = lane * kSubPerLane + i;
      if (c < p.C) W += __ldcg(&p.resid[(size_t)b * p.C + c]);
    }
    W = warp_sum_f64(W);
    // Zero residual mass (p == q up to rounding): draw from p instead.
    mode = W > 0.0 ? 0 : 1;
    row = a;
    slot = 0;
    u = uniform(p.seed, (uint32_t)b, step_of(p), (uint32_t)(L + a + 1),
                ISD_STREAM_RESAMPLE);
  } else {
    if (wi >= N) return;
    slot = wi;                  // 0: the bonus; >= 1: drafts
    row = n + wi - 1;
    prow = p.lc + ((size_t)b * K + row) * p.V;
    if (p.argmax && wi >= 1) {
      // Argmax draft: the first sub-chunk whose max is the row max holds
      // the first maximal index (exact compares of the same values).
      const size_t o = ((size_t)b * p.RU + row) * p.C;
      const float m = p.rmax[b * K + row];
      int first = INT_MAX;
#pragma unroll
      for (int i = kSubPerLane - 1; i >= 0; --i) {
        const int c = lane * kSubPerLane + i;
        if (c < p.C && p.cmax[o + c] == m) first = c;
      }
      first = warp_min_int(first);
      if (lane == 0) p.pending_out[b * N + wi] = first < p.C ? p.cidx[o + first] : -1;
      return;
    }
    mode = 1;
    u = uniform(p.seed, (uint32_t)b, step_of(p), (uint32_t)(L + n + wi),
                wi == 0 ? ISD_STREAM_RESAMPLE : ISD_STREAM_DRAFT);
  }
  const int tok = warp_draw<T, kVec>(p, b, mode, row, rr, prow, qrow, u);
  if (lane == 0) p.pending_out[b * N + slot] = tok;
}

// ---------------------------------------------------------------------------
// Host-side launcher (called from the C ABI after validation).

struct AcceptLayout {
  size_t csum, cmax, cidx, rsum, rmax, resid, decision, count, total;
};

static AcceptLayout accept_layout(int B, int N, int K, int V) {
  const size_t C = (V + kSub - 1) / kSub;
  const size_t RU = 2 * N - 1;
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
  l.rsum = take((size_t)B * K * 8);
  l.rmax = take((size_t)B * K * 4);
  l.resid = take((size_t)B * C * 8);
  l.decision = take((size_t)B * 4 * 4);
  l.count = take((size_t)B * 4);
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

template <typename T>
static int launch_accept_t(const isd_accept_args* a, cudaStream_t st) {
  AcceptDev<T> p;
  p.B = a->B; p.N = a->N; p.K = a->K; p.V = a->V;
  p.C = (a->V + kSub - 1) / kSub;
  p.RU = 2 * a->N - 1;
  if (p.C > kMaxSub) return ISD_ERR_UNSUPPORTED;
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
  p.rsum = reinterpret_cast<double*>(ws + l.rsum);
  p.rmax = reinterpret_cast<float*>(ws + l.rmax);
  p.resid = reinterpret_cast<double*>(ws + l.resid);
  p.decision = reinterpret_cast<int32_t*>(ws + l.decision);
  p.count = reinterpret_cast<int32_t*>(ws + l.count);
  p.argmax = a->proposal == ISD_PROPOSAL_ARGMAX;

  const int sms = num_sms();
  if (sms <= 0) return ISD_ERR_CUDA;
  const long long items = (long long)p.B * p.RU * p.C;
  // Bulk copies need 16-byte aligned rows (logits_cur itself is checked on
  // the host) and whole 16-byte multiples.
  if (((size_t)a->V * sizeof(T)) % 16 == 0) {
    auto kern = accept_stats_kernel<T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStatsSmem) != cudaSuccess)
      return ISD_ERR_CUDA;
    const int S = kCopyBytes / (kSub * (int)sizeof(T));
    const long long copies = (long long)p.B * p.RU * ((p.C + S - 1) / S);
    const int grid = (int)std::min<long long>(sms, copies);
    if (launch_pdl(kern, dim3(grid), dim3(kStatsThreads), kStatsSmem, st, p) !=
        cudaSuccess)
      return ISD_ERR_CUDA;
  } else {
    const int grid = (int)std::min<long long>(8LL * sms, (items + 7) / 8);
    if (launch_pdl(accept_stats_plain_kernel<T>, dim3(grid), dim3(256), 0, st,
                   p) != cudaSuccess)
      return ISD_ERR_CUDA;
  }
  if (launch_pdl(accept_decide_kernel<T>, dim3(p.B), dim3(32 * p.RU), 0, st,
                 p) != cudaSuccess)
    return ISD_ERR_CUDA;
  const dim3 g_draw(p.B, (std::max(p.C, p.N) + kDrawWarps - 1) / kDrawWarps);
  const cudaError_t e =
      (a->V % 8) == 0
          ? launch_pdl(accept_draw_kernel<T, true>, g_draw,
                       dim3(kDrawWarps * 32), 0, st, p)
          : launch_pdl(accept_draw_kernel<T, false>, g_draw,
                       dim3(kDrawWarps * 32), 0, st, p);
  return e == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

size_t accept_workspace_bytes(int B, int N, int K, int V) {
  return accept_layout(B, N, K, V).total;
}

int launch_accept(const isd_accept_args* a, cudaStream_t st) {
  if (a->dtype == ISD_BF16) return launch_accept_t<__nv_bfloat16>(a, st);
  return launch_accept_t<float>(a, st);
}

}  // namespace isd
