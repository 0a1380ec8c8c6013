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
// Four kernels, one stream, no inter-CTA waiting:
//   stats     grid (C, 2N-1, B): per 8192-element chunk of each used row,
//             chunk max and sum of exp(l - chunk max)            [HBM bound]
//   decide    one warp per sequence: merge chunk stats into row (m, s),
//             ratio tests, ballot for the first rejection, next state
//   residual  grid (C, B), rejected sequences only: chunk sums of
//             max(0, p - q)                                       [HBM bound]
//   sample    grid (N, B): chunk located from the chunk masses, then a
//             block-wide ordered scan inside the chunk
// Element masses are fp32 (MUFU exp2 of exactly formed differences); every
// sum that places a sampling boundary or normalises a probability is
// accumulated in fp64 in a fixed order, so draws agree with an fp64
// reference except within a few 1e-8 of a boundary, and every run is
// bitwise reproducible.
#include "common.cuh"

namespace isd {

constexpr int kChunk = 8192;             // vocabulary elements per chunk
constexpr int kAThreads = 256;           // threads per stats/sample CTA
constexpr int kRound = kAThreads * 8;    // elements per round (8 per thread)
constexpr int kRounds = kChunk / kRound; // 4

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
  double* csum;        // [B][RU][C] chunk sum of exp(l - chunk max)
  double* rsum;        // [B][K] row normaliser s
  double* resid;       // [B][C] residual chunk mass
  float* cmax;         // [B][RU][C] chunk max
  float* rmax;         // [B][K] row max m
  int32_t* decision;   // [B][4]: valid, rejected, a, n
  int32_t* cidx;       // [B][RU][C] first index of the chunk max (argmax)
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
template <typename T, bool kVec>
__global__ void __launch_bounds__(kAThreads)
    accept_stats_kernel(AcceptDev<T> p) {
  __shared__ float red[32];
  __shared__ double redd[32];
  const int c = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  if (!state_ok(p, b)) return;
  if (j >= p.n_in[b] + p.N - 1) return;
  const T* row = p.lc + ((size_t)b * p.K + j) * p.V;
  const int lo = c * kChunk, hi = min(p.V, lo + kChunk);
  float v[kRounds][8];
#pragma unroll
  for (int r = 0; r < kRounds; ++r)
    load_row8<T, kVec>(row, lo + (r * kAThreads + threadIdx.x) * 8, hi, v[r]);
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < kRounds; ++r)
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, v[r][k]);
  m = block_reduce<true>(m, red);
  double s = 0.0;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    float t = 0.0f;  // 8 terms in fp32, then fp64 across groups
#pragma unroll
    for (int k = 0; k < 8; ++k) t += ex2((v[r][k] - m) * kLog2e);
    s += (double)t;
  }
  s = block_sum(s, redd);
  const size_t o = ((size_t)b * p.RU + j) * p.C + c;
  if (p.argmax) {
    // First index of the chunk max (exact compare of the same values).
    int first = INT_MAX;
#pragma unroll
    for (int r = kRounds - 1; r >= 0; --r)
#pragma unroll
      for (int k = 7; k >= 0; --k)
        if (v[r][k] == m) first = lo + (r * kAThreads + threadIdx.x) * 8 + k;
    first = block_min_int(first, reinterpret_cast<int*>(red));
    if (threadIdx.x == 0) p.cidx[o] = first;
  }
  if (threadIdx.x == 0) {
    p.cmax[o] = m;
    p.csum[o] = s;
  }
}

// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) accept_decide_kernel(AcceptDev<T> p) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (b >= p.B) return;
  const int N = p.N, K = p.K;
  const int n = p.n_in[b];
  const int L = p.seq_len[b];
  const int tok = lane < N ? p.pending_in[b * N + lane] : 0;
  bool ok = (n == 1 || n == N) && L >= 0;
  if (ok && lane < n) ok = tok >= 0 && tok < p.V;
  if (ok && lane >= 1 && lane < n) {
    const int qr = p.q_row_in[b * N + lane];
    ok = qr >= 0 && qr < K;
  }
  ok = __all_sync(0xffffffffu, ok);
  int32_t* dec = p.decision + b * 4;
  if (!ok) {
    if (lane == 0) {
      if (p.status) *p.status = ISD_ERR_BAD_STATE;
      p.n_commit[b] = 0;
      p.n_out[b] = n;
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
  // Row statistics: lane l merges the chunks of row l in a fixed order.
  const int rows_used = n + N - 1;
  float m = 0.0f;
  double s = 1.0;
  if (lane < rows_used) {
    const size_t o = ((size_t)b * p.RU + lane) * p.C;
    m = -INFINITY;
    for (int c = 0; c < p.C; ++c) m = fmaxf(m, p.cmax[o + c]);
    s = 0.0;
    for (int c = 0; c < p.C; ++c)
      s += p.csum[o + c] * exp((double)(p.cmax[o + c] - m));
    p.rmax[b * K + lane] = m;
    p.rsum[b * K + lane] = s;
    if (p.row_stats_out) {
      p.row_stats_out[(b * K + lane) * 2] = m;
      p.row_stats_out[(b * K + lane) * 2 + 1] = (float)s;
    }
  }
  // Ratio test of drafts 1..n-1: lane i verifies draft i with row i-1.
  // l - m is exact in fp32 (both are logits); p, q and the ratio in fp64.
  const float m_prev = __shfl_up_sync(0xffffffffu, m, 1);
  const double s_prev = __shfl_up_sync(0xffffffffu, s, 1);
  bool acc = true;
  if (lane >= 1 && lane < n) {
    const float lx = to_f(p.lc[((size_t)b * K + lane - 1) * p.V + tok]);
    const double px = exp((double)(lx - m_prev)) / s_prev;
    double qx = 1.0;      // argmax drafts: the proposal is a point mass
    if (!p.argmax) {
      const int qr = p.q_row_in[b * N + lane];
      const float mq = p.q_stats_in[(b * N + lane) * 2];
      const float sq = p.q_stats_in[(b * N + lane) * 2 + 1];
      const float lqx = to_f(p.lp[((size_t)b * K + qr) * p.V + tok]);
      qx = exp((double)(lqx - mq)) / (double)sq;
    }
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
  if (lane < N) p.commit_tokens[b * N + lane] = lane <= a ? tok : -1;
  // Next drafts' q rows and their statistics (lane j reads row n + j - 1).
  const int src = min(n + lane - 1, 31);
  const float mq_next = __shfl_sync(0xffffffffu, m, src);
  const double sq_next = __shfl_sync(0xffffffffu, s, src);
  if (lane < N) {
    const bool has = !rejected && lane >= 1;
    p.q_row_out[b * N + lane] = has ? n + lane - 1 : -1;
    p.q_stats_out[(b * N + lane) * 2] = has ? mq_next : 0.0f;
    p.q_stats_out[(b * N + lane) * 2 + 1] = has ? (float)sq_next : 0.0f;
  }
  if (lane == 0) {
    p.n_commit[b] = a + 1;
    p.n_out[b] = rejected ? 1 : N;
    dec[0] = 1; dec[1] = rejected ? 1 : 0; dec[2] = a; dec[3] = n;
  }
}

// ---------------------------------------------------------------------------
// Residual element weight max(0, p - q), shared by the chunk sums and the
// in-chunk scan so both see the same per-element values.
// With argmax drafts q is a point mass at the rejected draft x, so the
// residual is p without x.
struct ResidRows {
  float mp, inv_sp, mq, inv_sq;
  int x;          // rejected draft (argmax proposals), else -1
};
ISD_DEV float resid_w(const ResidRows& r, float lpv, float lqv, int v) {
  if (r.x >= 0) return v == r.x ? 0.0f : ex2((lpv - r.mp) * kLog2e) * r.inv_sp;
  return fmaxf(0.0f, ex2((lpv - r.mp) * kLog2e) * r.inv_sp -
                         ex2((lqv - r.mq) * kLog2e) * r.inv_sq);
}

template <typename T>
ISD_DEV ResidRows resid_rows(const AcceptDev<T>& p, int b, int a,
                             const T*& prow, const T*& qrow) {
  const int N = p.N, K = p.K;
  prow = p.lc + ((size_t)b * K + a) * p.V;
  ResidRows r;
  r.mp = p.rmax[b * K + a];
  r.inv_sp = (float)(1.0 / p.rsum[b * K + a]);
  if (p.argmax) {
    qrow = prow;                       // not read
    r.mq = 0.0f; r.inv_sq = 0.0f;
    r.x = p.pending_in[b * N + a + 1];
  } else {
    const int qr = p.q_row_in[b * N + a + 1];
    qrow = p.lp + ((size_t)b * K + qr) * p.V;
    r.mq = p.q_stats_in[(b * N + a + 1) * 2];
    r.inv_sq = 1.0f / p.q_stats_in[(b * N + a + 1) * 2 + 1];
    r.x = -1;
  }
  return r;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kAThreads)
    accept_residual_kernel(AcceptDev<T> p) {
  __shared__ double redd[32];
  const int c = blockIdx.x, b = blockIdx.y;
  const int32_t* dec = p.decision + b * 4;
  if (dec[0] == 0 || dec[1] == 0) return;
  const T *prow, *qrow;
  const ResidRows rr = resid_rows(p, b, dec[2], prow, qrow);
  const int lo = c * kChunk, hi = min(p.V, lo + kChunk);
  double s = 0.0;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int idx = lo + (r * kAThreads + threadIdx.x) * 8;
    float vp[8], vq[8];
    load_row8<T, kVec>(prow, idx, hi, vp);
    if (rr.x < 0) load_row8<T, kVec>(qrow, idx, hi, vq);
    float t = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += resid_w(rr, vp[k], vq[k], idx + k);
    s += (double)t;
  }
  s = block_sum(s, redd);
  if (threadIdx.x == 0) p.resid[(size_t)b * p.C + c] = s;
}

// ---------------------------------------------------------------------------
template <typename T, bool kVec>
__global__ void __launch_bounds__(kAThreads)
    accept_sample_kernel(AcceptDev<T> p) {
  __shared__ double sh[32];
  __shared__ int s_chunk, s_found, s_last;
  __shared__ double s_target;
  const int t = blockIdx.x, b = blockIdx.y;
  const int N = p.N, K = p.K;
  const int32_t* dec = p.decision + b * 4;
  if (dec[0] == 0) return;  // malformed state: decide copied it through
  const bool rejected = dec[1] != 0;
  const int a = dec[2], n = dec[3];
  const int L = p.seq_len[b];
  if (t >= 1 && rejected) {
    if (threadIdx.x == 0) p.pending_out[b * N + t] = -1;
    return;
  }
  // What is drawn: 0 = residual, 1 = p/q row with row statistics.
  int mode, row;
  uint32_t pos, stream;
  if (t == 0 && rejected) {
    mode = 0; row = a; pos = L + a + 1; stream = ISD_STREAM_RESAMPLE;
  } else if (t == 0) {
    mode = 1; row = n - 1; pos = L + n; stream = ISD_STREAM_RESAMPLE;
  } else {
    mode = 1; row = n + t - 1; pos = L + n + t; stream = ISD_STREAM_DRAFT;
  }
  const int C = p.C;
  if (p.argmax && t >= 1) {
    // Argmax draft: the first chunk whose max is the row max holds the
    // first maximal index (exact compares of the same values).
    if (threadIdx.x == 0) {
      const size_t o = ((size_t)b * p.RU + row) * C;
      const float m = p.rmax[b * K + row];
      int tok = -1;
      for (int cc = 0; cc < C && tok < 0; ++cc)
        if (p.cmax[o + cc] == m) tok = p.cidx[o + cc];
      p.pending_out[b * N + t] = tok;
    }
    return;
  }
  if (mode == 0) {  // zero residual mass: draw from p instead
    double W = 0.0;
    for (int c = 0; c < C; ++c) W += p.resid[(size_t)b * C + c];
    if (!(W > 0.0)) mode = 1;
  }
  const float u = uniform(p.seed, (uint32_t)b, step_of(p), pos, stream);
  const T* prow = p.lc + ((size_t)b * K + row) * p.V;
  const T* qrow = nullptr;
  ResidRows rr{};
  float m_row = 0.0f;
  if (mode == 0) {
    rr = resid_rows(p, b, a, prow, qrow);
  } else {
    m_row = p.rmax[b * K + row];
  }
  // Locate the chunk: warp 0, one lane per chunk (C <= 32 is checked on
  // the host), an inclusive fp64 scan in a fixed shuffle tree, so the
  // choice is deterministic.  Chunk masses are in units of exp(l - m_row)
  // for p/q rows, probability units for residuals.
  if (threadIdx.x < 32) {
    const int ln = threadIdx.x;
    const size_t o = ((size_t)b * p.RU + row) * C;
    double mc = 0.0;
    if (ln < C)
      mc = mode == 0 ? p.resid[(size_t)b * C + ln]
                     : p.csum[o + ln] * exp((double)(p.cmax[o + ln] - m_row));
    double incl = mc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, off);
      if (ln >= off) incl += y;
    }
    const double total = __shfl_sync(0xffffffffu, incl, 31);
    const double target = (double)u * total;
    // Exclusive prefix = the previous lane's inclusive value, bit for bit.
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (ln == 0) excl = 0.0;
    // First chunk whose inclusive sum exceeds the target (rounding past
    // the end: the last chunk with positive mass, scanned to its end).
    const uint32_t hit = __ballot_sync(0xffffffffu, ln < C && incl > target);
    const uint32_t pos = __ballot_sync(0xffffffffu, ln < C && mc > 0.0);
    const int chosen = hit ? (__ffs(hit) - 1) : (pos ? 31 - __clz(pos) : 0);
    const double ex_ch = __shfl_sync(0xffffffffu, excl, chosen);
    if (ln == 0) {
      s_chunk = chosen;
      s_target = hit ? target - ex_ch : INFINITY;
      s_found = -1;
      s_last = -1;
    }
  }
  __syncthreads();
  const int c = s_chunk;
  double rem = s_target;
  const int lo = c * kChunk, hi = min(p.V, lo + kChunk);
  // All four rounds' loads are issued before the scans.
  float w[kRounds][8];
#pragma unroll
  for (int r = 0; r < kRounds; ++r)
    load_row8<T, kVec>(prow, lo + (r * kAThreads + threadIdx.x) * 8, hi, w[r]);
  if (mode == 0) {
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const int idx = lo + (r * kAThreads + threadIdx.x) * 8;
      float vq[8];
      if (rr.x < 0) load_row8<T, kVec>(qrow, idx, hi, vq);
#pragma unroll
      for (int k = 0; k < 8; ++k) w[r][k] = resid_w(rr, w[r][k], vq[k], idx + k);
    }
  } else {
#pragma unroll
    for (int r = 0; r < kRounds; ++r)
#pragma unroll
      for (int k = 0; k < 8; ++k) w[r][k] = ex2((w[r][k] - m_row) * kLog2e);
  }
  int my_last = -1;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int idx = lo + (r * kAThreads + threadIdx.x) * 8;
    float own32 = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      own32 += w[r][k];
      if (w[r][k] > 0.0f) my_last = idx + k;
    }
    double total, excl;
    const double incl = block_inclusive_scan<double>((double)own32, sh, excl,
                                                     total);
    if (rem < total) {
      if (incl > rem && excl <= rem) {
        double run = excl;
        int pick = -1, lastp = -1;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          run += (double)w[r][k];
          if (w[r][k] > 0.0f) lastp = idx + k;
          if (pick < 0 && run > rem) pick = idx + k;
        }
        atomicMax(&s_found, pick >= 0 ? pick : lastp);
      }
      __syncthreads();
      break;
    }
    rem -= total;
  }
  // Rounding left the target past every running sum: last positive entry.
  atomicMax(&s_last, my_last);
  __syncthreads();
  if (threadIdx.x == 0) {
    const int tok = s_found >= 0 ? s_found : s_last;
    p.pending_out[b * N + t] = tok;
  }
}

// ---------------------------------------------------------------------------
// Host-side launcher (called from the C ABI after validation).

struct AcceptLayout {
  size_t csum, rsum, resid, cmax, rmax, decision, cidx, total;
};

static AcceptLayout accept_layout(int B, int N, int K, int V) {
  const size_t C = (V + kChunk - 1) / kChunk;
  const size_t RU = 2 * N - 1;
  AcceptLayout l;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) & ~size_t(255);
    return at;
  };
  l.csum = take((size_t)B * RU * C * 8);
  l.rsum = take((size_t)B * K * 8);
  l.resid = take((size_t)B * C * 8);
  l.cmax = take((size_t)B * RU * C * 4);
  l.rmax = take((size_t)B * K * 4);
  l.decision = take((size_t)B * 4 * 4);
  l.cidx = take((size_t)B * RU * C * 4);
  l.total = off;
  return l;
}

template <typename T>
static int launch_accept_t(const isd_accept_args* a, cudaStream_t st) {
  AcceptDev<T> p;
  p.B = a->B; p.N = a->N; p.K = a->K; p.V = a->V;
  p.C = (a->V + kChunk - 1) / kChunk;
  p.RU = 2 * a->N - 1;
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
  p.rsum = reinterpret_cast<double*>(ws + l.rsum);
  p.resid = reinterpret_cast<double*>(ws + l.resid);
  p.cmax = reinterpret_cast<float*>(ws + l.cmax);
  p.rmax = reinterpret_cast<float*>(ws + l.rmax);
  p.decision = reinterpret_cast<int32_t*>(ws + l.decision);
  p.cidx = reinterpret_cast<int32_t*>(ws + l.cidx);
  p.argmax = a->proposal == ISD_PROPOSAL_ARGMAX;
  const bool vec = (a->V % 8) == 0;
  dim3 g_stats(p.C, p.RU, p.B), g_res(p.C, p.B), g_samp(p.N, p.B);
  if (vec) {
    accept_stats_kernel<T, true><<<g_stats, kAThreads, 0, st>>>(p);
    accept_decide_kernel<T><<<(p.B + 3) / 4, 128, 0, st>>>(p);
    accept_residual_kernel<T, true><<<g_res, kAThreads, 0, st>>>(p);
    accept_sample_kernel<T, true><<<g_samp, kAThreads, 0, st>>>(p);
  } else {
    accept_stats_kernel<T, false><<<g_stats, kAThreads, 0, st>>>(p);
    accept_decide_kernel<T><<<(p.B + 3) / 4, 128, 0, st>>>(p);
    accept_residual_kernel<T, false><<<g_res, kAThreads, 0, st>>>(p);
    accept_sample_kernel<T, false><<<g_samp, kAThreads, 0, st>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

size_t accept_workspace_bytes(int B, int N, int K, int V) {
  return accept_layout(B, N, K, V).total;
}

int launch_accept(const isd_accept_args* a, cudaStream_t st) {
  if (a->dtype == ISD_BF16) return launch_accept_t<__nv_bfloat16>(a, st);
  return launch_accept_t<float>(a, st);
}

}  // namespace isd
