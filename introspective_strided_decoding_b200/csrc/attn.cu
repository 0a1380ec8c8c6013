// isd_attn_strided kernels: strided-query causal GQA attention over a paged
// KV cache.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io): strict causal attention with a logit shift ("Méthodologie"),
// a paged KV cache and a paged-only attention kernel ("Serving (SGLang)"),
// one forward pass carrying the verify rows and the MASK rows of a stride
// ("Introspective Strided Decoding").  Row r of sequence b (position
// L_b + r) attends to cached positions [0, L_b) and stride rows 0..r.
//
// bf16 path for head dim 64 (mma.sync tensor cores; head dim 128 runs on
// the tcgen05 kernel of attn_tc.cu).  Work is a flat list of "units": for every
// (sequence b, KV head h), one unit per cached page plus one tail unit for
// the stride's own rows.  Each persistent CTA takes an equal contiguous
// range of that list (no per-sequence imbalance, whatever the lengths).
// Inside a CTA four loader warps walk the range and copy each unit's K and
// V tiles (16 tokens x d, 128-byte-swizzled layout) into a ring of
// mbarrier-guarded stages with 16-byte cp.async; consumer warps compute
// S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32 accumulate)
// and an online softmax in base 2.  All K*g query rows of a KV head share every K/V tile,
// which is read from HBM exactly once.  Consumer warps split the rows into
// groups of 16*MW and, when rows are few, split the units of a segment
// round-robin and merge through shared memory at the segment's end.  A
// (b, h) whose units straddle CTAs leaves fp32 partials (unnormalised O,
// running max, running sum) that a combine kernel merges in CTA order.
//
// fp32 path (SIMT, exact fp32 arithmetic): one warp per query row.
#include "common.cuh"

namespace isd {

int launch_attn_combine(const isd_attn_args* a, int G, cudaStream_t st);

constexpr int kStages = 16;                     // power of two
constexpr uint64_t kWaitCycles = 4000000000ull; // ~2 s at boost clock

struct AttnDev {
  int B, Hq, Hkv, K, g, M, P, stride, RG, KS;
  float scale_log2;   // softmax scale * log2(e)
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;   // [P][Hkv][16][D]
  const __nv_bfloat16* vc;
  const __nv_bfloat16* kn;   // [B][K][Hkv][D]
  const __nv_bfloat16* vn;
  __nv_bfloat16* out;
  float* lse;
  const int32_t* page_table;
  const int32_t* seq_len;
  int32_t* status;
  float* part_o;      // [G][2][M][D]: unnormalised O of split segments
  float* part_ml;     // [G][2][2][M]: their raw row max, then row sum
  int32_t* ws_int;    // [B + 1] unit prefix, then G
};

// Bounded mbarrier wait (clock deadline); false on timeout.
ISD_DEV bool wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if ((uint64_t)(clock64() - t0) > kWaitCycles) return false;
  return true;
}

ISD_DEV int pages_of(const AttnDev& p, int b, bool* bad) {
  int L = p.seq_len[b];
  if (L < 0) { *bad = true; L = 0; }
  int n = (L + kPage - 1) / kPage;
  if (n > p.stride) { *bad = true; n = p.stride; }
  return n;
}

// Sequence b of unit u (prefix[b] <= u < prefix[b+1]).
ISD_DEV int find_seq(const int* prefix, int B, int u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Threads per CTA: NW consumer warps + NL loader warps.
template <int NW, int NL> constexpr int attn_threads() { return (NW + NL) * 32; }

template <int D, int MW, int NW, int NL>
__global__ void __launch_bounds__(attn_threads<NW, NL>(), 1)
    attn_bf16_kernel(AttnDev p) {
  constexpr int kTile = 16 * D * 2;            // one K or V tile, bytes
  constexpr int kStage = 2 * kTile;
  constexpr int RW = 16 * MW;                  // rows per consumer warp
  constexpr int kRedRow = D + 8;               // conflict-free float2 rows
  constexpr int kRedWarp = RW * kRedRow + 2 * RW;
  constexpr int KK = D / 16;                   // k-steps of Q K^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * kStage);
  uint64_t* empty = full + kStages;
  float* red = reinterpret_cast<float*>(empty + kStages);
  int* prefix = reinterpret_cast<int*>(red + NW * kRedWarp);
  __shared__ int scan_sh[33];
  __shared__ int s_bad;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, Hkv = p.Hkv;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  const int T = block_exclusive_scan_int(
      B,
      [&](int b) {
        bool bad = false;
        const int n = pages_of(p, b, &bad);
        if (bad) s_bad = 1;
        return Hkv * (n + 1);
      },
      prefix, scan_sh);
  if (tid == 0) prefix[B] = T;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = split_point(prefix, B, T, Hkv, c, G);
  const int u1 = split_point(prefix, B, T, Hkv, c + 1, G);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], NL * 32);
      mbar_init(&empty[s], p.RG);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (c == 0) {
    for (int i = tid; i <= B; i += blockDim.x) p.ws_int[i] = prefix[i];
    if (tid == 0) {
      p.ws_int[B + 1] = G;
      p.ws_int[B + 2 + G] = T;
      if (s_bad && p.status) *p.status = ISD_ERR_PAGE_TABLE_FULL;
    }
  }
  if (tid == 0) p.ws_int[B + 2 + c] = u0;   // range starts, for the combine
  if (u0 >= u1) return;

  // --------------------------------------------------------------- loaders
  // NL loader warps copy every unit's K and V tiles into the stage with
  // 16-byte cp.async (many independent requests per SM: a 4 KB gather
  // streams at HBM rate only with this much memory-level parallelism),
  // writing the 128-byte-swizzled layout the consumers' ldmatrix expects.
  // Each loader thread arrives on the stage's full barrier when its own
  // copies land.  Units are resolved 32 at a time per warp (sequence,
  // head, page id from one coalesced page-table load), one batch ahead.
  if (warp >= NW) {
    constexpr int kLT = NL * 32;
    constexpr int kCPR = D / 8;                  // 16-byte chunks per row
    constexpr int kCPT = 16 * kCPR;              // chunks per tile
    constexpr int kPer = 2 * kCPT / kLT;         // chunks per thread per unit
    static_assert((2 * kCPT) % kLT == 0, "loader split");
    const int lt = tid - NW * 32;
    uint32_t soff[kPer];
    int srow[kPer], scol[kPer], sten[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int q = lt + i * kLT;
      sten[i] = q / kCPT;
      const int w = q - sten[i] * kCPT;
      srow[i] = w / kCPR;
      scol[i] = w - srow[i] * kCPR;
      soff[i] = sten[i] * kTile + (scol[i] >> 3) * 2048 + srow[i] * 128 +
                (((scol[i] & 7) ^ (srow[i] & 7)) << 4);
    }
    auto resolve = [&](int u, int& bb, int& hh, int& page) {
      // page >= 0: cached page id; -1: the tail unit; -2: bad page id.
      if (u >= u1) { bb = 0; hh = 0; page = -2; return; }
      bb = find_seq(prefix, B, u);
      const int units = (prefix[bb + 1] - prefix[bb]) / Hkv;
      const int rel = u - prefix[bb];
      hh = rel / units;
      const int idx = rel - hh * units;
      if (idx == units - 1) {
        page = -1;
      } else {
        page = p.page_table[(size_t)bb * p.stride + idx];
        if (page < 0 || page >= p.P) {
          if (p.status) *p.status = ISD_ERR_BAD_PAGE;
          page = -2;  // read as zeros
        }
      }
    };
    int cb, ch, cp, nb, nh, np;
    resolve(u0 + lane, cb, ch, cp);
    bool failed = false;
    for (int base = u0; base < u1; base += 32) {
      resolve(base + 32 + lane, nb, nh, np);
      const int cnt = min(32, u1 - base);
      for (int j = 0; j < cnt; ++j) {
        const int b = __shfl_sync(0xffffffffu, cb, j);
        const int h = __shfl_sync(0xffffffffu, ch, j);
        const int page = __shfl_sync(0xffffffffu, cp, j);
        const int it = base - u0 + j;
        const int s = it & (kStages - 1);
        if (!failed && !wait_bounded(&empty[s], ((it / kStages) & 1) ^ 1)) {
          failed = true;
          if (p.status) *p.status = ISD_ERR_CUDA;
        }
        const uint32_t stage = smem_u32(ring + s * kStage);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const __nv_bfloat16* src;
          uint32_t bytes = 16;
          if (page >= 0) {
            src = (sten[i] ? p.vc : p.kc) +
                  (((size_t)page * Hkv + h) * kPage + srow[i]) * D + scol[i] * 8;
          } else if (page == -1 && srow[i] < p.K) {
            src = (sten[i] ? p.vn : p.kn) +
                  (((size_t)b * p.K + srow[i]) * Hkv + h) * D + scol[i] * 8;
          } else {
            src = p.kc;  // tail rows >= K, bad page: zero-fill, nothing read
            bytes = 0;
          }
          cp_async_16(stage + soff[i], src, bytes);
        }
        cp_async_arrive(&full[s]);
      }
      cb = nb; ch = nh; cp = np;
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int KS = p.KS;
  const int rg = warp / KS, ks = warp - (warp / KS) * KS;
  const int g = p.g, K = p.K, Hq = p.Hq;
  const float c2 = p.scale_log2;
  float* my_red = red + warp * kRedWarp;
  // Per-lane ldmatrix offsets inside a 16 x D tile (128-byte swizzle:
  // 16-byte chunk index XOR row % 8; 64-column boxes 2048 bytes apart).
  // K (non-transposed, B operand of Q K^T): matrices (keys 0-7 | 8-15) x
  // (chunk 2kk | 2kk+1).  V (transposed, B operand of P V): matrices
  // (keys 0-7 | 8-15) x (chunk 2np | 2np+1).
  const int k_key = ((lane >> 4) << 3) + (lane & 7);
  const int k_c0 = (lane >> 3) & 1;
  const int v_key = (((lane >> 3) & 1) << 3) + (lane & 7);
  const int v_c0 = lane >> 4;
  const uint32_t k_row = k_key * 128, v_row = v_key * 128;
  const int k_x = (k_key & 7), v_x = (v_key & 7);
  bool failed = false;
  int u = u0, it = 0;
  while (u < u1) {
    const int b = find_seq(prefix, B, u);
    const int units = (prefix[b + 1] - prefix[b]) / Hkv;
    const int rel = u - prefix[b];
    const int h = rel / units, idx0 = rel - h * units;
    const int bh_end = prefix[b] + (h + 1) * units;
    const int seg_end = min(u1, bh_end);
    const int nseg = seg_end - u;
    const bool complete = idx0 == 0 && seg_end == bh_end;
    const int npg = units - 1;
    const int L = p.seq_len[b];

    // Q fragments of this warp's rows (A operand, row-major m16 x k16).
    uint32_t qa[MW][KK][4];
    int rrow[MW][2];
#pragma unroll
    for (int mt = 0; mt < MW; ++mt) {
      const int m0 = rg * RW + mt * 16 + (lane >> 2);
      const int m1 = m0 + 8;
      rrow[mt][0] = m0 / g;
      rrow[mt][1] = m1 / g;
      const __nv_bfloat16* q0 =
          p.q + (((size_t)b * K + m0 / g) * Hq + h * g + m0 % g) * D;
      const __nv_bfloat16* q1 =
          p.q + (((size_t)b * K + m1 / g) * Hq + h * g + m1 % g) * D;
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
        const int col = kk * 16 + 2 * (lane & 3);
        qa[mt][kk][0] = *reinterpret_cast<const uint32_t*>(q0 + col);
        qa[mt][kk][1] = *reinterpret_cast<const uint32_t*>(q1 + col);
        qa[mt][kk][2] = *reinterpret_cast<const uint32_t*>(q0 + col + 8);
        qa[mt][kk][3] = *reinterpret_cast<const uint32_t*>(q1 + col + 8);
      }
    }
    float acc[MW][D / 8][4];
    float mrow[MW][2], lrow[MW][2];
#pragma unroll
    for (int mt = 0; mt < MW; ++mt) {
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
      mrow[mt][0] = mrow[mt][1] = -INFINITY;
      lrow[mt][0] = lrow[mt][1] = 0.0f;
    }

    // This warp's units: k = first, first + KS, ... (unit it + k is owned
    // by key split (it + k) % KS).
    int first = (ks - it) % KS;
    if (first < 0) first += KS;
    for (int k = first; k < nseg; k += KS) {
      const int itk = it + k;
      const int s = itk & (kStages - 1);
      if (!failed && !wait_bounded(&full[s], (itk / kStages) & 1)) {
        failed = true;
        if (p.status) *p.status = ISD_ERR_CUDA;
      }
      const int uidx = idx0 + k;
      const bool tail = uidx == npg;
      const int valid = tail ? K : min(kPage, L - uidx * kPage);
      const bool masked = tail || valid < kPage;
      const uint32_t kb = smem_u32(ring + s * kStage);
      const uint32_t vb = kb + kTile;

      // S = Q K^T for this tile's 16 keys; with 16-row warps the even and
      // odd k-steps accumulate separately to halve the dependent-mma chains.
      float sc[MW][2][4], sd[MW][2][4];
#pragma unroll
      for (int mt = 0; mt < MW; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[mt][nt][e] = sd[mt][nt][e] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
        const int chunk = 2 * kk + k_c0;
        const uint32_t addr = kb + (chunk >> 3) * 2048 + k_row +
                              (((chunk & 7) ^ k_x) << 4);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(addr, b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MW; ++mt) {
          if (MW == 1 && (kk & 1)) {
            mma_bf16_16816(sd[mt][0], qa[mt][kk], b0, b1);
            mma_bf16_16816(sd[mt][1], qa[mt][kk], b2, b3);
          } else {
            mma_bf16_16816(sc[mt][0], qa[mt][kk], b0, b1);
            mma_bf16_16816(sc[mt][1], qa[mt][kk], b2, b3);
          }
        }
      }
      if (MW == 1) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[0][nt][e] += sd[0][nt][e];
      }
      if (masked) {
        // Tail: row r sees stride rows 0..r; partial page: slots < valid.
#pragma unroll
        for (int mt = 0; mt < MW; ++mt)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int lim = tail ? min(valid - 1, rrow[mt][hf]) : valid - 1;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                if (nt * 8 + 2 * (lane & 3) + e > lim)
                  sc[mt][nt][hf * 2 + e] = -INFINITY;
          }
      }
      // Online softmax in base 2 on raw scores: p = 2^(s*c - m*c).
      bool grew = false;
      float mnew[MW][2];
#pragma unroll
      for (int mt = 0; mt < MW; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float mx = fmaxf(fmaxf(sc[mt][0][hf * 2], sc[mt][0][hf * 2 + 1]),
                           fmaxf(sc[mt][1][hf * 2], sc[mt][1][hf * 2 + 1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          mnew[mt][hf] = fmaxf(mrow[mt][hf], mx);
          grew |= mnew[mt][hf] > mrow[mt][hf];
        }
      if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
        for (int mt = 0; mt < MW; ++mt)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const float alpha = ex2((mrow[mt][hf] - mnew[mt][hf]) * c2);
            lrow[mt][hf] *= alpha;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
              acc[mt][nt][hf * 2] *= alpha;
              acc[mt][nt][hf * 2 + 1] *= alpha;
            }
            mrow[mt][hf] = mnew[mt][hf];
          }
      }
      uint32_t pa[MW][4];
#pragma unroll
      for (int mt = 0; mt < MW; ++mt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float off = mrow[mt][hf] * c2;
          float ls = 0.0f;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float& x = sc[mt][nt][hf * 2 + e];
              x = ex2(fmaf(x, c2, -off));
              ls += x;
            }
          lrow[mt][hf] += ls;
        }
        pa[mt][0] = pack_bf16(sc[mt][0][0], sc[mt][0][1]);
        pa[mt][1] = pack_bf16(sc[mt][0][2], sc[mt][0][3]);
        pa[mt][2] = pack_bf16(sc[mt][1][0], sc[mt][1][1]);
        pa[mt][3] = pack_bf16(sc[mt][1][2], sc[mt][1][3]);
      }
      // O += P V.  V rows of unwritten slots (a partial page) may hold any
      // bits; zero them in the fragments so 0 * NaN cannot reach O.
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (masked) {
        const int k0 = 2 * (lane & 3);
        mlo = (k0 < valid ? 0x0000FFFFu : 0u) |
              (k0 + 1 < valid ? 0xFFFF0000u : 0u);
        mhi = (k0 + 8 < valid ? 0x0000FFFFu : 0u) |
              (k0 + 9 < valid ? 0xFFFF0000u : 0u);
      }
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int chunk = 2 * np + v_c0;
        const uint32_t addr = vb + (chunk >> 3) * 2048 + v_row +
                              (((chunk & 7) ^ v_x) << 4);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(addr, b0, b1, b2, b3);
        b0 &= mlo; b1 &= mhi; b2 &= mlo; b3 &= mhi;
#pragma unroll
        for (int mt = 0; mt < MW; ++mt) {
          mma_bf16_16816(acc[mt][2 * np], pa[mt], b0, b1);
          mma_bf16_16816(acc[mt][2 * np + 1], pa[mt], b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // Row sums across the quad of threads sharing a row.
#pragma unroll
    for (int mt = 0; mt < MW; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float l = lrow[mt][hf];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        lrow[mt][hf] = l;
      }

    const int slot = (u == u0) ? 0 : 1;
    float* part = p.part_o + ((size_t)(c * 2 + slot)) * p.M * D;
    float* pml = p.part_ml + ((size_t)(c * 2 + slot)) * 2 * p.M;
    if (KS == 1) {
      // Write this warp's rows straight from registers.
#pragma unroll
      for (int mt = 0; mt < MW; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int m = rg * RW + mt * 16 + (lane >> 2) + hf * 8;
          const int r = m / g, j = m % g;
          const float mr = mrow[mt][hf], l = lrow[mt][hf];
          if (complete) {
            const float inv = 1.0f / l;
            __nv_bfloat16* o =
                p.out + (((size_t)b * K + r) * Hq + h * g + j) * D;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
              const int col = nt * 8 + 2 * (lane & 3);
              *reinterpret_cast<uint32_t*>(o + col) =
                  pack_bf16(acc[mt][nt][hf * 2] * inv,
                            acc[mt][nt][hf * 2 + 1] * inv);
            }
            if (p.lse && (lane & 3) == 0)
              p.lse[((size_t)b * K + r) * Hq + h * g + j] =
                  (mr * c2 + log2f(l)) * kLn2;
          } else {
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
              const int col = nt * 8 + 2 * (lane & 3);
              *reinterpret_cast<float2*>(part + (size_t)m * D + col) =
                  make_float2(acc[mt][nt][hf * 2], acc[mt][nt][hf * 2 + 1]);
            }
            if ((lane & 3) == 0) {
              pml[m] = mr;
              pml[p.M + m] = l;
            }
          }
        }
    } else {
      // Merge the KS key splits of each row group through shared memory.
#pragma unroll
      for (int mt = 0; mt < MW; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int rl = mt * 16 + (lane >> 2) + hf * 8;
#pragma unroll
          for (int nt = 0; nt < D / 8; ++nt) {
            const int col = nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(my_red + rl * kRedRow + col) =
                make_float2(acc[mt][nt][hf * 2], acc[mt][nt][hf * 2 + 1]);
          }
          if ((lane & 3) == 0) {
            my_red[RW * kRedRow + rl] = mrow[mt][hf];
            my_red[RW * kRedRow + RW + rl] = lrow[mt][hf];
          }
        }
      asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));
      const int cols = D / KS;
      for (int e = lane; e < RW * cols; e += 32) {
        const int rl = e / cols, col = ks * cols + (e - rl * cols);
        float mstar = -INFINITY;
        for (int q2 = 0; q2 < KS; ++q2) {
          const float* rw = red + (rg * KS + q2) * kRedWarp;
          mstar = fmaxf(mstar, rw[RW * kRedRow + rl]);
        }
        float o = 0.0f, l = 0.0f;
        for (int q2 = 0; q2 < KS; ++q2) {
          const float* rw = red + (rg * KS + q2) * kRedWarp;
          const float mq = rw[RW * kRedRow + rl];
          const float wgt = mq == -INFINITY ? 0.0f : ex2((mq - mstar) * c2);
          o += rw[rl * kRedRow + col] * wgt;
          l += rw[RW * kRedRow + RW + rl] * wgt;
        }
        const int m = rg * RW + rl;
        const int r = m / g, j = m % g;
        if (complete) {
          p.out[(((size_t)b * K + r) * Hq + h * g + j) * D + col] =
              __float2bfloat16_rn(o / l);
          if (p.lse && col == 0)
            p.lse[((size_t)b * K + r) * Hq + h * g + j] =
                (mstar * c2 + log2f(l)) * kLn2;
        } else {
          part[(size_t)m * D + col] = o;
          if (col == ks * cols) {
            pml[m] = mstar;
            pml[p.M + m] = l;
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(NW * 32));
    }
    it += nseg;
    u = seg_end;
  }
}

// Merges the split-KV partials of each (b, h) segment that straddles CTAs:
// O = sum_k w_k O_k / sum_k w_k l_k with w_k = 2^((m_k - m*) c) over the
// CTAs k holding a part (m* = max_k m_k).  One block per (b, h); the CTA
// ranges come from the starts the attention kernel recorded.  Per 32-row
// chunk the normalised weights w_k / L are computed once into shared
// memory, then each thread accumulates float4 columns with independent
// loads (no dependent load chains per element).
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(AttnDev p) {
  // Shared: [G] partial indices, [G][32] weights, [G + 1] range starts.
  extern __shared__ int s_dyn[];
  __shared__ int s_n;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int B = p.B;
  const int* prefix = p.ws_int;
  const int G = p.ws_int[B + 1];
  const int units = (prefix[b + 1] - prefix[b]) / p.Hkv;
  const int s = prefix[b] + h * units, e = s + units;
  // The range starts are searched in shared memory: a binary search over
  // global memory would chain ~log2(G) dependent loads.
  int* starts = s_dyn + G * 33;
  for (int i = tid; i <= G; i += blockDim.x) starts[i] = p.ws_int[B + 2 + i];
  __syncthreads();
  // CTAs whose range holds unit s and unit e - 1: the last c with
  // starts[c] <= unit (empty ranges have equal neighbouring starts).
  auto owner = [&](int u) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (starts[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  const int cf = owner(s), cl = owner(e - 1);
  if (cf == cl) return;
  int* s_part = s_dyn;
  float* s_w = reinterpret_cast<float*>(s_dyn + G);
  const int M = p.M, g = p.g, K = p.K, Hq = p.Hq;
  if (tid == 0) {
    int n = 0;
    for (int cc = cf; cc <= cl; ++cc) {
      if (starts[cc] == starts[cc + 1]) continue;   // empty range
      // slot 0: the part that starts at the CTA's own first unit.
      s_part[n++] = cc * 2 + (starts[cc] < s ? 1 : 0);
    }
    s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const float c2 = p.scale_log2;
  for (int r0 = 0; r0 < M; r0 += 32) {
    const int rows = min(32, M - r0);
    if (tid < rows) {
      const int m = r0 + tid;
      float mstar = -INFINITY;
      for (int k = 0; k < n; ++k)
        mstar = fmaxf(mstar, p.part_ml[(size_t)s_part[k] * 2 * M + m]);
      float l = 0.0f;
      for (int k = 0; k < n; ++k) {
        const float* ml = p.part_ml + (size_t)s_part[k] * 2 * M;
        const float w = ml[m] == -INFINITY ? 0.0f : ex2((ml[m] - mstar) * c2);
        s_w[k * 32 + tid] = w;
        l += ml[M + m] * w;
      }
      const float inv = 1.0f / l;
      for (int k = 0; k < n; ++k) s_w[k * 32 + tid] *= inv;
      if (p.lse) {
        const int r = m / g, j = m - r * g;
        p.lse[((size_t)b * K + r) * Hq + h * g + j] =
            (mstar * c2 + log2f(l)) * kLn2;
      }
    }
    __syncthreads();
    for (int q = tid; q < rows * (D / 4); q += blockDim.x) {
      const int rl = q / (D / 4), col = (q - rl * (D / 4)) * 4;
      const int m = r0 + rl;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < n; ++k) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(
            p.part_o + ((size_t)s_part[k] * M + m) * D + col));
        const float w = s_w[k * 32 + rl];
        acc.x += v.x * w; acc.y += v.y * w; acc.z += v.z * w; acc.w += v.w * w;
      }
      const int r = m / g, j = m - r * g;
      __nv_bfloat16* o = p.out + (((size_t)b * K + r) * Hq + h * g + j) * D + col;
      *reinterpret_cast<uint2*>(o) =
          make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// fp32 SIMT path: one warp per (b, r, hq) query row, exact fp32 arithmetic.
template <int DPL>  // d / 32 elements per lane
__global__ void __launch_bounds__(128)
    attn_f32_kernel(int B, int Hq, int Hkv, int K, int stride, int P,
                    float scale, const float* q, const float* k_new,
                    const float* v_new, const float* k_cache,
                    const float* v_cache, const int32_t* page_table,
                    const int32_t* seq_len, float* out, float* lse,
                    int32_t* status) {
  constexpr int D = DPL * 32;
  const int lane = threadIdx.x & 31;
  const int wg = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (wg >= B * K * Hq) return;
  const int hq = wg % Hq, r = (wg / Hq) % K, b = wg / (Hq * K);
  const int g = Hq / Hkv, h = hq / g;
  int L = seq_len[b];
  if (L < 0 || (L + kPage - 1) / kPage > stride) {
    if (status && lane == 0) *status = ISD_ERR_PAGE_TABLE_FULL;
    L = max(0, min(L, stride * kPage));
  }
  float qv[DPL], o[DPL];
  const float* qp = q + (((size_t)b * K + r) * Hq + hq) * D;
#pragma unroll
  for (int i = 0; i < DPL; ++i) { qv[i] = qp[lane + 32 * i]; o[i] = 0.0f; }
  float m = -INFINITY, l = 0.0f;
  const int total = L + r + 1;
  for (int t = 0; t < total; ++t) {
    const float *kp, *vp;
    if (t < L) {
      const int page = page_table[(size_t)b * stride + t / kPage];
      if (page < 0 || page >= P) {
        if (status && lane == 0) *status = ISD_ERR_BAD_PAGE;
        continue;
      }
      const size_t off = (((size_t)page * Hkv + h) * kPage + t % kPage) * D;
      kp = k_cache + off;
      vp = v_cache + off;
    } else {
      const size_t off = (((size_t)b * K + (t - L)) * Hkv + h) * D;
      kp = k_new + off;
      vp = v_new + off;
    }
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) dot = fmaf(qv[i], kp[lane + 32 * i], dot);
    dot = warp_sum(dot) * scale;
    const float mn = fmaxf(m, dot);
    const float alpha = expf(m - mn);
    const float pr = expf(dot - mn);
    l = l * alpha + pr;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = fmaf(o[i], alpha, pr * vp[lane + 32 * i]);
    m = mn;
  }
  float* op = out + (((size_t)b * K + r) * Hq + hq) * D;
#pragma unroll
  for (int i = 0; i < DPL; ++i) op[lane + 32 * i] = o[i] / l;
  if (lse && lane == 0) lse[((size_t)b * K + r) * Hq + hq] = m + logf(l);
}

// ---------------------------------------------------------------------------
// Host side.

// Consumer warps of each instantiation: 16-row warps (MW = 1) run eight
// consumers (two per SM sub-partition); 32-row warps (MW = 2) run four.
// Every instantiation adds kLoaderWarps loader warps.
constexpr int nw_of(int MW) { return MW == 1 ? 8 : 4; }
constexpr int kLoaderWarps = 4;

size_t attn_smem_bytes(int D, int MW, int B) {
  const int RW = 16 * MW;
  const size_t red = (size_t)nw_of(MW) * (RW * (D + 8) + 2 * RW) * 4;
  return 1024 + (size_t)kStages * 2 * (16 * D * 2) + 2 * kStages * 8 + red +
         (size_t)(B + 1) * 4;
}

// Workspace: the unit prefix (ints), then the split-segment partials
// part_o [G][2][M][D] and part_ml [G][2][2][M] (fp32).
// Integers: the unit prefix [B + 1], G, then the CTA range starts [G + 1].
static size_t ws_ints_bytes(int B, int G) {
  return ((size_t)(B + G + 3) * 4 + 255) & ~size_t(255);
}

size_t attn_workspace_bytes_impl(int B, int M, int D, int G) {
  return ws_ints_bytes(B, G) + (size_t)G * 2 * M * (D + 2) * 4;
}

void attn_partial_ptrs(const isd_attn_args* a, int G, float** part_o,
                       float** part_ml) {
  const int M = a->K * (a->Hq / a->Hkv);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  *part_o = reinterpret_cast<float*>(ws + ws_ints_bytes(a->B, G));
  *part_ml = *part_o + (size_t)G * 2 * M * a->d;
}

template <int D, int MW>
static int launch_bf16(const isd_attn_args* a, int G, cudaStream_t st) {
  constexpr int NW = nw_of(MW);
  constexpr int NL = kLoaderWarps;
  AttnDev p;
  p.B = a->B; p.Hq = a->Hq; p.Hkv = a->Hkv; p.K = a->K;
  p.g = a->Hq / a->Hkv; p.M = a->K * p.g; p.P = a->num_pages;
  p.stride = a->page_table_stride;
  p.RG = p.M / (16 * MW); p.KS = NW / p.RG;
  if (p.KS < 1 || p.RG * p.KS != NW) return ISD_ERR_UNSUPPORTED;
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
  attn_partial_ptrs(a, G, &p.part_o, &p.part_ml);
  const size_t smem = attn_smem_bytes(D, MW, a->B);
  auto kern = attn_bf16_kernel<D, MW, NW, NL>;
  // The shared-memory opt-in is per device; it is set on every call (a
  // host-side attribute, no device work).
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  kern<<<G, attn_threads<NW, NL>(), smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ISD_ERR_CUDA;
  return launch_attn_combine(a, G, st);
}

// Merges the split-KV partials any attention kernel left in the workspace
// (same partial layout for the mma.sync and the tcgen05 kernels).
int launch_attn_combine(const isd_attn_args* a, int G, cudaStream_t st) {
  AttnDev p{};
  p.B = a->B; p.Hq = a->Hq; p.Hkv = a->Hkv; p.K = a->K;
  p.g = a->Hq / a->Hkv; p.M = a->K * p.g;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.lse = a->lse;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  p.ws_int = reinterpret_cast<int32_t*>(ws);
  attn_partial_ptrs(a, G, &p.part_o, &p.part_ml);
  // Shared memory: G partial indices, G x 32 weights, G + 1 range starts.
  const size_t smem = (size_t)G * 136 + 4;
  auto kern = a->d == 128 ? attn_combine_kernel<128> : attn_combine_kernel<64>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  kern<<<dim3(a->Hkv, a->B), 256, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

bool attn_tc_supported(const isd_attn_args* a);
int launch_attn_tc(const isd_attn_args* a, int G, cudaStream_t st);

// Head dim 128 runs on the tcgen05 kernel (every shape the host check
// admits), head dim 64 on the mma.sync kernel.
int launch_attn_bf16(const isd_attn_args* a, int G, cudaStream_t st) {
  if (attn_tc_supported(a)) return launch_attn_tc(a, G, st);
  if (a->d != 64) return ISD_ERR_UNSUPPORTED;
  const int M = a->K * (a->Hq / a->Hkv);
  return M <= 32 ? launch_bf16<64, 1>(a, G, st) : launch_bf16<64, 2>(a, G, st);
}

int launch_attn_f32(const isd_attn_args* a, cudaStream_t st) {
  const int rows = a->B * a->K * a->Hq;
  const int blocks = (rows + 3) / 4;
#define ISD_F32_CASE(DPL)                                                     \
  attn_f32_kernel<DPL><<<blocks, 128, 0, st>>>(                               \
      a->B, a->Hq, a->Hkv, a->K, a->page_table_stride, a->num_pages,          \
      a->softmax_scale, (const float*)a->q, (const float*)a->k_new,           \
      (const float*)a->v_new, (const float*)a->k_cache,                       \
      (const float*)a->v_cache, a->page_table, a->seq_len, (float*)a->out,    \
      a->lse, a->status)
  switch (a->d / 32) {
    case 1: ISD_F32_CASE(1); break;
    case 2: ISD_F32_CASE(2); break;
    case 3: ISD_F32_CASE(3); break;
    case 4: ISD_F32_CASE(4); break;
    default: return ISD_ERR_UNSUPPORTED;
  }
#undef ISD_F32_CASE
  return cudaGetLastError() == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

}  // namespace isd
