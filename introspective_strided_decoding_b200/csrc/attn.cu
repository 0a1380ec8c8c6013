// isd_attn_strided kernels besides the tcgen05 one (attn_tc.cu): the merge
// of split-KV partials and the exact-fp32 SIMT path.
//
// Method: "Introspective Diffusion Language Models", project summary
// (hada.io): strict causal attention with a logit shift ("Méthodologie"),
// a paged KV cache and a paged-only attention kernel ("Serving (SGLang)"),
// one forward pass carrying the verify rows and the MASK rows of a stride
// ("Introspective Strided Decoding").  Row r of sequence b (position
// L_b + r) attends to cached positions [0, L_b) and stride rows 0..r.
//
// The bf16 path (head dim 128) cuts the flat list of (sequence, KV head,
// page) units into one contiguous range per persistent CTA; a (b, h) whose
// units straddle CTAs leaves fp32 partials (unnormalised O, running max,
// running sum) that attn_combine_kernel merges.
//
// fp32 path (SIMT, exact fp32 arithmetic): one warp per query row.
#include "common.cuh"

namespace isd {

struct AttnDev {
  int B, Hq, Hkv, K, g, M;
  float scale_log2;   // softmax scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  float* part_o;      // [G][2][M][D]: unnormalised O of split segments
  float* part_ml;     // [G][2][2][M]: their raw row max, then row sum
  int32_t* ws_int;    // [B + 1] unit prefix, G, [G + 1] CTA range starts
};

// Merges the split-KV partials of each (b, h) segment that straddles CTAs:
// O = sum_k w_k O_k / sum_k w_k l_k with w_k = 2^((m_k - m*) c) over the
// CTAs k holding a part (m* = max_k m_k).  Block c looks at the boundary
// between CTAs c and c + 1 and merges the segment that boundary cuts when
// it is the first boundary inside that segment (so each split segment has
// one block).  The unit prefix and the CTA range starts come into shared
// memory in one pass; every later load is independent of the others in its
// step (the part maxima and sums of a row, the float4 rows of every part).
constexpr int kCombineThreads = 256;
constexpr int kCombineChunk = 64;         // parts whose weights are staged

__global__ void __launch_bounds__(kCombineThreads)
    attn_combine_kernel(AttnDev p) {
  extern __shared__ int s_dyn[];
  const int B = p.B, G = gridDim.x, c = blockIdx.x, tid = threadIdx.x;
  const int M = p.M, Hkv = p.Hkv;
  int* prefix = s_dyn;                    // [B + 1]
  int* starts = prefix + B + 1;           // [G + 1]
  int* parts = starts + G + 1;            // [G] part rows
  float* rowf = reinterpret_cast<float*>(parts + G);   // [2][128]: m* c, 1 / l
  float* w = rowf + 256;                  // [kCombineChunk][128]
  __shared__ int s_n;
  grid_dep_wait();
  for (int i = tid; i <= B; i += blockDim.x) prefix[i] = p.ws_int[i];
  for (int i = tid; i <= G; i += blockDim.x) starts[i] = p.ws_int[B + 2 + i];
  __syncthreads();
  const int T = starts[G];
  const int e = starts[c + 1];            // first unit after CTA c
  if (c + 1 >= G || e >= T) return;
  int lo = 0, hi = B - 1;                 // the sequence holding unit e
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= e) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int units = (prefix[b + 1] - prefix[b]) / Hkv;
  const int h = (e - prefix[b]) / units;
  const int s0 = prefix[b] + h * units, s1 = s0 + units;
  // No cut at this boundary, or an earlier boundary cuts the segment too.
  if (e == s0 || starts[c] > s0) return;
  if (tid == 0) {
    int n = 0;
    for (int cc = c; cc < G && starts[cc] < s1; ++cc) {
      if (starts[cc] == starts[cc + 1]) continue;      // empty range
      const int slot = cc == c && starts[c] < s0 ? 1 : 0;
      parts[n++] = (cc * 2 + slot) * M;
    }
    s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const float c2 = p.scale_log2;
  // Row m = tid: the maximum and the normaliser over the parts.  Up to 8
  // parts (the usual case) their maxima and sums are loaded once and the
  // weights come straight from registers.
  if (tid < M) {
    float mk[8], lk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool ok = j < n;
      const float* ml = p.part_ml + 2 * (size_t)parts[ok ? j : 0];
      mk[j] = ok ? __ldcg(ml + tid) : -INFINITY;
      lk[j] = ok ? __ldcg(ml + M + tid) : 0.0f;
    }
    float mstar = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) mstar = fmaxf(mstar, mk[j]);
    for (int k0 = 8; k0 < n; ++k0)
      mstar = fmaxf(mstar, __ldcg(p.part_ml + 2 * (size_t)parts[k0] + tid));
    float l = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mk[j] = mk[j] == -INFINITY ? 0.0f : ex2((mk[j] - mstar) * c2);
      l += lk[j] * mk[j];
    }
    for (int k0 = 8; k0 < n; ++k0) {
      const float* ml = p.part_ml + 2 * (size_t)parts[k0];
      const float m1 = __ldcg(ml + tid);
      if (m1 != -INFINITY) l += __ldcg(ml + M + tid) * ex2((m1 - mstar) * c2);
    }
    rowf[tid] = mstar;
    rowf[128 + tid] = 1.0f / l;
    if (n <= kCombineChunk) {
      // Weights of the first chunk now (the loop below skips them).
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < n) w[j * 128 + tid] = mk[j] / l;
      for (int j = 8; j < n; ++j) {
        const float m1 = __ldcg(p.part_ml + 2 * (size_t)parts[j] + tid);
        w[j * 128 + tid] = m1 == -INFINITY ? 0.0f : ex2((m1 - mstar) * c2) / l;
      }
    }
    if (p.lse) {
      const int r = tid / p.g, j = tid - r * p.g;
      p.lse[((size_t)b * p.K + r) * p.Hq + h * p.g + j] =
          (mstar * c2 + log2f(l)) * kLn2;
    }
  }
  // O: thread (rg, q) owns columns 4q..4q+3 of rows rg + 8i (i < 16).
  const int q = tid & 31, rg = tid >> 5;
  float4 acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < n; k0 += kCombineChunk) {
    const int kn = min(kCombineChunk, n - k0);
    __syncthreads();                      // rowf ready / w free again
    if (tid < M && n > kCombineChunk) {
      for (int j = 0; j < kn; ++j) {
        const float mk = __ldcg(p.part_ml + 2 * (size_t)parts[k0 + j] + tid);
        w[j * 128 + tid] = mk == -INFINITY
                               ? 0.0f
                               : ex2((mk - rowf[tid]) * c2) * rowf[128 + tid];
      }
    }
    __syncthreads();
    for (int j = 0; j < kn; ++j) {
      const float* po = p.part_o + ((size_t)parts[k0 + j] + rg) * 128 + 4 * q;
      float4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = rg + 8 * i < M
                   ? __ldcg(reinterpret_cast<const float4*>(po + i * 1024))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float wk = w[j * 128 + min(rg + 8 * i, M - 1)];
        acc[i].x += wk * v[i].x; acc[i].y += wk * v[i].y;
        acc[i].z += wk * v[i].z; acc[i].w += wk * v[i].w;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int m = rg + 8 * i;
    if (m < M) {
      const int r = m / p.g, j = m - r * p.g;
      *reinterpret_cast<uint2*>(
          p.out + (((size_t)b * p.K + r) * p.Hq + h * p.g + j) * 128 + 4 * q) =
          make_uint2(pack_bf16(acc[i].x, acc[i].y),
                     pack_bf16(acc[i].z, acc[i].w));
    }
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
  grid_dep_wait();
  if (wg >= B * K * Hq) return;
  const int hq = wg % Hq, r = (wg / Hq) % K, b = wg / (Hq * K);
  const int g = Hq / Hkv, h = hq / g;
  int L = seq_len[b];
  if (L < 0 || (L + kPage - 1) / kPage > stride) {
    if (lane == 0) report(status, ISD_ERR_PAGE_TABLE_FULL);
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
        if (lane == 0) report(status, ISD_ERR_BAD_PAGE);
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

// Merges the split-KV partials the tcgen05 kernel left in the workspace.
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
  // Shared memory: prefix, starts, part rows, row factors, staged weights.
  const size_t smem = (size_t)(a->B + 1 + 2 * G + 1) * 4 + 256 * 4 +
                      (size_t)kCombineChunk * 128 * 4;
  if (cudaFuncSetAttribute(attn_combine_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  return launch_pdl(attn_combine_kernel, dim3(G), dim3(kCombineThreads), smem,
                    st, p) == cudaSuccess
             ? ISD_OK
             : ISD_ERR_CUDA;
}

bool attn_tc_supported(const isd_attn_args* a);
int launch_attn_tc(const isd_attn_args* a, int G, cudaStream_t st);

// bf16 runs on the tcgen05 kernel (head dim 128, every shape the host
// check admits).
int launch_attn_bf16(const isd_attn_args* a, int G, cudaStream_t st) {
  if (!attn_tc_supported(a)) return ISD_ERR_UNSUPPORTED;
  return launch_attn_tc(a, G, st);
}

int launch_attn_f32(const isd_attn_args* a, cudaStream_t st) {
  const int rows = a->B * a->K * a->Hq;
  const int blocks = (rows + 3) / 4;
  cudaError_t err = cudaSuccess;
#define ISD_F32_CASE(DPL)                                                     \
  err = launch_pdl(attn_f32_kernel<DPL>, dim3(blocks), dim3(128), 0, st,      \
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
  return err == cudaSuccess ? ISD_OK : ISD_ERR_CUDA;
}

}  // namespace isd
