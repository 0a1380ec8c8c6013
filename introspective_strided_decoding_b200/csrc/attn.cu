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
  grid_dep_wait();
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
  // Shared memory: G partial indices, G x 32 weights, G + 1 range starts.
  const size_t smem = (size_t)G * 136 + 4;
  auto kern = attn_combine_kernel<128>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return ISD_ERR_CUDA;
  return launch_pdl(kern, dim3(a->Hkv, a->B), dim3(256), smem, st, p) ==
                 cudaSuccess
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
