// Device helpers shared by the ISD kernels (sm_100a).
#pragma once

#include <climits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "isd.h"

#define ISD_DEV __device__ __forceinline__

namespace isd {

constexpr int kPage = ISD_PAGE_SIZE;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11): round function on (c0, c1, c2, c3) with key
// (k0, k1) and multipliers M0, M1; Weyl key bump between rounds.

struct U4 { uint32_t x, y, z, w; };

ISD_DEV U4 philox4x32_10(U4 c, uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += W0; k1 += W1; }
    const uint32_t hi0 = __umulhi(M0, c.x), lo0 = M0 * c.x;
    const uint32_t hi1 = __umulhi(M1, c.z), lo1 = M1 * c.z;
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
  }
  return c;
}

// U(seed, seq, step, pos, stream) = (x0 >> 8) * 2^-24, exact in fp32.
ISD_DEV float uniform(uint64_t seed, uint32_t seq, uint32_t step, uint32_t pos,
                      uint32_t stream) {
  const U4 o = philox4x32_10(U4{seq, step, pos, stream}, (uint32_t)seed,
                             (uint32_t)(seed >> 32));
  return (float)(o.x >> 8) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// Device-side error reporting.  The caller's status word keeps the FIRST
// error recorded in it: a kernel never clears it and never overwrites an
// error that an earlier kernel (or call) left there, so a step's three calls
// may share one word and the host reads the earliest failure after the step.

// Kept out of line: it sits on the failure path of every bounded wait, and
// an inlined atomic there slows the wait loops themselves (measured: the
// attention kernel ran 2% slower).
static __device__ __noinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), ISD_OK, code);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of a step is launched with
// programmatic stream serialisation and waits (grid_dep_wait) for the
// kernel before it on the stream to finish, its memory visible, before it
// reads anything; work that does not depend on it (barrier set-up) comes
// first.  No kernel triggers its dependents early: measured on the C=64
// step, letting the next grid launch while the current one still runs put
// waiting CTAs beside the running ones and cost more than it saved, while
// the serialised form with these waits still shortens every boundary.
// Without a programmatic predecessor the wait returns at once.

ISD_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// The one early trigger: the commit inside isd_accept_commit triggers right
// after its wait, and the draw kernel launched behind it does not wait
// before its work, so the draws run beside the commit.  Safe because the
// trigger comes after the commit's own wait (everything ahead of the
// commit, the decide kernel included, has finished when the draw grid
// launches) and the two touch disjoint memory.  One draw CTA waits at its
// end, so the draw grid completes only after the commit.
ISD_DEV void grid_dep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches `kern` on `st` with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block,
                              size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Fast base-2 exponential (MUFU).  Used where per-element rounding averages
// out in a sum; decision values use expf.

ISD_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Element loads.

template <typename T> ISD_DEV float to_f(T v);
template <> ISD_DEV float to_f<float>(float v) { return v; }
template <> ISD_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// 8 consecutive elements starting at p (16-byte aligned for bf16, 32 for f32).
ISD_DEV void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
ISD_DEV void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Streaming variant for data read exactly once (bypasses L1 allocation).
ISD_DEV void load8_stream(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 u;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
ISD_DEV void load8_stream(const float* p, float (&v)[8]) { load8(p, v); }

// ---------------------------------------------------------------------------
// Warp / block reductions with a fixed tree (deterministic).

ISD_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
ISD_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan of ints over the block (loops for n > blockDim), in index
// order: store(i, sum_{j<i} in(j)) for every i < n; returns the total.
// Every thread of the block must call it.  `sh` >= 33 ints.
template <typename F, typename S>
ISD_DEV int block_exclusive_scan_int(int n, F in, S store, int* sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = i < n ? in(i) : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) sh[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = lane < nw ? sh[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) sh[lane] = w;
    }
    __syncthreads();
    const int excl = x - v + (wid > 0 ? sh[wid - 1] : 0);
    if (i < n) store(i, carry + excl);
    carry += sh[nw - 1];
    __syncthreads();
  }
  return carry;
}

// ---------------------------------------------------------------------------
// Work split of the attention kernels.  The flat unit list (per sequence b,
// per KV head h: its cached pages, then one tail unit) is cut into G
// contiguous ranges of equal cost, a unit costing 1 and each (b, h) segment
// kSegCost more for its fixed work (Q load, first-block max, epilogue), so
// CTAs that meet many short sequences get fewer pages.  Measured on the
// C=64 step: a segment boundary costs about what 30-40 pages of streaming
// do (per-CTA times fitted against blocks and segments), and costs of 32 to
// 40 balance the CTAs best (36: attention 4% faster than 16).

constexpr int kSegCost = 36;

// First unit of CTA c (c = G gives T).  prefix[b] = first unit of sequence
// b for b < B; T = total units; every segment of b has the same length.
// Nondecreasing in c.
ISD_DEV int split_point(const int* prefix, int B, int T, int Hkv, int c,
                        int G) {
  const long long seg = (long long)kSegCost * Hkv;
  const long long ctot = (long long)T + seg * B;
  const long long x = (long long)c * ctot / G;
  if (x >= ctot) return T;
  int lo = 0, hi = B - 1;   // last b whose cost prefix is <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)prefix[mid] + seg * mid <= x) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int end_b = b + 1 < B ? prefix[b + 1] : T;
  const long long ub = (end_b - prefix[b]) / Hkv;   // units per segment
  const long long rem = x - ((long long)prefix[b] + seg * b);
  const long long h = rem / (ub + kSegCost);
  if (h >= Hkv) return end_b;
  const long long r = rem - h * (ub + kSegCost);
  const long long off = r <= kSegCost ? 0 : min(r - kSegCost, ub);
  return (int)(prefix[b] + h * ub + off);
}

// ---------------------------------------------------------------------------
// mbarrier / TMA wrappers (inline PTX, sm_90+ forms).

ISD_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

ISD_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count));
}
ISD_DEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
ISD_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// Adds `bytes` to the transaction count the current phase waits for,
// without arriving.
ISD_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
ISD_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
ISD_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// 4-D tiled TMA load into shared memory, completion on `bar` (tx bytes).
ISD_DEV void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar,
                         int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cta.global.tile.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1),
      "r"(c2), "r"(c3)
      : "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only); `src_bytes` < 16
// zero-fills the rest (0 reads nothing).
ISD_DEV void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
               "l"(src), "r"(src_bytes)
               : "memory");
}
ISD_DEV uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace isd
