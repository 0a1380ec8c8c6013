// Device helpers shared by the ISD kernels (sm_100a).
#pragma once

#include <climits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

// Block-wide reduction; `red` holds >= 32 values; all threads get the result.
template <bool kMax>
ISD_DEV float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = kMax ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : (kMax ? -INFINITY : 0.0f);
  r = kMax ? warp_max(r) : warp_sum(r);
  return r;
}

// Block-wide minimum of ints; `red` holds >= 32 ints; all threads get it.
ISD_DEV int block_min_int(int v, int* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  int r = lane < nw ? red[lane] : INT_MAX;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r = min(r, __shfl_xor_sync(0xffffffffu, r, o));
  return r;
}

ISD_DEV double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  double r = lane < nw ? red[lane] : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  return r;
}

// Inclusive scan over the block of one value per thread (fixed order).
// Returns the inclusive prefix; `excl` gets exactly the previous thread's
// inclusive prefix (0 for thread 0) and `total` the block sum.  `sh` >= 32.
template <typename T>
ISD_DEV T block_inclusive_scan(T v, T* sh, T& excl, T& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  T prev = __shfl_up_sync(0xffffffffu, x, 1);
  __syncthreads();
  if (lane == 31) sh[wid] = x;
  __syncthreads();
  // Warp totals are scanned sequentially: sh[w] = sh[w-1] + total_w is then
  // the very addition the last thread of warp w performs below.
  if (threadIdx.x == 0)
    for (int w = 1; w < nw; ++w) sh[w] = sh[w - 1] + sh[w];
  __syncthreads();
  total = sh[nw - 1];
  const T base = wid > 0 ? sh[wid - 1] : T(0);
  if (lane == 0) prev = T(0);
  // Apply the warp offset to both prefixes with the same single addition,
  // so thread i's excl equals thread i-1's result bit for bit.
  excl = (lane == 0) ? base : (wid > 0 ? base + prev : prev);
  return wid > 0 ? base + x : x;
}

// Exclusive scan of ints over the block (loops for n > blockDim).
// out[i] = sum_{j<i} in(j), returns the total.  `sh` >= 33 ints.
template <typename F>
ISD_DEV int block_exclusive_scan_int(int n, F in, int* out, int* sh) {
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
    if (i < n) out[i] = carry + excl;
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
// CTAs that meet many short sequences get fewer pages.

constexpr int kSegCost = 16;

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
// mbarrier / TMA / ldmatrix / mma wrappers (inline PTX, sm_90+ forms).

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

// Bounded wait: gives up after `limit` polls and reports false.  Every
// wait in this library is bounded so that a broken invariant ends the
// kernel with an error status instead of hanging the device.
ISD_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

ISD_DEV void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m))
               : "memory");
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
// Arrive on `bar` once every cp.async this thread issued so far completes
// (counts as one of the barrier's expected arrivals).
ISD_DEV void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

ISD_DEV void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                         uint32_t& r2, uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}
ISD_DEV void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                               uint32_t& r2, uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
ISD_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                            uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

ISD_DEV uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace isd
