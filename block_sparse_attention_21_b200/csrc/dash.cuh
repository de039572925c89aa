// dash.cuh -- DashAttention chunk routing ("Resumen Tecnico: DashAttention",
// stage 1 with its GQA rule): per query block i of KV head h, every query head
// g of the group scores the complete earlier chunks j < i with the mean query
// of block i against the chunk's mean key,
//   z_gj = gamma * scale * qmean_g(i) . kbar_j,
// turns the scores into a sparse distribution with alpha-entmax,
//   p_gj = [(alpha - 1) z_gj - tau_g]_+ ^ (1 / (alpha - 1)),  sum_j p_gj = 1,
// and the group shares w_j = mean_g p_gj.  The support (w_j > 0, plus the
// diagonal chunk i, which is not routed) is written as a bit mask.
//
// One CTA per (i, h, b), 256 threads:
//   1. the G per-head query means of block i (16-byte loads, fp32 sums);
//   2. a thread per chunk j < i: its mean key against the G query means;
//   3. a warp per head: the entmax threshold by bisection in fp32 until the
//      bracket stops shrinking, then p normalised to sum 1;
//   4. w (the full row, zeros from i on) and the mask words.
#pragma once

#include "pool_select.cuh"
#include "sm100.cuh"
#include "softmax_util.cuh"

namespace ssa {

struct DashRouteParams {
  int B, S, Hq, Hkv, G, n, W;
  float am1;        // alpha - 1
  float inv_am1;    // 1 / (alpha - 1)
  int pw_mode;      // 0: exponent 2 (alpha = 1.5), 1: exponent 1 (alpha = 2), 2: general
  float zscale;     // gamma * softmax scale
  const __nv_bfloat16* q;  // [B][S][Hq][D]
  const float* kbar;       // [B][Hkv][n][D]
  float* w;                // [B][Hkv][n][n]
  uint32_t* mask;          // [B][Hkv][n][W]
};

// Dynamic shared memory of dash_route_kernel (floats: query means, per-head
// scores, the group weights).
__host__ __device__ constexpr size_t dash_route_smem(int G, int D, int n) {
  return (static_cast<size_t>(G) * D + static_cast<size_t>(G) * n + n) * sizeof(float);
}

__device__ __forceinline__ float dash_pow(float t, int mode, float inv) {
  if (t <= 0.f) return 0.f;
  if (mode == 0) return t * t;
  if (mode == 1) return t;
  return exp2f(log2f(t) * inv);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int D>
__global__ void __launch_bounds__(256) dash_route_kernel(const DashRouteParams p) {
  extern __shared__ float route_smem[];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = p.G, GD = G * D, n = p.n;
  float* qm = route_smem;            // [G * D] query means
  float* x = qm + GD;         // [G][n] (alpha - 1) z, then p
  float* wj = x + G * n;      // [n] group weights
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  pdl_wait();  // the mean keys may still be in flight from the pooling kernel

  // 1. per-head query means of block i: C 16-byte chunks per token row; R
  //    row groups of threads, each summing every R-th token, then combined
  const int C = GD / 8;
  const int R = 256 / C;
  for (int e = tid; e < GD; e += 256) qm[e] = 0.f;
  __syncthreads();
  const bool loader = tid < R * C;
  const int c = tid % C, r0 = tid / C;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (loader) {
    const size_t row = static_cast<size_t>(p.Hq) * D;
    const __nv_bfloat16* base = p.q + (static_cast<size_t>(b) * p.S + 64 * i) * row +
                                static_cast<size_t>(h) * GD + c * 8;
    for (int t = r0; t < 64; t += R) add_bf16x8(acc, ld_stream16(base + t * row));
  }
  for (int r = 0; r < R; ++r) {  // row groups add in a fixed order
    if (loader && r0 == r)
#pragma unroll
      for (int e = 0; e < 8; ++e) qm[c * 8 + e] += acc[e];
    __syncthreads();
  }
  for (int e = tid; e < GD; e += 256) qm[e] *= (1.f / 64.f);
  __syncthreads();

  // 2. scores of the earlier chunks, x = (alpha - 1) * z
  const float xs = p.am1 * p.zscale;
  const float* kb = p.kbar + (static_cast<size_t>(b) * p.Hkv + h) * n * D;
  for (int j = tid; j < i; j += 256) {
    const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
    float acc[kDashMaxG];
#pragma unroll
    for (int g = 0; g < kDashMaxG; ++g) acc[g] = 0.f;
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = __ldg(kr + d4);
#pragma unroll
      for (int g = 0; g < kDashMaxG; ++g) {
        if (g < G) {
          const float4 qv = reinterpret_cast<const float4*>(qm + g * D)[d4];
          acc[g] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc[g]))));
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kDashMaxG; ++g)
      if (g < G) x[g * n + j] = xs * acc[g];
  }
  __syncthreads();

  // 3. alpha-entmax per head: bisection on tau in [max x - 1, max x - i^(1-alpha)]
  //    (the sum is >= 1 at the lower end and <= 1 at the upper end)
  if (i > 0) {
    for (int g = warp; g < G; g += 8) {
      float* xg = x + g * n;
      float mx = -INFINITY;
      for (int j = lane; j < i; j += 32) mx = fmaxf(mx, xg[j]);
      mx = warp_max(mx);
      float lo = mx - 1.f;
      float hi = mx - exp2f(-p.am1 * log2f(static_cast<float>(i)));
      for (int it = 0; it < 64; ++it) {
        const float mid = 0.5f * (lo + hi);
        if (mid <= lo || mid >= hi) break;  // the bracket no longer shrinks
        float f = 0.f;
        for (int j = lane; j < i; j += 32) f += dash_pow(xg[j] - mid, p.pw_mode, p.inv_am1);
        f = warp_sum(f);  // identical in every lane (xor butterfly)
        if (f >= 1.f) lo = mid; else hi = mid;
      }
      const float tau = 0.5f * (lo + hi);
      float s = 0.f;
      for (int j = lane; j < i; j += 32) {
        const float pj = dash_pow(xg[j] - tau, p.pw_mode, p.inv_am1);
        xg[j] = pj;
        s += pj;
      }
      s = warp_sum(s);
      const float inv = 1.f / s;
      for (int j = lane; j < i; j += 32) xg[j] *= inv;
    }
  }
  __syncthreads();

  // 4. the group's weights and the support bits
  const float invg = 1.f / static_cast<float>(G);
  float* wrow = p.w + ((static_cast<size_t>(b) * p.Hkv + h) * n + i) * n;
  for (int j = tid; j < n; j += 256) {
    float s = 0.f;
    if (j < i) {
      for (int g = 0; g < G; ++g) s += x[g * n + j];
      s *= invg;
    }
    wj[j] = s;
    wrow[j] = s;
  }
  __syncthreads();
  uint32_t* mrow = p.mask + ((static_cast<size_t>(b) * p.Hkv + h) * n + i) * p.W;
  for (int wd = tid; wd < p.W; wd += 256) {
    uint32_t bits = 0u;
    for (int bit = 0; bit < 32; ++bit) {
      const int j = wd * 32 + bit;
      if ((j < i && wj[j] > 0.f) || j == i) bits |= 1u << bit;
    }
    mrow[wd] = bits;
  }
}

}  // namespace ssa
