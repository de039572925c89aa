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
//   3. a warp per head: the entmax threshold in fp32 (Newton steps for
//      alpha <= 2, bisection otherwise), then p normalised to sum 1;
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
  int newton;       // alpha <= 2: Newton steps on the convex threshold equation
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

// t^(k-1) for t > 0, the derivative's power (k = 1/(alpha-1))
__device__ __forceinline__ float dash_pow_m1(float t, int mode, float inv) {
  if (mode == 0) return t;
  if (mode == 1) return 1.f;
  return exp2f(log2f(t) * (inv - 1.f));
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

template <int D, int G>
__global__ void __launch_bounds__(256) dash_route_kernel(const DashRouteParams p) {
  extern __shared__ float route_smem[];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  constexpr int GD = G * D;
  const int n = p.n;
  float* qm = route_smem;     // [G * D] query means
  float* x = qm + GD;         // [G][n] (alpha - 1) z, then p
  float* wj = x + G * n;      // [n] group weights
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  pdl_wait();  // the mean keys may still be in flight from the pooling kernel

  // 1. per-head query means of block i: C 16-byte chunks per token row; R
  //    row groups of threads, each summing every R-th token with all of its
  //    loads in flight (eight at a time), then combined in a fixed order
  constexpr int C = GD / 8;
  constexpr int R = 256 / C;
  constexpr int TPT = 64 / R;               // tokens per thread
  constexpr int U = TPT < 8 ? TPT : 8;
  static_assert(C <= 256 && 256 % C == 0 && 64 % R == 0, "query slab layout");
  for (int e = tid; e < GD; e += 256) qm[e] = 0.f;
  __syncthreads();
  const int c = tid % C, r0 = tid / C;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  {
    const size_t row = static_cast<size_t>(p.Hq) * D;
    const __nv_bfloat16* base = p.q + (static_cast<size_t>(b) * p.S + 64 * i + r0) * row +
                                static_cast<size_t>(h) * GD + c * 8;
#pragma unroll
    for (int t0 = 0; t0 < TPT; t0 += U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = ld_stream16(base + static_cast<size_t>((t0 + u) * R) * row);
#pragma unroll
      for (int u = 0; u < U; ++u) add_bf16x8(acc, v[u]);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {  // row groups add in a fixed order
    if (r0 == r)
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
    float sacc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sacc[g] = 0.f;
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = __ldg(kr + d4);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 qv = reinterpret_cast<const float4*>(qm + g * D)[d4];
        sacc[g] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, sacc[g]))));
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) x[g * n + j] = xs * sacc[g];
  }
  __syncthreads();

  // 3. alpha-entmax per head.  f(tau) = sum_j [x_j - tau]_+^k - 1 (k =
  //    1/(alpha-1)) falls from >= 0 at tau = max x - 1 to <= 0 at
  //    max x - i^(1-alpha).  For alpha <= 2 (k >= 1) f is convex, so Newton
  //    steps from the lower end climb monotonically to the root and stop when
  //    the step vanishes in fp32; otherwise the bracket is bisected until it
  //    stops shrinking.  Every warp sum is bit-identical in all lanes (xor
  //    butterfly), so the loop exits are warp-uniform.
  if (i > 0) {
    for (int g = warp; g < G; g += 8) {
      float* xg = x + g * n;
      float mx = -INFINITY;
      for (int j = lane; j < i; j += 32) mx = fmaxf(mx, xg[j]);
      mx = warp_max(mx);
      float tau;
      if (p.newton) {
        tau = mx - 1.f;
        for (int it = 0; it < 64; ++it) {
          float f = 0.f, df = 0.f;
          for (int j = lane; j < i; j += 32) {
            const float t = xg[j] - tau;
            if (t > 0.f) {
              f += dash_pow(t, p.pw_mode, p.inv_am1);
              df += dash_pow_m1(t, p.pw_mode, p.inv_am1);
            }
          }
          f = warp_sum(f) - 1.f;
          df = warp_sum(df) * p.inv_am1;
          const float step = f / df;
          if (!(step > 0.f)) break;           // at the root, to rounding
          const float nt = tau + step;
          if (nt <= tau) break;               // the step vanished in fp32
          tau = nt;
        }
      } else {
        float lo = mx - 1.f;
        float hi = mx - exp2f(-p.am1 * log2f(static_cast<float>(i)));
        for (int it = 0; it < 64; ++it) {
          const float mid = 0.5f * (lo + hi);
          if (mid <= lo || mid >= hi) break;  // the bracket no longer shrinks
          float f = 0.f;
          for (int j = lane; j < i; j += 32) f += dash_pow(xg[j] - mid, p.pw_mode, p.inv_am1);
          f = warp_sum(f);
          if (f >= 1.f) lo = mid; else hi = mid;
        }
        tau = 0.5f * (lo + hi);
      }
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
  constexpr float invg = 1.f / static_cast<float>(G);
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
