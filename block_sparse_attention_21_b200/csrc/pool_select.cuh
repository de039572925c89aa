// pool_select.cuh -- block summaries and top-k block selection (the bandwidth
// bound front of the SSA sparse stream).
//
// Block pooling: the mean of the 64 keys of each block, and the mean of the
// 64 queries x G heads of each query block's GQA group ("SSA: Guida a Sparse
// Sparse Attention per LLM", section "Block-sparse attention e Receptive
// Field": a mean representation of each block).  Selection: per query block,
// the diagonal plus the k-1 earlier blocks of highest pooled score (same
// section: keep only the top-k most relevant blocks).
#pragma once

#include "sm100.cuh"

namespace ssa {

struct PoolParams {
  const __nv_bfloat16* k;
  const __nv_bfloat16* q;  // may be null
  float* kbar;
  float* qbar;  // may be null
  int S, Hq, Hkv, G, n;
};

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] += __uint_as_float(w[e] << 16);
    acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One CTA of 256 threads per (block j, KV head h, batch b, role): role 0 pools
// the 64 keys of block j, role 1 the 64 queries x G heads of query block j.
// Each thread owns one 16-byte chunk column of the slab and sums a strided
// subset of its rows in fp32 (8 loads in flight); a shared-memory pass then
// adds the row lanes (and, for queries, the G heads of the group).  Requires
// CH = (row width in elements) / 8 to divide 256.
template <int D>
__global__ void __launch_bounds__(256) block_pool_kernel(const PoolParams p) {
  __shared__ float part[256][9];
  const int j = blockIdx.x, h = blockIdx.y >> 1, role = blockIdx.y & 1, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t out_off = ((static_cast<size_t>(b) * p.Hkv + h) * p.n + j) * D;
  if (role == 1 && (p.q == nullptr || p.qbar == nullptr)) return;
  const int width = role ? p.G * D : D;                     // elements per row of the slab
  const size_t row_stride = role ? static_cast<size_t>(p.Hq) * D : static_cast<size_t>(p.Hkv) * D;
  const __nv_bfloat16* slab =
      role ? p.q + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hq + h * p.G) * D
           : p.k + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D;
  const int CH = width / 8;
  const int NTL = 256 / CH;
  const int ch = tid % CH, tl = tid / CH;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const __nv_bfloat16* base = slab + ch * 8;
  for (int t0 = tl; t0 < 64; t0 += 8 * NTL) {
    uint4 v[8];
#pragma unroll
    for (int x = 0; x < 8; ++x)
      if (t0 + x * NTL < 64) v[x] = ld_stream16(base + static_cast<size_t>(t0 + x * NTL) * row_stride);
#pragma unroll
    for (int x = 0; x < 8; ++x)
      if (t0 + x * NTL < 64) add_bf16x8(acc, v[x]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[tid][e] = acc[e];
  __syncthreads();
  const int G = role ? p.G : 1;
  const float inv = role ? 1.0f / (64.0f * static_cast<float>(p.G)) : 1.0f / 64.0f;
  float* out = role ? p.qbar : p.kbar;
  for (int d = tid; d < D; d += 256) {
    float s = 0.f;
    for (int l = 0; l < NTL; ++l)
      for (int g = 0; g < G; ++g) s += part[l * CH + g * (D / 8) + d / 8][d % 8];
    out[out_off + d] = s * inv;
  }
}

struct SelectParams {
  const float* qbar;
  const float* kbar;
  int32_t* idx;
  int n, topk, rows;  // rows = B * Hkv * n
};

constexpr int kSelectWarps = 4;
constexpr int kSelectMaxPerLane = 256;  // n <= 8192

// Order-preserving map of fp32 onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t f32_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp per (b, h, query block i).
//  1. score(i, j) = q_pooled[i] . k_pooled[j] in fp32 for j < i; lane l owns
//     the candidates j = l, l + 32, ... (kept in shared memory), each dot
//     product over D with all loads of four candidates in flight.
//  2. The (k-1)-th largest score T is found exactly by a 32-step radix search
//     on order-preserving keys: the largest key T with #(key >= T) >= k-1.
//  3. Chosen = {j : key > T} plus the lowest j with key == T up to k-1 in all
//     (higher score first, lower block index on ties), plus i itself; written
//     in ascending order and -1 padded.
template <int D>
__global__ void __launch_bounds__(32 * kSelectWarps) block_select_kernel(const SelectParams p) {
  extern __shared__ uint32_t sel_keys[];  // [warps][n] order keys of the scores
  __shared__ float4 qs_all[kSelectWarps][D / 4];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * kSelectWarps + warp;
  if (row >= p.rows) return;
  const int i = row % p.n;
  const size_t bh = static_cast<size_t>(row / p.n);
  int32_t* out = p.idx + static_cast<size_t>(row) * p.topk;
  if (i + 1 <= p.topk) {  // every causal block
    for (int r = lane; r < p.topk; r += 32) out[r] = (r <= i) ? r : -1;
    return;
  }
  float4* qs = qs_all[warp];
  const float4* qrow = reinterpret_cast<const float4*>(p.qbar + static_cast<size_t>(row) * D);
  for (int d4 = lane; d4 < D / 4; d4 += 32) qs[d4] = __ldg(qrow + d4);
  __syncwarp();
  uint32_t* key = sel_keys + static_cast<size_t>(warp) * p.n;
  const float* kb = p.kbar + bh * p.n * D;
  for (int j0 = lane; j0 < i; j0 += 4 * 32) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 q4 = qs[d4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 32 * u;
        if (j < i) {
          const float4 k4 = __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D) + d4);
          acc[u] = fmaf(q4.x, k4.x, acc[u]);
          acc[u] = fmaf(q4.y, k4.y, acc[u]);
          acc[u] = fmaf(q4.z, k4.z, acc[u]);
          acc[u] = fmaf(q4.w, k4.w, acc[u]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j0 + 32 * u < i) key[j0 + 32 * u] = f32_order_key(acc[u]);
  }
  __syncwarp();
  // radix search for the (k-1)-th largest key
  const int need = p.topk - 1;
  uint32_t T = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < i; j += 32) cnt += (key[j] >= cand) ? 1 : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (cnt >= need) T = cand;
  }
  // ties at T: the lowest block indices first
  int above = 0;
  for (int j = lane; j < i; j += 32) above += (key[j] > T) ? 1 : 0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) above += __shfl_xor_sync(0xffffffffu, above, off);
  int ties_left = need - above;
  int written = 0;
  for (int c = 0; c * 32 <= i; ++c) {
    const int j = c * 32 + lane;
    const uint32_t kj = (j < i) ? key[j] : 0u;
    const bool tie = (j < i) && kj == T;
    const uint32_t tm = __ballot_sync(0xffffffffu, tie);
    const int tie_rank = __popc(tm & ((1u << lane) - 1u));
    const bool chosen = (j == i) || (j < i && (kj > T || (tie && tie_rank < ties_left)));
    ties_left -= __popc(tm);
    const uint32_t m = __ballot_sync(0xffffffffu, chosen);
    const int pos = written + __popc(m & ((1u << lane) - 1u));
    if (chosen && pos < p.topk) out[pos] = j;
    written += __popc(m);
  }
  for (int r = written + lane; r < p.topk; r += 32) out[r] = -1;
}

}  // namespace ssa
