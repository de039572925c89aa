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

// One CTA of 256 threads per (block j, KV head h, batch b).  Each thread owns
// one 16-byte chunk column of the 64-row slab and sums a strided subset of the
// rows in fp32; a shared-memory pass then adds the row lanes (and, for Q, the
// G heads of the group).  Requires CH = (row width)/8 to divide 256.
template <int D>
__global__ void __launch_bounds__(256) block_pool_kernel(const PoolParams p) {
  __shared__ float part[256][9];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t out_off = ((static_cast<size_t>(b) * p.Hkv + h) * p.n + j) * D;

  // ---- keys: slab of 64 rows x D, row stride Hkv*D
  {
    constexpr int CH = D / 8;
    constexpr int NTL = 256 / CH;
    const int ch = tid % CH, tl = tid / CH;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const __nv_bfloat16* base =
        p.k + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D + ch * 8;
#pragma unroll
    for (int t = tl; t < 64; t += NTL)
      add_bf16x8(acc, ld_stream16(base + static_cast<size_t>(t) * p.Hkv * D));
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tid][e] = acc[e];
    __syncthreads();
    for (int d = tid; d < D; d += 256) {
      float s = 0.f;
      for (int l = 0; l < NTL; ++l) s += part[l * CH + d / 8][d % 8];
      p.kbar[out_off + d] = s * (1.0f / 64.0f);
    }
    __syncthreads();
  }
  if (p.q == nullptr || p.qbar == nullptr) return;

  // ---- queries: slab of 64 rows x (G*D) contiguous, row stride Hq*D
  {
    const int CH = p.G * (D / 8);
    const int NTL = 256 / CH;
    const int ch = tid % CH, tl = tid / CH;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const __nv_bfloat16* base =
        p.q + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hq + h * p.G) * D + ch * 8;
    if (tl < NTL) {
#pragma unroll 4
      for (int t = tl; t < 64; t += NTL)
        add_bf16x8(acc, ld_stream16(base + static_cast<size_t>(t) * p.Hq * D));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tid][e] = acc[e];
    __syncthreads();
    const float inv = 1.0f / (64.0f * static_cast<float>(p.G));
    for (int d = tid; d < D; d += 256) {
      float s = 0.f;
      for (int l = 0; l < NTL; ++l)
        for (int g = 0; g < p.G; ++g) s += part[l * CH + g * (D / 8) + d / 8][d % 8];
      p.qbar[out_off + d] = s * inv;
    }
  }
}

struct SelectParams {
  const float* qbar;
  const float* kbar;
  int32_t* idx;
  int n, D, topk, rows;  // rows = B * Hkv * n
};

constexpr int kSelectWarps = 4;

// One warp per (b, h, query block i).  Scores q_pooled[i] . k_pooled[j] for
// j < i in fp32, then k-1 rounds of a warp arg-max (higher score first, lower
// j on ties), then the chosen set plus i written in ascending order, -1 padded.
// Dynamic shared memory per warp: n scores, n/32 taken-bits, D pooled query.
__global__ void __launch_bounds__(32 * kSelectWarps) block_select_kernel(const SelectParams p) {
  extern __shared__ float sel_smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * kSelectWarps + warp;
  if (row >= p.rows) return;
  const int words = (p.n + 31) / 32;
  float* sc = sel_smem + static_cast<size_t>(warp) * (p.n + words + p.D);
  uint32_t* taken = reinterpret_cast<uint32_t*>(sc + p.n);
  float* qs = sc + p.n + words;
  const int i = row % p.n;
  const size_t bh = static_cast<size_t>(row / p.n);
  int32_t* out = p.idx + static_cast<size_t>(row) * p.topk;

  if (i + 1 <= p.topk) {  // every causal block
    for (int r = lane; r < p.topk; r += 32) out[r] = (r <= i) ? r : -1;
    return;
  }
  for (int d = lane; d < p.D; d += 32) qs[d] = p.qbar[static_cast<size_t>(row) * p.D + d];
  for (int w = lane; w < words; w += 32) taken[w] = 0u;
  __syncwarp();
  for (int j = lane; j < i; j += 32) {
    const float4* kj = reinterpret_cast<const float4*>(p.kbar + (bh * p.n + j) * p.D);
    float s = 0.f;
    for (int d4 = 0; d4 < p.D / 4; ++d4) {
      const float4 kv = __ldg(kj + d4);
      s = fmaf(qs[4 * d4 + 0], kv.x, s);
      s = fmaf(qs[4 * d4 + 1], kv.y, s);
      s = fmaf(qs[4 * d4 + 2], kv.z, s);
      s = fmaf(qs[4 * d4 + 3], kv.w, s);
    }
    sc[j] = s;
  }
  __syncwarp();
  for (int r = 0; r < p.topk - 1; ++r) {
    float bs = -INFINITY;
    int bj = 0x7fffffff;
    for (int j = lane; j < i; j += 32) {
      if (taken[j >> 5] & (1u << (j & 31))) continue;
      const float s = sc[j];
      if (s > bs || (s == bs && j < bj)) { bs = s; bj = j; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
      if (os > bs || (os == bs && oj < bj)) { bs = os; bj = oj; }
    }
    if (bj >= i) break;  // nothing comparable left (non-finite scores)
    if (lane == 0) taken[bj >> 5] |= 1u << (bj & 31);
    __syncwarp();
  }
  __syncwarp();
  int written = 0;
  for (int c = 0; c * 32 <= i; ++c) {
    const int j = c * 32 + lane;
    const bool chosen = (j == i) || (j < i && (taken[j >> 5] & (1u << (j & 31))));
    const uint32_t m = __ballot_sync(0xffffffffu, chosen);
    const int pos = written + __popc(m & ((1u << lane) - 1u));
    if (chosen && pos < p.topk) out[pos] = j;
    written += __popc(m);
  }
  for (int r = written + lane; r < p.topk; r += 32) out[r] = -1;
}

}  // namespace ssa
