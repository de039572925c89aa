// decode.cuh -- one decoding step of the SSA sparse stream against a KV cache.
//
// Each sequence b has `len` cached tokens; the newest one, t = len - 1, is the
// query.  Its block c = t / 64 may be partial.  The selection follows the
// block-sparse rule of "SSA: Guida a Sparse Sparse Attention per LLM"
// (section "Block-sparse attention e Receptive Field": each query keeps the
// blocks whose mean representation scores highest) applied to one query:
// the query of the KV head's group, averaged over its G heads, is scored
// against the cached mean keys K-bar of the complete blocks j < c, the top
// k - 1 are kept with block c itself (causal up to t), and attention runs over
// those tokens only ("Resumen Tecnico: SSA", section 4: inference in the
// sparse mode reads only the selected blocks).
//
//   decode_select_kernel   one CTA per (b, KV head): pooled query, scores of
//                          the complete blocks, exact top-(k-1) by a radix
//                          search on order-preserving keys (ties: lower j),
//                          ascending table with c last.
//   decode_attn_kernel     one CTA per (b, KV head, selected block): scores of
//                          the G query heads against the block's 64 keys, a
//                          partial softmax (max, sum, unnormalised output).
//   decode_combine_kernel  one CTA per (b, query head): merges the partials.
//
// The work is a few rows per KV head, far below a 128-row tensor-core tile,
// and it is bound by the HBM reads of K-bar and of the selected K/V blocks;
// it runs on the CUDA cores with 16-byte loads.
#pragma once

#include "sm100.cuh"

namespace ssa {

struct DecodeParams {
  int B, S, Hq, Hkv, G, n, topk;
  float scale_log2;               // softmax scale * log2(e)
  const __nv_bfloat16* q;         // [B][Hq][D]
  const __nv_bfloat16* k;         // [B][S][Hkv][D] cache
  const __nv_bfloat16* v;         // [B][S][Hkv][D] cache
  const float* kbar;              // [B][Hkv][n][D] mean keys (complete blocks are read)
  const int32_t* len;             // [B] cached tokens per sequence, 1..S
  int32_t* idx;                   // [B][Hkv][topk] selected blocks, ascending, -1 padded
  float* part;                    // [B][Hkv][topk][G][D + 2]: m, l, o (log2 units)
  __nv_bfloat16* o;               // [B][Hq][D]
  float* lse;                     // [B][Hq] natural log
};

constexpr int kDecodeSelThreads = 256;

__device__ __forceinline__ uint32_t dec_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Sum over the CTA (kDecodeSelThreads threads); red holds 8 ints.
__device__ __forceinline__ unsigned cta_sum(unsigned x, unsigned* red) {
  x = __reduce_add_sync(0xffffffffu, x);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  unsigned s = 0;
#pragma unroll
  for (int w = 0; w < kDecodeSelThreads / 32; ++w) s += red[w];
  return s;
}

// dynamic shared memory: 4 * n bytes of keys
template <int D>
__global__ void __launch_bounds__(kDecodeSelThreads) decode_select_kernel(const DecodeParams p) {
  extern __shared__ uint32_t dkey[];
  __shared__ float qs[D];
  __shared__ unsigned red[kDecodeSelThreads / 32];
  const int bh = blockIdx.x, b = bh / p.Hkv, h = bh % p.Hkv;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int L = p.len[b];
  int32_t* out = p.idx + static_cast<size_t>(bh) * p.topk;
  if (L < 1 || L > p.S) {  // a length outside the cache: no block, error reported
    for (int r = threadIdx.x; r < p.topk; r += blockDim.x) out[r] = -1;
    if (threadIdx.x == 0) {
      atomicOr(&g_error_word, kErrBadInput);
      atomicExch(&g_error_site, 0xd01);
    }
    return;
  }
  const int t = L - 1, c = t / 64;
  if (c + 1 <= p.topk) {  // every causal block
    for (int r = threadIdx.x; r < p.topk; r += blockDim.x) out[r] = (r <= c) ? r : -1;
    return;
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < p.G; ++g)
      s += __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * p.G + g) * D + d]);
    qs[d] = s / static_cast<float>(p.G);
  }
  __syncthreads();
  // scores of the complete blocks j < c: a warp per block, lanes over D
  const float* kb = p.kbar + static_cast<size_t>(bh) * p.n * D;
  for (int j = warp; j < c; j += kDecodeSelThreads / 32) {
    float acc = 0.f;
#pragma unroll
    for (int d = lane; d < D; d += 32) acc = fmaf(qs[d], kb[static_cast<size_t>(j) * D + d], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dkey[j] = dec_order_key(acc);
  }
  __syncthreads();
  // the (k-1)-th largest key, by a 32-step radix search
  const unsigned need = static_cast<unsigned>(p.topk - 1);
  uint32_t T = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    unsigned cnt = 0;
    for (int j = threadIdx.x; j < c; j += blockDim.x) cnt += (dkey[j] >= cand) ? 1u : 0u;
    if (cta_sum(cnt, red) >= need) T = cand;
  }
  unsigned above = 0;
  for (int j = threadIdx.x; j < c; j += blockDim.x) above += (dkey[j] > T) ? 1u : 0u;
  above = cta_sum(above, red);
  // ordered compaction by warp 0: keys above T, then ties at T by lower j
  if (warp == 0) {
    int ties_left = static_cast<int>(need) - static_cast<int>(above);
    int written = 0;
    for (int j0 = 0; j0 < c; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t kj = (j < c) ? dkey[j] : 0u;
      const bool tie = (j < c) && kj == T;
      const uint32_t tm = __ballot_sync(0xffffffffu, tie);
      const int tie_rank = __popc(tm & ((1u << lane) - 1u));
      const bool chosen = (j < c) && (kj > T || (tie && tie_rank < ties_left));
      ties_left -= __popc(tm);
      const uint32_t m = __ballot_sync(0xffffffffu, chosen);
      const int pos = written + __popc(m & ((1u << lane) - 1u));
      if (chosen && pos < p.topk - 1) out[pos] = j;
      written += __popc(m);
    }
    if (lane == 0) out[p.topk - 1] = c;  // the query's own block, last (ascending)
  }
}

// Dynamic shared memory of decode_attn_kernel: the block's K (rows padded by
// one float against bank conflicts) and V in fp32, up to 16 queries, scores.
template <int D>
constexpr int decode_attn_smem() {
  return (64 * (D + 1) + 64 * D + 16 * D + 16 * 64) * 4;
}

// 128 threads; G <= 16.
template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(const DecodeParams p) {
  extern __shared__ float dsm[];
  float (*ks)[D + 1] = reinterpret_cast<float (*)[D + 1]>(dsm);
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(dsm + 64 * (D + 1));
  float (*qs)[D] = reinterpret_cast<float (*)[D]>(dsm + 64 * (D + 1) + 64 * D);
  float (*sc)[64] = reinterpret_cast<float (*)[64]>(dsm + 64 * (D + 1) + 64 * D + 16 * D);
  const int slot = blockIdx.x % p.topk;
  const int bh = blockIdx.x / p.topk, b = bh / p.Hkv, h = bh % p.Hkv;
  const int G = p.G;
  float* part = p.part + (static_cast<size_t>(bh) * p.topk + slot) * G * (D + 2);
  const int j = p.idx[static_cast<size_t>(bh) * p.topk + slot];
  if (j < 0) {  // padding: an empty partial
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
      part[g * (D + 2)] = -INFINITY;
      part[g * (D + 2) + 1] = 0.f;
    }
    return;
  }
  const int t = p.len[b] - 1;
  const int nkeys = (j == t / 64) ? (t - 64 * j + 1) : 64;  // causal inside the query's block
  // K and V rows of the block: 16-byte loads, D / 8 per row
  for (int e = threadIdx.x; e < 64 * (D / 8); e += blockDim.x) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    const size_t off = ((static_cast<size_t>(b) * p.S + 64 * j + r) * p.Hkv + h) * D + c8 * 8;
    uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (r < nkeys) {
      kk = *reinterpret_cast<const uint4*>(p.k + off);
      vv = *reinterpret_cast<const uint4*>(p.v + off);
    }
    const uint32_t wk[4] = {kk.x, kk.y, kk.z, kk.w}, wv[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      ks[r][c8 * 8 + 2 * x] = __uint_as_float(wk[x] << 16);
      ks[r][c8 * 8 + 2 * x + 1] = __uint_as_float(wk[x] & 0xFFFF0000u);
      vs[r][c8 * 8 + 2 * x] = __uint_as_float(wv[x] << 16);
      vs[r][c8 * 8 + 2 * x + 1] = __uint_as_float(wv[x] & 0xFFFF0000u);
    }
  }
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, d = e % D;
    qs[g][d] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * D + d]) * p.scale_log2;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * 64; e += blockDim.x) {
    const int g = e / 64, r = e % 64;
    float acc = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) acc = fmaf(qs[g][d], ks[r][d], acc);
    sc[g][r] = (r < nkeys) ? acc : -INFINITY;
  }
  __syncthreads();
  // per head: max and sum by one warp each (warp w takes heads w, w + 4, ...)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int g = warp; g < G; g += 4) {
    const float a = sc[g][lane], c2 = sc[g][lane + 32];
    float m = fmaxf(a, c2);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float pa = exp2f(a - m), pb = exp2f(c2 - m);
    sc[g][lane] = pa;
    sc[g][lane + 32] = pb;
    float l = pa + pb;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      part[g * (D + 2)] = m;
      part[g * (D + 2) + 1] = l;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, d = e % D;
    float acc = 0.f;
#pragma unroll 8
    for (int r = 0; r < 64; ++r) acc = fmaf(sc[g][r], vs[r][d], acc);
    part[g * (D + 2) + 2 + d] = acc;
  }
}

// One CTA of D threads per (b, query head): o = sum_s 2^(m_s - M) o_s / l.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int bq = blockIdx.x, b = bq / p.Hq, hq = bq % p.Hq;
  const int h = hq / p.G, g = hq % p.G;
  const float* base = p.part + (static_cast<size_t>(b) * p.Hkv + h) * p.topk * p.G * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < p.topk; ++s) M = fmaxf(M, base[(s * p.G + g) * (D + 2)]);
  float l = 0.f, acc = 0.f;
  for (int s = 0; s < p.topk; ++s) {
    const float* ps = base + (s * p.G + g) * (D + 2);
    const float m = ps[0];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    l = fmaf(w, ps[1], l);
    acc = fmaf(w, ps[2 + threadIdx.x], acc);
  }
  // l == 0 only for a length the selection rejected: zeros and -inf
  p.o[static_cast<size_t>(bq) * D + threadIdx.x] = __float2bfloat16_rn(l > 0.f ? acc / l : 0.f);
  if (threadIdx.x == 0) p.lse[bq] = l > 0.f ? (M + log2f(l)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace ssa
