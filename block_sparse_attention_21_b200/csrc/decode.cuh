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
//   decode_attn_kernel     one warp per (b, KV head, selected block): scores
//                          of the G query heads against the block's 64 keys,
//                          a partial softmax (max, sum, unnormalised output).
//   decode_combine_kernel  one CTA per (b, query head): merges the partials
//                          (row groups of threads over the partials).
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
  // scores of the complete blocks j < c: a thread per block, its mean-key row
  // read with 16-byte loads, eight in flight
  const float* kb = p.kbar + static_cast<size_t>(bh) * p.n * D;
  for (int j = threadIdx.x; j < c; j += blockDim.x) {
    const float4* row = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int d4 = 0; d4 < D / 4; d4 += 8) {
      float4 r[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) r[x] = __ldg(row + d4 + x);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int d = 4 * (d4 + x);
        acc0 = fmaf(qs[d], r[x].x, acc0);
        acc1 = fmaf(qs[d + 1], r[x].y, acc1);
        acc0 = fmaf(qs[d + 2], r[x].z, acc0);
        acc1 = fmaf(qs[d + 3], r[x].w, acc1);
      }
    }
    dkey[j] = dec_order_key(acc0 + acc1);
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

// Warps per CTA of decode_attn_kernel, and its dynamic shared memory: per
// warp the block's K and V (rows padded by 16 bytes, so lanes reading
// different rows hit different banks), the G <= 16 queries and probabilities.
constexpr int kDecodeWarps = 2;
template <int D>
__host__ __device__ constexpr int decode_row_bytes() {
  return D * 2 + 16;
}
template <int D>
__host__ __device__ constexpr int decode_warp_smem() {
  return 2 * 64 * decode_row_bytes<D>() + 16 * D * 4 + 16 * 64 * 4;
}
template <int D>
__host__ __device__ constexpr int decode_attn_smem() {
  return kDecodeWarps * decode_warp_smem<D>();
}

__device__ __forceinline__ void dec_cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

__device__ __forceinline__ uint64_t dec_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t dec_f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ float dec_f2_sum(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}
// bf16 pair (low = even element) -> packed fp32 pair
__device__ __forceinline__ uint64_t dec_bf2(uint32_t w) {
  return dec_f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// One warp per (b, KV head, selected block), G query heads (template, so no
// work is spent on absent heads).  The warp first copies the block's K and V
// rows into shared memory with cp.async (one round trip for all of them);
// lane l scores keys l and l + 32 against the G queries with packed f32x2
// FMAs and 16-byte query loads; a per-head max and sum run over the warp; then
// lane l accumulates its output columns of every head over the 64 keys.
template <int D, int G>
__global__ void __launch_bounds__(32 * kDecodeWarps) decode_attn_kernel(const DecodeParams p) {
  constexpr int CPL = D / 32;                 // output columns per lane
  constexpr int RB = decode_row_bytes<D>();
  extern __shared__ __align__(16) uint8_t dsm[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint8_t* ks = dsm + warp * decode_warp_smem<D>();
  uint8_t* vs = ks + 64 * RB;
  float (*qs)[D] = reinterpret_cast<float (*)[D]>(vs + 64 * RB);
  float (*pr)[64] = reinterpret_cast<float (*)[64]>(vs + 64 * RB + 16 * D * 4);
  const int item = blockIdx.x * kDecodeWarps + warp;
  if (item >= p.B * p.Hkv * p.topk) return;
  const int slot = item % p.topk;
  const int bh = item / p.topk, b = bh / p.Hkv, h = bh % p.Hkv;
  float* part = p.part + static_cast<size_t>(item) * G * (D + 2);
  const int j = p.idx[static_cast<size_t>(bh) * p.topk + slot];
  if (j < 0) {  // padding: an empty partial
    if (lane < G) {
      part[lane * (D + 2)] = -INFINITY;
      part[lane * (D + 2) + 1] = 0.f;
    }
    return;
  }
  const int t = p.len[b] - 1;
  const int nkeys = (j == t / 64) ? (t - 64 * j + 1) : 64;  // causal inside the query's block
  // K and V rows of the block -> shared memory, 16 bytes per copy; rows past
  // the causal end are zeroed (their probabilities are 0)
  const size_t rstride = static_cast<size_t>(p.Hkv) * D;
  const __nv_bfloat16* kg = p.k + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D;
  const __nv_bfloat16* vg = p.v + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D;
  for (int e = lane; e < 64 * (D / 8); e += 32) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    if (r < nkeys) {
      dec_cp_async16(ks + r * RB + c8 * 16, kg + r * rstride + c8 * 8);
      dec_cp_async16(vs + r * RB + c8 * 16, vg + r * rstride + c8 * 8);
    } else {
      *reinterpret_cast<uint4*>(ks + r * RB + c8 * 16) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(vs + r * RB + c8 * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int e = lane; e < G * D; e += 32)
    qs[e / D][e % D] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * G) * D + e]) * p.scale_log2;
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();
  // scores of keys lane and lane + 32 against every head, 64 columns at a time
  float sc[2][G];
#pragma unroll
  for (int x = 0; x < 2; ++x)
#pragma unroll
    for (int g = 0; g < G; ++g) sc[x][g] = 0.f;
#pragma unroll
  for (int d0 = 0; d0 < D; d0 += 64) {
    uint64_t kp[2][32];  // the two keys' 64 columns as fp32 pairs
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint4* krow = reinterpret_cast<const uint4*>(ks + (lane + 32 * x) * RB + 2 * d0);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 kv = krow[c8];
        kp[x][4 * c8] = dec_bf2(kv.x);
        kp[x][4 * c8 + 1] = dec_bf2(kv.y);
        kp[x][4 * c8 + 2] = dec_bf2(kv.z);
        kp[x][4 * c8 + 3] = dec_bf2(kv.w);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint64_t a0 = 0, a1 = 0;
      const float4* qrow = reinterpret_cast<const float4*>(&qs[g][d0]);
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 q4 = qrow[c4];
        const uint64_t qa = dec_f2(q4.x, q4.y), qb = dec_f2(q4.z, q4.w);
        a0 = dec_f2_fma(qa, kp[0][2 * c4], a0);
        a0 = dec_f2_fma(qb, kp[0][2 * c4 + 1], a0);
        a1 = dec_f2_fma(qa, kp[1][2 * c4], a1);
        a1 = dec_f2_fma(qb, kp[1][2 * c4 + 1], a1);
      }
      sc[0][g] += dec_f2_sum(a0);
      sc[1][g] += dec_f2_sum(a1);
    }
  }
  // per head: max and sum over the warp, probabilities to shared memory
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float a = lane < nkeys ? sc[0][g] : -INFINITY;
    const float c2 = lane + 32 < nkeys ? sc[1][g] : -INFINITY;
    float m = fmaxf(a, c2);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float pa = exp2f(a - m), pb = exp2f(c2 - m);
    pr[g][lane] = pa;
    pr[g][lane + 32] = pb;
    float l = pa + pb;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      part[g * (D + 2)] = m;
      part[g * (D + 2) + 1] = l;
    }
  }
  __syncwarp();
  // o[g][d] for the lane's columns d = CPL * lane .. + CPL - 1, four keys at a time
  float acc[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[g][c] = 0.f;
  for (int r0 = 0; r0 < 64; r0 += 4) {
    float vv[4][CPL];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const uint8_t* vrow = vs + (r0 + x) * RB + 2 * CPL * lane;
      if constexpr (CPL == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(vrow);
        vv[x][0] = __uint_as_float(w << 16);
        vv[x][1] = __uint_as_float(w & 0xFFFF0000u);
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(vrow);
        vv[x][0] = __uint_as_float(w.x << 16);
        vv[x][1] = __uint_as_float(w.x & 0xFFFF0000u);
        vv[x][2] = __uint_as_float(w.y << 16);
        vv[x][3] = __uint_as_float(w.y & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 p4 = *reinterpret_cast<const float4*>(&pr[g][r0]);
      const float pw[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[g][c] = fmaf(pw[x], vv[x][c], acc[g][c]);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < CPL; ++c) part[g * (D + 2) + 2 + CPL * lane + c] = acc[g][c];
}

// One CTA of NT threads per (b, query head): o = sum_s 2^(m_s - M) o_s / l
// over the partials s.  M first (a strided max), then the threads split into
// D/4 float4 columns x R row groups; each row group walks every R-th partial
// with eight loads in flight, and the row groups' sums are added in a fixed
// order in shared memory.  NT = 256 for many partials, 64 for a few.
template <int D, int NT>
__global__ void __launch_bounds__(NT) decode_combine_kernel(const DecodeParams p) {
  constexpr int C4 = D / 4;                  // float4 columns
  constexpr int R = NT / C4;                 // row groups
  constexpr int U = 8;
  static_assert(R >= 1 && NT % 32 == 0, "combine layout");
  __shared__ float red[NT / 32];
  __shared__ float4 osum[R][C4];
  __shared__ float lsum[R];
  const int bq = blockIdx.x, b = bq / p.Hq, hq = bq % p.Hq;
  const int h = hq / p.G, g = hq % p.G;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const size_t stride = static_cast<size_t>(p.G) * (D + 2);   // floats between partials
  const float* base = p.part + (static_cast<size_t>(b) * p.Hkv + h) * p.topk * stride + g * (D + 2);

  float mx = -INFINITY;
  for (int s = tid; s < p.topk; s += NT) mx = fmaxf(mx, base[s * stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w]);

  const int c = tid % C4, r = tid / C4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float l = 0.f;
  if (M != -INFINITY) {
    for (int s0 = r; s0 < p.topk; s0 += R * U) {
      float m[U], ls[U];
      float4 ov[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = s0 + u * R;
        if (s < p.topk) {
          const float* ps = base + s * stride;
          m[u] = ps[0];
          ls[u] = ps[1];
          ov[u] = make_float4(ps[2 + 4 * c], ps[3 + 4 * c], ps[4 + 4 * c], ps[5 + 4 * c]);
        } else {
          m[u] = -INFINITY;
          ls[u] = 0.f;
          ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float w = m[u] == -INFINITY ? 0.f : exp2f(m[u] - M);
        l = fmaf(w, ls[u], l);
        acc.x = fmaf(w, ov[u].x, acc.x);
        acc.y = fmaf(w, ov[u].y, acc.y);
        acc.z = fmaf(w, ov[u].z, acc.z);
        acc.w = fmaf(w, ov[u].w, acc.w);
      }
    }
  }
  osum[r][c] = acc;
  if (c == 0) lsum[r] = l;
  __syncthreads();
  if (tid < C4) {
    float4 o = osum[0][tid];
    float lt = lsum[0];
    for (int rr = 1; rr < R; ++rr) {
      const float4 v = osum[rr][tid];
      o.x += v.x;
      o.y += v.y;
      o.z += v.z;
      o.w += v.w;
      lt += lsum[rr];
    }
    // l == 0 only for a length the selection rejected: zeros and -inf
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    __nv_bfloat16* out = p.o + static_cast<size_t>(bq) * D + 4 * tid;
    out[0] = __float2bfloat16_rn(o.x * inv);
    out[1] = __float2bfloat16_rn(o.y * inv);
    out[2] = __float2bfloat16_rn(o.z * inv);
    out[3] = __float2bfloat16_rn(o.w * inv);
    if (tid == 0) p.lse[bq] = lt > 0.f ? (M + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace ssa
