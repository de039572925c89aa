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
//   decode_score_kernel    long caches only: the block scores over many CTAs.
//   decode_select_kernel   one CTA per (b, KV head): pooled query, scores of
//                          the complete blocks, exact top-(k-1) by a radix
//                          search (8-bit digits) on order-preserving keys
//                          (ties: lower j),
//                          ascending table with c last.
//   decode_attn_kernel     one CTA per (b, KV head, selected block): scores
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
  uint32_t* keys;                 // [B][Hkv][n] order keys of the scores, or null (scored in the selection)
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

// The group-mean query of (b, h) into qs[D] (a CTA-wide loop; the caller
// synchronises before reading it).
template <int D>
__device__ __forceinline__ void decode_group_query(const DecodeParams& p, int b, int h, float* qs) {
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < p.G; ++g)
      s += __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * p.G + g) * D + d]);
    qs[d] = s / static_cast<float>(p.G);
  }
}

// Order key of block j's score against the group-mean query: its mean-key
// row read with 16-byte loads, eight in flight.
template <int D>
__device__ __forceinline__ uint32_t decode_score_key(const float* kb, int j, const float* qs) {
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
  return dec_order_key(acc0 + acc1);
}

// Long caches: the scores of the complete blocks spread over many CTAs (a
// thread per block), written as order keys for the selection kernel.
// grid (ceil((n - 1) / kDecodeSelThreads), B * Hkv).
template <int D>
__global__ void __launch_bounds__(kDecodeSelThreads) decode_score_kernel(const DecodeParams p) {
  __shared__ float qs[D];
  const int bh = blockIdx.y, b = bh / p.Hkv, h = bh % p.Hkv;
  const int L = p.len[b];
  if (L < 1 || L > p.S) return;  // reported by the selection kernel
  const int c = (L - 1) / 64;   // complete blocks before the query's own
  if (c + 1 <= p.topk) return;   // every causal block is kept: no ranking
  const int j0 = blockIdx.x * kDecodeSelThreads;
  if (j0 >= c) return;           // the whole CTA: nothing to score here
  decode_group_query<D>(p, b, h, qs);
  __syncthreads();
  const int j = j0 + threadIdx.x;
  if (j < c) p.keys[static_cast<size_t>(bh) * p.n + j] = decode_score_key<D>(p.kbar + static_cast<size_t>(bh) * p.n * D, j, qs);
}

// dynamic shared memory: 4 * n bytes of keys
template <int D>
__global__ void __launch_bounds__(kDecodeSelThreads) decode_select_kernel(const DecodeParams p) {
  extern __shared__ uint32_t dkey[];
  __shared__ float qs[D];
  __shared__ unsigned red[kDecodeSelThreads / 32];
  __shared__ unsigned hist[256];
  __shared__ unsigned sel_digit[2];
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
  if (p.keys != nullptr) {
    // scored by decode_score_kernel
    const uint32_t* kin = p.keys + static_cast<size_t>(bh) * p.n;
    for (int j = threadIdx.x; j < c; j += blockDim.x) dkey[j] = kin[j];
  } else {
    decode_group_query<D>(p, b, h, qs);
    __syncthreads();
    // scores of the complete blocks j < c: a thread per block
    const float* kb = p.kbar + static_cast<size_t>(bh) * p.n * D;
    for (int j = threadIdx.x; j < c; j += blockDim.x) dkey[j] = decode_score_key<D>(kb, j, qs);
  }
  __syncthreads();
  // the (k-1)-th largest key, by a radix search over 8-bit digits (most
  // significant first): a histogram of the keys that match the digits found so
  // far, then warp 0 finds the digit holding the wanted rank
  const unsigned need = static_cast<unsigned>(p.topk - 1);
  // top-k 1 keeps only the query's own block: no key is chosen (T above all)
  uint32_t T = need == 0 ? 0xFFFFFFFFu : 0u, tmask = 0;
  unsigned rank = need;  // wanted rank among the keys matching T on tmask
  for (int shift = 24; shift >= 0 && need > 0; shift -= 8) {
    for (int x = threadIdx.x; x < 256; x += blockDim.x) hist[x] = 0u;
    __syncthreads();
    // lanes with the same digit add once per warp (scores of similar size
    // share their leading digits, so a plain atomic per key would serialise)
    for (int j0 = 0; j0 < c; j0 += blockDim.x) {
      const int j = j0 + static_cast<int>(threadIdx.x);
      const uint32_t kj = j < c ? dkey[j] : 0u;
      const bool in = j < c && (kj & tmask) == T;
      const unsigned digit = in ? (kj >> shift) & 255u : 256u;  // 256: not counted
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], static_cast<unsigned>(__popc(peers)));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8 l down to 248 - 8 l (descending)
      unsigned cnt[8], local = 0;
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        cnt[x] = hist[255 - 8 * lane - x];
        local += cnt[x];
      }
      unsigned incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned excl = incl - local;
      if (excl < rank && rank <= incl) {  // exactly one lane
        unsigned acc = excl, left = 0;
        int digit = 0;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          if (acc + cnt[x] >= rank) {
            digit = 255 - 8 * lane - x;
            left = rank - acc;
            break;
          }
          acc += cnt[x];
        }
        sel_digit[0] = static_cast<unsigned>(digit);
        sel_digit[1] = left;
      }
    }
    __syncthreads();
    T |= sel_digit[0] << shift;
    tmask |= 255u << shift;
    rank = sel_digit[1];
    __syncthreads();  // sel_digit and hist are rewritten by the next pass
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

// decode_attn_kernel: one CTA of kDecodeThreads threads per kept block.
constexpr int kDecodeThreads = 128;
template <int D>
__host__ __device__ constexpr int decode_row_bytes() {
  return D * 2 + 16;  // a K or V row padded by 16 B: lane-per-row reads spread over the banks
}
// K and V rows, the G scaled queries, the G x 64 probabilities, and the
// per-warp maxima and sums of the two key warps
template <int D, int G>
__host__ __device__ constexpr int decode_attn_smem() {
  return 2 * 64 * decode_row_bytes<D>() + G * D * 4 + G * 64 * 4 + 2 * 2 * G * 4;
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

// One CTA of 128 threads per (b, KV head, selected block), G query heads
// (template, so no work is spent on absent heads).  The CTA copies the
// block's K and V rows into shared memory with cp.async (one round trip), then
//   scores: thread (key tid % 64, heads of half tid / 64) dots its key row with
//           the scaled queries using packed f32x2 FMAs;
//   softmax: per head, max and sum over the 64 keys (two warps, combined in
//           shared memory), probabilities to shared memory;
//   P V:     thread (column pair, head group) accumulates over the 64 keys.
// A partial (m, l, o) per head goes to the workspace for the combine.
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads) decode_attn_kernel(const DecodeParams p) {
  constexpr int RB = decode_row_bytes<D>();
  constexpr int GH = G / 2;                      // heads per score thread (G >= 2)
  constexpr int CP = D / 2;                      // output column pairs
  constexpr int HG = kDecodeThreads / CP;        // head groups in P V
  constexpr int GPH = (G + HG - 1) / HG;         // heads per P V thread
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t* ks = dsm;
  uint8_t* vs = ks + 64 * RB;
  float* qs = reinterpret_cast<float*>(vs + 64 * RB);   // [G][D]
  float* ps = qs + G * D;                               // [G][64]
  float* red = ps + G * 64;                             // [2 warps][G] max, then [2][G] sum
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int item = blockIdx.x;
  const int slot = item % p.topk;
  const int bh = item / p.topk, b = bh / p.Hkv, h = bh % p.Hkv;
  float* part = p.part + static_cast<size_t>(item) * G * (D + 2);
  const int j = p.idx[static_cast<size_t>(bh) * p.topk + slot];
  if (j < 0) {  // padding: an empty partial
    if (tid < G) {
      part[tid * (D + 2)] = -INFINITY;
      part[tid * (D + 2) + 1] = 0.f;
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
  for (int e = tid; e < 64 * (D / 8); e += kDecodeThreads) {
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
  for (int e = tid; e < G * D; e += kDecodeThreads)
    qs[e] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * G) * D + e]) * p.scale_log2;
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // scores of key k against heads g0 .. g0 + GH - 1
  const int k = tid & 63, g0 = (tid >> 6) * GH;
  uint64_t a2[GH];
#pragma unroll
  for (int x = 0; x < GH; ++x) a2[x] = 0;
  const uint4* krow = reinterpret_cast<const uint4*>(ks + k * RB);
#pragma unroll 4
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const uint4 kv = krow[c8];
    const uint64_t k0 = dec_bf2(kv.x), k1 = dec_bf2(kv.y), k2 = dec_bf2(kv.z), k3 = dec_bf2(kv.w);
#pragma unroll
    for (int x = 0; x < GH; ++x) {
      const float4* q4 = reinterpret_cast<const float4*>(qs + (g0 + x) * D + c8 * 8);
      const float4 qa = q4[0], qb = q4[1];
      a2[x] = dec_f2_fma(dec_f2(qa.x, qa.y), k0, a2[x]);
      a2[x] = dec_f2_fma(dec_f2(qa.z, qa.w), k1, a2[x]);
      a2[x] = dec_f2_fma(dec_f2(qb.x, qb.y), k2, a2[x]);
      a2[x] = dec_f2_fma(dec_f2(qb.z, qb.w), k3, a2[x]);
    }
  }
  // per head: max and sum over the 64 keys, held by warps (tid >> 5) and its pair
  float sc[GH];
#pragma unroll
  for (int x = 0; x < GH; ++x) {
    sc[x] = k < nkeys ? dec_f2_sum(a2[x]) : -INFINITY;
    float m = sc[x];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[(warp & 1) * G + g0 + x] = m;
  }
  __syncthreads();
  float* red_l = red + 2 * G;
#pragma unroll
  for (int x = 0; x < GH; ++x) {
    const float m = fmaxf(red[g0 + x], red[G + g0 + x]);
    const float pk = exp2f(sc[x] - m);  // 0 for keys past the causal end
    ps[(g0 + x) * 64 + k] = pk;
    float l = pk;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) red_l[(warp & 1) * G + g0 + x] = l;
  }
  __syncthreads();
  if (tid < G) {
    part[tid * (D + 2)] = fmaxf(red[tid], red[G + tid]);
    part[tid * (D + 2) + 1] = red_l[tid] + red_l[G + tid];
  }

  // o[g][2c .. 2c + 1] over the 64 keys for the heads of this thread's group
  const int cp = tid % CP, hg = tid / CP;
  uint64_t acc[GPH];
#pragma unroll
  for (int x = 0; x < GPH; ++x) acc[x] = 0;
  // four keys at a time: their V pairs, then each head's four probabilities
  // with one 16-byte load
#pragma unroll 2
  for (int r0 = 0; r0 < 64; r0 += 4) {
    uint64_t v2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v2[u] = dec_bf2(*reinterpret_cast<const uint32_t*>(vs + (r0 + u) * RB + 4 * cp));
#pragma unroll
    for (int x = 0; x < GPH; ++x) {
      const int g = hg * GPH + x;
      if (g < G) {
        const float4 p4 = *reinterpret_cast<const float4*>(ps + g * 64 + r0);
        acc[x] = dec_f2_fma(dec_f2(p4.x, p4.x), v2[0], acc[x]);
        acc[x] = dec_f2_fma(dec_f2(p4.y, p4.y), v2[1], acc[x]);
        acc[x] = dec_f2_fma(dec_f2(p4.z, p4.z), v2[2], acc[x]);
        acc[x] = dec_f2_fma(dec_f2(p4.w, p4.w), v2[3], acc[x]);
      }
    }
  }
#pragma unroll
  for (int x = 0; x < GPH; ++x) {
    const int g = hg * GPH + x;
    if (g < G) {
      float lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[x]));
      *reinterpret_cast<float2*>(part + g * (D + 2) + 2 + 2 * cp) = make_float2(lo, hi);
    }
  }
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
