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
  const __nv_bfloat16* k;  // may be null (queries only)
  const __nv_bfloat16* q;  // may be null (keys only)
  float* kbar;
  float* qbar;  // may be null
  int S, Hq, Hkv, G, n;
  int j0;       // the grid's first block (blocks j0 .. j0 + gridDim.x - 1)
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
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Loads rows t0, t0 + step, ... (up to R of them, below 64) of one slab
// column chunk.
template <int R>
__device__ __forceinline__ void slab_load(uint4 (&v)[R], const __nv_bfloat16* base, size_t row_stride,
                                          int t0, int step) {
#pragma unroll
  for (int x = 0; x < R; ++x)
    if (t0 + x * step < 64) v[x] = ld_stream16(base + static_cast<size_t>(t0 + x * step) * row_stride);
}

template <int R>
__device__ __forceinline__ void slab_add(float (&acc)[8], const uint4 (&v)[R], int t0, int step) {
#pragma unroll
  for (int x = 0; x < R; ++x)
    if (t0 + x * step < 64) add_bf16x8(acc, v[x]);
}

// Threads per CTA: 256 pool the query slab, KW = D / 64 more warps the key
// slab; loads in flight per round and CTAs per SM, per head dim.
template <int D>
struct PoolConfig {
  static constexpr int KW = D / 64;
  static constexpr int THREADS = 256 + 32 * KW;
  static constexpr int QR = (D == 64) ? 8 : 16;   // query loads per round
  static constexpr int CHK = D / 8;                // 16-byte chunks per key row
  static constexpr int KTL = 32 * KW / CHK;        // key row lanes (4)
  static constexpr int KR = 64 / KTL;              // key rows per thread (16)
  static constexpr int MIN_CTAS = (D == 64) ? 4 : 2;
};

// One CTA per (block j, KV head h, batch b) pools the 64 keys of block j and
// the 64 queries x G heads of query block j (the group's heads are adjacent
// in memory), so every CTA streams the same amount.  Each thread owns one
// 16-byte column chunk of a slab and sums a strided subset of its rows in
// fp32, QR loads in flight per round; the first 256 threads take the query
// slab and the last KW warps the key slab, so both are in flight together.
// A shared-memory pass then adds the row lanes (and, for queries, the G
// heads).
template <int D>
__global__ void __launch_bounds__(PoolConfig<D>::THREADS, PoolConfig<D>::MIN_CTAS)
    block_pool_kernel(const PoolParams p) {
  using C = PoolConfig<D>;
  __shared__ float partq[256][9];
  __shared__ float partk[32 * C::KW][9];
  pdl_launch_dependents();
  pdl_wait();
  const int j = p.j0 + static_cast<int>(blockIdx.x), h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t out_off = ((static_cast<size_t>(b) * p.Hkv + h) * p.n + j) * D;
  const bool with_q = p.q != nullptr && p.qbar != nullptr;
  const bool with_k = p.k != nullptr && p.kbar != nullptr;
  const int chq = p.G * D / 8, ntlq = 256 / chq;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (tid < 256) {
    if (with_q) {
      const __nv_bfloat16* qbase =
          p.q + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hq + h * p.G) * D + (tid % chq) * 8;
      const size_t qstride = static_cast<size_t>(p.Hq) * D;
      for (int t = tid / chq; t < 64; t += C::QR * ntlq) {
        uint4 v[C::QR];
        slab_load<C::QR>(v, qbase, qstride, t, ntlq);
        slab_add<C::QR>(acc, v, t, ntlq);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) partq[tid][e] = acc[e];
  } else if (with_k) {
    const int tk = tid - 256;
    const __nv_bfloat16* kbase =
        p.k + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D + (tk % C::CHK) * 8;
    const size_t kstride = static_cast<size_t>(p.Hkv) * D;
    constexpr int R = C::KR < C::QR ? C::KR : C::QR;
    for (int t = tk / C::CHK; t < 64; t += R * C::KTL) {
      uint4 v[R];
      slab_load<R>(v, kbase, kstride, t, C::KTL);
      slab_add<R>(acc, v, t, C::KTL);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) partk[tk][e] = acc[e];
  }
  __syncthreads();
  if (with_k) {
    for (int d = tid; d < D; d += C::THREADS) {
      float s = 0.f;
      for (int l = 0; l < C::KTL; ++l) s += partk[l * C::CHK + d / 8][d % 8];
      p.kbar[out_off + d] = s * (1.0f / 64.0f);
    }
  }
  if (with_q) {
    const float inv = 1.0f / (64.0f * static_cast<float>(p.G));
    for (int d = tid; d < D; d += C::THREADS) {
      float s = 0.f;
      for (int l = 0; l < ntlq; ++l)
        for (int g = 0; g < p.G; ++g) s += partq[l * chq + g * (D / 8) + d / 8][d % 8];
      p.qbar[out_off + d] = s * inv;
    }
  }
}

struct SelectParams {
  const float* qbar;
  const float* kbar;
  int32_t* idx;
  int n, topk;
  int i0, i1;  // rows i0 .. i1 - 1 (query blocks); the grid covers them in fours
};

constexpr int kSelectWarps = 4;

template <int D>
struct SelectConfig {
  static constexpr int CJ = (D == 64) ? 128 : 64;  // pooled-key rows per staged chunk
  static constexpr int RS = D + 4;                 // padded row stride in floats
  static constexpr int CHUNK_FLOATS = CJ * RS;
  static constexpr int KBUF_BYTES = 2 * CHUNK_FLOATS * 4;  // double buffer
  // dynamic shared memory for n query blocks
  static size_t smem_bytes(int n) { return KBUF_BYTES + static_cast<size_t>(kSelectWarps) * n * 4; }
};

// Order-preserving map of fp32 onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t f32_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One CTA per (b, h, four consecutive query blocks), one warp per query
// block i.
//  1. The CTA stages the pooled keys its rows need (rows 0 .. i_max - 1 of
//     (b, h)) through a double-buffered shared-memory chunk with cp.async,
//     all threads copying, so the loads overlap instead of forming one
//     warp's dependent chain.
//  2. score(i, j) = q_pooled[i] . k_pooled[j] in fp32 for j < i: lane l owns
//     the candidates j = l, l + 32, ... of each chunk; rows are padded by 4
//     floats so the lanes' 16-byte reads fall in distinct banks.  The scores
//     are kept as order-preserving keys in shared memory.
//  3. The (k-1)-th largest key T is found exactly by a 32-step radix search:
//     the largest T with #(key >= T) >= k-1, counted with one redux.sync per
//     step.  When n <= 32 * KPL each lane first moves its keys (j = lane +
//     32u) into registers, so a step is KPL compares and one redux; KPL = 0
//     reads them from shared memory (long sequences).
//  4. Chosen = {j : key > T} plus the lowest j with key == T up to k-1 in all
//     (higher score first, lower block index on ties), plus i itself; written
//     in ascending order and -1 padded.
template <int D, int KPL>
__global__ void __launch_bounds__(32 * kSelectWarps) block_select_kernel(const SelectParams p) {
  using C = SelectConfig<D>;
  extern __shared__ __align__(16) float sel_smem[];
  __shared__ float4 qs_all[kSelectWarps][D / 4];
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int i = p.i0 + static_cast<int>(blockIdx.x) * kSelectWarps + warp;
  const bool valid = i < p.i1;
  const bool active = valid && i + 1 > p.topk;  // needs a real selection
  int32_t* out = p.idx + (static_cast<size_t>(bh) * p.n + i) * p.topk;
  if (valid && !active)  // every causal block
    for (int r = lane; r < p.topk; r += 32) out[r] = (r <= i) ? r : -1;
  const int imax = min(p.i1 - 1, p.i0 + static_cast<int>(blockIdx.x) * kSelectWarps + kSelectWarps - 1);
  const int need_rows = (imax + 1 > p.topk) ? imax : 0;  // CTA-uniform
  if (need_rows == 0) return;

  float* kbuf = sel_smem;
  uint32_t* key = reinterpret_cast<uint32_t*>(sel_smem + 2 * C::CHUNK_FLOATS) + warp * p.n;
  float4* qs = qs_all[warp];
  if (active) {
    const float4* qrow =
        reinterpret_cast<const float4*>(p.qbar + (static_cast<size_t>(bh) * p.n + i) * D);
    for (int d4 = lane; d4 < D / 4; d4 += 32) qs[d4] = __ldg(qrow + d4);
  }
  const float* kb = p.kbar + static_cast<size_t>(bh) * p.n * D;
  const int nchunks = (need_rows + C::CJ - 1) / C::CJ;
  auto stage = [&](int c) {
    const int r0 = c * C::CJ;
    const int nr = min(C::CJ, need_rows - r0);
    float* dst = kbuf + (c & 1) * C::CHUNK_FLOATS;
    for (int x = threadIdx.x; x < nr * (D / 4); x += blockDim.x) {
      const int r = x / (D / 4), c4 = x % (D / 4);
      cp_async16(dst + r * C::RS + c4 * 4, kb + static_cast<size_t>(r0 + r) * D + c4 * 4);
    }
    cp_async_commit();
  };
  stage(0);
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) {
      stage(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (active) {
      const float* kc = kbuf + (c & 1) * C::CHUNK_FLOATS;
      const int r0 = c * C::CJ;
      const int nr = min(C::CJ, i - r0);  // this row's candidates in the chunk
      for (int u0 = lane; u0 < nr; u0 += 4 * 32) {
        float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
        for (int d4 = 0; d4 < D / 4; ++d4) {
          const float4 q4 = qs[d4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = u0 + 32 * u;
            if (r < nr) {
              const float4 k4 = *reinterpret_cast<const float4*>(kc + r * C::RS + d4 * 4);
              float& a = acc[u][d4 & 1];
              a = fmaf(q4.x, k4.x, a);
              a = fmaf(q4.y, k4.y, a);
              a = fmaf(q4.z, k4.z, a);
              a = fmaf(q4.w, k4.w, a);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (u0 + 32 * u < nr) key[r0 + u0 + 32 * u] = f32_order_key(acc[u][0] + acc[u][1]);
      }
    }
    __syncthreads();  // the buffer is refilled two chunks later
  }
  if (!active) return;
  __syncwarp();
  const unsigned need = static_cast<unsigned>(p.topk - 1);
  uint32_t T = 0;
  int written = 0;
  if constexpr (KPL > 0) {
    uint32_t kr[KPL];  // this lane's keys j = lane + 32u; 0 (below every real key) past i
#pragma unroll
    for (int u = 0; u < KPL; ++u) {
      const int j = lane + 32 * u;
      kr[u] = (j < i) ? key[j] : 0u;
    }
    // radix search for the (k-1)-th largest key
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned cnt = 0;
#pragma unroll
      for (int u = 0; u < KPL; ++u) cnt += (kr[u] >= cand) ? 1u : 0u;
      if (__reduce_add_sync(0xffffffffu, cnt) >= need) T = cand;
    }
    // ties at T: the lowest block indices first
    unsigned above = 0;
#pragma unroll
    for (int u = 0; u < KPL; ++u) above += (kr[u] > T) ? 1u : 0u;
    int ties_left = static_cast<int>(need) - static_cast<int>(__reduce_add_sync(0xffffffffu, above));
#pragma unroll
    for (int u = 0; u < KPL; ++u) {
      if (u * 32 > i) break;
      const int j = u * 32 + lane;
      const uint32_t kj = kr[u];
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
  } else {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned cnt = 0;
      for (int j = lane; j < i; j += 32) cnt += (key[j] >= cand) ? 1u : 0u;
      if (__reduce_add_sync(0xffffffffu, cnt) >= need) T = cand;
    }
    unsigned above = 0;
    for (int j = lane; j < i; j += 32) above += (key[j] > T) ? 1u : 0u;
    int ties_left = static_cast<int>(need) - static_cast<int>(__reduce_add_sync(0xffffffffu, above));
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
  }
  for (int r = written + lane; r < p.topk; r += 32) out[r] = -1;
}

}  // namespace ssa
