// softmax_util.cuh -- pieces shared by the forward attention kernels: the
// parameter block, packed-fp32 helpers and the per-row online-softmax steps
// (row maximum, exp2 with the scale folded into one packed FMA, bf16 packing).
#pragma once

#include "sm100.cuh"

namespace ssa {

// Limits of the DashAttention path: chunks per sequence (the routed list of a
// query block lives in shared memory) and query heads per KV head.
constexpr int kDashMaxN = 1024;
constexpr int kDashMaxG = 16;

struct FwdParams {
  int B, S, Hq, Hkv, G, n, topk, slices;
  // the plain (persistent) sparse stream computes query blocks i_lo .. i_hi - 1
  // only (0 .. n - 1 from the C entry points); the other modes use 0, n
  int i_lo, i_hi;
  float scale_log2;  // softmax scale * log2(e)
  const int32_t* idx;
  __nv_bfloat16* o;      // sparse output
  float* lse;            // sparse log-sum-exp (natural log)
  __nv_bfloat16* o_full; // MASS: dense causal output
  float* lse_full;       // MASS
  float* dropped;        // MASS: dropped attention mass
  uint64_t timeout_ns;
  // early stop (sparse forward only): the pooled queries and keys that order
  // the visit, the stop threshold, and the blocks visited per M-tile
  const float* qbar;     // [B][Hkv][n][D]
  const float* kbar;     // [B][Hkv][n][D]
  float tau;
  int32_t* visited;      // [B][Hq][n], or null
  // DashAttention (prior-induced softmax): the routed chunks of each query
  // block as a bit mask, their group weights, and the prior strength
  const uint32_t* dmask; // [B][Hkv][n][ceil(n / 32)]
  const float* dw;       // [B][Hkv][n][n]
  float sigma;
};

__host__ __device__ constexpr int pow2_at_least(int x) {
  return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512;
}

// DashAttention: warp-wide decode of query block i's routed chunks (KV head
// h, batch b) into an ascending list with per-chunk biases sigma * log2 w_j,
// followed by the diagonal chunk i with bias 0; *count receives the length.
__device__ __forceinline__ void dash_build_list(const FwdParams& p, int b, int h, int i, int lane,
                                                int32_t* dord, float* dbias, int* dcount) {
  // only chunks before the diagonal whose bit is set and whose weight is
  // positive are visited, in ascending order, and the diagonal chunk last
  // (its own branch, bias 0) whatever its bit says.  Lane l holds mask word
  // l (n <= 32 * 32); the weights are read eight words at a time, coalesced,
  // and each word's chunks are placed with a ballot.
  const int W = (p.n + 31) / 32;
  const size_t rowid = (static_cast<size_t>(b) * p.Hkv + h) * p.n + i;
  const float* wrow = p.dw + rowid * p.n;
  const uint32_t myword = lane < W ? p.dmask[rowid * W + lane] : 0u;
  int base = 0;
  for (int w0 = 0; w0 * 32 < i; w0 += 8) {
    float wv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = (w0 + u) * 32 + lane;
      wv[u] = j < i ? wrow[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int wd = w0 + u;
      const uint32_t word = __shfl_sync(0xffffffffu, myword, wd & 31);
      const int j = wd * 32 + lane;
      const bool on = j < i && ((word >> lane) & 1u) != 0u && wv[u] > 0.f && wv[u] < INFINITY;
      const uint32_t bal = __ballot_sync(0xffffffffu, on);
      if (on) {
        const int pos = base + __popc(bal & ((1u << lane) - 1u));
        dord[pos] = j;
        dbias[pos] = p.sigma * log2f(wv[u]);
      }
      base += __popc(bal);
    }
  }
  if (lane == 0) {
    dord[base] = i;
    dbias[base] = 0.f;
    *dcount = base + 1;
  }
}

// Early stop: the visiting order of query block i (KV head h, batch b) into
// ord[0 .. nsel - 1], by the whole warp: the diagonal block i first, then the
// other selected blocks (idx_row[0 .. nsel - 2], all below i) by descending
// pooled score q_pooled[i] . k_pooled[j] in fp32, ties to the lower block.
// esc and ej are scratch of nsel - 1 entries.
template <int D>
__device__ __forceinline__ void early_visit_order(const FwdParams& p, int b, int h, int i, int nsel,
                                                  const int32_t* idx_row, int lane, int32_t* ord, float* esc,
                                                  int32_t* ej) {
  // visiting order: the diagonal block i first, then the other selected
  // blocks (idx_row[0 .. nsel - 2], all below i) by descending pooled score
  // q_pooled[i] . k_pooled[j] in fp32, ties to the lower block
  // Each lane holds D/32 values of the pooled query; eight rows' dot
  // products are in flight at once and summed across the warp.
  constexpr int QV = D / 32;
  const int ne = nsel - 1;
  const float* qb = p.qbar + ((static_cast<size_t>(b) * p.Hkv + h) * p.n + i) * D + lane * QV;
  const float* kb = p.kbar + (static_cast<size_t>(b) * p.Hkv + h) * p.n * D + lane * QV;
  float qf[QV];
#pragma unroll
  for (int c = 0; c < QV; ++c) qf[c] = __ldg(qb + c);
  for (int c0 = 0; c0 < ne; c0 += 32) {
    const int cnt = min(32, ne - c0);
    const int jl = lane < cnt ? idx_row[c0 + lane] : 0;
    if (lane < cnt) ej[c0 + lane] = jl;
    for (int r = 0; r < cnt; r += 8) {  // r + 7 <= 31
      float part[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        // clamped: a malformed table entry reads a valid row, not past the buffer
        const int ju = min(max(__shfl_sync(0xffffffffu, jl, r + u), 0), p.n - 1);
        const float* kr = kb + static_cast<size_t>(ju) * D;
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < QV; ++c) a = fmaf(qf[c], __ldg(kr + c), a);
        part[u] = a;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (lane == u && r + u < cnt) esc[c0 + r + u] = part[u];
    }
  }
  __syncwarp();
  for (int r = lane; r < ne; r += 32) {
    const float sr = esc[r];
    const int jr = ej[r];
    int rank = 0;
    for (int r2 = 0; r2 < ne; ++r2) rank += (esc[r2] > sr || (esc[r2] == sr && ej[r2] < jr)) ? 1 : 0;
    ord[1 + rank] = jr;
  }
  if (lane == 0) ord[0] = i;
  __syncwarp();
}

// Packed fp32 pair helpers (Blackwell f32x2 FMA-pipe instructions).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Row maximum of 32 raw scores; on the diagonal block keys past the row's own
// token (column c0 + c > tq) are excluded.  Four independent max3 chains keep
// the dependency depth short.
template <bool DIAG>
__device__ __forceinline__ float row_max32(const float* s, int c0, int tq, float m) {
  float x[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) x[c] = (DIAG && c0 + c > tq) ? -INFINITY : s[c];
  float m0 = max3f(m, x[0], x[1]), m1 = max3f(x[2], x[3], x[4]);
  float m2 = max3f(x[5], x[6], x[7]), m3 = max3f(x[8], x[9], x[10]);
#pragma unroll
  for (int c = 11; c + 7 < 32; c += 8) {
    m0 = max3f(m0, x[c], x[c + 1]);
    m1 = max3f(m1, x[c + 2], x[c + 3]);
    m2 = max3f(m2, x[c + 4], x[c + 5]);
    m3 = max3f(m3, x[c + 6], x[c + 7]);
  }
  // c = 27..31
  m0 = max3f(m0, x[27], x[28]);
  m1 = max3f(m1, x[29], x[30]);
  m2 = fmaxf(m2, x[31]);
  return max3f(m0, m1, fmaxf(m2, m3));
}

// 2^x for a pair of inputs on the FMA pipe, to take part of the softmax's
// exponentials off the MUFU unit.  x = j + f with j = round(x) and f in
// [-1/2, 1/2]: adding 1.5 * 2^23 rounds x to an integer held in the low
// mantissa bits, so j << 23 is those bits shifted into the exponent field;
// 2^f is a degree-3 polynomial whose coefficients were fitted to minimise the
// relative error on [-1/2, 1/2] by Lawson's iteratively reweighted least
// squares (maximum relative error 7.5e-5, well below half a bf16 ulp, 2^-9).
// Inputs below -125 are clamped: 2^-125 (about 2e-38) stands in for 0.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = f2_add(x, f2_pack(kRound, kRound));
  const uint64_t j = f2_add(t, f2_pack(-kRound, -kRound));            // round(x), exact
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), x);               // x - round(x), exact
  uint64_t q = f2_fma(f2_pack(0.0551716685f, 0.0551716685f), f, f2_pack(0.2426111400f, 0.2426111400f));
  q = f2_fma(q, f, f2_pack(0.6932609677f, 0.6932609677f));
  q = f2_fma(q, f, f2_pack(0.9999280572f, 0.9999280572f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// p = 2^(s * scale_log2 - m_ref) for 32 scores, summed into the pair
// accumulator (two independent partial sums) and packed to 16 bf16 pairs.
// POLY of every 8 pairs take the FMA-pipe polynomial instead of MUFU ex2
// (off the diagonal block only, where no score is masked): it pays where the
// softmax is bound by the MUFU rate (head_dim 128), not where it is bound by
// latency (head_dim 64).
template <bool DIAG, int POLY = 0>
__device__ __forceinline__ void exp_pack32(const float* s, int c0, int tq, uint64_t scale2,
                                           uint64_t negm2, uint64_t& acc, uint32_t* pk) {
  uint64_t acc_b = f2_pack(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const uint64_t x = f2_fma(f2_pack(s[c], s[c + 1]), scale2, negm2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    float p0, p1;
    if (DIAG) {
      if (c0 + c > tq) x0 = -INFINITY;
      if (c0 + c + 1 > tq) x1 = -INFINITY;
      p0 = ex2(x0);
      p1 = ex2(x1);
    } else if ((c / 2) % 8 >= 8 - POLY) {
      exp2_poly2(x0, x1, p0, p1);
    } else {
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    if ((c / 2) & 1) acc_b = f2_add(acc_b, f2_pack(p0, p1));
    else acc = f2_add(acc, f2_pack(p0, p1));
    pk[c / 2] = pack_bf16x2(p0, p1);
  }
  acc = f2_add(acc, acc_b);
}

// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core reads P through a shared-memory descriptor).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace ssa
