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
// One kernel, decode_kernel<D, G>, with a thread-block cluster of ns CTAs per
// (b, KV head):
//   selection  CTA r scores the r-th slice of the complete blocks (the
//              group-mean query against K-bar) and keeps the slice's top
//              k - 1 as candidates in its shared memory.  After a cluster
//              barrier every CTA reads all the cluster's candidates through
//              distributed shared memory and picks the same exact top k - 1,
//              so the table never goes through HBM.  Candidates are 64-bit
//              keys (order-preserving bits of the fp32 score, then ~j), so
//              ties go to the lower j and every key is distinct.
//   attention  each warp of the cluster takes every (ns * 4)-th entry of the
//              table (the warp that holds block c starts loading it before
//              the selection ends).  A warp streams its blocks' K and V
//              halves through a private ring of cp.async slots and runs the
//              block on the tensor cores with mma.sync m16n8k16: the G query
//              heads are the rows (padded to 16), S = Q K^T over the 64 keys,
//              an online softmax on the accumulator fragments, O += P V.
//   merge      each warp leaves (m, l, o) per head in shared memory; the CTA
//              merges its warps, and after a cluster barrier CTA 0 merges the
//              ns CTAs in rank order and writes o and the LSE.
//
// The block contractions are 16 x 64 x D, far below a tcgen05 tile (M >= 64
// rows of one operand); the warp-level MMA keeps the instruction count per
// block small so that the kernel stays bound by the HBM reads of K-bar and of
// the kept K/V blocks.
#pragma once

#include <cooperative_groups.h>

#include "sm100.cuh"

namespace ssa {

struct DecodeParams {
  int B, S, Hq, Hkv, G, n, topk;
  int ns;                         // CTAs per (b, KV head): the cluster size, 1..8
  int slice_cap;                  // complete blocks one CTA scores at most
  int cand_cap;                   // candidates of a whole cluster at most
  float scale_log2;               // softmax scale * log2(e)
  const __nv_bfloat16* q;         // [B][Hq][D]
  const __nv_bfloat16* k;         // [B][S][Hkv][D] cache
  const __nv_bfloat16* v;         // [B][S][Hkv][D] cache
  const float* kbar;              // [B][Hkv][n][D] mean keys (complete blocks are read)
  const int32_t* len;             // [B] cached tokens per sequence, 1..S
  int32_t* idx;                   // [B][Hkv][topk] kept blocks, ascending, -1 padded; or null
  __nv_bfloat16* o;               // [B][Hq][D]
  float* lse;                     // [B][Hq] natural log
};

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr int kDecodeSlots = 3;      // K or V halves of 64 rows in each warp's ring
constexpr int kDecodeMaxCluster = 8;
// Up to this many keys (one per thread) the top-k is picked by counting
// ranks; beyond, by a radix search.
constexpr int kDecodeRankMax = kDecodeThreads;

__host__ __device__ constexpr int decode_al16(int x) { return (x + 15) & ~15; }
__host__ __device__ constexpr int decode_imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int decode_imax(int a, int b) { return a > b ? a : b; }

// Dynamic shared memory of decode_kernel<D, G>, byte offsets.  A warp's ring
// also holds its partial (m, l, o) once its blocks are done.
struct DecodeSmem {
  int ring, qm, part, list, bits, skey, cand, gath, misc, total;
};

template <int D, int G>
__host__ __device__ inline DecodeSmem decode_smem(int n, int topk, int slice_cap, int cand_cap) {
  DecodeSmem L;
  int o = 0;
  L.ring = o;  o += kDecodeWarps * kDecodeSlots * 64 * D * 2;        // per warp: slots of 64 rows
  L.qm = o;    o += decode_al16(D * 4);                               // group-mean query
  L.part = o;  o += decode_al16(G * (D + 2) * 4);                     // the CTA's (m, l, o) per head
  L.list = o;  o += decode_al16(decode_imin(topk, n) * 4);           // the kept blocks
  L.bits = o;  o += decode_al16(((n + 31) / 32) * 4);                 // chosen blocks, a bit each
  L.skey = o;  o += decode_al16(8 * (slice_cap + 8));                 // this slice's 64-bit keys
  L.cand = o;  o += decode_al16(8 * decode_imin(topk - 1, slice_cap));  // its candidates
  L.gath = o;  o += decode_al16(8 * (cand_cap + 8));                  // the cluster's candidates
  L.misc = o;  o += decode_al16((256 + 4) * 4);                       // radix histogram, scratch
  L.total = o;
  return L;
}

__device__ __forceinline__ uint32_t dec_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Larger is better: the score's order key, then the lower block index.
__device__ __forceinline__ unsigned long long dec_comp(uint32_t key, int j) {
  return (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(j));
}
__device__ __forceinline__ int dec_comp_j(unsigned long long comp) {
  return static_cast<int>(~static_cast<uint32_t>(comp));
}

// The group-mean query of (b, h) into qm[D] (a CTA-wide loop; the caller
// synchronises before reading it).  The G loads of an entry are issued
// together, then summed in head order.
template <int D, int G>
__device__ __forceinline__ void decode_group_query(const DecodeParams& p, int b, int h, float* qm) {
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float x[G];
#pragma unroll
    for (int g = 0; g < G; ++g) x[g] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * D + d]);
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) s += x[g];
    qm[d] = s / static_cast<float>(G);
  }
}

// Scores of the complete blocks lo .. lo + m - 1 against the group-mean query,
// as 64-bit keys into skey[0 .. m).  A warp reads two consecutive K-bar rows
// (2 D fp32, contiguous) per load instruction, half a warp per row, and sums
// each row's partial dots over its half-warp by shuffles.  load() issues one
// batch of row pairs (pairs p0, p0 + 4, ...); consume() finishes it.
template <int D>
struct DecScorer {
  static constexpr int FL = D / 64;      // 16-byte loads per lane per row
  static constexpr int BATCH = 16 / FL;  // row pairs per warp per batch
  float4 v[BATCH][FL];
  __device__ __forceinline__ void load(const float* kb, int lo, int m, int p0) {
    const int lane = threadIdx.x & 31, half = lane >> 4, q = lane & 15;
#pragma unroll
    for (int bi = 0; bi < BATCH; ++bi) {
      const int row = 2 * (p0 + kDecodeWarps * bi) + half;
      const float4* rp = reinterpret_cast<const float4*>(kb + static_cast<size_t>(lo + (row < m ? row : 0)) * D);
#pragma unroll
      for (int f = 0; f < FL; ++f) v[bi][f] = __ldg(rp + q + 16 * f);
    }
  }
  __device__ __forceinline__ void consume(int lo, int m, int p0, const float* qm, unsigned long long* skey) {
    const int lane = threadIdx.x & 31, half = lane >> 4, q = lane & 15;
#pragma unroll
    for (int bi = 0; bi < BATCH; ++bi) {
      float acc = 0.f;
#pragma unroll
      for (int f = 0; f < FL; ++f) {
        const float4 qv = *reinterpret_cast<const float4*>(qm + 4 * (q + 16 * f));
        acc = fmaf(qv.x, v[bi][f].x, acc);
        acc = fmaf(qv.y, v[bi][f].y, acc);
        acc = fmaf(qv.z, v[bi][f].z, acc);
        acc = fmaf(qv.w, v[bi][f].w, acc);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const int row = 2 * (p0 + kDecodeWarps * bi) + half;
      if (q == 0 && row < m) skey[row] = dec_comp(dec_order_key(acc), lo + row);
    }
  }
};

// Rank of each key = keys above it (one key per thread, M <= kDecodeRankMax);
// the first `need` are emitted at their rank.  comp is padded with zeros to a
// multiple of 8 entries.
template <class Emit>
__device__ __forceinline__ void dec_rank_pick(const unsigned long long* comp, int M, int need, Emit emit) {
  const int i = threadIdx.x;
  const unsigned long long mine = i < M ? comp[i] : ~0ull;
  int rank = 0;
  const ulonglong2* c2 = reinterpret_cast<const ulonglong2*>(comp);
  for (int x = 0; x < (M + 7) / 8; ++x) {
    ulonglong2 pr[4];
#pragma unroll
    for (int y = 0; y < 4; ++y) pr[y] = c2[4 * x + y];
#pragma unroll
    for (int y = 0; y < 4; ++y) rank += (pr[y].x > mine) + (pr[y].y > mine);
  }
  if (i < M && rank < need) emit(i, rank);
}

// The top `need` of the M distinct 64-bit keys comp[0 .. M) (M <= need: all).
// emit(i, slot) is called once per chosen key with distinct slots
// 0 .. min(need, M) - 1.  comp[M .. M + 7] must be readable and 0 (below every
// key).  All threads of the CTA call it with the same M and need >= 1;
// `misc` holds 260 words of scratch.
template <class Emit>
__device__ void dec_pick(const unsigned long long* comp, int M, int need, Emit emit, unsigned* misc) {
  const int tid = threadIdx.x, lane = tid % 32;
  if (M <= need) {
    for (int i = tid; i < M; i += blockDim.x) emit(i, i);
    return;
  }
  if (M <= kDecodeRankMax) {
    dec_rank_pick(comp, M, need, emit);
    return;
  }
  // A threshold T with exactly `need` keys >= T, by a radix search over 8-bit
  // digits (most significant first): a histogram of the keys that match the
  // digits found so far, then warp 0 finds the digit d holding the wanted
  // rank.  If every key of d's bucket is wanted, T is the prefix with d and
  // zeros below, and the search stops; else it goes on inside the bucket.
  // Keys are distinct, so the last digit always ends it.
  unsigned* hist = misc;
  unsigned* sel = misc + 256;  // [0] digit, [1] rank left, [2] slots taken, [3] done
  unsigned long long T = 0ull, tmask = 0ull;
  unsigned rank = static_cast<unsigned>(need);
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int x = tid; x < 256; x += blockDim.x) hist[x] = 0u;
    __syncthreads();
    for (int i0 = 0; i0 < M; i0 += blockDim.x) {
      const int i = i0 + tid;
      const unsigned long long ki = i < M ? comp[i] : 0ull;
      const bool in = i < M && (ki & tmask) == T;
      const unsigned digit = in ? static_cast<unsigned>(ki >> shift) & 255u : 256u;  // 256: not counted
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], static_cast<unsigned>(__popc(peers)));
    }
    __syncthreads();
    if (tid < 32) {
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
        unsigned acc = excl;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          if (acc + cnt[x] >= rank) {
            sel[0] = static_cast<unsigned>(255 - 8 * lane - x);
            sel[1] = rank - acc;
            sel[3] = (rank - acc == cnt[x]) ? 1u : 0u;
            break;
          }
          acc += cnt[x];
        }
      }
      if (lane == 0) sel[2] = 0u;
    }
    __syncthreads();
    T |= static_cast<unsigned long long>(sel[0]) << shift;
    tmask |= 255ull << shift;
    rank = sel[1];
    const bool done = sel[3] != 0u;
    __syncthreads();  // sel and hist are rewritten by the next pass
    if (done) break;
  }
  for (int i = tid; i < M; i += blockDim.x)
    if (comp[i] >= T) emit(i, static_cast<int>(atomicAdd(&sel[2], 1u)));
}

__device__ __forceinline__ void dec_cp_async16(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void dec_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void dec_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void dec_ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// d += a b: A 16 x 16 bf16 (row), B 16 x 8 bf16 (col), D 16 x 8 fp32
__device__ __forceinline__ void dec_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t dec_pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// One cluster of ns CTAs (kDecodeWarps warps each) per (b, KV head); grid
// B * Hkv * ns, cluster (ns, 1, 1); dynamic shared memory
// decode_smem<D, G>(...).total.  Every thread runs the same cluster barriers
// and CTA barriers; with one CTA per (b, KV head) the cluster barriers become
// CTA barriers and the CTA writes its outputs itself.
//
// A warp's MMA fragments (lane = 4 qr + qc): rows qr and qr + 8 are query
// heads, so each lane holds two heads' running maximum and sum; columns
// 2 qc, 2 qc + 1 of each 8-wide tile are keys (S, P) or head-dim entries (O).
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const DecodeParams p) {
  namespace cg = cooperative_groups;
  constexpr int W = kDecodeWarps;
  constexpr int NSL = kDecodeSlots;
  constexpr int HALF = 64 * D * 2;     // bytes of 64 K or V rows
  constexpr int CH = D / 8;            // 16-byte chunks per row
  constexpr int KS = D / 16;           // k-steps of S = Q K^T
  constexpr int NT = D / 8;            // n-tiles of O
  static_assert(G >= 2 && G <= 16, "query heads per KV head");
  extern __shared__ __align__(128) uint8_t dsm[];
  cg::cluster_group cluster = cg::this_cluster();
  const DecodeSmem SL = decode_smem<D, G>(p.n, p.topk, p.slice_cap, p.cand_cap);
  uint8_t* ring = dsm + SL.ring;
  float* qm = reinterpret_cast<float*>(dsm + SL.qm);
  float* part = reinterpret_cast<float*>(dsm + SL.part);
  int* list = reinterpret_cast<int*>(dsm + SL.list);
  unsigned* bits = reinterpret_cast<unsigned*>(dsm + SL.bits);
  unsigned long long* skey = reinterpret_cast<unsigned long long*>(dsm + SL.skey);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(dsm + SL.cand);
  unsigned long long* gath = reinterpret_cast<unsigned long long*>(dsm + SL.gath);
  unsigned* misc = reinterpret_cast<unsigned*>(dsm + SL.misc);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int ns = p.ns;
  const int r = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / ns, b = bh / p.Hkv, h = bh % p.Hkv;
  const int len = p.len[b];
  const bool valid = len >= 1 && len <= p.S;
  const int t = len - 1, c = valid ? t / 64 : 0;
  const int need = p.topk - 1;
  const bool search = valid && c + 1 > p.topk;         // else every block 0..c is kept
  const int kept = !valid ? 0 : (search ? p.topk : c + 1);
  // this warp's table entries: gw, gw + NW, ...; entry kept - 1 (block c) is
  // its last if it has it, and then goes first, before the table exists
  const int NW = ns * W, gw = r * W + warp;
  const int nbw = kept > gw ? (kept - 1 - gw) / NW + 1 : 0;
  const bool wc = nbw > 0 && (kept - 1) % NW == gw;

  // half-step hh of this warp: the K (even) or V (odd) rows of its block
  // hh / 2 into slot hh % NSL, rows past the causal end zeroed; 16-byte chunk
  // x of row y sits at chunk x ^ (y & 7), so ldmatrix's eight rows hit
  // distinct banks
  const size_t rstride = static_cast<size_t>(p.Hkv) * D;
  const uint32_t wring = smem_u32(ring) + warp * (NSL * HALF);
  auto block_of = [&](int i) { return (wc && i == 0) ? c : list[gw + (wc ? i - 1 : i) * NW]; };
  auto issue = [&](int hh) {
    if (hh < 2 * nbw) {
      const int j = block_of(hh >> 1);
      const int nk = (j == c) ? t - 64 * c + 1 : 64;
      const uint32_t dst = wring + (hh % NSL) * HALF;
      const __nv_bfloat16* src = ((hh & 1) ? p.v : p.k) + ((static_cast<size_t>(b) * p.S + 64 * j) * p.Hkv + h) * D;
#pragma unroll 4
      for (int e = lane; e < 64 * CH; e += 32) {
        const int row = e / CH, x = e % CH;
        const uint32_t a = dst + row * (D * 2) + ((x ^ (row & 7)) * 16);
        if (row < nk)
          dec_cp_async16(a, src + row * rstride + x * 8);
        else
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
      }
    }
    dec_cp_commit();  // one group per half-step, empty past the end: the waits count half-steps
  };

  // block c's K and V go first, before the selection; so does the first
  // batch of this CTA's K-bar rows (slice lo .. lo + m - 1), while the
  // group-mean query forms
  const int pre = wc ? decode_imin(NSL - 1, 2) : 0;
  for (int hh = 0; hh < pre; ++hh) issue(hh);
  const bool scoring = search && need > 0;
  const int chunk = search ? (c + ns - 1) / ns : 0;
  const int lo = r * chunk;
  const int m = scoring ? decode_imax(0, decode_imin(c, lo + chunk) - lo) : 0;
  const float* kbh = p.kbar + static_cast<size_t>(bh) * p.n * D;
  DecScorer<D> scorer;
  if (m > 0) scorer.load(kbh, lo, m, warp);
  for (int x = tid; x < (p.n + 31) / 32; x += kDecodeThreads) bits[x] = 0u;
  if (scoring) decode_group_query<D, G>(p, b, h, qm);
  __syncthreads();

  // ---- selection, part 1: the top k - 1 of this CTA's slice
  if (m > 0) {
    const int np = (m + 1) / 2;
    for (int base = 0; base < np; base += kDecodeWarps * DecScorer<D>::BATCH) {
      if (base > 0) scorer.load(kbh, lo, m, base + warp);
      scorer.consume(lo, m, base + warp, qm, skey);
    }
    if (tid < 8) skey[m + tid] = 0ull;
    __syncthreads();
    if (ns == 1)  // the slice is every complete block: its top k - 1 is the answer
      dec_pick(
          skey, m, need,
          [&](int i, int) {
            const int j = dec_comp_j(skey[i]);
            atomicOr(&bits[j >> 5], 1u << (j & 31));
          },
          misc);
    else
      dec_pick(skey, m, need, [&](int i, int slot) { cand[slot] = skey[i]; }, misc);
  }
  // a cluster barrier only when there are other CTAs (it costs about a
  // microsecond even for a cluster of one)
  auto csync = [&]() {
    if (ns > 1)
      cluster.sync();
    else
      __syncthreads();
  };
  csync();  // every slice's candidates are in place

  // ---- selection, part 2: the exact top k - 1 of all candidates, in every CTA
  if (search && need > 0) {
    // candidates of CTA s: entries off[s] .. off[s] + nl[s] - 1 of gath, one
    // remote load each, all in flight together
    int off[kDecodeMaxCluster + 1];
    off[0] = 0;
#pragma unroll
    for (int s = 0; s < kDecodeMaxCluster; ++s) {
      const int ms = s < ns ? decode_imax(0, decode_imin(c, s * chunk + chunk) - s * chunk) : 0;
      off[s + 1] = off[s] + decode_imin(need, ms);
    }
    const int M = off[kDecodeMaxCluster];
    if (ns > 1) {
      for (int f = tid; f < M; f += kDecodeThreads) {
        int s = 0, base = 0;
#pragma unroll
        for (int x = 1; x < kDecodeMaxCluster; ++x)
          if (f >= off[x]) {
            s = x;
            base = off[x];
          }
        gath[f] = cluster.map_shared_rank(cand, s)[f - base];
      }
      if (tid < 8) gath[M + tid] = 0ull;
      __syncthreads();
      dec_pick(
          gath, M, need,
          [&](int i, int) {
            const int j = dec_comp_j(gath[i]);
            atomicOr(&bits[j >> 5], 1u << (j & 31));
          },
          misc);
      __syncthreads();
    }
    // the chosen blocks in ascending order, then c
    if (warp == 0) {
      const int words = (c + 31) / 32;
      int written = 0;
      for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        unsigned word = w < words ? bits[w] : 0u;
        const int cw = __popc(word);
        int incl = cw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int pos = written + incl - cw;
        while (word != 0u) {
          const int bit = __ffs(word) - 1;
          word &= word - 1u;
          if (pos < need) list[pos] = w * 32 + bit;
          ++pos;
        }
        written += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) list[need] = c;
    }
  } else if (search) {
    if (tid == 0) list[0] = c;  // top-k 1: the query's own block only
  } else if (valid) {
    for (int i = tid; i <= c; i += kDecodeThreads) list[i] = i;
  }
  __syncthreads();
  if (r == 0) {
    if (p.idx != nullptr)
      for (int i = tid; i < p.topk; i += kDecodeThreads)
        p.idx[static_cast<size_t>(bh) * p.topk + i] = i < kept ? list[i] : -1;
    if (!valid && tid == 0) {  // a length outside the cache: no block, error reported
      atomicOr(&g_error_word, kErrBadInput);
      atomicExch(&g_error_site, 0xd01);
    }
  }

  // ---- attention: this warp's blocks
  for (int hh = pre; hh < NSL - 1; ++hh) issue(hh);
  const int qr = lane >> 2, qc = lane & 3;
  // Q fragments (A, 16 x 16 per k-step): heads qr, qr + 8; zero rows past G
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qb = p.q + (static_cast<size_t>(b) * p.Hq + h * G) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int d0 = 16 * ks + 2 * qc;
      qa[ks][0] = qr < G ? *reinterpret_cast<const uint32_t*>(qb + qr * D + d0) : 0u;
      qa[ks][1] = qr + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (qr + 8) * D + d0) : 0u;
      qa[ks][2] = qr < G ? *reinterpret_cast<const uint32_t*>(qb + qr * D + d0 + 8) : 0u;
      qa[ks][3] = qr + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (qr + 8) * D + d0 + 8) : 0u;
    }
  }
  float oacc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads qr, qr + 8 (log2 units)
  uint32_t pa[4][4];  // P as A fragments, 4 k-steps of 16 keys
  const float sl2 = p.scale_log2;
  for (int hh = 0; hh < 2 * nbw; ++hh) {
    asm volatile("cp.async.wait_group %0;" ::"n"(NSL - 2) : "memory");
    __syncwarp();  // half-step hh's rows are in; every lane is past half-step hh - 1
    issue(hh + NSL - 1);
    const uint32_t sb = wring + (hh % NSL) * HALF;
    if ((hh & 1) == 0) {
      // S = Q K^T: n-tile nt is keys 8 nt .. 8 nt + 7; one ldmatrix.x4 gives
      // chunks 2 ks .. 2 ks + 3 of those eight key rows (two k-steps)
      const int j = block_of(hh >> 1);
      const int nk = (j == c) ? t - 64 * c + 1 : 64;
      float s[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        const int row = 8 * nt + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < KS; ks += 2) {
          const int x = 2 * ks + (lane >> 3);
          uint32_t b0, b1, b2, b3;
          dec_ldsm_x4(sb + row * (D * 2) + ((x ^ (row & 7)) * 16), b0, b1, b2, b3);
          dec_mma(s[nt], qa[ks], b0, b1);
          dec_mma(s[nt], qa[ks + 1], b2, b3);
        }
      }
      // online softmax per head row, in log2 units
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int key = 8 * nt + 2 * qc;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = key + e < nk;
          s[nt][e] = ok ? s[nt][e] * sl2 : -INFINITY;
          s[nt][2 + e] = ok ? s[nt][2 + e] * sl2 : -INFINITY;
          mx0 = fmaxf(mx0, s[nt][e]);
          mx1 = fmaxf(mx1, s[nt][2 + e]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float a0 = exp2f(m0 - n0), a1 = exp2f(m1 - n1);  // 0 on the first block
      m0 = n0;
      m1 = n1;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(s[nt][0] - n0), p1 = exp2f(s[nt][1] - n0);
        const float p2 = exp2f(s[nt][2] - n1), p3 = exp2f(s[nt][3] - n1);
        sum0 += p0 + p1;
        sum1 += p2 + p3;
        // n-tiles 2 kk and 2 kk + 1 are keys 16 kk .. 16 kk + 15 of P's k-step kk
        pa[nt >> 1][(nt & 1) * 2 + 0] = dec_pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = dec_pack_bf16(p2, p3);
      }
      l0 = fmaf(l0, a0, sum0);
      l1 = fmaf(l1, a1, sum1);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        oacc[nt][0] *= a0;
        oacc[nt][1] *= a0;
        oacc[nt][2] *= a1;
        oacc[nt][3] *= a1;
      }
    } else {
      // O += P V: k-step kk is keys 16 kk .. 16 kk + 15; one ldmatrix.x4.trans
      // gives the two key halves of chunks nd, nd + 1 (two n-tiles)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int row = 16 * kk + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
        for (int nd = 0; nd < NT; nd += 2) {
          const int x = nd + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          dec_ldsm_x4_t(sb + row * (D * 2) + ((x ^ (row & 7)) * 16), b0, b1, b2, b3);
          dec_mma(oacc[nd], pa[kk], b0, b1);
          dec_mma(oacc[nd + 1], pa[kk], b2, b3);
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();

  // ---- merge: the warp's partial into its own ring, then the CTA's, then the cluster's
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* wp = reinterpret_cast<float*>(ring + warp * (NSL * HALF));  // [G][D + 2]: m, l, o
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int g = qr + 8 * half;
    if (g < G) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float2*>(wp + g * (D + 2) + 2 + 8 * nt + 2 * qc) =
            make_float2(oacc[nt][2 * half], oacc[nt][2 * half + 1]);
      if (qc == 0) {
        wp[g * (D + 2)] = half ? m1 : m0;
        wp[g * (D + 2) + 1] = half ? l1 : l0;
      }
    }
  }
  __syncthreads();
  for (int it = tid; it < G * (D / 2); it += kDecodeThreads) {
    const int g = it / (D / 2), c2 = it % (D / 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, reinterpret_cast<const float*>(ring + w * (NSL * HALF))[g * (D + 2)]);
    float l = 0.f, o0 = 0.f, o1 = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float* pp = reinterpret_cast<const float*>(ring + w * (NSL * HALF)) + g * (D + 2);
        const float wt = exp2f(pp[0] - M);  // 0 for a warp without blocks
        l = fmaf(wt, pp[1], l);
        o0 = fmaf(wt, pp[2 + 2 * c2], o0);
        o1 = fmaf(wt, pp[3 + 2 * c2], o1);
      }
    }
    if (ns == 1) {
      // l == 0 only for a length the selection rejected: zeros and -inf
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t row = static_cast<size_t>(b) * p.Hq + h * G + g;
      *reinterpret_cast<__nv_bfloat162*>(p.o + row * D + 2 * c2) = __floats2bfloat162_rn(o0 * inv, o1 * inv);
      if (c2 == 0) p.lse[row] = l > 0.f ? (M + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      continue;
    }
    part[g * (D + 2) + 2 + 2 * c2] = o0;
    part[g * (D + 2) + 3 + 2 * c2] = o1;
    if (c2 == 0) {
      part[g * (D + 2)] = M;
      part[g * (D + 2) + 1] = l;
    }
  }
  if (ns == 1) return;  // uniform over the launch: no cluster barriers follow
  cluster.sync();  // every CTA's partial is in place
  if (r == 0) {
    for (int it = tid; it < G * (D / 2); it += kDecodeThreads) {
      const int g = it / (D / 2), c2 = it % (D / 2);
      float ms[kDecodeMaxCluster];
#pragma unroll
      for (int s = 0; s < kDecodeMaxCluster; ++s)
        ms[s] = s < ns ? cluster.map_shared_rank(part, s)[g * (D + 2)] : -INFINITY;
      float M = -INFINITY;
#pragma unroll
      for (int s = 0; s < kDecodeMaxCluster; ++s) M = fmaxf(M, ms[s]);
      float l = 0.f, o0 = 0.f, o1 = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int s = 0; s < kDecodeMaxCluster; ++s) {
          if (s < ns) {
            const float* pp = cluster.map_shared_rank(part, s) + g * (D + 2);
            const float wt = exp2f(ms[s] - M);  // 0 for a CTA without blocks
            l = fmaf(wt, pp[1], l);
            o0 = fmaf(wt, pp[2 + 2 * c2], o0);
            o1 = fmaf(wt, pp[3 + 2 * c2], o1);
          }
        }
      }
      // l == 0 only for a length the selection rejected: zeros and -inf
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t row = static_cast<size_t>(b) * p.Hq + h * G + g;
      *reinterpret_cast<__nv_bfloat162*>(p.o + row * D + 2 * c2) = __floats2bfloat162_rn(o0 * inv, o1 * inv);
      if (c2 == 0) p.lse[row] = l > 0.f ? (M + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  cluster.sync();  // the partials stay readable until CTA 0 has merged them
}

}  // namespace ssa
