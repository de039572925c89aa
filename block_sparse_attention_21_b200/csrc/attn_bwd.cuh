// attn_bwd.cuh -- sparse attention backward: dQ, dK, dV over the selected
// (query block, key block) pairs only.
//
// The gradient of exact softmax attention restricted to the selected blocks
// ("Resumen Tecnico: SSA", section 1: tokens the sparse stream drops receive
// zero gradient; the top-k selection itself is not differentiated).  With
// P_ts = exp(scale q_t.k_s - LSE_t) from the forward's log-sum-exp:
//   D_t  = dO_t . O_t
//   dV_s = sum_t P_ts dO_t            dS_ts = P_ts (dO_t . v_s - D_t)
//   dK_s = scale sum_t dS_ts q_t      dQ_t  = scale sum_s dS_ts k_s
// where t runs over the query rows of every head of the KV head's group.
//
// Four launches, no floating-point atomics (results are deterministic):
//   bwd_prep_kernel    D_t for every row, and the reverse index: for each key
//                      block j the query blocks whose selection contains j,
//                      ascending (CSR in the workspace).
//   attn_bwd_dkdv_kernel  kDkdvSplit CTAs per (batch, KV head, key block j),
//                      sharing out the query tiles (query block x head pair)
//                      of j's reverse list; S = Q K_j^T and dP = dO V_j^T on
//                      tcgen05, the elementwise warps form P and dS into shared
//                      memory, then dV += P^T dO and dK += dS^T Q as M = 64 MMAs
//                      with both operands MN-major in shared memory; each CTA
//                      writes fp32 partial sums.
//   bwd_dkdv_reduce_kernel  adds the partials in a fixed order into dK, dV.
//   attn_bwd_dq_kernel one CTA per (batch, KV head, query block, head pairs):
//                      walks the selected blocks like the forward; dS goes to
//                      TMEM (columns of its own at head_dim 64, over S at 128)
//                      and dQ += dS K_j reads it as the A operand.
#pragma once

#include "sm100.cuh"
#include "softmax_util.cuh"

namespace ssa {

// The dK/dV work of one key block is split into this many CTAs (tile x goes
// to CTA x % kDkdvSplit), so the key blocks that many query blocks select do
// not leave one CTA running long after the rest; each CTA writes fp32 partial
// sums, which a reduction kernel adds in a fixed order.
constexpr int kDkdvSplit = 4;

struct BwdParams {
  int B, S, Hq, Hkv, G, n, topk, slices;
  int dense;         // 1: every causal block counts as selected (dense causal
                     // attention): no index table and no reverse index are read
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
  const __nv_bfloat16* o;
  const __nv_bfloat16* d_o;
  const float* lse;       // [B][Hq][S] natural log
  const int32_t* idx;     // [B][Hkv][n][topk]
  float* dt;              // workspace: D_t [B][Hq][S]
  int32_t* rev_off;       // workspace: [B][Hkv][n + 1]
  int32_t* rev;           // workspace: [B][Hkv][n * topk]
  float* part;            // workspace: [B][Hkv][n][kDkdvSplit][dV, dK][64][D]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint64_t timeout_ns;
};

__host__ __device__ inline size_t bwd_align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct BwdWorkspace {
  size_t dt, rev_off, rev, part, total;
};

__host__ __device__ inline BwdWorkspace bwd_workspace_layout(int B, int S, int Hq, int Hkv, int n,
                                                            int topk, int D) {
  BwdWorkspace w;
  w.dt = 0;
  w.rev_off = bwd_align256(static_cast<size_t>(B) * Hq * S * sizeof(float));
  w.rev = w.rev_off + bwd_align256(static_cast<size_t>(B) * Hkv * (n + 1) * sizeof(int32_t));
  w.part = w.rev + bwd_align256(static_cast<size_t>(B) * Hkv * n * topk * sizeof(int32_t));
  w.total = w.part + bwd_align256(static_cast<size_t>(B) * Hkv * n * kDkdvSplit * 2 * 64 * D * sizeof(float));
  return w;
}

// Index-table entries the reverse-index CTAs stage in shared memory at a time.
constexpr int kRevStage = 2048;
// Tokens of one (b, query head) per D_t CTA of bwd_prep_kernel.
constexpr int kDtRows = 256;

// Dynamic shared memory of bwd_prep_kernel for n key blocks.
__host__ __device__ inline size_t bwd_prep_smem(int n) {
  return static_cast<size_t>(2 * n + 1 + kRevStage) * sizeof(int32_t);
}

// Blocks 0 .. B*Hkv - 1: the reverse index of one (b, KV head); the rest: D_t.
//  - reverse index: for each key block j, the query blocks i whose selection
//    holds j, ascending (CSR).  Counts come from shared-memory atomics over
//    the table, offsets from a warp scan; then one warp walks the rows in
//    ascending i (staged through shared memory) and appends i to the list of
//    each of its blocks.  A row's blocks are distinct, so the lanes of one row
//    never touch the same list, and the lists come out in ascending order
//    without sorting: deterministic.
//  - D_t: kDtRows tokens of one (b, query head) per CTA; each row's D
//    elements are read by D / 8 lanes (16 B each) and reduced with shuffles;
//    every lane group has four rows' loads in flight.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p, int rev_blocks) {
  if (static_cast<int>(blockIdx.x) < rev_blocks) {
    extern __shared__ int32_t rsm[];
    const int n = p.n, k = p.topk;
    int32_t* off = rsm;             // [n + 1]: counts, then offsets
    int32_t* fill = off + n + 1;    // [n]
    int32_t* stage = fill + n;      // [kRevStage]
    const int bh = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int32_t* idx = p.idx + static_cast<size_t>(bh) * n * k;
    for (int j = threadIdx.x; j <= n; j += blockDim.x) off[j] = 0;
    for (int j = threadIdx.x; j < n; j += blockDim.x) fill[j] = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < n * k; e += blockDim.x) {
      const int j = idx[e];
      if (j >= 0 && j < n) atomicAdd(&off[j + 1], 1);
    }
    __syncthreads();
    if (warp == 0) {  // inclusive scan of off[1..n]
      const int per = (n + 31) / 32, base = 1 + lane * per;
      int sum = 0;
      for (int x = 0; x < per; ++x)
        if (base + x <= n) sum += off[base + x];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
      for (int x = 0; x < per; ++x)
        if (base + x <= n) {
          run += off[base + x];
          off[base + x] = run;
        }
    }
    __syncthreads();
    int32_t* goff = p.rev_off + static_cast<size_t>(bh) * (n + 1);
    for (int j = threadIdx.x; j <= n; j += blockDim.x) goff[j] = off[j];
    int32_t* rev = p.rev + static_cast<size_t>(bh) * n * k;
    const int rows_per_chunk = k <= kRevStage ? kRevStage / k : 1;
    for (int i0 = 0; i0 < n; i0 += rows_per_chunk) {
      const int rows = min(rows_per_chunk, n - i0);
      for (int e = threadIdx.x; e < rows * k; e += blockDim.x)
        stage[e] = idx[static_cast<size_t>(i0) * k + e];
      __syncthreads();
      if (warp == 0) {
        for (int ii = 0; ii < rows; ++ii) {
          for (int r = lane; r < k; r += 32) {
            const int j = stage[ii * k + r];
            if (j >= 0 && j < n) {
              rev[off[j] + fill[j]] = i0 + ii;
              fill[j] += 1;
            }
          }
          __syncwarp();
        }
      }
      __syncthreads();
    }
    return;
  }
  // ---- D_t: CTA c covers kDtRows consecutive tokens of one (b, query head),
  //      so the D_t writes are coalesced and no per-row index division is
  //      needed; each row's D elements are read by D / 8 lanes (16 B each) and
  //      reduced with shuffles, four steps' loads in flight.
  constexpr int LPR = D / 8;            // lanes per row
  constexpr int RPW = 32 / LPR;         // rows per warp per step
  constexpr int RPC = RPW * 8;          // rows per CTA per step (256 threads)
  constexpr int U = 4;                  // steps whose loads are in flight together
  const int c = static_cast<int>(blockIdx.x) - rev_blocks;
  const int tiles = (p.S + kDtRows - 1) / kDtRows;
  const int bhq = c / tiles;
  const int t0 = (c % tiles) * kDtRows;
  const int b = bhq / p.Hq, hq = bhq % p.Hq;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int sub = lane / LPR, part = lane % LPR;
  const size_t rstride = static_cast<size_t>(p.Hq) * D;
  const __nv_bfloat16* ob = p.o + (static_cast<size_t>(b) * p.S * p.Hq + hq) * D + part * 8;
  const __nv_bfloat16* gb = p.d_o + (static_cast<size_t>(b) * p.S * p.Hq + hq) * D + part * 8;
  float* dtrow = p.dt + static_cast<size_t>(bhq) * p.S;
  for (int s0 = 0; s0 < kDtRows; s0 += U * RPC) {
    uint4 a[U], g[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + s0 + u * RPC + warp * RPW + sub;
      if (t < p.S) {
        a[u] = *reinterpret_cast<const uint4*>(ob + static_cast<size_t>(t) * rstride);
        g[u] = *reinterpret_cast<const uint4*>(gb + static_cast<size_t>(t) * rstride);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + s0 + u * RPC + warp * RPW + sub;
      float acc = 0.f;
      if (t < p.S) {
        const uint32_t wa[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, wg[4] = {g[u].x, g[u].y, g[u].z, g[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(__uint_as_float(wa[e] << 16), __uint_as_float(wg[e] << 16), acc);
          acc = fmaf(__uint_as_float(wa[e] & 0xFFFF0000u), __uint_as_float(wg[e] & 0xFFFF0000u), acc);
        }
      }
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (t < p.S && part == 0) dtrow[t] = acc;
    }
  }
}

template <int D>
struct DkdvConfig {
  static constexpr int NP = D / 64;
  static constexpr int QTILE = 128 * D * 2;    // Q or dO tile: 128 rows = 2 heads x 64 tokens
  static constexpr int KVT = 64 * D * 2;       // K or V block
  static constexpr int PTILE = 128 * 64 * 2;   // P or dS tile
  static constexpr int NQ = 2;                 // Q/dO ring stages
  static constexpr int TMEM_COLS = pow2_at_least(128 + 2 * D);
  static constexpr int THREADS = 256;          // warp 0 producer, 1-2 issuers, 4..7 elementwise
  static constexpr int NBARS = 1 + 2 * NQ + 7;
  // no alignment slack: the dynamic shared memory of a kernel without static
  // shared memory starts 1024-byte aligned (the kernel checks it), which lets
  // two CTAs share an SM at head_dim 64 (TMEM 256 columns each)
  static constexpr int SMEM_BYTES = 2 * KVT + NQ * 2 * QTILE + 2 * PTILE + NBARS * 8 + 16;
  static constexpr int MIN_CTAS = (TMEM_COLS <= 256 && SMEM_BYTES + 1024 <= 116736) ? 2 : 1;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// kDkdvSplit CTAs per (batch b, KV head h, key block j), CTA sp taking tiles
// sp, sp + kDkdvSplit, ... of j's list.  TMEM: S at +0 and dP at +64
// (128 lanes x 64 fp32 each), then one M = 128, N = 2D accumulator at +128:
// dV and dK come from a single MMA per K-step with the operands stacked,
//   A = [P^T ; dS^T]  (128 x 16: the P tile then the dS tile, MN-major)
//   B = [Q | dO]      (16 x 2D: the Q tile then the dO tile, MN-major)
// so lanes 0..63 hold P^T Q | P^T dO and lanes 64..127 dS^T Q | dS^T dO:
// dV = P^T dO sits in lanes 0..63, columns D..2D-1, and dK = dS^T Q in lanes
// 64..127, columns 0..D-1 (the other two quadrants are discarded).  One
// M = 128 MMA in place of two M = 64 ones halves the instructions of this
// step, which is bound by their issue, at the cost of tensor work that is
// not used.  Key row r of dV is lane r, of dK lane 64 + r.
template <int D>
__global__ void __launch_bounds__(256, DkdvConfig<D>::MIN_CTAS)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const BwdParams p) {
  using C = DkdvConfig<D>;
  constexpr int NP = C::NP, QTILE = C::QTILE, KVT = C::KVT, PTILE = C::PTILE, NQ = C::NQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) {
      atomicOr(&g_error_word, kErrTimeout);
      atomicExch(&g_error_site, 0x8fe);
    }
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;
  uint8_t* sV = sK + KVT;
  // stage qs holds its Q tile, then its dO tile: the B operand [Q | dO] of
  // the dV/dK MMA steps through the 64-column panels of both at one stride
  uint8_t* sQ = sV + KVT;              // [NQ][Q tile, dO tile]
  uint8_t* sdO = sQ + QTILE;
  uint8_t* sP = sQ + NQ * 2 * QTILE;   // P tile, then dS tile
  uint8_t* sdS = sP + PTILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + PTILE);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;      // [NQ]
  uint64_t* q_empty = q_full + NQ;     // [NQ]
  uint64_t* s_full = q_empty + NQ;     // S and dP of a tile in TMEM
  uint64_t* s_free = s_full + 1;       // ... read by the elementwise warps
  uint64_t* p_full = s_free + 1;       // P and dS in shared memory
  uint64_t* p_done = p_full + 1;       // dV, dK MMAs of the tile completed
  uint64_t* o_done = p_done + 1;       // all MMAs completed
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int sp = blockIdx.x % kDkdvSplit;  // this CTA's share: tiles sp, sp + kDkdvSplit, ...
  const int bhn = blockIdx.x / kDkdvSplit;
  const int j = bhn % p.n;
  const int h = (bhn / p.n) % p.Hkv;
  const int b = bhn / (p.n * p.Hkv);
  const int HP = p.G / 2;                                   // head pairs per group
  const size_t bh = static_cast<size_t>(b) * p.Hkv + h;
  const int32_t* off = p.rev_off + bh * (p.n + 1);
  const int32_t* rev = p.rev + bh * p.n * p.topk;
  // query blocks whose selection holds j: the reverse list, or all i >= j (dense)
  const int first_q = p.dense ? 0 : off[j];
  const int nq = p.dense ? (p.n - j) : (off[j + 1] - first_q);
  const int ntiles_all = nq * HP;
  const int ntiles = ntiles_all > sp ? (ntiles_all - sp + kDkdvSplit - 1) / kDkdvSplit : 0;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 2);  // released by both issuers
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(p_done, 1);
    mbar_init(o_done, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      mbar_arrive_expect_tx(kv_full, 2 * KVT);
      for (int pn = 0; pn < NP; ++pn) {
        tma_load_4d(sK + pn * (64 * 128), &tm_k, kv_full, 64 * pn, h, 64 * j, b);
        tma_load_4d(sV + pn * (64 * 128), &tm_v, kv_full, 64 * pn, h, 64 * j, b);
      }
      int issued = 0;
      for (int x = 0; x < ntiles; ++x) {
        const int qs = x % NQ;
        if (x >= NQ && !mbar_wait(&q_empty[qs], ((x / NQ) - 1) & 1, abort_flag, tmo, 0x801)) break;
        const int gx = sp + x * kDkdvSplit;
        const int i = p.dense ? j + gx / HP : rev[first_q + gx / HP];
        const int hq0 = h * p.G + 2 * (gx % HP);
        mbar_arrive_expect_tx(&q_full[qs], 2 * QTILE);
        for (int hh = 0; hh < 2; ++hh)
          for (int pn = 0; pn < NP; ++pn) {
            tma_load_4d(sQ + qs * 2 * QTILE + pn * (128 * 128) + hh * (64 * 128), &tm_q, &q_full[qs],
                        64 * pn, hq0 + hh, 64 * i, b);
            tma_load_4d(sdO + qs * 2 * QTILE + pn * (128 * 128) + hh * (64 * 128), &tm_do, &q_full[qs],
                        64 * pn, hq0 + hh, 64 * i, b);
          }
        ++issued;
      }
      if (*abort_flag) {  // loads already issued land before the CTA exits
        volatile int never = 0;
        mbar_wait(kv_full, 0, &never, 1000000ull, 0x8ff);
        for (int x = (issued > NQ ? issued - NQ : 0); x < issued; ++x)
          mbar_wait(&q_full[x % NQ], (x / NQ) & 1, &never, 1000000ull, 0x8ff);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Two issuing threads, so that the issue cost of one tile's dV/dK MMAs
    // overlaps that of the next tile's S and dP (each thread's tcgen05.mma
    // issue, not the tensor pipe, bounds this kernel):
    //   warp 1  S(x+1) = Q K^T and dP(x+1) = dO V^T once the elementwise
    //           warps hold tile x's (they write TMEM columns 0..127 only)
    //   warp 2  the dV/dK MMAs of tile x once P(x) and dS(x) are in shared
    //           memory (they write the accumulator at column 128 only)
    // Each releases a Q/dO stage once its own MMAs on it have completed.
    if (lane == 0 && ntiles > 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO),
                     aP = smem_u32(sP);
      bool ok = true;
      if (warp == 1) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false);
        const uint32_t tS = tmem, tdP = tmem + 64;
        auto issue_scores = [&](int x) {
          const int qs = x % NQ;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            const uint32_t ok_ = (kk / 4) * (64 * 128) + (kk % 4) * 32;
            mma_ss(tS, sdesc_sw128(aQ + qs * 2 * QTILE + o, 16, 1024), sdesc_sw128(aK + ok_, 16, 1024),
                   idesc_s, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            const uint32_t ok_ = (kk / 4) * (64 * 128) + (kk % 4) * 32;
            mma_ss(tdP, sdesc_sw128(adO + qs * 2 * QTILE + o, 16, 1024), sdesc_sw128(aV + ok_, 16, 1024),
                   idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          tc_commit(&q_empty[qs]);  // this thread's reads of the stage
        };
        ok = mbar_wait(kv_full, 0, abort_flag, tmo, 0x901) && mbar_wait(&q_full[0], 0, abort_flag, tmo, 0x902);
        if (ok) {
          tc_fence_after();
          issue_scores(0);
        }
        for (int x = 0; ok && x + 1 < ntiles; ++x) {
          // the next tile's S and dP once the elementwise warps hold this one's
          if (!mbar_wait(s_free, x & 1, abort_flag, tmo, 0x903) ||
              !mbar_wait(&q_full[(x + 1) % NQ], ((x + 1) / NQ) & 1, abort_flag, tmo, 0x904)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_scores(x + 1);
        }
      } else {
        // M = 128 (P^T over dS^T), N = 2D (Q then dO), both operands MN-major
        // (bit 15: A, bit 16: B)
        constexpr uint32_t idesc_kv = idesc_bf16_f32(128, 2 * D, true) | (1u << 15);
        const uint32_t tKV = tmem + 128;
        for (int x = 0; ok && x < ntiles; ++x) {
          const int qs = x % NQ;
          if (!mbar_wait(p_full, x & 1, abort_flag, tmo, 0x905) ||
              !mbar_wait(&q_full[qs], (x / NQ) & 1, abort_flag, tmo, 0x906)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // [P^T ; dS^T] [Q | dO] over the tile's 128 rows (8 K-steps of 16
          // rows = 2048 B): A's second 64-row chunk (dS) sits PTILE after the
          // first (P), B's 64-column panels (Q, then dO) are 128 x 128 B apart
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (x > 0 || kk > 0) ? 1u : 0u;
            mma_ss(tKV, sdesc_sw128(aP + kk * 2048, PTILE, 1024),
                   sdesc_sw128(aQ + qs * 2 * QTILE + kk * 2048, 128 * 128, 1024), idesc_kv, acc);
          }
          tc_commit(p_done);
          tc_commit(&q_empty[qs]);
        }
        if (ok) tc_commit(o_done);
      }
      if (!ok) {
        // every MMA this thread issued completes before TMEM is released
        uint64_t* dr = &drain[warp - 1];
        tc_commit(dr);
        volatile int never = 0;
        mbar_wait(dr, 0, &never, tmo, 0x9ff);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- elementwise warps
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int hh = r / 64, tq = r % 64;
    const uint32_t row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint8_t* prow = sP + r * 128;
    uint8_t* dsrow = sdS + r * 128;
    constexpr float kLog2e = 1.4426950408889634f;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int x = 0; x < ntiles; ++x) {
      const int gx = sp + x * kDkdvSplit;
      const int i = p.dense ? j + gx / HP : rev[first_q + gx / HP];
      const int hq = h * p.G + 2 * (gx % HP) + hh;
      const size_t lrow = (static_cast<size_t>(b) * p.Hq + hq) * p.S + 64 * i + tq;
      const float nlse = -p.lse[lrow] * kLog2e;
      const float dt = p.dt[lrow];
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, x & 1, abort_flag, tmo, 0xa01))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld32_to(row, s);
      tmem_ld32_to(row + 32, s + 32);
      tmem_ld32_to(row + 64, dp);
      tmem_ld32_to(row + 96, dp + 32);
      tc_fence_before();
      mbar_arrive(s_free);
      const bool diag = (i == j);
      uint32_t pp[32], dd[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float p0 = ex2(fmaf(s[c], sl2, nlse)), p1 = ex2(fmaf(s[c + 1], sl2, nlse));
        if (diag) {
          if (c > tq) p0 = 0.f;
          if (c + 1 > tq) p1 = 0.f;
        }
        pp[c / 2] = pack_bf16x2(p0, p1);
        dd[c / 2] = pack_bf16x2(p0 * (dp[c] - dt), p1 * (dp[c + 1] - dt));
      }
      if (x > 0 && !__all_sync(0xffffffffu, mbar_wait(p_done, (x - 1) & 1, abort_flag, tmo, 0xa02))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const int sw = (cc ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pp[4 * cc], pp[4 * cc + 1], pp[4 * cc + 2], pp[4 * cc + 3]);
        *reinterpret_cast<uint4*>(dsrow + sw) = make_uint4(dd[4 * cc], dd[4 * cc + 1], dd[4 * cc + 2], dd[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(p_full);
    }
    // ---------------------------------------------------------- epilogue
    // lanes 0..63 (warps wq 0, 1) hold dV's key rows in columns D..2D-1,
    // lanes 64..127 (wq 2, 3) dK's in columns 0..D-1: this CTA's fp32 partial
    // sums of dV and dK (dK not yet scaled)
    const int which = wq / 2;                  // 0: dV, 1: dK
    const int kr = 32 * (wq % 2) + lane;       // key row
    float* part = p.part + (static_cast<size_t>(bhn) * kDkdvSplit + sp) * 2 * 64 * D;
    float* out_row = part + (which * 64 + kr) * D;
    if (ntiles == 0) {
      for (int d = 0; d < D; d += 4)
        *reinterpret_cast<float4*>(out_row + d) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, 0, abort_flag, tmo, 0xa03))) {
      tc_fence_after();
      const uint32_t base = row + 128 + (which == 0 ? D : 0);
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        float o[32];
        tmem_ld32(base + ch * 32, o);
        float4* out = reinterpret_cast<float4*>(out_row + ch * 32);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          out[v4] = make_float4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// dV = sum of the kDkdvSplit partials, dK = scale * sum, in a fixed order
// (deterministic); one CTA per (b, KV head, key block).
template <int D>
__global__ void __launch_bounds__(256) bwd_dkdv_reduce_kernel(const BwdParams p) {
  const int bhn = blockIdx.x;
  const int j = bhn % p.n, h = (bhn / p.n) % p.Hkv, b = bhn / (p.n * p.Hkv);
  constexpr int PER = 2 * 64 * D / 4;  // float4 per partial
  const float4* part = reinterpret_cast<const float4*>(p.part + static_cast<size_t>(bhn) * kDkdvSplit * 2 * 64 * D);
  for (int e = threadIdx.x; e < PER; e += blockDim.x) {
    float4 a = part[e];
#pragma unroll
    for (int x = 1; x < kDkdvSplit; ++x) {
      const float4 c = part[x * PER + e];
      a.x += c.x;
      a.y += c.y;
      a.z += c.z;
      a.w += c.w;
    }
    const int which = e / (64 * D / 4);  // 0: dV, 1: dK
    const int rem = e % (64 * D / 4);
    const int kr = rem / (D / 4), d4 = rem % (D / 4);
    const float mul = which ? p.scale : 1.f;
    __nv_bfloat16* dst = (which ? p.dk : p.dv) + ((static_cast<size_t>(b) * p.S + 64 * j + kr) * p.Hkv + h) * D + 4 * d4;
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(a.x * mul, a.y * mul), pack_bf16x2(a.z * mul, a.w * mul));
  }
}

template <int D, int T_>
struct DqConfig {
  static constexpr int T = T_;                 // M-tiles (head pairs) per CTA
  static constexpr int NP = D / 64;
  static constexpr int QTILE = 128 * D * 2;
  static constexpr int KVT = 64 * D * 2;
  static constexpr int NS = (D == 64) ? 4 : 2;
  // SEP: dS in TMEM columns of its own (S +0, dP +64, dQ +128, dS +128 + D),
  // so the next block's S and dP need only wait for S and dP to be read;
  // else dS over S's first columns (S +0, dP +64, dQ +128)
  static constexpr bool SEP = (D == 64);
  static constexpr int DS_COL = 128 + D;
  static constexpr int TSTRIDE = 128 + D + (SEP ? 32 : 0);
  static constexpr int TMEM_COLS = pow2_at_least(T * TSTRIDE);
  static constexpr int THREADS = 128 * (T + 1);
  static constexpr int NBARS = 1 + 3 * NS + 5 * T + 1;
  static constexpr int SMEM_BYTES = 1024 + 2 * T * QTILE + 2 * NS * KVT + NBARS * 8 + 16;
  // two CTAs share an SM when both fit in TMEM and shared memory: one CTA's
  // prologue and epilogue overlap the other's main loop
  static constexpr int MIN_CTAS = (TMEM_COLS <= 256 && SMEM_BYTES + 1024 <= 116736) ? 2 : 1;
  static_assert(T * TSTRIDE <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// One CTA per (batch b, KV head h, query block i, T head pairs of h's group).
// For each selected block jj (in the index table's order) and tile t:
//   issuer:      wait dS_t(jj);  dQ_t += dS_t(jj) K(jj);  S_t = Q_t K(jj+1)^T,
//                dP_t = dO_t V(jj+1)^T
//   elementwise: S_t, dP_t -> P = exp2(S scale log2e - LSE log2e),
//                dS = P (dP - D) -> bf16 into TMEM.
// At head_dim 64 (SEP) dS has TMEM columns of its own: the issuer issues
// S(jj+1) and dP(jj+1) as soon as the elementwise warps have loaded S(jj) and
// dP(jj) (s_free), then dQ(jj) once dS(jj) is stored; the elementwise warps
// store dS(jj+1) once the dQ MMAs of jj have read dS(jj) (ds_free).  So the
// next block's score MMAs overlap this block's exponentials.  At head_dim 128
// dS goes over S's first 32 columns, and S(jj+1) is issued after dQ(jj) (the
// tensor pipe runs one thread's MMAs in issue order).
template <int D, int T_>
__global__ void __launch_bounds__(DqConfig<D, T_>::THREADS, DqConfig<D, T_>::MIN_CTAS)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p) {
  using C = DqConfig<D, T_>;
  constexpr int T = C::T, NP = C::NP, QTILE = C::QTILE, KVT = C::KVT, NS = C::NS, TS = C::TSTRIDE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                  // [T][QTILE]
  uint8_t* sdO = sQ + T * QTILE;       // [T][QTILE]
  uint8_t* sK = sdO + T * QTILE;       // [NS][KVT]
  uint8_t* sV = sK + NS * KVT;         // [NS][KVT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NS * KVT);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;       // [NS]
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* s_full = kv_empty + NS;    // [T]
  uint64_t* ds_full = s_full + T;      // [T]
  uint64_t* q_done = ds_full + T;      // [T] last dQ MMA completed
  uint64_t* s_free = q_done + T;       // [T] SEP: S and dP read into registers
  uint64_t* ds_free = s_free + T;      // [T] SEP: the dQ MMAs of the block read dS
  uint64_t* drain = ds_free + T;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int per_i = p.B * p.Hkv * p.slices;
  const int i = p.n - 1 - static_cast<int>(blockIdx.x) / per_i;
  int rem = static_cast<int>(blockIdx.x) % per_i;
  const int slice = rem % p.slices;
  rem /= p.slices;
  const int h = rem % p.Hkv;
  const int b = rem / p.Hkv;
  const int hq0 = h * p.G + slice * 2 * T;
  const int nblk = min(p.topk, i + 1);
  const int32_t* idx_row = p.idx + ((static_cast<size_t>(b) * p.Hkv + h) * p.n + i) * p.topk;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < T; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&ds_full[t], 128);
      mbar_init(&q_done[t], 1);
      mbar_init(&s_free[t], 128);
      mbar_init(&ds_free[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * T * QTILE);
      for (int t = 0; t < T; ++t)
        for (int hh = 0; hh < 2; ++hh)
          for (int pn = 0; pn < NP; ++pn) {
            const uint32_t o = t * QTILE + pn * (128 * 128) + hh * (64 * 128);
            tma_load_4d(sQ + o, &tm_q, q_full, 64 * pn, hq0 + 2 * t + hh, 64 * i, b);
            tma_load_4d(sdO + o, &tm_do, q_full, 64 * pn, hq0 + 2 * t + hh, 64 * i, b);
          }
      int issued = 0;
      for (int jj = 0; jj < nblk; ++jj) {
        const int st = jj % NS, use = jj / NS;
        if (use > 0 && !mbar_wait(&kv_empty[st], (use - 1) & 1, abort_flag, tmo, 0xb01)) break;
        const int j = p.dense ? jj : idx_row[jj];
        mbar_arrive_expect_tx(&k_full[st], KVT);
        for (int pn = 0; pn < NP; ++pn)
          tma_load_4d(sK + st * KVT + pn * (64 * 128), &tm_k, &k_full[st], 64 * pn, h, 64 * j, b);
        mbar_arrive_expect_tx(&v_full[st], KVT);
        for (int pn = 0; pn < NP; ++pn)
          tma_load_4d(sV + st * KVT + pn * (64 * 128), &tm_v, &v_full[st], 64 * pn, h, 64 * j, b);
        ++issued;
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int jj = (issued > NS ? issued - NS : 0); jj < issued; ++jj)
          mbar_wait(&v_full[jj % NS], (jj / NS) & 1, &never, 1000000ull, 0xbff);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true);  // B = K block, MN-major
      const uint32_t aQ = smem_u32(sQ), adO = smem_u32(sdO), aK = smem_u32(sK), aV = smem_u32(sV);
      auto issue_scores = [&](int t, int st) {
        const uint32_t tS = tmem + t * TS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oq = t * QTILE + (kk / 4) * (128 * 128) + (kk % 4) * 32;
          const uint32_t ok_ = st * KVT + (kk / 4) * (64 * 128) + (kk % 4) * 32;
          mma_ss(tS, sdesc_sw128(aQ + oq, 16, 1024), sdesc_sw128(aK + ok_, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oq = t * QTILE + (kk / 4) * (128 * 128) + (kk % 4) * 32;
          const uint32_t ok_ = st * KVT + (kk / 4) * (64 * 128) + (kk % 4) * 32;
          mma_ss(tS + 64, sdesc_sw128(adO + oq, 16, 1024), sdesc_sw128(aV + ok_, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, tmo, 0xc01) &&
                mbar_wait(&k_full[0], 0, abort_flag, tmo, 0xc02) &&
                mbar_wait(&v_full[0], 0, abort_flag, tmo, 0xc03);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < T; ++t) {
          issue_scores(t, 0);
          tc_commit(&s_full[t]);
        }
      }
      for (int jj = 0; ok && jj < nblk; ++jj) {
        const int st = jj % NS;
        const bool more = jj + 1 < nblk;
        const int st1 = (jj + 1) % NS;
        if (more && (!mbar_wait(&k_full[st1], ((jj + 1) / NS) & 1, abort_flag, tmo, 0xc04) ||
                     !mbar_wait(&v_full[st1], ((jj + 1) / NS) & 1, abort_flag, tmo, 0xc05)))
          break;
        for (int t = 0; t < T; ++t) {
          const uint32_t tS = tmem + t * TS;
          if (C::SEP && more) {
            // the next block's S and dP once this block's are in registers
            if (!mbar_wait(&s_free[t], jj & 1, abort_flag, tmo, 0xc07)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_scores(t, st1);
            tc_commit(&s_full[t]);
          }
          if (!mbar_wait(&ds_full[t], jj & 1, abort_flag, tmo, 0xc06)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_sw128(aK + st * KVT + kk * (16 * 128), 64 * 128, 1024);
            mma_ts(tS + 128, tS + (C::SEP ? C::DS_COL : 0) + kk * 8, bd, idesc_dq, (jj == 0 && kk == 0) ? 0u : 1u);
          }
          if (!more) {
            tc_commit(&q_done[t]);
          } else if (C::SEP) {
            tc_commit(&ds_free[t]);
          } else {
            issue_scores(t, st1);
            tc_commit(&s_full[t]);
          }
        }
        if (!ok) break;
        tc_commit(&kv_empty[st]);
      }
      if (!ok || *abort_flag) {
        tc_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, tmo, 0xcff);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- elementwise warps
    const int t = (warp - 4) / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int hh = r / 64, tq = r % 64;
    const int hq = hq0 + 2 * t + hh;
    const int tok = 64 * i + tq;
    const uint32_t row = tmem + (static_cast<uint32_t>(wq * 32) << 16) + t * TS;
    constexpr float kLog2e = 1.4426950408889634f;
    const float sl2 = p.scale_log2;
    const size_t lrow = (static_cast<size_t>(b) * p.Hq + hq) * p.S + tok;
    const float nlse = -p.lse[lrow] * kLog2e;
    const float dt = p.dt[lrow];
    bool ok = true;
    for (int jj = 0; jj < nblk; ++jj) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], jj & 1, abort_flag, tmo, 0xd01))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld32_to(row, s);
      tmem_ld32_to(row + 32, s + 32);
      tmem_ld32_to(row + 64, dp);
      tmem_ld32_to(row + 96, dp + 32);
      if (C::SEP) {  // S and dP are in registers: the next block's may be issued
        tc_fence_before();
        mbar_arrive(&s_free[t]);
      }
      const bool diag = (jj == nblk - 1);
      uint32_t dd[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float p0 = ex2(fmaf(s[c], sl2, nlse)), p1 = ex2(fmaf(s[c + 1], sl2, nlse));
        if (diag) {
          if (c > tq) p0 = 0.f;
          if (c + 1 > tq) p1 = 0.f;
        }
        dd[c / 2] = pack_bf16x2(p0 * (dp[c] - dt), p1 * (dp[c + 1] - dt));
      }
      if (C::SEP) {
        // dS into its own columns once the previous block's dQ MMAs read them
        if (jj > 0 && !__all_sync(0xffffffffu, mbar_wait(&ds_free[t], (jj - 1) & 1, abort_flag, tmo, 0xd03))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(row + C::DS_COL, dd);
      } else {
        tmem_st32(row, dd);  // dS (bf16 pairs) over S columns 0..31, already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ds_full[t]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&q_done[t], 0, abort_flag, tmo, 0xd02))) {
      tc_fence_after();
      const size_t orow = ((static_cast<size_t>(b) * p.S + tok) * p.Hq + hq) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        float o[32];
        tmem_ld32(row + 128 + ch * 32, o);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = pack_bf16x2(o[2 * c] * p.scale, o[2 * c + 1] * p.scale);
        uint4* dst = reinterpret_cast<uint4*>(p.dq + orow + ch * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace ssa
