// attn_fwd_psmem.cuh -- block-sparse causal attention forward on tcgen05 tensor
// cores, with P in TMEM columns of its own, so each tile's next scores are
// computed while it exponentiates (the variant used at head_dim 128).
//
// A work unit is one query block i (64 tokens) of one batch entry for 2*T
// query heads that share KV head h; a CTA takes one unit, or in the plain
// sparse stream a sequence of them (persistent CTAs, below).  A unit's rows
// form T M-tiles of 128 rows (2 heads x 64 tokens).  The KV blocks it visits are either the selected
// blocks of the index table (sparse stream: "SSA: Guida a Sparse Sparse
// Attention per LLM", section "Block-sparse attention e Receptive Field",
// attention computed only over the tokens of the selected blocks) or, with
// MASS, every causal block 0..i, each one's P.V going to the selected or the
// unselected accumulator against one shared running maximum, which yields the
// dense counterpart, the sparse output and the dropped attention mass from
// one pass ("Resumen Tecnico: SSA", section 2, "Alineacion Bidireccional",
// and section 1 on the dropped mass).
//
// Two more modes reuse the pipeline:
//   DASH   the routed chunks of a DashAttention mask, each block's scores
//          offset by sigma * log2 w_j ("Resumen Tecnico: DashAttention",
//          stage 2, prior-induced softmax); see dash_build_list.
//   EARLY  the selected blocks in descending pooled score after the diagonal,
//          each head's query segment (the 64 rows of one head in a tile)
//          stopping once a block adds less than tau times the mass gathered
//          before it to every one of its rows (the "S2O" summary, section 2);
//          a stopped head's P is zero from then on, and the tile ends its
//          block loop once both of its heads have stopped; see
//          early_visit_order.
//
// Pipeline per M-tile t and visited block jj:
//   S_t(jj) = Q_t K(jj)^T          tensor core, fp32 in TMEM
//   softmax warps load S_t(jj) into registers and release it at once, so the
//   issuer can start S_t(jj+1) while they exponentiate
//   P_t(jj) (bf16 pairs) -> TMEM columns of its own
//   O_t += P_t(jj) V(jj)           tensor core, A from TMEM, B from shared memory
// so the score MMA of the next block and the P.V of this block both overlap
// the softmax.  O is rescaled in TMEM (lazily, see below) after the previous
// P.V has completed.
//
// Warp roles (128 * (T + 1) threads):
//   warp 0      TMA producer: the Q tiles once, then K and V of each visited
//               block through an NS-stage ring (index-guided loads).
//   issuers     one warp per M-tile (warps 1, 2, 3 and, for a fourth tile,
//               the warp after the softmax warpgroups); one elected thread
//               issues that tile's tcgen05.mma in order, waiting (suspended,
//               no issue slots taken) on its "S consumed" and "P ready"
//               barriers.  Warp 1 also allocates TMEM; warp 3 first builds
//               the selection bitmap (MASS).
//   warps 4..   one warpgroup per M-tile: thread r owns row r of the tile;
//               online softmax in the exp2 domain with lazy rescaling (the
//               reference maximum only moves when the row maximum exceeds it
//               by more than 8, i.e. a factor 256), and the epilogue.
//
// TMEM per M-tile t (stride 96 + D, or 96 + 2D with MASS): S at +0 (64 fp32
// columns), P at +64 (64 keys as 32 columns of bf16 pairs), O (O_selected
// with MASS) at +96, O_unselected at +96 + D.  Two tiles take 448 of the 512
// columns at head_dim 128.  Keeping P out of shared memory leaves the shared
// memory bandwidth to the operand reads of the MMAs (P was written and then
// read again as the P.V MMA's A operand: 32 KB per tile and block).
//
// Persistent CTAs (plain sparse stream).  One CTA per SM takes the work units
// blockIdx.x, blockIdx.x + gridDim.x, ... (heaviest query blocks first) and
// every barrier keeps counting across units: the K/V ring, the score, P and
// P.V barriers by the CTA's running block count, the Q and output barriers by
// its running unit count.  So the producer loads the next unit's first K/V
// block, and its Q as soon as both tiles' last score MMA has read the old Q
// (bar_qfree); each issuer starts the next unit's first score MMA while the
// softmax warps still write the previous unit's output; and the next unit's
// first P.V (which overwrites O) waits on P, which the softmax warps store only
// after their epilogue has read O.  With one CTA per SM, a new CTA per unit
// would leave the SM idle for the unit's prologue and epilogue.  The other
// modes run one unit per CTA through the same code.
#pragma once

#include "sm100.cuh"
#include "softmax_util.cuh"

namespace ssa {

template <int D, int T, bool MASS, bool DASH = false, bool EARLY = false>
struct PsFwdConfig {
  static constexpr int NP = D / 64;               // 64-column panels per row
  static constexpr int QTILE = 128 * D * 2;       // bytes of one Q M-tile
  static constexpr int KVT = 64 * D * 2;          // bytes of one K (or V) block
  static constexpr int NS = 4;                    // K/V ring stages
  // TMEM columns per M-tile: S (64 fp32), P (32: 64 keys as bf16 pairs), O
  // (O_selected with MASS), O_unselected (MASS)
  static constexpr int TSTRIDE = 96 + (MASS ? 2 : 1) * D;
  static constexpr int TMEM_COLS = pow2_at_least(T * TSTRIDE);
  static constexpr int POLY = 4;                  // exp2 pairs of 8 on the FMA pipe
  // warps: 0 producer, 1..3 issuers, 4.. softmax (4 per tile), then the
  // issuer of a fourth tile
  static constexpr int THREADS = 128 * (T + 1) + (T > 3 ? 32 : 0);
  // barriers: q, kfull/vfull/empty[NS], sfull/sfree/pfull/pvdone/odone/drain/turn[T], qfree
  static constexpr int NBARS = 1 + 3 * NS + 7 * T + 1;
  // shared memory: Q tiles, K ring, V ring, barriers, tmem slot,
  // abort flag, selection bitmap (up to 8192 blocks); DASH: the routed chunk
  // list and its biases (kDashMaxN each) and the count
  static constexpr int SMEM_TILES = T * QTILE + 2 * NS * KVT;
  // EARLY: 2 KB of visiting-order scratch and 128 B of stop flags
  static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + NBARS * 8 + 16 + 1024 + (DASH ? 8 * kDashMaxN + 16 : 0) +
                                    (EARLY ? 2048 + 128 : 0);
  static_assert(T * TSTRIDE <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Warp that issues the MMAs of M-tile t.
template <int T>
__device__ __forceinline__ int ps_issuer_warp(int t) {
  return t < 3 ? 1 + t : 4 + 4 * T;
}

template <int D, int T, bool MASS, bool DASH = false, bool EARLY = false>
__global__ void __launch_bounds__(PsFwdConfig<D, T, MASS, DASH, EARLY>::THREADS, 1)
    attn_fwd_psmem_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = PsFwdConfig<D, T, MASS, DASH, EARLY>;
  static_assert(!(MASS && DASH), "the routed softmax is a mode of its own");
  static_assert(!(EARLY && (MASS || DASH)), "the early stop applies to the sparse stream only");
  constexpr int NP = C::NP, QTILE = C::QTILE, KVT = C::KVT, NS = C::NS, TSTRIDE = C::TSTRIDE;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                 // [T][QTILE]
  uint8_t* sK = sQ + T * QTILE;       // [NS][KVT]
  uint8_t* sV = sK + NS * KVT;        // [NS][KVT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NS * KVT);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bar_q + 1;              // [NS]
  uint64_t* bar_vfull = bar_kfull + NS;
  uint64_t* bar_empty = bar_vfull + NS;
  uint64_t* bar_sfull = bar_empty + NS;         // [T] scores in TMEM
  uint64_t* bar_sfree = bar_sfull + T;          // [T] scores read by the softmax
  uint64_t* bar_pfull = bar_sfree + T;          // [T] P stored in TMEM (O rescaled)
  uint64_t* bar_pvdone = bar_pfull + T;         // [T] P.V completed
  uint64_t* bar_odone = bar_pvdone + T;         // [T] last P.V completed
  uint64_t* bar_drain = bar_odone + T;          // [T] issuer's MMAs drained (abort)
  uint64_t* bar_turn = bar_drain + T;           // [T] tile t may exponentiate (T = 2)
  uint64_t* bar_qfree = bar_turn + T;           // every tile's last score MMA of a unit read Q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_qfree + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* selbits = tmem_slot + 4;
  // DASH: routed chunks in ascending order then the diagonal, their biases
  // (sigma * log2 w, in the exp2 domain of the scores), and their count
  int32_t* dord = reinterpret_cast<int32_t*>(selbits + 256);
  float* dbias = reinterpret_cast<float*>(dord + kDashMaxN);
  int* dcount = reinterpret_cast<int*>(dbias + kDashMaxN);
  // EARLY: visiting order (over the bitmap area), score scratch, stop flags
  int32_t* ord = reinterpret_cast<int32_t*>(selbits);
  float* esc = reinterpret_cast<float*>(selbits + 256);       // [256] scores
  int32_t* ej = reinterpret_cast<int32_t*>(esc + 256);        // [256] their blocks
  volatile int* all_stop = reinterpret_cast<volatile int*>(ej + 256);
  volatile int* tile_stop = all_stop + 1;                     // [T]
  volatile int* wflag = all_stop + 4;                         // [T][2][4]
  int* nstopped = const_cast<int*>(all_stop) + 24;            // tiles stopped so far

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // work units, heaviest query blocks first; the plain sparse stream runs
  // persistent CTAs over units blockIdx.x, blockIdx.x + gridDim.x, ..., the
  // other modes one unit per CTA
  constexpr bool PERSIST = !MASS && !DASH && !EARLY;
  const int per_i = p.B * p.Hkv * p.slices;
  const int n_units = PERSIST ? (p.i_hi - p.i_lo) * per_i : static_cast<int>(blockIdx.x) + 1;
  struct Unit {
    int i, b, h, slice, hq0, nsel;
    const int32_t* idx_row;
  };
  auto unit_of = [&](int u) {
    Unit w;
    w.i = p.i_hi - 1 - u / per_i;
    int rem = u % per_i;
    w.slice = rem % p.slices;
    rem /= p.slices;
    w.h = rem % p.Hkv;
    w.b = rem / p.Hkv;
    w.hq0 = w.h * p.G + w.slice * 2 * T;
    w.nsel = min(p.topk, w.i + 1);
    w.idx_row = p.idx + ((static_cast<size_t>(w.b) * p.Hkv + w.h) * p.n + w.i) * p.topk;
    return w;
  };
  const Unit u0 = unit_of(static_cast<int>(blockIdx.x));
  const int i = u0.i, b = u0.b, h = u0.h, hq0 = u0.hq0, nsel = u0.nsel;
  int nblk = MASS ? (i + 1) : nsel;  // DASH: the routed count, known after the prologue
  const int32_t* idx_row = u0.idx_row;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_kfull[s], 1);
      mbar_init(&bar_vfull[s], 1);
      mbar_init(&bar_empty[s], T);  // released by each tile's issuer
    }
    for (int t = 0; t < T; ++t) {
      mbar_init(&bar_sfull[t], 1);
      mbar_init(&bar_sfree[t], 128);
      mbar_init(&bar_pfull[t], 128);
      mbar_init(&bar_pvdone[t], 1);
      mbar_init(&bar_odone[t], 1);
      mbar_init(&bar_drain[t], 1);
      mbar_init(&bar_turn[t], 128);
    }
    mbar_init(bar_qfree, T);  // one commit per tile's issuer and unit
    *abort_flag = 0;
    fence_mbar_init();
  }
  // launched with programmatic serialization: the index table may still be
  // in flight from the selection kernel until here
  pdl_wait();
  if (MASS && warp == 3) {
    const int words = (p.n + 31) / 32;
    for (int w = lane; w < words; w += 32) selbits[w] = 0u;
    __syncwarp();
    for (int r = lane; r < nsel; r += 32) {
      const int j = idx_row[r];
      if (j >= 0 && j <= i) atomicOr(&selbits[j >> 5], 1u << (j & 31));
    }
  }
  if (DASH && warp == 2) dash_build_list(p, b, h, i, lane, dord, dbias, dcount);
  if (EARLY && threadIdx.x == 0) {
    *all_stop = 0;
    *nstopped = 0;
    for (int t = 0; t < T; ++t) tile_stop[t] = 0;
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
  if (DASH) nblk = *dcount;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    auto load_kv = [&](int st, int j) {
      mbar_arrive_expect_tx(&bar_kfull[st], KVT);
      for (int pn = 0; pn < NP; ++pn)
        tma_load_4d(sK + st * KVT + pn * (64 * 128), &tm_k, &bar_kfull[st], 64 * pn, h, 64 * j, b);
      mbar_arrive_expect_tx(&bar_vfull[st], KVT);
      for (int pn = 0; pn < NP; ++pn)
        tma_load_4d(sV + st * KVT + pn * (64 * 128), &tm_v, &bar_vfull[st], 64 * pn, h, 64 * j, b);
    };
    if (PERSIST) {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        // per unit: its first K/V block, then its Q once both tiles' last
        // score MMA of the previous unit has read the old Q, then the rest
        int g = 0, k = 0;  // K/V blocks and units loaded so far
        int qk = -1;       // the last unit whose Q was loaded
        bool alive = true;
        for (int u = static_cast<int>(blockIdx.x); alive && u < n_units; u += gridDim.x, ++k) {
          const Unit w = unit_of(u);
          for (int s = 0; s < w.nsel; ++s) {
            const int st = g % NS, use = g / NS;
            if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, abort_flag, tmo, 0x101)) {
              alive = false;
              break;
            }
            const int j = w.idx_row[s];
            mbar_arrive_expect_tx(&bar_kfull[st], KVT);
            for (int pn = 0; pn < NP; ++pn)
              tma_load_4d(sK + st * KVT + pn * (64 * 128), &tm_k, &bar_kfull[st], 64 * pn, w.h, 64 * j, w.b);
            mbar_arrive_expect_tx(&bar_vfull[st], KVT);
            for (int pn = 0; pn < NP; ++pn)
              tma_load_4d(sV + st * KVT + pn * (64 * 128), &tm_v, &bar_vfull[st], 64 * pn, w.h, 64 * j, w.b);
            ++g;
            if (s == 0) {
              if (k > 0 && !mbar_wait(bar_qfree, (k - 1) & 1, abort_flag, tmo, 0x102)) {
                alive = false;
                break;
              }
              mbar_arrive_expect_tx(bar_q, T * QTILE);
              for (int t = 0; t < T; ++t)
                for (int hh = 0; hh < 2; ++hh)
                  for (int pn = 0; pn < NP; ++pn)
                    tma_load_4d(sQ + t * QTILE + pn * (128 * 128) + hh * (64 * 128), &tm_q, bar_q,
                                64 * pn, w.hq0 + 2 * t + hh, 64 * w.i, w.b);
              qk = k;
            }
          }
        }
        // on abort, the loads already issued are waited for (bounded) before exit
        if (*abort_flag) {
          volatile int never = 0;
          for (int gj = (g > NS ? g - NS : 0); gj < g; ++gj) {
            mbar_wait(&bar_kfull[gj % NS], (gj / NS) & 1, &never, 1000000ull, 0x1fe);
            mbar_wait(&bar_vfull[gj % NS], (gj / NS) & 1, &never, 1000000ull, 0x1ff);
          }
          if (qk >= 0) mbar_wait(bar_q, qk & 1, &never, 1000000ull, 0x1fd);
        }
      }
    } else {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_arrive_expect_tx(bar_q, T * QTILE);
        for (int t = 0; t < T; ++t)
          for (int hh = 0; hh < 2; ++hh)
            for (int pn = 0; pn < NP; ++pn)
              tma_load_4d(sQ + t * QTILE + pn * (128 * 128) + hh * (64 * 128), &tm_q, bar_q,
                          64 * pn, hq0 + 2 * t + hh, 64 * i, b);
        if (EARLY) load_kv(0, i);  // the diagonal block is visited first
      }
      if (EARLY) early_visit_order<D>(p, b, h, i, nsel, idx_row, lane, ord, esc, ej);
      if (lane == 0) {
        int issued = EARLY ? 1 : 0;
        for (int jj = issued; jj < nblk; ++jj) {
          const int st = jj % NS, use = jj / NS;
          if (EARLY && *all_stop) break;  // every tile stopped: no more blocks
          // EARLY: once every tile stopped, the stage may never be released;
          // the stop flag ends the wait instead
          if (use > 0 && !(EARLY ? mbar_wait_or(&bar_empty[st], (use - 1) & 1, abort_flag, all_stop, tmo, 0x101)
                                 : mbar_wait(&bar_empty[st], (use - 1) & 1, abort_flag, tmo, 0x101)))
            break;
          load_kv(st, MASS ? jj : (DASH ? dord[jj] : (EARLY ? ord[jj] : idx_row[jj])));
          ++issued;
        }
        // on abort or an early stop, loads already issued are waited for
        // (bounded) before exit
        if (*abort_flag || (EARLY && issued < nblk)) {
          volatile int never = 0;
          for (int jj = (issued > NS ? issued - NS : 0); jj < issued; ++jj) {
            mbar_wait(&bar_kfull[jj % NS], (jj / NS) & 1, &never, 1000000ull, 0x1fe);
            mbar_wait(&bar_vfull[jj % NS], (jj / NS) & 1, &never, 1000000ull, 0x1ff);
          }
        }
      }
    }  // one unit
  } else if (warp != 0 && (warp < 4 || warp >= 4 + 4 * T)) {
    // ------------------------------------------------------------ MMA issuers
    int t = -1;
#pragma unroll
    for (int x = 0; x < T; ++x)
      if (ps_issuer_warp<T>(x) == warp) t = x;
    if (lane == 0 && t >= 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint32_t s_tmem = tmem + t * TSTRIDE;
      auto issue_qk = [&](int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32;  // 16 bf16 = 32 B inside the 128 B row
          const uint64_t a = sdesc_sw128(sQa + t * QTILE + (kk / 4) * (128 * 128) + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKa + st * KVT + (kk / 4) * (64 * 128) + off, 16, 1024);
          mma_ss(s_tmem, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // Per unit: S(0) once its Q and first K/V block landed and the softmax
      // read the previous unit's last scores; then for s = 0, 1, ...:
      //   [S(s) read]  S(s+1);   [P(s) stored]  O += P(s) V(s)
      // Parities count the CTA's blocks (g + s) and units (k).
      bool ok = true;
      int g = 0, k = 0;
      for (int u = static_cast<int>(blockIdx.x); ok && u < n_units; u += gridDim.x, ++k) {
        const int nb = PERSIST ? unit_of(u).nsel : nblk;
        ok = mbar_wait(bar_q, k & 1, abort_flag, tmo, 0x201) &&
             mbar_wait(&bar_kfull[g % NS], (g / NS) & 1, abort_flag, tmo, 0x202) &&
             (g == 0 || mbar_wait(&bar_sfree[t], (g - 1) & 1, abort_flag, tmo, 0x203));
        if (!ok) break;
        tc_fence_after();
        issue_qk(g % NS);
        tc_commit(&bar_sfull[t]);
        if (PERSIST && nb == 1) tc_commit(bar_qfree);  // the unit's last score MMA read Q
        bool first_sel = true, first_uns = true;
        for (int s = 0; ok && s < nb; ++s) {
          const int gs = g + s;
          if (s + 1 < nb) {
            // S(s+1) as soon as the softmax has read S(s)
            const int st1 = (gs + 1) % NS;
            if (!mbar_wait(&bar_sfree[t], gs & 1, abort_flag, tmo, 0x203) ||
                !mbar_wait(&bar_kfull[st1], ((gs + 1) / NS) & 1, abort_flag, tmo, 0x204)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(st1);
            tc_commit(&bar_sfull[t]);
            if (PERSIST && s + 2 == nb) tc_commit(bar_qfree);
          }
          // P(s).V once P(s) is stored
          const int st = gs % NS;
          if (!mbar_wait(&bar_pfull[t], gs & 1, abort_flag, tmo, 0x205) ||
              !mbar_wait(&bar_vfull[st], (gs / NS) & 1, abort_flag, tmo, 0x206)) {
            ok = false;
            break;
          }
          tc_fence_after();
          bool is_sel = true;
          if (MASS) is_sel = (selbits[s >> 5] >> (s & 31)) & 1u;
          const bool first = MASS ? (is_sel ? first_sel : first_uns) : (s == 0);
          const uint32_t o_col = s_tmem + 96 + ((MASS && !is_sel) ? D : 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 keys of P (8 TMEM columns) per MMA
            const uint64_t bd = sdesc_sw128(sVa + st * KVT + kk * (16 * 128), 64 * 128, 1024);
            mma_ts(o_col, s_tmem + 64 + kk * 8, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(&bar_pvdone[t]);
          // EARLY: the softmax records the position of the block it stops at
          // before it arrives on that block's pfull.  The issuer compares with
          // its own position: S(s+1) is already issued here, so the softmax
          // may have decided a stop at s+1 before this thread reads the flag.
          const bool stop_now = EARLY && tile_stop[t] == s + 1;
          if (s + 1 == nb || stop_now) tc_commit(&bar_odone[t]);
          tc_commit(&bar_empty[st]);
          if (MASS) {
            if (is_sel) first_sel = false; else first_uns = false;
          }
          if (EARLY && stop_now) {
            // the other tiles still need every stage released by this tile too:
            // release each remaining block's stage once it is loaded, until the
            // last block or until every tile has stopped (the producer then
            // loads nothing more)
            if (atomicAdd(nstopped, 1) + 1 == T) *all_stop = 1;
            for (int s2 = g + s + 1; s2 < g + nb; ++s2) {
              if (!mbar_wait_or(&bar_vfull[s2 % NS], (s2 / NS) & 1, abort_flag, all_stop, tmo, 0x207)) break;
              tc_commit(&bar_empty[s2 % NS]);
            }
            break;
          }
        }
        g += nb;
      }
      if (!ok) {
        // every MMA this thread issued completes before TMEM is released
        tc_commit(&bar_drain[t]);
        volatile int never = 0;
        mbar_wait(&bar_drain[t], 0, &never, tmo, 0x2ff);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int hh = r / 64, tq = r % 64;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16) + t * TSTRIDE;
    const uint32_t tS = lane_base, tP = lane_base + 64, tO = lane_base + 96;
    const uint32_t tOu = tO + D;
    const float sl2 = p.scale_log2;
    const uint64_t scale2 = f2_pack(sl2, sl2);
    bool ok = true;
    // parities count the CTA's blocks (g + jj) and units (k)
    int g = 0, k = 0;
    for (int u = static_cast<int>(blockIdx.x); ok && u < n_units; u += gridDim.x, ++k) {
      const Unit w = PERSIST ? unit_of(u) : u0;
      const int nb = PERSIST ? w.nsel : nblk;
      const int hq = w.hq0 + 2 * t + hh;
      float m_ref = -INFINITY;  // reference maximum, scaled (log2) units
      float l_sel = 0.f, l_uns = 0.f;
      // EARLY: each head of the tile (64-row half: warps wq 0-1 and 2-3)
      // stops on its own; a stopped head's P is stored as zeros, so P.V adds
      // nothing to its rows and its maximum, mass and O stay as they were
      bool hstop = false;       // this thread's head has stopped
      int hvis = 0;             // blocks this thread's head visited
      for (int jj = 0; jj < nb; ++jj) {
        const int gj = g + jj;
        // waits are made warp-uniform: the tcgen05.ld/st below are .sync.aligned
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_sfull[t], gj & 1, abort_flag, tmo, 0x301))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // warp-uniform: both warps of a head stop together
        const bool live = !EARLY || !hstop;
        float sA[32], sB[32];
        if (live) {
          tmem_ld32(tS, sA);
          tmem_ld32(tS + 32, sB);
        }
        // the scores are in registers: the issuer may overwrite S with the next block's
        tc_fence_before();
        mbar_arrive(&bar_sfree[t]);
        // the diagonal block comes last in the ascending table, first in the
        // early-stop order
        const bool diag = EARLY ? (jj == 0) : (jj == nb - 1);
        bool is_sel = true;
        if (MASS) is_sel = (selbits[jj >> 5] >> (jj & 31)) & 1u;
        // with two tiles, their exponential phases alternate: tile 1's block jj
        // follows tile 0's block jj, tile 0's block jj + 1 follows tile 1's
        // block jj, so one tile's MMAs run while the other exponentiates (not
        // with the early stop, where one tile may stop before the other); the
        // order runs on across units
        if (T == 2 && !EARLY && (t == 1 || gj > 0) &&
            !__all_sync(0xffffffffu, mbar_wait(&bar_turn[t], (t == 1 ? gj : gj - 1) & 1, abort_flag, tmo,
                                               0x305))) {
          ok = false;
          break;
        }
        float alpha = 1.f;
        bool moved = false;
        uint64_t acc2 = f2_pack(0.f, 0.f);
        uint32_t pk[32];
        if (live) {
          float mx = diag ? row_max32<true>(sB, 32, tq, -INFINITY) : row_max32<false>(sB, 32, tq, -INFINITY);
          mx = diag ? row_max32<true>(sA, 0, tq, mx) : row_max32<false>(sA, 0, tq, mx);
          // DASH: the chunk's prior adds sigma * log2 w_j to every score of the block
          const float bias = DASH ? dbias[jj] : 0.f;
          const float mx_s = mx * sl2 + bias;
          moved = mx_s > m_ref + 8.f;
          if (moved) {
            alpha = ex2(m_ref - mx_s);
            m_ref = mx_s;
          }
          const uint64_t negm2 = f2_pack(bias - m_ref, bias - m_ref);
          if (diag) {
            exp_pack32<true>(sA, 0, tq, scale2, negm2, acc2, pk);
            exp_pack32<true>(sB, 32, tq, scale2, negm2, acc2, pk + 16);
          } else {
            exp_pack32<false, C::POLY>(sA, 0, tq, scale2, negm2, acc2, pk);
            exp_pack32<false, C::POLY>(sB, 32, tq, scale2, negm2, acc2, pk + 16);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        }
        if (T == 2 && !EARLY) mbar_arrive(&bar_turn[1 - t]);
        float r0, r1;
        f2_unpack(acc2, r0, r1);
        bool stop = false;
        if (EARLY && jj > 0 && p.tau > 0.f) {
          // this block's mass against the mass accumulated before it (both in
          // the current reference); a head stops when none of its rows gained
          // at least tau times what it had, the tile when both heads have
          // stopped (tau = 0 never stops: no decision is taken).  A stopped
          // head votes 0.
          const bool cont_row = live && (r0 + r1) >= p.tau * (l_sel * alpha);
          volatile int* wf = wflag + (t * 2 + (jj & 1)) * 4;
          const bool wcont = __any_sync(0xffffffffu, cont_row);
          if (lane == 0) wf[wq] = wcont ? 1 : 0;
          named_bar_sync(1 + t, 128);
          const bool head_stop = !(wf[2 * hh] | wf[2 * hh + 1]);
          stop = !(wf[0] | wf[1] | wf[2] | wf[3]);
          if (stop && r == 0) tile_stop[t] = jj + 1;  // read by the issuer after pfull
          if (live && head_stop) hstop = true;       // this block is the head's last
        }
        l_sel *= alpha;
        l_uns *= alpha;
        if (is_sel) l_sel += r0 + r1; else l_uns += r0 + r1;
        if (jj > 0) {
          // P(jj-1).V has finished: the P tile may be overwritten and O is stable
          // (for jj = 0 the previous unit's epilogue waited for its last P.V)
          if (!__all_sync(0xffffffffu, mbar_wait(&bar_pvdone[t], (gj - 1) & 1, abort_flag, tmo, 0x302))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, moved)) {
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int acc = 0; acc < (MASS ? 2 : 1); ++acc) {
              const uint32_t base = acc ? tOu : tO;
#pragma unroll
              for (int ch = 0; ch < D / 16; ++ch) {
                float o[16];
                uint32_t w[16];
                tmem_ld16(base + ch * 16, o);
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                  float lo, hi;
                  f2_unpack(f2_mul(f2_pack(o[c], o[c + 1]), a2), lo, hi);
                  w[c] = __float_as_uint(lo);
                  w[c + 1] = __float_as_uint(hi);
                }
                tmem_st16(base + ch * 16, w);
              }
            }
            tmem_wait_st();
          }
        }
        tmem_st16(tP, pk);       // keys 0..31
        tmem_st16(tP + 16, pk + 16);  // keys 32..63
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_pfull[t]);
        if (EARLY && live) hvis = jj + 1;
        if (stop) break;
      }
      // ---------------------------------------------------------- epilogue
      // (O is read here before this tile's next P store, which the next unit's
      // first P.V waits for: so that P.V never overwrites O still being read)
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&bar_odone[t], k & 1, abort_flag, tmo, 0x303))) ok = false;
      if (ok) {
        tc_fence_after();
        const int tok = 64 * w.i + tq;
        const size_t orow = ((static_cast<size_t>(w.b) * p.S + tok) * p.Hq + hq) * D;
        const size_t lrow = (static_cast<size_t>(w.b) * p.Hq + hq) * p.S + tok;
        const bool has_uns = MASS && (nb > w.nsel);
        const float inv_sel = 1.f / l_sel;
        const float l_all = l_sel + (has_uns ? l_uns : 0.f);
        const float inv_all = 1.f / l_all;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          float o[32];
          tmem_ld32(tO + ch * 32, o);
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) w[c] = pack_bf16x2(o[2 * c] * inv_sel, o[2 * c + 1] * inv_sel);
          uint4* dst = reinterpret_cast<uint4*>(p.o + orow + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
          if (MASS) {
            if (has_uns) {
              float ou[32];
              tmem_ld32(tOu + ch * 32, ou);
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] += ou[c];
            }
#pragma unroll
            for (int c = 0; c < 16; ++c)
              w[c] = pack_bf16x2(o[2 * c] * inv_all, o[2 * c + 1] * inv_all);
            uint4* dstf = reinterpret_cast<uint4*>(p.o_full + orow + ch * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dstf[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
          }
        }
        constexpr float kLn2 = 0.69314718055994530942f;
        p.lse[lrow] = (m_ref + log2f(l_sel)) * kLn2;
        if (EARLY && tq == 0 && p.visited != nullptr)
          p.visited[(static_cast<size_t>(w.b) * p.Hq + hq) * p.n + w.i] = hvis;
        if (MASS) {
          p.lse_full[lrow] = (m_ref + log2f(l_all)) * kLn2;
          p.dropped[lrow] = has_uns ? (l_uns / l_all) : 0.f;
        }
      }
      g += nb;
    }  // units
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace ssa
