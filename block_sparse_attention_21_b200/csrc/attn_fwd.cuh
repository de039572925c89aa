// attn_fwd.cuh -- block-sparse causal attention forward on tcgen05 tensor cores.
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
// Two CTAs share an SM when T = 2 (256 TMEM columns each), so one CTA's
// prologue and epilogue overlap the other's main loop.
//
// Persistent CTAs (plain sparse stream): as many CTAs as fit on the GPU take
// the work units blockIdx.x, blockIdx.x + gridDim.x, ... (heaviest query
// blocks first), and every barrier keeps counting across units (the K/V ring,
// score and P barriers by the CTA's running block count, the Q and output
// barriers by its running unit count).  The producer loads the next unit's
// first K/V block, and its Q once the last score MMAs of the previous unit
// have read the old Q (bar_qfree); the issuer starts the next unit's score
// MMAs right after the previous unit's last P.V (one thread's MMAs execute in
// order, so S never overwrites a P still being read); and the next unit's
// first P.V, which overwrites O, waits for P, which the softmax warps store
// only after their epilogue has read O.  The other modes run one unit per CTA
// through the same code.
//
// Warp roles (64 + 128 * T threads):
//   warp 0      builds the selection bitmap (MASS), then is the TMA producer:
//               the Q tiles once, then K and V of each visited block through
//               an NS-stage ring (index-guided loads).
//   warp 1      TMEM allocation and the tcgen05.mma issuer (one elected
//               thread), serving the M-tiles round-robin with suspending
//               waits; it releases a K/V stage with one commit once all
//               tiles are done with it.  Per visited block jj and M-tile t,
//               in this order:
//                 wait P_t(jj) keys 0..31;   O_t += P_t V(jj) over them;
//                 wait P_t(jj) keys 32..63;  O_t += P_t V(jj) over them;
//                 S_t = Q_t K(jj+1)^T
//               so one commit of S_t(jj+1) also tells the softmax warps that
//               O_t is stable.  P_t lives in the first 32 TMEM columns of S_t;
//               the tensor pipe executes one thread's MMAs in issue order, so
//               S_t(jj+1) overwrites P_t(jj) only after P.V has read it.
//   warps 2..   one warpgroup per M-tile (TMEM lane quarter = warp % 4):
//               thread r owns row r of the tile; all 64 scores of a block
//               come in with one TMEM load; online softmax in the exp2 domain
//               with lazy rescaling (the reference maximum only moves when the
//               row maximum exceeds it by more than 8, i.e. a factor 256), P
//               written back to TMEM as bf16 pairs in two halves, O rescaled in
//               TMEM when the maximum moved, and the epilogue.
//
// TMEM per M-tile t (stride 64 + D, or 64 + 2D with MASS): S/P at +0
// (64 columns of fp32 scores; P overwrites columns 0..31 as bf16 pairs),
// O (O_selected with MASS) at +64, O_unselected at +64 + D (MASS only).
#pragma once

#include "sm100.cuh"
#include "softmax_util.cuh"

namespace ssa {

// Largest top-k of the early-stop variant (its visiting order lives in the
// 1 KB selection-bitmap area).
constexpr int kEarlyMaxTopk = 256;

template <int D, int T, bool MASS, bool EARLY = false, bool DASH = false>
struct FwdConfig {
  static constexpr int NP = D / 64;               // 64-column panels per row
  static constexpr int QTILE = 128 * D * 2;       // bytes of one Q M-tile
  static constexpr int KVT = 64 * D * 2;          // bytes of one K (or V) block
  static constexpr int NS = (D == 64) ? 4 : 3;    // K/V ring stages
  static constexpr int TSTRIDE = 64 + (MASS ? 2 : 1) * D;  // TMEM columns per M-tile
  static constexpr int TMEM_COLS = pow2_at_least(T * TSTRIDE);
  static constexpr int THREADS = 64 + 128 * T;
  static constexpr int ISS = 1;                   // MMA issuer warps (warp 1)
  static constexpr int POLY = (D == 128) ? 3 : (MASS ? 0 : 1);  // exp2 pairs of 8 on the FMA pipe
  static constexpr int NBARS = 1 + ISS + 3 * NS + 4 * T + 1;
  // shared memory: Q tiles, K ring, V ring, barriers, tmem slot, abort flag,
  // selection bitmap (up to 8192 blocks)
  static constexpr int SMEM_TILES = T * QTILE + 2 * NS * KVT;
  // EARLY: 2 KB of score scratch and 128 B of stop flags after the bitmap area;
  // DASH: the routed chunk list and its biases (kDashMaxN each) and the count
  static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + NBARS * 8 + 16 + 1024 + (EARLY ? 2048 + 128 : 0) +
                                    (DASH ? 8 * kDashMaxN + 16 : 0);
  // two CTAs share an SM when both fit in TMEM (256 columns each) and in
  // shared memory: one CTA's prologue and epilogue overlap the other's loop
  static constexpr int MIN_CTAS = (TMEM_COLS <= 256 && SMEM_BYTES <= 113 * 1024) ? 2 : 1;
  static_assert(T * TSTRIDE <= 512, "TMEM budget");
};

template <int D, int T, bool MASS, bool EARLY = false, bool DASH = false>
__global__ void __launch_bounds__(FwdConfig<D, T, MASS, EARLY, DASH>::THREADS,
                                  FwdConfig<D, T, MASS, EARLY, DASH>::MIN_CTAS)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdConfig<D, T, MASS, EARLY, DASH>;
  static_assert(!(MASS && EARLY), "the early stop applies to the sparse stream only");
  static_assert(!(DASH && (MASS || EARLY)), "the routed softmax is a mode of its own");
  constexpr int NP = C::NP, QTILE = C::QTILE, KVT = C::KVT, NS = C::NS, TSTRIDE = C::TSTRIDE;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + T * QTILE;
  uint8_t* sV = sK + NS * KVT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NS * KVT);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_vfull = bar_kfull + NS;
  uint64_t* bar_empty = bar_vfull + NS;
  uint64_t* bar_sfull = bar_empty + NS;
  uint64_t* bar_phalf = bar_sfull + T;  // P columns 0..15 (keys 0..31) stored, O rescaled
  uint64_t* bar_pfull = bar_phalf + T;  // all of P stored
  uint64_t* bar_odone = bar_pfull + T;
  uint64_t* bar_drain = bar_odone + T;
  uint64_t* bar_qfree = bar_drain + C::ISS;  // the last score MMAs of a unit read Q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_qfree + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* selbits = tmem_slot + 4;
  // EARLY: visiting order (over the bitmap area), score scratch, stop flags
  int32_t* ord = reinterpret_cast<int32_t*>(selbits);
  float* esc = reinterpret_cast<float*>(selbits + 256);       // [256] scores
  int32_t* ej = reinterpret_cast<int32_t*>(esc + 256);        // [256] their blocks
  volatile int* all_stop = reinterpret_cast<volatile int*>(ej + 256);
  volatile int* tile_stop = all_stop + 1;                     // [T]
  volatile int* wflag = all_stop + 4;                         // [T][2][4]
  // DASH: routed chunks in ascending order then the diagonal, their biases
  // (sigma * log2 w, in the exp2 domain of the scores), and their count
  int32_t* dord = reinterpret_cast<int32_t*>(selbits + 256);
  float* dbias = reinterpret_cast<float*>(dord + kDashMaxN);
  int* dcount = reinterpret_cast<int*>(dbias + kDashMaxN);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // work units, heaviest query blocks first; the plain sparse stream runs
  // persistent CTAs over units blockIdx.x, blockIdx.x + gridDim.x, ..., the
  // other modes one unit per CTA
  constexpr bool PERSIST = !MASS && !EARLY && !DASH;
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
      mbar_init(&bar_empty[s], C::ISS);  // released once per issuer
    }
    for (int t = 0; t < T; ++t) {
      mbar_init(&bar_sfull[t], 1);
      mbar_init(&bar_phalf[t], 128);
      mbar_init(&bar_pfull[t], 128);
      mbar_init(&bar_odone[t], 1);
    }
    for (int x = 0; x < C::ISS; ++x) mbar_init(&bar_drain[x], 1);
    mbar_init(bar_qfree, C::ISS);  // one commit per issuer and unit
    *abort_flag = 0;
    fence_mbar_init();
    if (PERSIST) {
      // thread 0 is the producer: the first unit's Q and diagonal block do
      // not depend on the index table, so they load before the wait below,
      // while the selection kernel may still run (only the pooling and
      // selection kernels let their dependents start early, and neither
      // writes Q, K or V)
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bar_kfull[0], KVT);
      for (int pn = 0; pn < NP; ++pn)
        tma_load_4d(sK + pn * (64 * 128), &tm_k, &bar_kfull[0], 64 * pn, h, 64 * i, b);
      mbar_arrive_expect_tx(&bar_vfull[0], KVT);
      for (int pn = 0; pn < NP; ++pn)
        tma_load_4d(sV + pn * (64 * 128), &tm_v, &bar_vfull[0], 64 * pn, h, 64 * i, b);
      mbar_arrive_expect_tx(bar_q, T * QTILE);
      for (int t = 0; t < T; ++t)
        for (int hh = 0; hh < 2; ++hh)
          for (int pn = 0; pn < NP; ++pn)
            tma_load_4d(sQ + t * QTILE + pn * (128 * 128) + hh * (64 * 128), &tm_q, bar_q, 64 * pn,
                        hq0 + 2 * t + hh, 64 * i, b);
    }
  }
  // launched with programmatic serialization: the index table may still be
  // in flight from the selection kernel until here
  pdl_wait();
  if (MASS && warp == 0) {
    const int words = (p.n + 31) / 32;
    for (int w = lane; w < words; w += 32) selbits[w] = 0u;
    __syncwarp();
    for (int r = lane; r < nsel; r += 32) {
      const int j = idx_row[r];
      if (j >= 0 && j <= i) atomicOr(&selbits[j >> 5], 1u << (j & 31));
    }
  }
  if (DASH && warp == 0) dash_build_list(p, b, h, i, lane, dord, dbias, dcount);
  if (EARLY && threadIdx.x == 0) {
    *all_stop = 0;
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
        // per unit: its first K/V block, then its Q once the previous unit's
        // last score MMAs have read the old Q, then the rest of its blocks
        int g = 0, k = 0;  // K/V blocks and units loaded so far
        int qk = 0;        // the last unit whose Q was loaded (unit 0: before the table wait)
        bool alive = true;
        for (int u = static_cast<int>(blockIdx.x); alive && u < n_units; u += gridDim.x, ++k) {
          const Unit w = unit_of(u);
          // the diagonal block first (the table's last entry), then the others
          // in table order
          for (int s = 0; s < w.nsel; ++s) {
            const int st = g % NS, use = g / NS;
            if (k == 0 && s == 0) {  // issued with Q before the table wait
              ++g;
              continue;
            }
            if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, abort_flag, tmo, 0x101)) {
              alive = false;
              break;
            }
            const int j = s == 0 ? w.i : w.idx_row[s - 1];
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
          // EARLY: once every tile stopped, the stage is never released; the
          // stop flag ends the wait instead
          if (use > 0 && !(EARLY ? mbar_wait_or(&bar_empty[st], (use - 1) & 1, abort_flag, all_stop, tmo, 0x101)
                                 : mbar_wait(&bar_empty[st], (use - 1) & 1, abort_flag, tmo, 0x101)))
            break;
          load_kv(st, MASS ? jj : (EARLY ? ord[jj] : (DASH ? dord[jj] : idx_row[jj])));
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
  } else if (warp >= 1 && warp <= C::ISS) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer warp w owns M-tiles t = w - 1, w - 1 + ISS, ...  Every tile
    // advances one block per round, so the issuer serves its tiles round-robin
    // with suspending waits (no issue slots taken from the softmax warps while
    // it waits).  Operand descriptors are built once; an operand offset is
    // added to the descriptor's address field (byte offset / 16).  A K/V stage
    // is released once all of the issuer's tiles committed their P.V on it.
    if (lane == 0) {
      constexpr int ISS = C::ISS;
      constexpr int MT = (T + ISS - 1) / ISS;  // tiles per issuer
      const int me = warp - 1;
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 64 * 128, 1024);
      auto issue_qk = [&](int t, int st) {
        const uint32_t d = tmem + t * TSTRIDE;
        const uint64_t a0 = dQ + ((t * QTILE) >> 4), b0 = dK + ((st * KVT) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 bf16 = 32 B inside a 128 B row; 64-column panels
          const uint32_t oa = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
          const uint32_t ob = ((kk / 4) * (64 * 128) + (kk % 4) * 32) >> 4;
          mma_ss(d, a0 + oa, b0 + ob, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // Per unit: the score MMAs of its first block once its Q and first K/V
      // block landed (S and P of every tile are free: this thread issued the
      // previous unit's last P.V before them), then block by block as above.
      // Parities count the CTA's blocks (g + jj) and units (k).
      bool ok = true;
      int g = 0, k = 0;
      for (int u = static_cast<int>(blockIdx.x); ok && u < n_units; u += gridDim.x, ++k) {
        const int nb = PERSIST ? unit_of(u).nsel : nblk;
        ok = mbar_wait(bar_q, k & 1, abort_flag, tmo, 0x201) &&
             mbar_wait(&bar_kfull[g % NS], (g / NS) & 1, abort_flag, tmo, 0x202);
        if (!ok) break;
        tc_fence_after();
        for (int t = me; t < T; t += ISS) {
          issue_qk(t, g % NS);
          tc_commit(&bar_sfull[t]);
        }
        if (PERSIST && nb == 1) tc_commit(bar_qfree);  // the unit's last score MMAs read Q
        bool first_sel[MT], first_uns[MT], stopped[MT];
#pragma unroll
        for (int x = 0; x < MT; ++x) first_sel[x] = first_uns[x] = true, stopped[x] = false;
        for (int jj = 0; ok && jj < nb; ++jj) {
          const int gj = g + jj;
          const int st = gj % NS;
          const bool more = jj + 1 < nb;
          const int st1 = (gj + 1) % NS;
          if (!mbar_wait(&bar_vfull[st], (gj / NS) & 1, abort_flag, tmo, 0x203) ||
              (more && !mbar_wait(&bar_kfull[st1], ((gj + 1) / NS) & 1, abort_flag, tmo, 0x204))) {
            ok = false;
            break;
          }
          bool is_sel = true;
          if (MASS) is_sel = (selbits[jj >> 5] >> (jj & 31)) & 1u;
          const uint64_t v0 = dV + ((st * KVT) >> 4);
#pragma unroll
          for (int x = 0; x < MT; ++x) {
            const int t = me + x * ISS;
            if (t >= T || !ok || (EARLY && stopped[x])) continue;
            // keys 0..31 as soon as the first half of P is stored
            if (!mbar_wait(&bar_phalf[t], gj & 1, abort_flag, tmo, 0x205)) {
              ok = false;
              continue;
            }
            tc_fence_after();
            const bool first = MASS ? (is_sel ? first_sel[x] : first_uns[x]) : (jj == 0);
            const uint32_t base = tmem + t * TSTRIDE;
            const uint32_t o_col = base + 64 + ((MASS && !is_sel) ? D : 0);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // 16 keys per MMA: 16 rows of 128 B
              mma_ts(o_col, base + kk * 8, v0 + ((kk * (16 * 128)) >> 4), idesc_pv,
                     (first && kk == 0) ? 0u : 1u);
            if (!mbar_wait(&bar_pfull[t], gj & 1, abort_flag, tmo, 0x206)) {
              ok = false;
              continue;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 2; kk < 4; ++kk)
              mma_ts(o_col, base + kk * 8, v0 + ((kk * (16 * 128)) >> 4), idesc_pv, 1u);
            // EARLY: the softmax records the position of the block it stops at
            // before it arrives on that block's pfull (the same rule as the
            // head_dim-128 kernel, where the next S is issued before this read)
            const bool stop_now = EARLY && tile_stop[t] == jj + 1;
            if (more && !stop_now) {
              issue_qk(t, st1);
              tc_commit(&bar_sfull[t]);
            } else {
              tc_commit(&bar_odone[t]);
              if (EARLY) stopped[x] = true;
            }
            if (MASS) {
              if (is_sel) first_sel[x] = false; else first_uns[x] = false;
            }
          }
          if (PERSIST && ok && jj + 2 == nb) tc_commit(bar_qfree);  // every tile's last S issued
          if (ok) tc_commit(&bar_empty[st]);  // this issuer's tiles are all done with the stage
          if (EARLY) {
            bool all = true;
#pragma unroll
            for (int x = 0; x < MT; ++x)
              if (me + x * ISS < T && !stopped[x]) all = false;
            if (all) {  // no tile visits more blocks: the producer stops too
              *all_stop = 1;
              break;
            }
          }
        }
        g += nb;
      }
      if (!ok) {
        // every MMA this thread issued completes before TMEM is released
        tc_commit(&bar_drain[me]);
        volatile int never = 0;
        mbar_wait(&bar_drain[me], 0, &never, tmo, 0x2ff);
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int hh = r / 64, tq = r % 64;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16) + t * TSTRIDE;
    const uint32_t tS = lane_base, tO = lane_base + 64;
    const uint32_t tOu = tO + D;
    const float sl2 = p.scale_log2;
    const uint64_t scale2 = f2_pack(sl2, sl2);
    bool ok = true;
    // parities count the CTA's blocks (g + jj) and units (k)
    int g = 0, k = 0;
    for (int u = static_cast<int>(blockIdx.x); ok && u < n_units; u += gridDim.x, ++k) {
      const int nb = PERSIST ? min(p.topk, p.i_hi - u / per_i) : nblk;
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
        // the diagonal block comes first in the plain (persistent) and the
        // early-stop orders, last in the other modes' ascending orders
        const bool diag = (EARLY || PERSIST) ? (jj == 0) : (jj == nb - 1);
        bool is_sel = true;
        if (MASS) is_sel = (selbits[jj >> 5] >> (jj & 31)) & 1u;
        // all 64 scores with one TMEM round trip, then the raw row maximum
        float sv[64];
        float alpha = 1.f;
        bool moved = false;
        uint64_t negm2 = 0, acc2 = f2_pack(0.f, 0.f);
        uint32_t pk[16];
        if (live) {
          tmem_ld64(tS, sv);
          float mx = diag ? row_max32<true>(sv + 32, 32, tq, -INFINITY)
                          : row_max32<false>(sv + 32, 32, tq, -INFINITY);
          mx = diag ? row_max32<true>(sv, 0, tq, mx) : row_max32<false>(sv, 0, tq, mx);
          // DASH: the chunk's prior adds sigma * log2 w_j to every score of the block
          const float bias = DASH ? dbias[jj] : 0.f;
          const float mx_s = mx * sl2 + bias;
          moved = mx_s > m_ref + 8.f;
          if (moved) {
            alpha = ex2(m_ref - mx_s);
            m_ref = mx_s;
          }
          negm2 = f2_pack(bias - m_ref, bias - m_ref);
          if (diag) exp_pack32<true>(sv, 0, tq, scale2, negm2, acc2, pk);
          else exp_pack32<false, C::POLY>(sv, 0, tq, scale2, negm2, acc2, pk);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
        }
        // O is stable here (S(jj) was committed after P(jj-1).V) and is read by
        // the tensor core only after phalf: rescale it when the maximum moved
        if (jj > 0 && __any_sync(0xffffffffu, moved)) {
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
        }
        tmem_st16(tS, pk);  // P columns 0..15 over S columns 0..15 (already read)
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_phalf[t]);
        if (live) {
          if (diag) exp_pack32<true>(sv + 32, 32, tq, scale2, negm2, acc2, pk);
          else exp_pack32<false, C::POLY>(sv + 32, 32, tq, scale2, negm2, acc2, pk);
        }
        tmem_st16(tS + 16, pk);  // P columns 16..31
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
        const Unit w = PERSIST ? unit_of(u) : u0;  // this unit's rows
        const int hq = w.hq0 + 2 * t + hh;
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
