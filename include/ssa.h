/*
 * ssa.h -- C ABI of libssa, the B200 (sm_100a) SSA sparse-stream kernels.
 *
 * SSA ("Sparse Sparse Attention") trains a model with a block-sparse attention
 * stream and a full attention stream side by side.  This library implements
 * the data-parallel hot path of the sparse stream on one GPU:
 *
 *   ssa_block_pool               mean-pooled block summaries of K (and of the
 *                                GQA-group queries)
 *   ssa_block_select             top-k block selection per query block, the
 *                                diagonal block always kept
 *   ssa_sparse_attn_fwd          exact softmax attention over the selected
 *                                blocks only (online softmax, tcgen05 + TMEM)
 *   ssa_full_attn_fwd_with_mass  the dense causal counterpart, the sparse
 *                                output and the dropped attention mass, all
 *                                from one launch
 *   ssa_sparse_attn_bwd          dQ, dK, dV over the selected pairs only
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named q, k, v, o, d_o, dq, dk, dv, ... are DEVICE pointers owned
 *    by the caller.  The library never allocates, frees or retains device
 *    memory.  bf16 tensors are passed as ssa_bf16 (the 16-bit storage of
 *    IEEE-754 bfloat16); every tensor is dense and contiguous.
 *  - Layouts (row-major):
 *        q, o, d_o, dq           [B][S][Hq][D]     bf16
 *        k, v, dk, dv            [B][S][Hkv][D]    bf16
 *        k_pooled, q_pooled      [B][Hkv][n][D]    fp32    n = S / block_size
 *        block_idx               [B][Hkv][n][top_k] int32
 *        lse, lse_*, dropped     [B][Hq][S]        fp32
 *    Query head hq uses KV head hq / (Hq / Hkv).  Token t belongs to block
 *    t / block_size.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Arguments are validated on the host before anything is
 *    launched: a bad argument returns SSA_ERR_INVALID_ARG and a shape this
 *    build does not implement returns SSA_ERR_UNSUPPORTED, in both cases with
 *    nothing launched and no output touched.  A launch failure returns
 *    SSA_ERR_CUDA.  A kernel whose bounded wait ran out records the fact in a
 *    device error word and exits early; ssa_get_device_error() reports it.
 *  - Outputs are fully overwritten (dk and dv are written, not accumulated).
 *  - Device pointers must be 16-byte aligned (TMA and vector accesses).
 *
 * Supported shapes in this build: block_size = 64, head_dim in {64, 128},
 * causal = 1, seq_len a positive multiple of 64 up to 524288, Hq a multiple
 * of Hkv with an even group size G = Hq / Hkv (2, 4, 8 or 16), top_k >= 1.
 *
 * Passages cited below are from the pages this method is described on:
 *  [SSA-es]  "Resumen Tecnico: SSA (Sparse Sparse Attention)"
 *  [SSA-it]  "SSA: Guida a Sparse Sparse Attention per LLM"
 *  [Dash]    the DashAttention summary (hierarchical routing)
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, inconsistent sizes     */
  SSA_ERR_UNSUPPORTED = 2,     /* valid problem that this build does not implement */
  SSA_ERR_CUDA = 3,            /* a CUDA runtime/driver call or launch failed      */
  SSA_ERR_DEVICE_TIMEOUT = 4,  /* a kernel's bounded wait ran out (see below)      */
  SSA_ERR_WORKSPACE = 5        /* workspace missing or smaller than required        */
} ssa_status;

typedef uint16_t ssa_bf16;               /* bfloat16 storage                       */
typedef struct CUstream_st *ssa_stream;  /* same type as cudaStream_t              */

/* The problem statement: Q/K/V shapes, block size, top-k budget, causal mask
 * ([SSA-it] "Block-sparse attention e Receptive Field": contiguous blocks,
 * top-k blocks per query, receptive field = block size x blocks selected). */
typedef struct {
  int batch;          /* B  >= 1                                                */
  int seq_len;        /* S, multiple of block_size                               */
  int n_q_heads;      /* Hq, multiple of n_kv_heads                              */
  int n_kv_heads;     /* Hkv (GQA: fewer KV heads than query heads, [SSA-it]
                         "Approccio generale" / "Training recipe")               */
  int head_dim;       /* D                                                       */
  int block_size;     /* query block == key block; 64 in this build              */
  int top_k;          /* blocks per query block INCLUDING the diagonal, >= 1     */
  int causal;         /* must be 1                                               */
  float softmax_scale;/* <= 0 selects 1/sqrt(head_dim)                           */
} ssa_problem;

/* Mean pooling of blocks ([SSA-it] "Block-sparse attention e Receptive Field":
 * a mean representation of each block; [Dash] Stage 0: a zero-initialised
 * summary query is a uniform mean).
 *   k_pooled[b,h,j,:] = (1/64) * sum_{t in block j} k[b,t,h,:]
 *   q_pooled[b,h,i,:] = (1/(64*G)) * sum_{g<G} sum_{t in block i} q[b,t,h*G+g,:]
 * Sums and outputs are fp32.  q and q_pooled may both be NULL (keys only). */
ssa_status ssa_block_pool(const ssa_problem *p, const ssa_bf16 *k, const ssa_bf16 *q,
                          float *k_pooled, float *q_pooled, ssa_stream stream);

/* Top-k block selection ([SSA-it] same section: keep only the top-k most
 * relevant earlier blocks; [Dash] Stage 1: heads sharing a KV head share one
 * support, here by scoring the group-pooled query).  For query block i:
 *   score(i, j) = q_pooled[i] . k_pooled[j]  (fp32) for j < i;
 *   selected = {i} + the top_k - 1 highest-scoring j < i (ties: lower j first);
 *   when i + 1 <= top_k every block 0..i is selected.
 * block_idx[b,h,i,:] lists the selected blocks in ascending order, padded with
 * -1 after the min(top_k, i + 1) valid entries. */
ssa_status ssa_block_select(const ssa_problem *p, const float *q_pooled, const float *k_pooled,
                            int32_t *block_idx, ssa_stream stream);

/* Sparse attention forward ([SSA-es] section 2, sparse stream; [SSA-it]: the
 * attention is computed only over the tokens of the selected blocks).
 * For query t of block i and head hq (KV head h):
 *   o[t]   = sum_{s in sel(i), s <= t} softmax_s(scale * q_t . k_s) * v_s
 *   lse[t] = ln sum_{s in sel(i), s <= t} exp(scale * q_t . k_s)
 * block_idx must satisfy the ssa_block_select output contract (ascending,
 * diagonal present, min(top_k, i + 1) valid entries); it is trusted.
 * o is rounded to bf16 (nearest even); lse is the natural log, fp32. */
ssa_status ssa_sparse_attn_fwd(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k,
                               const ssa_bf16 *v, const int32_t *block_idx, ssa_bf16 *o,
                               float *lse, ssa_stream stream);

/* Bytes of device workspace ssa_sparse_attn_fwd_host needs for problem p (0
 * on an invalid problem): device copies of Q, K, V, O and LSE whole, the
 * pooled keys and queries, and the index table. */
size_t ssa_sparse_attn_fwd_host_workspace(const ssa_problem *p);

/* ssa_block_pool, ssa_block_select and ssa_sparse_attn_fwd on HOST buffers:
 * q [B][S][Hq][D], k and v [B][S][Hkv][D] bf16 in, o [B][S][Hq][D] bf16 and
 * lse [B][Hq][S] fp32 out, all in host memory (page-locked, or the copies do
 * not overlap).  `workspace` is caller-owned device memory of at least
 * ssa_sparse_attn_fwd_host_workspace(p) bytes, 256-byte aligned.  K and V are
 * copied in whole and the keys pooled; then the query blocks stream through
 * in chunks of consecutive blocks (every batch entry and head; at least 8 MB
 * of Q per chunk, at most sixteen chunks):
 * a chunk's Q rows are copied in on an internal stream, its queries pooled,
 * its rows selected and attended on `stream`, and its O rows and LSE columns
 * copied out on a second internal stream, so both copy directions and the
 * kernels of neighbouring chunks overlap.  The results equal the
 * device-buffer calls bit for bit.
 * `stream` is ordered after everything before the call and waits for the
 * last copy out, so synchronising it makes o and lse valid on the host.
 * Not capturable in a CUDA graph.  Errors: INVALID_ARG for null pointers,
 * WORKSPACE for a missing, misaligned or short workspace. */
ssa_status ssa_sparse_attn_fwd_host(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k, const ssa_bf16 *v,
                                    ssa_bf16 *o, float *lse, void *workspace, size_t ws_bytes, ssa_stream stream);

/* Full causal attention with its sparse counterpart and the dropped mass, in
 * one launch ([SSA-es] section 2 "Alineacion Bidireccional": the opposite-mode
 * output is computed alongside, for the alignment only; section 1: the error
 * of sparse attention grows linearly with the attention mass it drops).
 * Every causal block's contribution is accumulated either into the selected
 * or into the unselected accumulator, against one shared running maximum:
 *   o_sparse, lse_sparse  as ssa_sparse_attn_fwd
 *   o_full, lse_full      dense causal attention over all s <= t
 *   dropped[t]            = 1 - exp(lse_sparse[t] - lse_full[t])
 *                         = full-softmax weight on the causal tokens not selected */
ssa_status ssa_full_attn_fwd_with_mass(const ssa_problem *p, const ssa_bf16 *q,
                                       const ssa_bf16 *k, const ssa_bf16 *v,
                                       const int32_t *block_idx, ssa_bf16 *o_sparse,
                                       float *lse_sparse, ssa_bf16 *o_full, float *lse_full,
                                       float *dropped, ssa_stream stream);

/* The sparse forward with an early stop ("S2O" summary, section 2, "Regla de
 * Parada Temprana", applied to the sparse stream): each query block visits
 * its diagonal block first, then its other selected blocks in descending
 * pooled score q_pooled[i] . k_pooled[j] (fp32; ties: lower j).  The unit
 * that stops is one query segment of one head: query head hq, the 64 tokens
 * of query block i.  It stops after the first block that adds, for every one
 * of its rows, less than tau times the attention mass the row had
 * accumulated before it (that block still counts); the heads of a KV group
 * share the order and stop on their own.  tau = 0 visits every selected
 * block (the ssa_sparse_attn_fwd result, up to summation order).
 * q_pooled/k_pooled: the outputs of ssa_block_pool for the same q, k;
 * block_idx: ssa_block_select's table.  Outputs o, lse as for the sparse
 * forward, and, if visited is not NULL, the blocks each segment visited,
 * [B][Hq][n] int32.
 * Errors: INVALID_ARG for null/misaligned pointers or tau not finite and
 * >= 0; UNSUPPORTED for top_k > 256 and the cases of the sparse forward. */
ssa_status ssa_sparse_attn_fwd_early_stop(const ssa_problem *p, const ssa_bf16 *q,
                                          const ssa_bf16 *k, const ssa_bf16 *v,
                                          const float *q_pooled, const float *k_pooled,
                                          const int32_t *block_idx, float tau, ssa_bf16 *o,
                                          float *lse, int32_t *visited, ssa_stream stream);

/* DashAttention chunk routing ("Resumen Tecnico: DashAttention", stage 1 and
 * its GQA rule; chunks are the 64-token blocks, summarised by their mean key
 * -- stage 0 with its summary query at its zero initialisation).  For query
 * block i of KV head h, each query head g of the group scores the complete
 * earlier chunks j < i:
 *   z_gj = gamma * scale * qmean_g(i) . k_pooled[b][h][j]
 * (qmean_g(i): the mean of head g's 64 queries of block i; scale: the
 * problem's softmax scale), p_g = alpha-entmax(z_g), the distribution
 *   p_gj = [(alpha - 1) z_gj - tau_g]_+ ^ (1 / (alpha - 1)),  sum_j p_gj = 1,
 * and the group shares w_j = mean_g p_gj.  tau_g is found in fp32 by
 * bisection until its bracket stops shrinking; p_g is then normalised.
 *   q         [B][S][Hq][D] bf16
 *   k_pooled  [B][Hkv][n][D] fp32, ssa_block_pool's mean keys
 *   weights   [B][Hkv][n][n] fp32 out: row i holds w_j for j < i, 0 elsewhere
 *   mask      [B][Hkv][n][ceil(n / 32)] uint32 out: bit j of row i (word
 *             j / 32, bit j % 32) is set for j < i with w_j > 0, and bit i
 *             (the diagonal chunk, which is not routed) always.
 * top_k of the problem is not used.  Errors: INVALID_ARG for null/misaligned
 * pointers, alpha outside (1, 4] or gamma not finite and > 0; UNSUPPORTED for
 * more than 1024 chunks (n = S / 64). */
ssa_status ssa_dash_route(const ssa_problem *p, const ssa_bf16 *q, const float *k_pooled, float alpha,
                          float gamma, float *weights, uint32_t *mask, ssa_stream stream);

/* DashAttention's prior-induced sparse softmax ("Resumen Tecnico:
 * DashAttention", stage 2): softmax attention whose reference distribution
 * is a prior g over the keys instead of the uniform one, i.e. attention
 * weights proportional to g_s exp(z_s).  g is uniform inside a chunk and
 * proportional to w_j^sigma across the active chunks (sigma: the prior's
 * strength; 0 gives plain attention over the support), and 0 elsewhere.  For
 * query t of block i the active chunks are the j < i whose mask bit is set and
 * whose weight is finite and > 0, plus the diagonal chunk i (its own branch,
 * weight 1, causal), so the logits are
 *   scale * q_t . k_s + sigma * ln w_j(s)   over the active keys s <= t.
 * weights/mask: as written by ssa_dash_route (any values are accepted; bits
 * at or after the diagonal are ignored).  Outputs o [B][S][Hq][D] bf16 and lse
 * [B][Hq][S] fp32, the natural-log log-sum-exp of the biased logits.
 * top_k of the problem is not used.  Errors: INVALID_ARG for null/misaligned
 * pointers or sigma not finite and >= 0; UNSUPPORTED for more than 1024
 * chunks. */
ssa_status ssa_dash_attn_fwd(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k, const ssa_bf16 *v,
                             const float *weights, const uint32_t *mask, float sigma, ssa_bf16 *o, float *lse,
                             ssa_stream stream);

/* Bytes of device workspace ssa_sparse_attn_bwd needs for problem p (0 on an
 * invalid problem). */
size_t ssa_sparse_attn_bwd_workspace(const ssa_problem *p);

/* Sparse attention backward ([SSA-es] section 1: keys outside the selected
 * blocks receive zero gradient; the selection itself is not differentiated).
 * With P_ts = exp(scale * q_t . k_s - lse_t) over the selected causal pairs:
 *   D_t = d_o_t . o_t;  dv_s = sum_t P_ts d_o_t;  dS_ts = P_ts (d_o_t . v_s - D_t)
 *   dq_t = scale sum_s dS_ts k_s;  dk_s = scale sum_t dS_ts q_t
 * (sums over the G heads of a group go into dk, dv).  o and lse are the
 * outputs of ssa_sparse_attn_fwd for the same inputs.  `workspace` is a
 * caller-owned device buffer of at least ssa_sparse_attn_bwd_workspace(p)
 * bytes, 256-byte aligned; its contents on entry do not matter. */
ssa_status ssa_sparse_attn_bwd(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k,
                               const ssa_bf16 *v, const ssa_bf16 *o, const float *lse,
                               const ssa_bf16 *d_o, const int32_t *block_idx, ssa_bf16 *dq,
                               ssa_bf16 *dk, ssa_bf16 *dv, void *workspace, size_t ws_bytes,
                               ssa_stream stream);

/* Bytes of device workspace ssa_alignment_bwd needs for problem p (0 on an
 * invalid problem). */
size_t ssa_alignment_bwd_workspace(const ssa_problem *p);

/* Backward of one layer of SSA's training objective with the bidirectional
 * alignment loss ([SSA-es] section 2, "Alineacion Bidireccional"): the
 * gradient of
 *     <d_o, h_mode> + alpha * (L_sparsity + L_commit)
 * with respect to q, k and v, where h_sparse and h_full are the sparse and
 * the full (dense causal) attention outputs, d_o is the upstream gradient of
 * the stream this step trains (mode 0: the sparse output; mode 1: the full
 * output; the other output is the counterpart, computed for the alignment
 * only), and, reading the pages' unspecified distance as the mean squared
 * error over the N = B*S*Hq*D output elements with a stop-gradient (sg) on
 * the target,
 *     L_sparsity = mean (h_full - sg(h_sparse))^2   (full pulled to sparse)
 *     L_commit   = mean (h_sparse - sg(h_full))^2   (sparse pulled to full).
 * The output gradients are then d_o + c (h_sparse - h_full) for the sparse
 * stream (d_o only in mode 0) and c (h_full - h_sparse) for the full one
 * (plus d_o in mode 1), c = 2 alpha / N; each goes back through its stream's
 * attention (the full stream over every causal block) and dq, dk, dv are the
 * sums.  o_sparse/lse_sparse and o_full/lse_full are the outputs of
 * ssa_full_attn_fwd_with_mass for the same inputs and block_idx.  `workspace`
 * is a caller-owned device buffer of at least ssa_alignment_bwd_workspace(p)
 * bytes, 256-byte aligned; its contents on entry do not matter.
 * Errors: INVALID_ARG for a null or misaligned pointer, mode outside {0, 1}
 * or a non-finite alpha; WORKSPACE for a missing or short workspace. */
ssa_status ssa_alignment_bwd(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k,
                             const ssa_bf16 *v, const ssa_bf16 *o_sparse, const float *lse_sparse,
                             const ssa_bf16 *o_full, const float *lse_full, const ssa_bf16 *d_o,
                             int mode, float alpha, const int32_t *block_idx, ssa_bf16 *dq,
                             ssa_bf16 *dk, ssa_bf16 *dv, void *workspace, size_t ws_bytes,
                             ssa_stream stream);

/* Largest scratch (in bytes) that ssa_sparse_attn_bwd_noalloc can use. */
#define SSA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* ssa_sparse_attn_bwd without a workspace argument, for callers that cannot
 * allocate device memory: a plugin or runtime that is handed only its input
 * and output buffers, or a service that reserves all of its memory up front
 * and must not call an allocator while it serves (an allocation can block,
 * synchronise the device, fragment the heap or fail under memory pressure).
 * The pages have no counterpart for this call; it exists for such callers.
 *
 * Same arguments, layouts, results and errors as ssa_sparse_attn_bwd, minus
 * the workspace.  Its scratch is one array of SSA_NOALLOC_SCRATCH_BYTES that
 * the library holds in device memory on every GPU that loads it, for the
 * life of the process.  It allocates nothing and calls no allocator.
 *  - A problem whose scratch (ssa_sparse_attn_bwd_workspace) exceeds
 *    SSA_NOALLOC_SCRATCH_BYTES is rejected with SSA_ERR_WORKSPACE before
 *    anything is launched.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current, once, and keeps it.
 *    Make that first call before any stream capture on the device: the
 *    look-up may load the library's device code onto the device, which is
 *    not allowed while a stream is being captured.  A failed look-up
 *    returns SSA_ERR_CUDA.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; nothing in it has to start at zero.  Calls whose kernels
 *    overlap on the GPU (on different streams, or from several threads)
 *    race on it: order them on one stream or synchronise between them. */
ssa_status ssa_sparse_attn_bwd_noalloc(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k,
                                       const ssa_bf16 *v, const ssa_bf16 *o, const float *lse,
                                       const ssa_bf16 *d_o, const int32_t *block_idx,
                                       ssa_bf16 *dq, ssa_bf16 *dk, ssa_bf16 *dv,
                                       ssa_stream stream);

/* Bytes of device workspace ssa_decode_attn needs for problem p: 0, since
 * the table and the partial softmax states stay in shared memory.  Kept so
 * callers size every call's scratch the same way. */
size_t ssa_decode_attn_workspace(const ssa_problem *p);

/* One decoding step of the sparse stream against a KV cache ([SSA-it]
 * "Block-sparse attention e Receptive Field" applied to a single query;
 * [SSA-es] section 4: sparse-mode inference reads only the selected blocks).
 * p->seq_len is the cache capacity S (a multiple of 64), the other fields as
 * for the forward.  For sequence b with lengths[b] = L cached tokens
 * (1 <= L <= S), the query is token t = L - 1, already in the cache, with its
 * Hq heads in q [B][Hq][D] bf16.  Its block c = t / 64 may be partial.
 *  - Selection, per KV head h: the mean over the G heads of q is scored
 *    against k_pooled[b][h][j] for the complete blocks j < c (fp32, the mean
 *    keys ssa_block_pool writes, [B][Hkv][S/64][D]; rows j >= c are not
 *    read).  The top-(k-1) scores are kept (ties: lower j) together with block
 *    c.  If c + 1 <= k, every block 0..c is kept.
 *  - Attention: softmax(scale q.k) over the kept blocks' tokens, causal in
 *    block c (keys up to t), for each query head of the group.
 * k_cache, v_cache: [B][S][Hkv][D] bf16.  Outputs: o [B][Hq][D] bf16,
 * lse [B][Hq] fp32 (natural log), and, if block_idx is not NULL, the kept
 * blocks [B][Hkv][k] int32, ascending, -1 padded.  `workspace` and
 * `ws_bytes` are not read (ssa_decode_attn_workspace returns 0; NULL is fine).
 * One launch: a cluster of up to 8 CTAs per (b, KV head) scores, selects,
 * attends and merges; UNSUPPORTED if its shared memory (about 4 B per cached
 * block plus the K/V ring) exceeds 227 KB.
 * Errors: INVALID_ARG / UNSUPPORTED as for the other calls.  A
 * length outside 1..S is found on the device; that sequence's outputs become
 * 0 (lse -inf), and ssa_get_device_error then returns SSA_ERR_INVALID_ARG.
 * The pages have no decode kernel of their own; this call is the sparse
 * stream's selection and attention applied to one new token. */
ssa_status ssa_decode_attn(const ssa_problem *p, const ssa_bf16 *q, const ssa_bf16 *k_cache,
                           const ssa_bf16 *v_cache, const float *k_pooled, const int32_t *lengths,
                           ssa_bf16 *o, float *lse, int32_t *block_idx, void *workspace,
                           size_t ws_bytes, ssa_stream stream);

/* Synchronises `stream`, then reports and clears the device error word of the
 * current device: SSA_ERR_DEVICE_TIMEOUT if a kernel's bounded wait ran out
 * since the last call, SSA_ERR_INVALID_ARG if a kernel found a device-side
 * input outside its range (a decode length), SSA_ERR_CUDA if the stream
 * reported an error, else SSA_OK. */
ssa_status ssa_get_device_error(ssa_stream stream);

/* Site code of the most recent bounded wait that ran out on the current
 * device (0 if none since the library was loaded); for diagnostics.  The code
 * names the kernel role and the barrier; it is not cleared by
 * ssa_get_device_error. */
unsigned int ssa_get_device_error_site(void);

/* Launches one tiny kernel whose single wait can never be satisfied (an
 * mbarrier that nothing arrives on), bounded by timeout_us microseconds of
 * %globaltimer.  It exercises the timeout path without any fault: the kernel
 * records SSA_ERR_DEVICE_TIMEOUT in the device error word and returns. */
ssa_status ssa_debug_timeout_probe(int timeout_us, ssa_stream stream);

/* y[i] = 2^x[i] for n device floats, computed by the FMA-pipe polynomial the
 * forward kernels use for part of the softmax exponentials (instead of the
 * MUFU ex2 unit): maximum relative error 7.5e-5 for x in [-125, 64]; inputs
 * below -125 give 2^-125.  The pages have no counterpart: this call exists so
 * tests can check that approximation against exp2f.  INVALID_ARG for n < 0 or
 * null pointers with n > 0. */
ssa_status ssa_debug_exp2_poly(const float *x, float *y, int n, ssa_stream stream);

/* Static, human-readable name of a status code. */
const char *ssa_status_string(ssa_status s);

/* Number of kernels this library has launched since it was loaded (all
 * devices, all entry points); for accounting in benchmarks. */
uint64_t ssa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
