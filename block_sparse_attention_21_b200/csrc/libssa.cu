// libssa.cu -- host side of the C ABI declared in include/ssa.h: argument
// validation, TMA tensor-map construction, kernel dispatch and the device
// error word.  The whole library is one translation unit so that every kernel
// shares the one device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <vector>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "ssa.h"
#include "sm100.cuh"
#include "pool_select.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_psmem.cuh"
#include "attn_bwd.cuh"
#include "align_bwd.cuh"
#include "decode.cuh"
#include "dash.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;
constexpr int kMaxSeqLen = 524288;

uint64_t wait_timeout_ns() {
  static uint64_t ns = [] {
    const char* env = std::getenv("SSA_WAIT_TIMEOUT_MS");
    long ms = env ? std::atol(env) : 0;
    if (ms <= 0) ms = 2000;
    return static_cast<uint64_t>(ms) * 1000000ull;
  }();
  return ns;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

struct Dims {
  int B, S, Hq, Hkv, D, G, n, topk;
  float scale;
};

// Host-side validation shared by every entry point.
ssa_status check_problem(const ssa_problem* p, Dims* d) {
  if (p == nullptr) return SSA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->seq_len < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 ||
      p->head_dim < 1 || p->block_size < 1 || p->top_k < 1)
    return SSA_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return SSA_ERR_INVALID_ARG;
  if (p->seq_len % p->block_size != 0) return SSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale)) return SSA_ERR_INVALID_ARG;
  if (p->block_size != 64) return SSA_ERR_UNSUPPORTED;
  if (p->causal != 1) return SSA_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return SSA_ERR_UNSUPPORTED;
  const int G = p->n_q_heads / p->n_kv_heads;
  if (G != 2 && G != 4 && G != 8 && G != 16) return SSA_ERR_UNSUPPORTED;
  if (p->seq_len > kMaxSeqLen) return SSA_ERR_UNSUPPORTED;
  // grid and element counts stay far inside 32-bit launch limits
  const double rows = static_cast<double>(p->batch) * p->n_kv_heads * (p->seq_len / 64) * G;
  if (rows > 1.0e9) return SSA_ERR_UNSUPPORTED;
  d->B = p->batch;
  d->S = p->seq_len;
  d->Hq = p->n_q_heads;
  d->Hkv = p->n_kv_heads;
  d->D = p->head_dim;
  d->G = G;
  d->n = p->seq_len / 64;
  d->topk = p->top_k;
  d->scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
  return SSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor [d3][d2][d1][d0] (d0 innermost), box of 64 x 1 x 64 x 1 elements
// (64 columns of one head for 64 consecutive tokens), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int d0, int d1, int d2, int d3) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                              static_cast<cuuint64_t>(d2), static_cast<cuuint64_t>(d3)};
  const cuuint64_t strides[3] = {dims[0] * 2, dims[0] * dims[1] * 2, dims[0] * dims[1] * dims[2] * 2};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device).
template <typename K>
ssa_status ensure_smem(K kernel, int bytes, std::atomic<uint64_t>* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return SSA_ERR_CUDA;
  const uint64_t bit = 1ull << dev;
  if (done_mask->load() & bit) return SSA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return SSA_ERR_CUDA;
  done_mask->fetch_or(bit);
  return SSA_OK;
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static std::atomic<int> cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return 0;
  int c = cached[dev].load();
  if (c == 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(c);
  }
  return c;
}

ssa_status launch_result() {
  g_launches.fetch_add(1);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes; it calls pdl_wait before
// touching global memory.
template <typename... KArgs, typename... Args>
ssa_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  g_launches.fetch_add(1);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SSA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// blocks j0 .. j0 + nj - 1 (nj < 0: every block)
template <int D>
ssa_status launch_pool(const Dims& d, const void* k, const void* q, float* kb, float* qb,
                       cudaStream_t st, int j0 = 0, int nj = -1) {
  ssa::PoolParams pp;
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.kbar = kb;
  pp.qbar = qb;
  pp.S = d.S;
  pp.Hq = d.Hq;
  pp.Hkv = d.Hkv;
  pp.G = d.G;
  pp.n = d.n;
  pp.j0 = j0;
  if (nj < 0) nj = d.n;
  return launch_pdl(ssa::block_pool_kernel<D>, dim3(nj, d.Hkv, d.B), dim3(ssa::PoolConfig<D>::THREADS), 0,
                    st, pp);
}

template <int D, int KPL>
ssa_status launch_select(const Dims& d, const ssa::SelectParams& sp, cudaStream_t st) {
  static std::atomic<uint64_t> done{0};
  auto kernel = ssa::block_select_kernel<D, KPL>;
  const ssa_status s = ensure_smem(kernel, 200 * 1024, &done);
  if (s != SSA_OK) return s;
  const dim3 grid((sp.i1 - sp.i0 + ssa::kSelectWarps - 1) / ssa::kSelectWarps, d.B * d.Hkv);
  return launch_pdl(kernel, grid, dim3(32 * ssa::kSelectWarps), ssa::SelectConfig<D>::smem_bytes(d.n), st,
                    sp);
}

// Inputs of the routed (DashAttention) mode of the forward kernels.
struct DashIn {
  const uint32_t* mask = nullptr;
  const float* w = nullptr;
  float sigma = 0.f;
};

// EARLY: the early-stop variant (qbar, kbar, tau, visited are read only then);
// DASH: the routed softmax (dash is read only then)
template <int D, int T, bool MASS, bool EARLY = false, bool DASH = false>
ssa_status launch_fwd(const Dims& d, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* o, float* lse, void* of, float* lsef,
                      float* dropped, cudaStream_t st, const float* qbar = nullptr,
                      const float* kbar = nullptr, float tau = 0.f, int32_t* visited = nullptr,
                      DashIn dash = DashIn(), int i_lo = 0, int i_hi = -1) {
  using C = ssa::FwdConfig<D, T, MASS, EARLY, DASH>;
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = ssa::attn_fwd_kernel<D, T, MASS, EARLY, DASH>;
  ssa_status s = ensure_smem(kernel, C::SMEM_BYTES, &smem_done);
  if (s != SSA_OK) return s;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, d.Hq, d.S, d.B) || !make_map(&mk, k, D, d.Hkv, d.S, d.B) ||
      !make_map(&mv, v, D, d.Hkv, d.S, d.B))
    return SSA_ERR_CUDA;
  ssa::FwdParams fp;
  fp.B = d.B;
  fp.S = d.S;
  fp.Hq = d.Hq;
  fp.Hkv = d.Hkv;
  fp.G = d.G;
  fp.n = d.n;
  fp.topk = d.topk;
  fp.slices = (d.G / 2) / T;
  // query blocks i_lo .. i_hi - 1 (the plain mode only; the others take all)
  fp.i_lo = (MASS || EARLY || DASH) ? 0 : i_lo;
  fp.i_hi = (MASS || EARLY || DASH || i_hi < 0) ? d.n : i_hi;
  fp.scale_log2 = d.scale * 1.4426950408889634f;
  fp.idx = idx;
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.lse = lse;
  fp.o_full = static_cast<__nv_bfloat16*>(of);
  fp.lse_full = lsef;
  fp.dropped = dropped;
  fp.timeout_ns = wait_timeout_ns();
  fp.qbar = qbar;
  fp.kbar = kbar;
  fp.tau = tau;
  fp.visited = visited;
  fp.dmask = dash.mask;
  fp.dw = dash.w;
  fp.sigma = dash.sigma;
  // the plain sparse stream runs persistent CTAs, as many as are resident at
  // once, over the units; the other modes one CTA per unit
  const unsigned units = static_cast<unsigned>(d.B) * d.Hkv * (fp.i_hi - fp.i_lo) * fp.slices;
  const unsigned slots = static_cast<unsigned>(sm_count()) * C::MIN_CTAS;
  const bool persist = !MASS && !EARLY && !DASH;
  if (persist && slots == 0) return SSA_ERR_CUDA;
  const unsigned grid = persist ? std::min(units, slots) : units;
  return launch_pdl(kernel, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, mq, mk, mv, fp);
}

// The same launch for the kernel that stages P in shared memory.
template <int D, int T, bool MASS, bool DASH = false, bool EARLY = false>
ssa_status launch_psfwd(const Dims& d, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* o, float* lse, void* of, float* lsef,
                      float* dropped, cudaStream_t st, DashIn dash = DashIn(), const float* qbar = nullptr,
                      const float* kbar = nullptr, float tau = 0.f, int32_t* visited = nullptr,
                      int i_lo = 0, int i_hi = -1) {
  using C = ssa::PsFwdConfig<D, T, MASS, DASH, EARLY>;
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = ssa::attn_fwd_psmem_kernel<D, T, MASS, DASH, EARLY>;
  ssa_status s = ensure_smem(kernel, C::SMEM_BYTES, &smem_done);
  if (s != SSA_OK) return s;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, d.Hq, d.S, d.B) || !make_map(&mk, k, D, d.Hkv, d.S, d.B) ||
      !make_map(&mv, v, D, d.Hkv, d.S, d.B))
    return SSA_ERR_CUDA;
  ssa::FwdParams fp;
  fp.B = d.B;
  fp.S = d.S;
  fp.Hq = d.Hq;
  fp.Hkv = d.Hkv;
  fp.G = d.G;
  fp.n = d.n;
  fp.topk = d.topk;
  fp.slices = (d.G / 2) / T;
  // query blocks i_lo .. i_hi - 1 (the plain mode only; the others take all)
  fp.i_lo = (MASS || EARLY || DASH) ? 0 : i_lo;
  fp.i_hi = (MASS || EARLY || DASH || i_hi < 0) ? d.n : i_hi;
  fp.scale_log2 = d.scale * 1.4426950408889634f;
  fp.idx = idx;
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.lse = lse;
  fp.o_full = static_cast<__nv_bfloat16*>(of);
  fp.lse_full = lsef;
  fp.dropped = dropped;
  fp.timeout_ns = wait_timeout_ns();
  fp.qbar = qbar;
  fp.kbar = kbar;
  fp.tau = tau;
  fp.visited = visited;
  fp.dmask = dash.mask;
  fp.dw = dash.w;
  fp.sigma = dash.sigma;
  // the plain sparse stream runs persistent CTAs, one per SM, over the units;
  // the other modes one CTA per unit
  const unsigned units = static_cast<unsigned>(d.B) * d.Hkv * (fp.i_hi - fp.i_lo) * fp.slices;
  const unsigned sms = static_cast<unsigned>(sm_count());
  const bool persist = !MASS && !DASH && !EARLY;
  if (persist && sms == 0) return SSA_ERR_CUDA;
  const unsigned grid = persist ? std::min(units, sms) : units;
  return launch_pdl(kernel, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, mq, mk, mv, fp);
}

// ------------------------------------------------------- DashAttention route

template <int D, int G>
ssa_status launch_dash_route(const Dims& d, const void* q, const float* kbar, float alpha, float gamma,
                             float* w, uint32_t* mask, cudaStream_t st) {
  static std::atomic<uint64_t> done{0};
  auto kernel = ssa::dash_route_kernel<D, G>;
  const ssa_status s =
      ensure_smem(kernel, static_cast<int>(ssa::dash_route_smem(ssa::kDashMaxG, 128, ssa::kDashMaxN)), &done);
  if (s != SSA_OK) return s;
  ssa::DashRouteParams rp;
  rp.B = d.B;
  rp.S = d.S;
  rp.Hq = d.Hq;
  rp.Hkv = d.Hkv;
  rp.G = d.G;
  rp.n = d.n;
  rp.W = (d.n + 31) / 32;
  rp.am1 = alpha - 1.f;
  rp.inv_am1 = 1.f / (alpha - 1.f);
  rp.pw_mode = alpha == 1.5f ? 0 : (alpha == 2.f ? 1 : 2);
  rp.newton = alpha <= 2.f ? 1 : 0;
  rp.zscale = gamma * d.scale;
  rp.q = static_cast<const __nv_bfloat16*>(q);
  rp.kbar = kbar;
  rp.w = w;
  rp.mask = mask;
  return launch_pdl(kernel, dim3(d.n, d.Hkv, d.B), dim3(256), ssa::dash_route_smem(d.G, D, d.n), st, rp);
}

// ---------------------------------------------------------------- backward

size_t bwd_workspace_bytes(const Dims& d) {
  return ssa::bwd_workspace_layout(d.B, d.S, d.Hq, d.Hkv, d.n, d.topk, d.D).total;
}

// The dense causal backward needs no reverse index: its workspace layout is
// the sparse one with a one-entry table.
size_t dense_bwd_workspace_bytes(const Dims& d) {
  return ssa::bwd_workspace_layout(d.B, d.S, d.Hq, d.Hkv, d.n, 1, d.D).total;
}

template <int D, int TQ>
ssa_status launch_bwd(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* d_o, const int32_t* idx, void* dq, void* dk,
                      void* dv, void* workspace, cudaStream_t st, bool dense = false) {
  // dense: every causal block counts as selected; idx is not read
  const ssa::BwdWorkspace ws =
      ssa::bwd_workspace_layout(d.B, d.S, d.Hq, d.Hkv, d.n, dense ? 1 : d.topk, d.D);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  ssa::BwdParams bp;
  bp.B = d.B;
  bp.S = d.S;
  bp.Hq = d.Hq;
  bp.Hkv = d.Hkv;
  bp.G = d.G;
  bp.n = d.n;
  bp.topk = dense ? d.n : d.topk;
  bp.dense = dense ? 1 : 0;
  bp.slices = (d.G / 2) / TQ;
  bp.scale = d.scale;
  bp.scale_log2 = d.scale * 1.4426950408889634f;
  bp.o = static_cast<const __nv_bfloat16*>(o);
  bp.d_o = static_cast<const __nv_bfloat16*>(d_o);
  bp.lse = lse;
  bp.idx = dense ? reinterpret_cast<const int32_t*>(base) : idx;
  bp.dt = reinterpret_cast<float*>(base + ws.dt);
  bp.rev_off = reinterpret_cast<int32_t*>(base + ws.rev_off);
  bp.rev = reinterpret_cast<int32_t*>(base + ws.rev);
  bp.part = reinterpret_cast<float*>(base + ws.part);
  bp.dq = static_cast<__nv_bfloat16*>(dq);
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.timeout_ns = wait_timeout_ns();
  if (bp.slices < 1) return SSA_ERR_UNSUPPORTED;

  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, D, d.Hq, d.S, d.B) || !make_map(&mk, k, D, d.Hkv, d.S, d.B) ||
      !make_map(&mv, v, D, d.Hkv, d.S, d.B) || !make_map(&mdo, d_o, D, d.Hq, d.S, d.B))
    return SSA_ERR_CUDA;

  // 1. D_t and the reverse index
  const int dt_blocks = d.B * d.Hq * ((d.S + ssa::kDtRows - 1) / ssa::kDtRows);
  // the reverse-index CTAs first (they run longest), then the D_t CTAs; the
  // shared-memory attribute is set once, for the largest supported n
  static std::atomic<uint64_t> prep_done{0};
  ssa_status s = ensure_smem(ssa::bwd_prep_kernel<D>, static_cast<int>(ssa::bwd_prep_smem(kMaxSeqLen / 64)),
                             &prep_done);
  if (s != SSA_OK) return s;
  const int rev_blocks = dense ? 0 : d.B * d.Hkv;
  ssa::bwd_prep_kernel<D><<<rev_blocks + dt_blocks, 256, ssa::bwd_prep_smem(d.n), st>>>(bp, rev_blocks);
  s = launch_result();
  if (s != SSA_OK) return s;

  // 2. dK, dV: kDkdvSplit CTAs per (b, KV head, key block), then their sum
  {
    using C = ssa::DkdvConfig<D>;
    static std::atomic<uint64_t> done{0};
    auto kernel = ssa::attn_bwd_dkdv_kernel<D>;
    s = ensure_smem(kernel, C::SMEM_BYTES, &done);
    if (s != SSA_OK) return s;
    kernel<<<static_cast<unsigned>(d.B) * d.Hkv * d.n * ssa::kDkdvSplit, C::THREADS, C::SMEM_BYTES, st>>>(
        mq, mk, mv, mdo, bp);
    s = launch_result();
    if (s != SSA_OK) return s;
    ssa::bwd_dkdv_reduce_kernel<D><<<static_cast<unsigned>(d.B) * d.Hkv * d.n, 256, 0, st>>>(bp);
    s = launch_result();
    if (s != SSA_OK) return s;
  }
  // 3. dQ: one CTA per (b, KV head, query block, head pairs)
  {
    using C = ssa::DqConfig<D, TQ>;
    static std::atomic<uint64_t> done{0};
    auto kernel = ssa::attn_bwd_dq_kernel<D, TQ>;
    s = ensure_smem(kernel, C::SMEM_BYTES, &done);
    if (s != SSA_OK) return s;
    kernel<<<static_cast<unsigned>(d.B) * d.Hkv * d.n * bp.slices, C::THREADS, C::SMEM_BYTES, st>>>(
        mq, mk, mv, mdo, bp);
    return launch_result();
  }
}

// ------------------------------------------- backward without an allocation
// Scratch of ssa_sparse_attn_bwd_noalloc: one file-scope array per device.
// Host code must not use its name as a device address; the address is looked
// up once per device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SSA_NOALLOC_SCRATCH_BYTES];

void* noalloc_scratch_address() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = ptr;
  }
  return addr[dev];
}

__global__ void timeout_probe_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ssa::mbar_init(&bar, 1);
    abort_flag = 0;
    ssa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) ssa::mbar_wait(&bar, 0, &abort_flag, timeout_ns, 0x900);
}

// Applies the forward kernels' FMA-pipe exp2 to n inputs (pairs per thread).
__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float p0, p1;
  ssa::exp2_poly2(x0, x1, p0, p1);
  y[i] = p0;
  if (i + 1 < n) y[i + 1] = p1;
}

// Workspace of ssa_alignment_bwd: both streams' output gradients, the dense
// pass's input gradients, then the backward workspace both passes share.
struct AlignLayout {
  size_t do_s, do_f, dq2, dk2, dv2, bwd, total;
};

AlignLayout align_layout(const Dims& d) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t eq = static_cast<size_t>(d.B) * d.S * d.Hq * d.D * 2;
  const size_t ekv = static_cast<size_t>(d.B) * d.S * d.Hkv * d.D * 2;
  AlignLayout L;
  L.do_s = 0;
  L.do_f = L.do_s + al(eq);
  L.dq2 = L.do_f + al(eq);
  L.dk2 = L.dq2 + al(eq);
  L.dv2 = L.dk2 + al(ekv);
  L.bwd = L.dv2 + al(ekv);
  const size_t wb = bwd_workspace_bytes(d), wd = dense_bwd_workspace_bytes(d);
  L.total = L.bwd + (wb > wd ? wb : wd);
  return L;
}

template <int D, int TQ>
ssa_status launch_align_bwd(const Dims& d, const void* q, const void* k, const void* v,
                            const void* o_s, const float* lse_s, const void* o_f, const float* lse_f,
                            const void* d_o, int mode, float alpha, const int32_t* idx, void* dq,
                            void* dk, void* dv, void* workspace, cudaStream_t st) {
  const AlignLayout L = align_layout(d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* do_s = reinterpret_cast<__nv_bfloat16*>(ws + L.do_s);
  auto* do_f = reinterpret_cast<__nv_bfloat16*>(ws + L.do_f);
  const long long nq8 = static_cast<long long>(d.B) * d.S * d.Hq * d.D / 8;
  const long long nkv8 = static_cast<long long>(d.B) * d.S * d.Hkv * d.D / 8;
  const float c = static_cast<float>(2.0 * alpha / (8.0 * static_cast<double>(nq8)));
  auto grid_of = [](long long n8) {
    const long long g = (n8 + 255) / 256;
    return static_cast<unsigned>(g < 148 * 16 ? g : 148 * 16);
  };
  ssa::align_grad_kernel<<<grid_of(nq8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o_s), static_cast<const __nv_bfloat16*>(o_f),
      static_cast<const __nv_bfloat16*>(d_o), mode, c, do_s, do_f, nq8);
  ssa_status s = launch_result();
  if (s != SSA_OK) return s;
  // the sparse stream over the selected blocks, the full stream over every causal block
  s = launch_bwd<D, TQ>(d, q, k, v, o_s, lse_s, do_s, idx, dq, dk, dv, ws + L.bwd, st);
  if (s != SSA_OK) return s;
  s = launch_bwd<D, TQ>(d, q, k, v, o_f, lse_f, do_f, nullptr, ws + L.dq2, ws + L.dk2, ws + L.dv2,
                        ws + L.bwd, st, true);
  if (s != SSA_OK) return s;
  ssa::add_bf16_kernel<<<grid_of(nq8), 256, 0, st>>>(static_cast<__nv_bfloat16*>(dq),
                                                     reinterpret_cast<const __nv_bfloat16*>(ws + L.dq2), nq8);
  if ((s = launch_result()) != SSA_OK) return s;
  ssa::add_bf16_kernel<<<grid_of(nkv8), 256, 0, st>>>(static_cast<__nv_bfloat16*>(dk),
                                                      reinterpret_cast<const __nv_bfloat16*>(ws + L.dk2), nkv8);
  if ((s = launch_result()) != SSA_OK) return s;
  ssa::add_bf16_kernel<<<grid_of(nkv8), 256, 0, st>>>(static_cast<__nv_bfloat16*>(dv),
                                                      reinterpret_cast<const __nv_bfloat16*>(ws + L.dv2), nkv8);
  return launch_result();
}

// ssa_decode_attn: one launch of decode_kernel<D, G>, a cluster of ns CTAs per
// (b, KV head).  ns fills the resident CTA slots once (up to 8, and no more
// than the blocks a row keeps); the CTAs of a cluster split the scoring and
// the kept blocks between them.
struct DecodeLaunch {
  int ns, slice_cap, cand_cap, smem;
};

template <int D, int G>
DecodeLaunch decode_launch_shape(const Dims& d) {
  const int need = d.topk - 1;
  const bool can_search = d.topk < d.n;  // else every causal block is kept
  auto shape = [&](int ns) {
    DecodeLaunch s;
    s.ns = ns;
    s.slice_cap = can_search ? (d.n - 1 + ns - 1) / ns : 0;
    s.cand_cap = can_search ? std::min(d.n - 1, ns * std::min(need, s.slice_cap)) : 0;
    s.smem = ssa::decode_smem<D, G>(d.n, d.topk, s.slice_cap, s.cand_cap).total;
    return s;
  };
  const DecodeLaunch one = shape(1);
  const int per_sm = std::max(1, std::min(2048 / ssa::kDecodeThreads, (228 * 1024) / (one.smem + 1024)));
  const int slots = std::max(1, sm_count()) * per_sm;
  const int units = d.B * d.Hkv;
  int ns = std::max(1, std::min(ssa::kDecodeMaxCluster, slots / units));
  ns = std::min(ns, std::max(1, std::min(d.topk, d.n)));
  return shape(ns);
}

template <int D, int G>
ssa_status launch_decode_g(const Dims& d, ssa::DecodeParams dp, cudaStream_t st) {
  static std::atomic<uint64_t> smem_done{0};
  constexpr int kMaxSmem = 227 * 1024;
  auto kernel = ssa::decode_kernel<D, G>;
  const DecodeLaunch s = decode_launch_shape<D, G>(d);
  if (s.smem > kMaxSmem) return SSA_ERR_UNSUPPORTED;
  const ssa_status e0 = ensure_smem(kernel, kMaxSmem, &smem_done);
  if (e0 != SSA_OK) return e0;
  dp.ns = s.ns;
  dp.slice_cap = s.slice_cap;
  dp.cand_cap = s.cand_cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(d.B) * d.Hkv * s.ns);
  cfg.blockDim = dim3(ssa::kDecodeThreads);
  cfg.dynamicSmemBytes = s.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = s.ns;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, dp) != cudaSuccess) {
    cudaGetLastError();
    return SSA_ERR_CUDA;
  }
  return launch_result();  // counts the launch
}

template <int D>
ssa_status launch_decode(const Dims& d, const void* q, const void* k, const void* v, const float* kbar,
                         const int32_t* len, void* o, float* lse, int32_t* idx_out, cudaStream_t st) {
  ssa::DecodeParams dp;
  dp.B = d.B;
  dp.S = d.S;
  dp.Hq = d.Hq;
  dp.Hkv = d.Hkv;
  dp.G = d.G;
  dp.n = d.n;
  dp.topk = d.topk;
  dp.ns = 1;
  dp.slice_cap = 0;
  dp.cand_cap = 0;
  dp.scale_log2 = d.scale * 1.4426950408889634f;
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.k = static_cast<const __nv_bfloat16*>(k);
  dp.v = static_cast<const __nv_bfloat16*>(v);
  dp.kbar = kbar;
  dp.len = len;
  dp.idx = idx_out;
  dp.o = static_cast<__nv_bfloat16*>(o);
  dp.lse = lse;
  switch (d.G) {
    case 2: return launch_decode_g<D, 2>(d, dp, st);
    case 4: return launch_decode_g<D, 4>(d, dp, st);
    case 8: return launch_decode_g<D, 8>(d, dp, st);
    default: return launch_decode_g<D, 16>(d, dp, st);
  }
}

// ------------------------------------------------------------ host buffers
// ssa_sparse_attn_fwd_host: device copies of Q, K, V, O and LSE whole, the
// pooled keys and queries and the index table.  K and V are copied first and
// pooled; then chunks of consecutive query blocks (all batch entries and
// heads) stream through: a chunk's Q rows in (contiguous per batch entry),
// its queries pooled, its rows selected and attended, its O rows and LSE
// columns out, with the copies in, the kernels and the copies out of
// neighbouring chunks overlapping.
struct HostLayout {
  size_t kall, vall, qall, oall, lse, kb, qb, idx, total;
};

HostLayout host_layout(const Dims& d) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t B = d.B, S = d.S, D = d.D, n = d.n, k = d.topk;
  const size_t kv = B * S * d.Hkv * D * 2, qo = B * S * d.Hq * D * 2;
  HostLayout L;
  L.kall = 0;
  L.vall = L.kall + al(kv);
  L.qall = L.vall + al(kv);
  L.oall = L.qall + al(qo);
  L.lse = L.oall + al(qo);
  L.kb = L.lse + al(B * d.Hq * S * 4);
  L.qb = L.kb + al(B * d.Hkv * n * D * 4);
  L.idx = L.qb + al(B * d.Hkv * n * D * 4);
  L.total = L.idx + al(B * d.Hkv * n * k * 4);
  return L;
}

// Query blocks per chunk of the host-buffer path: at least 8 MB of Q per
// chunk (about 150 us of PCIe, which hides a chunk's launches and keeps many
// work units per forward launch), and at most sixteen chunks.
int host_chunk_blocks(const Dims& d) {
  const size_t row_bytes = static_cast<size_t>(d.B) * 64 * d.Hq * d.D * 2;  // one query block, all heads
  const int by_bytes = static_cast<int>(((8u << 20) + row_bytes - 1) / row_bytes);
  return std::min(d.n, std::max(by_bytes, (d.n + 15) / 16));
}

// The plain sparse forward over query blocks i0 .. i1 - 1.
ssa_status sparse_fwd_range(const Dims& d, const void* q, const void* k, const void* v, const int32_t* idx,
                            void* o, float* lse, cudaStream_t st, int i0, int i1) {
  if (d.D == 64)
    return d.G >= 4 ? launch_fwd<64, 2, false>(d, q, k, v, idx, o, lse, nullptr, nullptr, nullptr, st, nullptr,
                                               nullptr, 0.f, nullptr, DashIn(), i0, i1)
                    : launch_fwd<64, 1, false>(d, q, k, v, idx, o, lse, nullptr, nullptr, nullptr, st, nullptr,
                                               nullptr, 0.f, nullptr, DashIn(), i0, i1);
  return d.G >= 4 ? launch_psfwd<128, 2, false>(d, q, k, v, idx, o, lse, nullptr, nullptr, nullptr, st, DashIn(),
                                                nullptr, nullptr, 0.f, nullptr, i0, i1)
                  : launch_psfwd<128, 1, false>(d, q, k, v, idx, o, lse, nullptr, nullptr, nullptr, st, DashIn(),
                                                nullptr, nullptr, 0.f, nullptr, i0, i1);
}

// The selection of query blocks i0 .. i1 - 1.
ssa_status select_range(const Dims& d, const float* qb, const float* kb, int32_t* idx, cudaStream_t st, int i0,
                        int i1) {
  ssa::SelectParams sp;
  sp.qbar = qb;
  sp.kbar = kb;
  sp.idx = idx;
  sp.n = d.n;
  sp.topk = d.topk;
  sp.i0 = i0;
  sp.i1 = i1;
  if (d.D == 64)
    return d.n <= 128 ? launch_select<64, 4>(d, sp, st)
                      : (d.n <= 512 ? launch_select<64, 16>(d, sp, st) : launch_select<64, 0>(d, sp, st));
  return d.n <= 128 ? launch_select<128, 4>(d, sp, st)
                    : (d.n <= 512 ? launch_select<128, 16>(d, sp, st) : launch_select<128, 0>(d, sp, st));
}

// The copy-in and copy-out streams of the host-buffer path, one pair per
// device, created on first use and kept for the life of the process.
std::mutex g_pipe_mutex;
cudaStream_t g_pipe_in[kMaxDevices], g_pipe_out[kMaxDevices];

ssa_status pipe_streams(cudaStream_t* in, cudaStream_t* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return SSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  if (g_pipe_in[dev] == nullptr) {
    if (cudaStreamCreateWithFlags(&g_pipe_in[dev], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&g_pipe_out[dev], cudaStreamNonBlocking) != cudaSuccess)
      return SSA_ERR_CUDA;
  }
  *in = g_pipe_in[dev];
  *out = g_pipe_out[dev];
  return SSA_OK;
}

}  // namespace

extern "C" {

const char* ssa_status_string(ssa_status s) {
  switch (s) {
    case SSA_OK: return "SSA_OK";
    case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
    case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
    case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
    case SSA_ERR_DEVICE_TIMEOUT: return "SSA_ERR_DEVICE_TIMEOUT";
    case SSA_ERR_WORKSPACE: return "SSA_ERR_WORKSPACE";
  }
  return "SSA_ERR_UNKNOWN";
}

uint64_t ssa_launch_count(void) { return g_launches.load(); }

ssa_status ssa_block_pool(const ssa_problem* p, const ssa_bf16* k, const ssa_bf16* q,
                          float* k_pooled, float* q_pooled, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  if (k == nullptr || k_pooled == nullptr) return SSA_ERR_INVALID_ARG;
  if ((q == nullptr) != (q_pooled == nullptr)) return SSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(k_pooled) || !aligned16(q) || !aligned16(q_pooled))
    return SSA_ERR_INVALID_ARG;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  return d.D == 64 ? launch_pool<64>(d, k, q, k_pooled, q_pooled, st)
                   : launch_pool<128>(d, k, q, k_pooled, q_pooled, st);
}

ssa_status ssa_block_select(const ssa_problem* p, const float* q_pooled, const float* k_pooled,
                            int32_t* block_idx, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  if (q_pooled == nullptr || k_pooled == nullptr || block_idx == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q_pooled) || !aligned16(k_pooled) || !aligned16(block_idx)) return SSA_ERR_INVALID_ARG;
  ssa::SelectParams sp;
  sp.qbar = q_pooled;
  sp.kbar = k_pooled;
  sp.idx = block_idx;
  sp.n = d.n;
  sp.topk = d.topk;
  sp.i0 = 0;
  sp.i1 = d.n;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  // keys in registers while a lane's share (n / 32) is small
  if (d.D == 64)
    return d.n <= 128 ? launch_select<64, 4>(d, sp, st)
                      : (d.n <= 512 ? launch_select<64, 16>(d, sp, st) : launch_select<64, 0>(d, sp, st));
  return d.n <= 128 ? launch_select<128, 4>(d, sp, st)
                    : (d.n <= 512 ? launch_select<128, 16>(d, sp, st) : launch_select<128, 0>(d, sp, st));
}

ssa_status ssa_sparse_attn_fwd(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                               const ssa_bf16* v, const int32_t* block_idx, ssa_bf16* o,
                               float* lse, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, block_idx, o, lse};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  // head_dim 64: two M-tiles (4 query heads) per CTA and two CTAs per SM;
  // head_dim 128: P staged in shared memory, two M-tiles per CTA
  if (d.D == 64)
    return d.G >= 4
               ? launch_fwd<64, 2, false>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st)
               : launch_fwd<64, 1, false>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st);
  return d.G >= 4
             ? launch_psfwd<128, 2, false>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st)
             : launch_psfwd<128, 1, false>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st);
}

size_t ssa_sparse_attn_fwd_host_workspace(const ssa_problem* p) {
  Dims d;
  if (check_problem(p, &d) != SSA_OK) return 0;
  return host_layout(d).total;
}

ssa_status ssa_sparse_attn_fwd_host(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k, const ssa_bf16* v,
                                    ssa_bf16* o, float* lse, void* workspace, size_t ws_bytes, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, o, lse};
  for (const void* ptr : ptrs)
    if (ptr == nullptr) return SSA_ERR_INVALID_ARG;
  const HostLayout L = host_layout(d);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < L.total)
    return SSA_ERR_WORKSPACE;
  auto sc = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t sin = nullptr, sout = nullptr;
  s = pipe_streams(&sin, &sout);
  if (s != SSA_OK) return s;
  const int cb = host_chunk_blocks(d), chunks = (d.n + cb - 1) / cb;
  std::vector<cudaEvent_t> ev(3 + 2 * static_cast<size_t>(chunks), nullptr);
  bool ok = true;
  for (auto& e : ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    for (auto& e : ev)
      if (e != nullptr) cudaEventDestroy(e);
    return SSA_ERR_CUDA;
  }
  cudaEvent_t ev_start = ev[0], ev_kv = ev[1], ev_end = ev[2];
  cudaEvent_t* in_done = ev.data() + 3;
  cudaEvent_t* comp_done = in_done + chunks;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* dk = reinterpret_cast<ssa_bf16*>(ws + L.kall);
  auto* dv = reinterpret_cast<ssa_bf16*>(ws + L.vall);
  auto* dq = reinterpret_cast<ssa_bf16*>(ws + L.qall);
  auto* dout = reinterpret_cast<ssa_bf16*>(ws + L.oall);
  auto* dlse = reinterpret_cast<float*>(ws + L.lse);
  auto* dkb = reinterpret_cast<float*>(ws + L.kb);
  auto* dqb = reinterpret_cast<float*>(ws + L.qb);
  auto* didx = reinterpret_cast<int32_t*>(ws + L.idx);
  const size_t S = d.S, D = d.D, Hq = d.Hq, Hkv = d.Hkv;
  const size_t qtok = Hq * D * 2;  // bytes of one token's Q (or O) row, all heads
  ok = cudaEventRecord(ev_start, sc) == cudaSuccess && cudaStreamWaitEvent(sin, ev_start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(sout, ev_start, 0) == cudaSuccess;
  // K and V whole, then the pooled keys of every block
  const size_t kv_all = static_cast<size_t>(d.B) * S * Hkv * D * 2;
  ok = ok && cudaMemcpyAsync(dk, k, kv_all, cudaMemcpyHostToDevice, sin) == cudaSuccess &&
       cudaMemcpyAsync(dv, v, kv_all, cudaMemcpyHostToDevice, sin) == cudaSuccess &&
       cudaEventRecord(ev_kv, sin) == cudaSuccess && cudaStreamWaitEvent(sc, ev_kv, 0) == cudaSuccess;
  if (ok) s = d.D == 64 ? launch_pool<64>(d, dk, nullptr, dkb, nullptr, sc) : launch_pool<128>(d, dk, nullptr, dkb, nullptr, sc);
  for (int c = 0; ok && s == SSA_OK && c < chunks; ++c) {
    const int i0 = c * cb, i1 = std::min(d.n, i0 + cb);
    const size_t t0 = 64 * static_cast<size_t>(i0), nt = 64 * static_cast<size_t>(i1 - i0);
    // copy in: the chunk's Q rows of every batch entry
    for (size_t b = 0; ok && b < static_cast<size_t>(d.B); ++b)
      ok = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(dq) + (b * S + t0) * qtok,
                           reinterpret_cast<const uint8_t*>(q) + (b * S + t0) * qtok, nt * qtok,
                           cudaMemcpyHostToDevice, sin) == cudaSuccess;
    ok = ok && cudaEventRecord(in_done[c], sin) == cudaSuccess;
    // compute on the caller's stream: the chunk's pooled queries, selection
    // and attention
    ok = ok && cudaStreamWaitEvent(sc, in_done[c], 0) == cudaSuccess;
    if (ok) s = d.D == 64 ? launch_pool<64>(d, nullptr, dq, nullptr, dqb, sc, i0, i1 - i0)
                          : launch_pool<128>(d, nullptr, dq, nullptr, dqb, sc, i0, i1 - i0);
    if (ok && s == SSA_OK) s = select_range(d, dqb, dkb, didx, sc, i0, i1);
    if (ok && s == SSA_OK) s = sparse_fwd_range(d, dq, dk, dv, didx, dout, dlse, sc, i0, i1);
    ok = ok && s == SSA_OK && cudaEventRecord(comp_done[c], sc) == cudaSuccess;
    // copy out: the chunk's O rows of every batch entry, and its LSE columns
    // of every (batch entry, query head) row
    ok = ok && cudaStreamWaitEvent(sout, comp_done[c], 0) == cudaSuccess;
    for (size_t b = 0; ok && b < static_cast<size_t>(d.B); ++b)
      ok = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(o) + (b * S + t0) * qtok,
                           reinterpret_cast<const uint8_t*>(dout) + (b * S + t0) * qtok, nt * qtok,
                           cudaMemcpyDeviceToHost, sout) == cudaSuccess;
    ok = ok && cudaMemcpy2DAsync(lse + t0, S * 4, dlse + t0, S * 4, nt * 4, static_cast<size_t>(d.B) * Hq,
                                 cudaMemcpyDeviceToHost, sout) == cudaSuccess;
  }
  // the caller's stream continues after the last copies; copy-in waits too, so
  // a later call cannot overwrite buffers still being read
  ok = ok && cudaEventRecord(ev_end, sout) == cudaSuccess && cudaStreamWaitEvent(sc, ev_end, 0) == cudaSuccess &&
       cudaStreamWaitEvent(sin, ev_end, 0) == cudaSuccess;
  for (auto& e : ev) cudaEventDestroy(e);  // released once the streams are past them
  if (s != SSA_OK) return s;
  return ok ? SSA_OK : SSA_ERR_CUDA;
}

ssa_status ssa_full_attn_fwd_with_mass(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                                       const ssa_bf16* v, const int32_t* block_idx,
                                       ssa_bf16* o_sparse, float* lse_sparse, ssa_bf16* o_full,
                                       float* lse_full, float* dropped, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, block_idx, o_sparse, lse_sparse, o_full, lse_full, dropped};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (d.D == 64)
    return d.G >= 4
               ? launch_fwd<64, 2, true>(d, q, k, v, block_idx, o_sparse, lse_sparse, o_full, lse_full, dropped, st)
               : launch_fwd<64, 1, true>(d, q, k, v, block_idx, o_sparse, lse_sparse, o_full, lse_full, dropped, st);
  return launch_psfwd<128, 1, true>(d, q, k, v, block_idx, o_sparse, lse_sparse, o_full, lse_full, dropped, st);
}

size_t ssa_sparse_attn_bwd_workspace(const ssa_problem* p) {
  Dims d;
  if (check_problem(p, &d) != SSA_OK) return 0;
  return bwd_workspace_bytes(d);
}

ssa_status ssa_sparse_attn_bwd(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                               const ssa_bf16* v, const ssa_bf16* o, const float* lse,
                               const ssa_bf16* d_o, const int32_t* block_idx, ssa_bf16* dq,
                               ssa_bf16* dk, ssa_bf16* dv, void* workspace, size_t ws_bytes,
                               ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, o, lse, d_o, block_idx, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  const size_t need = bwd_workspace_bytes(d);
  if (workspace == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SSA_ERR_WORKSPACE;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  // dQ kernel: two head pairs per CTA when the group has them
  if (d.D == 64)
    return launch_bwd<64, 1>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, workspace, st);
  return d.G >= 4 ? launch_bwd<128, 2>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, workspace, st)
                  : launch_bwd<128, 1>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, workspace, st);
}

ssa_status ssa_sparse_attn_bwd_noalloc(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                                       const ssa_bf16* v, const ssa_bf16* o, const float* lse,
                                       const ssa_bf16* d_o, const int32_t* block_idx, ssa_bf16* dq,
                                       ssa_bf16* dk, ssa_bf16* dv, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, o, lse, d_o, block_idx, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if (bwd_workspace_bytes(d) > SSA_NOALLOC_SCRATCH_BYTES) return SSA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (scratch == nullptr) return SSA_ERR_CUDA;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (d.D == 64)
    return launch_bwd<64, 1>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, scratch, st);
  return d.G >= 4 ? launch_bwd<128, 2>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, scratch, st)
                  : launch_bwd<128, 1>(d, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, scratch, st);
}

size_t ssa_alignment_bwd_workspace(const ssa_problem* p) {
  Dims d;
  if (check_problem(p, &d) != SSA_OK) return 0;
  return align_layout(d).total;
}

ssa_status ssa_alignment_bwd(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                             const ssa_bf16* v, const ssa_bf16* o_sparse, const float* lse_sparse,
                             const ssa_bf16* o_full, const float* lse_full, const ssa_bf16* d_o,
                             int mode, float alpha, const int32_t* block_idx, ssa_bf16* dq,
                             ssa_bf16* dk, ssa_bf16* dv, void* workspace, size_t ws_bytes,
                             ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, o_sparse, lse_sparse, o_full, lse_full, d_o, block_idx, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if ((mode != 0 && mode != 1) || !std::isfinite(alpha)) return SSA_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace) || ws_bytes < align_layout(d).total)
    return SSA_ERR_WORKSPACE;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (d.D == 64)
    return launch_align_bwd<64, 1>(d, q, k, v, o_sparse, lse_sparse, o_full, lse_full, d_o, mode, alpha,
                                   block_idx, dq, dk, dv, workspace, st);
  return d.G >= 4 ? launch_align_bwd<128, 2>(d, q, k, v, o_sparse, lse_sparse, o_full, lse_full, d_o, mode,
                                             alpha, block_idx, dq, dk, dv, workspace, st)
                  : launch_align_bwd<128, 1>(d, q, k, v, o_sparse, lse_sparse, o_full, lse_full, d_o, mode,
                                             alpha, block_idx, dq, dk, dv, workspace, st);
}

ssa_status ssa_sparse_attn_fwd_early_stop(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k,
                                          const ssa_bf16* v, const float* q_pooled, const float* k_pooled,
                                          const int32_t* block_idx, float tau, ssa_bf16* o, float* lse,
                                          int32_t* visited, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, q_pooled, k_pooled, block_idx, o, lse};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if (visited != nullptr && !aligned16(visited)) return SSA_ERR_INVALID_ARG;
  if (!(tau >= 0.f) || !std::isfinite(tau)) return SSA_ERR_INVALID_ARG;
  if (d.topk > ssa::kEarlyMaxTopk) return SSA_ERR_UNSUPPORTED;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (d.D == 64)
    return d.G >= 4 ? launch_fwd<64, 2, false, true>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st,
                                                     q_pooled, k_pooled, tau, visited)
                    : launch_fwd<64, 1, false, true>(d, q, k, v, block_idx, o, lse, nullptr, nullptr, nullptr, st,
                                                     q_pooled, k_pooled, tau, visited);
  return d.G >= 4 ? launch_psfwd<128, 2, false, false, true>(d, q, k, v, block_idx, o, lse, nullptr, nullptr,
                                                             nullptr, st, DashIn(), q_pooled, k_pooled, tau, visited)
                  : launch_psfwd<128, 1, false, false, true>(d, q, k, v, block_idx, o, lse, nullptr, nullptr,
                                                             nullptr, st, DashIn(), q_pooled, k_pooled, tau, visited);
}

size_t ssa_decode_attn_workspace(const ssa_problem* p) {
  Dims d;
  (void)check_problem(p, &d);
  return 0;  // the selection and the partial softmax states stay on chip
}

ssa_status ssa_decode_attn(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k_cache,
                           const ssa_bf16* v_cache, const float* k_pooled, const int32_t* lengths,
                           ssa_bf16* o, float* lse, int32_t* block_idx, void* workspace, size_t ws_bytes,
                           ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k_cache, v_cache, k_pooled, lengths, o, lse};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if (block_idx != nullptr && !aligned16(block_idx)) return SSA_ERR_INVALID_ARG;
  (void)workspace;  // none is needed (ssa_decode_attn_workspace returns 0)
  (void)ws_bytes;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  return d.D == 64 ? launch_decode<64>(d, q, k_cache, v_cache, k_pooled, lengths, o, lse, block_idx, st)
                   : launch_decode<128>(d, q, k_cache, v_cache, k_pooled, lengths, o, lse, block_idx, st);
}

// ------------------------------------------------------------ DashAttention

ssa_status ssa_dash_route(const ssa_problem* p, const ssa_bf16* q, const float* k_pooled, float alpha,
                          float gamma, float* weights, uint32_t* mask, ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k_pooled, weights, mask};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if (!(alpha > 1.f) || !(alpha <= 4.f)) return SSA_ERR_INVALID_ARG;
  if (!(gamma > 0.f) || !std::isfinite(gamma)) return SSA_ERR_INVALID_ARG;
  if (d.n > ssa::kDashMaxN) return SSA_ERR_UNSUPPORTED;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  auto route = [&](auto dd, auto gg) {
    return launch_dash_route<decltype(dd)::value, decltype(gg)::value>(d, q, k_pooled, alpha, gamma, weights,
                                                                       mask, st);
  };
  using I64 = std::integral_constant<int, 64>;
  using I128 = std::integral_constant<int, 128>;
  switch (d.G) {
    case 2: return d.D == 64 ? route(I64(), std::integral_constant<int, 2>())
                             : route(I128(), std::integral_constant<int, 2>());
    case 4: return d.D == 64 ? route(I64(), std::integral_constant<int, 4>())
                             : route(I128(), std::integral_constant<int, 4>());
    case 8: return d.D == 64 ? route(I64(), std::integral_constant<int, 8>())
                             : route(I128(), std::integral_constant<int, 8>());
    default: return d.D == 64 ? route(I64(), std::integral_constant<int, 16>())
                              : route(I128(), std::integral_constant<int, 16>());
  }
}

ssa_status ssa_dash_attn_fwd(const ssa_problem* p, const ssa_bf16* q, const ssa_bf16* k, const ssa_bf16* v,
                             const float* weights, const uint32_t* mask, float sigma, ssa_bf16* o, float* lse,
                             ssa_stream stream) {
  Dims d;
  ssa_status s = check_problem(p, &d);
  if (s != SSA_OK) return s;
  const void* ptrs[] = {q, k, v, weights, mask, o, lse};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return SSA_ERR_INVALID_ARG;
  if (!(sigma >= 0.f) || !std::isfinite(sigma)) return SSA_ERR_INVALID_ARG;
  if (d.n > ssa::kDashMaxN) return SSA_ERR_UNSUPPORTED;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  DashIn dash;
  dash.mask = mask;
  dash.w = weights;
  dash.sigma = sigma;
  if (d.D == 64)
    return d.G >= 4 ? launch_fwd<64, 2, false, false, true>(d, q, k, v, nullptr, o, lse, nullptr, nullptr, nullptr,
                                                            st, nullptr, nullptr, 0.f, nullptr, dash)
                    : launch_fwd<64, 1, false, false, true>(d, q, k, v, nullptr, o, lse, nullptr, nullptr, nullptr,
                                                            st, nullptr, nullptr, 0.f, nullptr, dash);
  return d.G >= 4
             ? launch_psfwd<128, 2, false, true>(d, q, k, v, nullptr, o, lse, nullptr, nullptr, nullptr, st, dash)
             : launch_psfwd<128, 1, false, true>(d, q, k, v, nullptr, o, lse, nullptr, nullptr, nullptr, st, dash);
}

ssa_status ssa_get_device_error(ssa_stream stream) {
  const cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, ssa::g_error_word, sizeof(word)) != cudaSuccess)
    return SSA_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(ssa::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return SSA_ERR_CUDA;
  if (word & ssa::kErrTimeout) return SSA_ERR_DEVICE_TIMEOUT;
  if (word & ssa::kErrBadInput) return SSA_ERR_INVALID_ARG;
  return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

unsigned int ssa_get_device_error_site(void) {
  unsigned int site = 0;
  if (cudaMemcpyFromSymbol(&site, ssa::g_error_site, sizeof(site)) != cudaSuccess) return 0;
  return site;
}

ssa_status ssa_debug_timeout_probe(int timeout_us, ssa_stream stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return SSA_ERR_INVALID_ARG;
  timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  return launch_result();
}

ssa_status ssa_debug_exp2_poly(const float* x, float* y, int n, ssa_stream stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return SSA_ERR_INVALID_ARG;
  if (n == 0) return SSA_OK;
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_result();
}

}  // extern "C"
