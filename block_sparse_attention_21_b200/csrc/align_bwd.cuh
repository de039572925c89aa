// align_bwd.cuh -- elementwise pieces of the backward of SSA's alignment
// objective ("Resumen Tecnico: SSA", section 2, "Alineacion Bidireccional"):
// the output gradients of both attention streams, and the sum of the two
// streams' input gradients.
//
// Per layer the objective is  <dO, h_mode> + alpha * (L_sparsity + L_commit)
// with L_sparsity = mean (h_full - sg(h_sparse))^2 pulling the full output
// towards the sparse one, and L_commit = mean (h_sparse - sg(h_full))^2
// pulling the sparse output towards the full one (sg: stop-gradient; the mean
// runs over the N elements of h).  So, with c = 2 alpha / N,
//   dL/dh_sparse = c (h_sparse - h_full)  [+ dO when mode = 0]
//   dL/dh_full   = c (h_full - h_sparse)  [+ dO when mode = 1]
// where mode says which stream's output the upstream gradient dO belongs to
// (the other output is the counterpart, computed for the alignment only).
#pragma once

#include "sm100.cuh"

namespace ssa {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// n8 = elements / 8; every pointer 16-byte aligned.
__global__ void __launch_bounds__(256) align_grad_kernel(const __nv_bfloat16* o_sparse,
                                                         const __nv_bfloat16* o_full,
                                                         const __nv_bfloat16* d_o, int mode, float c,
                                                         __nv_bfloat16* do_sparse, __nv_bfloat16* do_full,
                                                         long long n8) {
  const uint4* os = reinterpret_cast<const uint4*>(o_sparse);
  const uint4* of = reinterpret_cast<const uint4*>(o_full);
  const uint4* g = reinterpret_cast<const uint4*>(d_o);
  uint4* ds = reinterpret_cast<uint4*>(do_sparse);
  uint4* df = reinterpret_cast<uint4*>(do_full);
  const float gs = mode == 0 ? 1.f : 0.f, gf = mode == 1 ? 1.f : 0.f;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n8;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 a = os[e], f = of[e], u = g[e];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wf[4] = {f.x, f.y, f.z, f.w}, wu[4] = {u.x, u.y, u.z, u.w};
    uint32_t rs[4], rf[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float d0 = bf16_lo(wa[x]) - bf16_lo(wf[x]), d1 = bf16_hi(wa[x]) - bf16_hi(wf[x]);
      const float u0 = bf16_lo(wu[x]), u1 = bf16_hi(wu[x]);
      rs[x] = pack_bf16x2(fmaf(gs, u0, c * d0), fmaf(gs, u1, c * d1));
      rf[x] = pack_bf16x2(fmaf(gf, u0, -c * d0), fmaf(gf, u1, -c * d1));
    }
    ds[e] = make_uint4(rs[0], rs[1], rs[2], rs[3]);
    df[e] = make_uint4(rf[0], rf[1], rf[2], rf[3]);
  }
}

// a += b over n8 * 8 bf16 elements (the sum in fp32, rounded once).
__global__ void __launch_bounds__(256) add_bf16_kernel(__nv_bfloat16* a, const __nv_bfloat16* b, long long n8) {
  uint4* pa = reinterpret_cast<uint4*>(a);
  const uint4* pb = reinterpret_cast<const uint4*>(b);
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n8;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 x = pa[e], y = pb[e];
    const uint32_t wx[4] = {x.x, x.y, x.z, x.w}, wy[4] = {y.x, y.y, y.z, y.w};
    uint32_t r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      r[k] = pack_bf16x2(bf16_lo(wx[k]) + bf16_lo(wy[k]), bf16_hi(wx[k]) + bf16_hi(wy[k]));
    pa[e] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

}  // namespace ssa
