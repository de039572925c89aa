// attn_bwd.cuh -- sparse attention backward (dQ, dK, dV over selected pairs).
#pragma once

#include "sm100.cuh"

static size_t ssa_bwd_workspace_bytes(int B, int S, int Hq, int Hkv, int n, int topk) {
  (void)B; (void)S; (void)Hq; (void)Hkv; (void)n; (void)topk;
  return 0;
}

static ssa_status ssa_bwd_launch(int, int, int, int, int, int, int, int, float, const void*,
                                 const void*, const void*, const void*, const float*,
                                 const void*, const int32_t*, void*, void*, void*, void*,
                                 cudaStream_t, uint64_t) {
  return SSA_ERR_UNSUPPORTED;
}
