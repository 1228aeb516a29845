// Internal launch interface between the C ABI (rra_api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rra {

// Problem geometry resolved from rra_params (all sizes in elements unless stated).
struct Geometry {
  int b, hq, hkv, L, d, B, S, shift;
  int g;            // hq / hkv
  int m;            // B / S sampled queries per block row
  int nb;           // L / B
  int ns;           // L / S
  int ntiles;       // ceil(ns / 128): 128-row tiles of sampled queries (and 128-stride key tiles)
  int64_t tri;      // nb (nb + 1) / 2 packed entries per (batch, head)
  float tau;
  float scale;      // resolved softmax scale
};

// Workspace carve-up (byte offsets from the workspace base).
struct WorkspaceLayout {
  size_t status;    // uint32 status word (first 256 bytes are the header)
  size_t khi, klo;  // pooled keys, bf16 hi / lo parts [b, hkv, ns, d]
  size_t est_e;     // estimate partial sums, float
  size_t est_ref;   // estimate per-tile row references, float
  size_t mass;      // fp32 masses when the caller of rra_prefill passes none
  size_t total;
  int est_slots;    // persistent CTAs of the estimate kernel
};

WorkspaceLayout workspace_layout(const Geometry &g, int num_sms);

// Time limit of the kernels' barrier waits, in ns (kWaitLimitNs unless rra_set_wait_limit_ns
// set another).
uint64_t wait_limit_ns();

// Driver entry point for tensor-map encoding (resolved once through the runtime).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// Each launcher returns cudaSuccess or the error of the failing CUDA call (tensor-map encoding
// failures are reported as cudaErrorInvalidValue).
cudaError_t launch_pool_keys(const Geometry &g, const void *k, void *khi, void *klo,
                             int num_sms, cudaStream_t stream);
cudaError_t launch_rr_estimate(const Geometry &g, const void *q, const void *khi,
                               const void *klo, float *mass, float *est_e, float *est_ref,
                               int slots, uint32_t *status, cudaStream_t stream);
cudaError_t launch_xattn_estimate(const Geometry &g, const void *q, const void *k, float *mass,
                                  float *est_e, float *est_ref, int slots, uint32_t *status,
                                  cudaStream_t stream);
cudaError_t launch_topt_select(const Geometry &g, const float *mass, int32_t *kept_idx,
                               int32_t *kept_cnt, int num_sms, cudaStream_t stream);
cudaError_t launch_sparse_attn(const Geometry &g, const void *q, const void *k, const void *v,
                               const int32_t *kept_idx, const int32_t *kept_cnt, void *out,
                               uint32_t *status, cudaStream_t stream);

}  // namespace rra
