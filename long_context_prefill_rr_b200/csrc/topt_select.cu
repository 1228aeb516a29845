// Standalone Top-tau select kernel: one warp per (batch, head, block row I) runs the row
// select of topt_select.cuh on masses read from global memory. Rows of up to 1024 blocks are
// held in registers, in a variant specialised to the row's chunk count; longer rows are re-read
// from memory in every pass. Three 256-thread blocks per SM (78 registers a thread, no spills):
// each bisection step waits on a warp reduction, so more resident warps hide that latency.
#include "common.cuh"
#include "rra_internal.h"
#include "topt_select.cuh"

namespace rra {

__global__ void __launch_bounds__(256, 3) topt_select_kernel(const float *__restrict__ mass,
                                                          int32_t *__restrict__ kept_idx,
                                                          int32_t *__restrict__ kept_cnt,
                                                          int64_t rows, int nb, int64_t tri,
                                                          float tau) {
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps_total) {
    const int64_t bh = row / nb;
    const int I = static_cast<int>(row - bh * nb);
    const int n = I + 1;
    const int64_t off = bh * tri + static_cast<int64_t>(I) * (I + 1) / 2;
    const float *a = mass + off;
    int32_t *out = kept_idx + off;
    int32_t *cnt = kept_cnt + row;
    select_row_any([a](int J) { return __ldg(a + J); }, out, cnt, n, I, tau, lane);
  }
}

cudaError_t launch_topt_select(const Geometry &g, const float *mass, int32_t *kept_idx,
                               int32_t *kept_cnt, int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(g.b) * g.hq * g.nb;
  const int threads = 256;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  topt_select_kernel<<<blocks, threads, 0, stream>>>(mass, kept_idx, kept_cnt, rows, g.nb, g.tri,
                                                     g.tau);
  return cudaGetLastError();
}

}  // namespace rra
