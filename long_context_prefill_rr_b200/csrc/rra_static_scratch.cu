// rra_estimate_static_scratch: the estimate step for callers that cannot allocate device memory.
//
// rra_estimate needs scratch space (pooled keys and per-row partial sums) that the caller
// normally provides as a workspace buffer. Some callers cannot obtain one: a serving process
// whose memory pool has already claimed the device and forbids further cudaMalloc, or code
// that must not call cudaMalloc / cudaFree because those calls can synchronise the whole
// device and stall unrelated work. This entry point keeps its scratch in a fixed array in the
// library's device image instead. The array is created when the library's module is loaded on
// a device and stays allocated on every device that uses the library until the process exits.
//
// Costs and limits:
//   - kStaticScratchBytes (48 MiB) bounds the problems it accepts; larger ones are refused with
//     RRA_ERR_WORKSPACE before anything is enqueued.
//   - All calls share the one array, so two calls whose kernels overlap on a GPU (different
//     streams, or different host threads) race and corrupt each other's results. Serialise
//     them, e.g. issue them on one stream.
//   - The first call on each device looks up the array's device address (a host-side query,
//     done once per device with that device current) and clears the array's status word; make
//     that first call before any stream capture begins.
//   - The status word is sticky, as a workspace's is: a kernel whose barrier wait timed out
//     sets it, later calls then enqueue kernels that exit at once, and
//     rra_static_scratch_status reads and clears it.
#include <mutex>

#include "rra.h"
#include "common.cuh"
#include "rra_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(48) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself. Host code must not pass `g_rra_static_scratch` to a kernel: on the host
// the name denotes a shadow variable, not device memory. Its device address comes from
// cudaGetSymbolAddress (see scratch_address).
static __device__ __align__(256) unsigned char g_rra_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device. The first call on a device looks
// it up and clears the status word at its start (enqueued on `stream`, ahead of any kernel that
// reads it).
cudaError_t scratch_address(void **out, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rra_static_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p, 0, 256, stream);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" rra_status rra_estimate_static_scratch(const rra_params *p, const void *q,
                                                  const void *k, float *mass,
                                                  rra_stream_t stream) {
  if (!p) return RRA_ERR_INVALID_ARG;
  if (p->batch == 0 || p->seqlen == 0) {
    // same validation as rra_estimate, which treats an empty problem as a no-op
    return rra_estimate(p, q, k, mass, nullptr, 0, stream);
  }
  if (!q || !k || !mass) return RRA_ERR_INVALID_ARG;
  // The scratch is laid out exactly like rra_estimate's workspace (whose trailing mass region
  // stays unused here), so the problem fits if rra_workspace_bytes does.
  const size_t need = rra_workspace_bytes(p);
  if (need == 0) {
    // invalid parameters: rra_estimate reports which check failed
    return rra_estimate(p, q, k, mass, nullptr, 0, stream);
  }
  if (need > kStaticScratchBytes) return RRA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (scratch_address(&scratch, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RRA_ERR_CUDA;
  // The array keeps the previous call's contents. Pooled keys and partial sums are rewritten
  // before they are read; the status word was cleared at set-up and stays set after a timeout
  // until rra_static_scratch_status reads it.
  return rra_estimate(p, q, k, mass, scratch, need, stream);
}

extern "C" rra_status rra_static_scratch_status(rra_stream_t stream, uint32_t *raw_word) {
  void *scratch = nullptr;
  if (scratch_address(&scratch, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RRA_ERR_CUDA;
  return rra_check_device_status(scratch, stream, raw_word);
}
