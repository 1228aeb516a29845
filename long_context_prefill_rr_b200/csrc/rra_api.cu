// C ABI of the RRAttention prefill hot path (declared in include/rra.h): argument validation,
// workspace carve-up, kernel launches and the chunked host-buffer pipeline. No memory is
// allocated here; the host pipeline creates its two streams and events once per device.
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "rra.h"
#include "common.cuh"
#include "rra_internal.h"

namespace rra {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

WorkspaceLayout workspace_layout(const Geometry &g, int num_sms) {
  WorkspaceLayout w{};
  size_t off = 256;   // header: status word
  w.status = 0;
  const size_t kbar = static_cast<size_t>(g.b) * g.hkv * g.ns * g.d * 2;
  w.khi = align_up(off, 1024);
  off = w.khi + kbar;
  w.klo = align_up(off, 1024);
  off = w.klo + kbar;
  const int64_t items = static_cast<int64_t>(g.b) * g.hq * g.ntiles;
  int slots = num_sms < 1 ? 1 : num_sms;
  if (items < slots) slots = static_cast<int>(items < 1 ? 1 : items);
  w.est_slots = slots;
  const int segs = g.m > 0 ? 128 / g.m : 0;
  // two scratch buffers per slot: one item is reduced while the next is computed
  w.est_e = align_up(off, 256);
  off = w.est_e + static_cast<size_t>(slots) * 2 * 128 * g.ntiles * segs * 4;
  w.est_ref = align_up(off, 256);
  off = w.est_ref + static_cast<size_t>(slots) * 2 * 128 * g.ntiles * 2 * 4;
  w.mass = align_up(off, 256);
  off = w.mass + static_cast<size_t>(g.b) * g.hq * g.tri * 4;
  w.total = align_up(off, 256);
  return w;
}

static std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace rra

using rra::Geometry;
using rra::WorkspaceLayout;

namespace {

enum Needs : unsigned { kNeedsStride = 1u, kNeedsHeadDim = 2u };

// Checks the shape parameters and resolves the geometry. `needs` says which kernel limits apply
// (the estimate needs a supported stride, the estimate and the attention a supported head_dim).
rra_status resolve(const rra_params *p, unsigned needs, Geometry *g) {
  if (!p) return RRA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->seqlen < 0 || p->heads_q < 1 || p->heads_kv < 1 ||
      p->heads_q % p->heads_kv != 0 || p->block <= 0 || p->stride <= 0 || p->head_dim <= 0)
    return RRA_ERR_INVALID_ARG;
  if (p->seqlen % p->block != 0 || p->block % p->stride != 0) return RRA_ERR_INVALID_ARG;
  if (!(p->tau > 0.f)) return RRA_ERR_INVALID_ARG;   // also rejects NaN
  if (p->block != 128) return RRA_ERR_UNSUPPORTED;
  if ((needs & kNeedsHeadDim) && p->head_dim != 64 && p->head_dim != 128)
    return RRA_ERR_UNSUPPORTED;
  if ((needs & kNeedsStride) && p->stride != 4 && p->stride != 8 && p->stride != 16 &&
      p->stride != 32)
    return RRA_ERR_UNSUPPORTED;
  // TMA coordinates and row indices are 32-bit
  const int64_t rows_q = static_cast<int64_t>(p->batch) * p->heads_q * p->seqlen;
  if (rows_q >= (static_cast<int64_t>(1) << 31)) return RRA_ERR_UNSUPPORTED;
  g->b = p->batch;
  g->hq = p->heads_q;
  g->hkv = p->heads_kv;
  g->L = p->seqlen;
  g->d = p->head_dim;
  g->B = p->block;
  g->S = p->stride;
  g->shift = ((p->shift % p->stride) + p->stride) % p->stride;
  g->g = p->heads_q / p->heads_kv;
  g->m = p->block / p->stride;
  g->nb = p->seqlen / p->block;
  g->ns = p->seqlen / p->stride;
  g->ntiles = (g->ns + 127) / 128;
  g->tri = static_cast<int64_t>(g->nb) * (g->nb + 1) / 2;
  g->tau = p->tau;
  g->scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->head_dim));
  return RRA_OK;
}

bool empty(const Geometry &g) { return g.b == 0 || g.L == 0; }

bool ptr_ok(const void *ptr) {
  return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

rra_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA; }

uint32_t *status_word(void *ws, const WorkspaceLayout &w) {
  return reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + w.status);
}

template <class T>
T *ws_at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// Pooled keys, then the estimate kernel; with kept_idx / kept_cnt, then the select kernel. (A
// select fused into the estimate kernel's reduction warps was measured slower at every size:
// the bisection then runs on 4 warps per SM instead of a grid of its own.)
rra_status run_estimate(const Geometry &g, const void *q, const void *k, float *mass, void *ws,
                        const WorkspaceLayout &w, int sms, cudaStream_t st,
                        int32_t *kept_idx = nullptr, int32_t *kept_cnt = nullptr) {
  cudaError_t e = rra::launch_pool_keys(g, k, ws_at<void>(ws, w.khi), ws_at<void>(ws, w.klo),
                                        sms, st);
  if (e != cudaSuccess) return RRA_ERR_CUDA;
  e = rra::launch_rr_estimate(g, q, ws_at<void>(ws, w.khi), ws_at<void>(ws, w.klo), mass,
                              ws_at<float>(ws, w.est_e), ws_at<float>(ws, w.est_ref),
                              w.est_slots, status_word(ws, w), st);
  if (e == cudaSuccess && kept_idx != nullptr)
    e = rra::launch_topt_select(g, mass, kept_idx, kept_cnt, sms, st);
  return cuda_status(e);
}

rra_status run_prefill(const Geometry &g, const void *q, const void *k, const void *v, void *out,
                       float *mass, int32_t *kept_idx, int32_t *kept_cnt, void *workspace,
                       const WorkspaceLayout &w, int sms, cudaStream_t st) {
  float *m = mass ? mass : ws_at<float>(workspace, w.mass);
  rra_status s = run_estimate(g, q, k, m, workspace, w, sms, st, kept_idx, kept_cnt);
  if (s != RRA_OK) return s;
  return cuda_status(rra::launch_sparse_attn(g, q, k, v, kept_idx, kept_cnt, out,
                                             status_word(workspace, w), st));
}

// Streams and events of rra_prefill_host, created once per device.
constexpr int kMaxHostChunks = 32;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kMaxHostChunks] = {};
  cudaEvent_t step_done[kMaxHostChunks] = {};
  bool ready = false;
};

HostPipe *host_pipe() {
  static std::mutex mu;
  static HostPipe pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  HostPipe &hp = pipes[dev];
  if (!hp.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.start, ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.end, ef) != cudaSuccess)
      return nullptr;
    for (int c = 0; c < kMaxHostChunks; ++c)
      if (cudaEventCreateWithFlags(&hp.in_done[c], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.step_done[c], ef) != cudaSuccess)
        return nullptr;
    hp.ready = true;
  }
  return &hp;
}

}  // namespace

extern "C" {

size_t rra_workspace_bytes(const rra_params *p) {
  Geometry g;
  if (resolve(p, 0, &g) != RRA_OK) return 0;
  const int sms = num_sms();
  if (sms <= 0) return 0;
  return rra::workspace_layout(g, sms).total;
}

rra_status rra_estimate(const rra_params *p, const void *q, const void *k, float *mass,
                        void *workspace, size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsStride | kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(mass) || !ptr_ok(workspace)) return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  const WorkspaceLayout w = rra::workspace_layout(g, sms);
  if (workspace_bytes < w.total) return RRA_ERR_WORKSPACE;
  return run_estimate(g, q, k, mass, workspace, w, sms, reinterpret_cast<cudaStream_t>(stream));
}

rra_status rra_estimate_select(const rra_params *p, const void *q, const void *k, float *mass,
                               int32_t *kept_idx, int32_t *kept_cnt, void *workspace,
                               size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsStride | kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(kept_idx) || !ptr_ok(kept_cnt) ||
      !ptr_ok(workspace) || (mass != nullptr && !ptr_ok(mass)))
    return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  const WorkspaceLayout w = rra::workspace_layout(g, sms);
  if (workspace_bytes < w.total) return RRA_ERR_WORKSPACE;
  float *m = mass ? mass : ws_at<float>(workspace, w.mass);
  return run_estimate(g, q, k, m, workspace, w, sms, reinterpret_cast<cudaStream_t>(stream),
                      kept_idx, kept_cnt);
}

rra_status rra_estimate_xattn(const rra_params *p, const void *q, const void *k, float *mass,
                              void *workspace, size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsStride | kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(mass) || !ptr_ok(workspace)) return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  const WorkspaceLayout w = rra::workspace_layout(g, sms);
  if (workspace_bytes < w.total) return RRA_ERR_WORKSPACE;
  return cuda_status(rra::launch_xattn_estimate(
      g, q, k, mass, ws_at<float>(workspace, w.est_e), ws_at<float>(workspace, w.est_ref),
      w.est_slots, status_word(workspace, w), reinterpret_cast<cudaStream_t>(stream)));
}

rra_status rra_select(const rra_params *p, const float *mass, int32_t *kept_idx,
                      int32_t *kept_cnt, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, 0, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(mass) || !ptr_ok(kept_idx) || !ptr_ok(kept_cnt)) return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  return cuda_status(rra::launch_topt_select(g, mass, kept_idx, kept_cnt, sms,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

rra_status rra_sparse_attn(const rra_params *p, const void *q, const void *k, const void *v,
                           const int32_t *kept_idx, const int32_t *kept_cnt, void *out,
                           void *workspace, size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(kept_idx) || !ptr_ok(kept_cnt) ||
      !ptr_ok(out) || !ptr_ok(workspace))
    return RRA_ERR_INVALID_ARG;
  if (workspace_bytes < 256) return RRA_ERR_WORKSPACE;   // only the status word is used
  return cuda_status(rra::launch_sparse_attn(g, q, k, v, kept_idx, kept_cnt, out,
                                             static_cast<uint32_t *>(workspace),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

rra_status rra_prefill(const rra_params *p, const void *q, const void *k, const void *v,
                       void *out, float *mass, int32_t *kept_idx, int32_t *kept_cnt,
                       void *workspace, size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsStride | kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(out) || !ptr_ok(kept_idx) ||
      !ptr_ok(kept_cnt) || !ptr_ok(workspace) || (mass != nullptr && !ptr_ok(mass)))
    return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  const WorkspaceLayout w = rra::workspace_layout(g, sms);
  if (workspace_bytes < w.total) return RRA_ERR_WORKSPACE;
  return run_prefill(g, q, k, v, out, mass, kept_idx, kept_cnt, workspace, w, sms,
                     reinterpret_cast<cudaStream_t>(stream));
}

rra_status rra_prefill_host(const rra_params *p, const void *q_host, const void *k_host,
                            const void *v_host, void *out_host, void *q_dev, void *k_dev,
                            void *v_dev, void *out_dev, int32_t *kept_idx, int32_t *kept_cnt,
                            void *workspace, size_t workspace_bytes, rra_stream_t stream) {
  Geometry g;
  rra_status s = resolve(p, kNeedsStride | kNeedsHeadDim, &g);
  if (s != RRA_OK) return s;
  if (empty(g)) return RRA_OK;
  if (!q_host || !k_host || !v_host || !out_host || !ptr_ok(q_dev) || !ptr_ok(k_dev) ||
      !ptr_ok(v_dev) || !ptr_ok(out_dev) || !ptr_ok(kept_idx) || !ptr_ok(kept_cnt) ||
      !ptr_ok(workspace))
    return RRA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return RRA_ERR_CUDA;
  if (workspace_bytes < rra::workspace_layout(g, sms).total) return RRA_ERR_WORKSPACE;
  HostPipe *hp = host_pipe();
  if (!hp) return RRA_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Chunks, each a whole sub-problem with contiguous inputs, outputs and kept lists. At batch 1:
  // groups of query heads within one KV head (a divisor gq of the GQA group, as small as keeps
  // the chunk count within kMaxHostChunks; a KV head's K and V travel with its first group), or
  // whole KV heads when there are more KV heads than chunks. Otherwise: groups of batch rows.
  struct Chunk {
    int b0, nb, h0, nh, kv0, nkv;
    bool copy_kv;
  };
  Chunk ch[kMaxHostChunks];
  int nch = 0;
  if (g.b == 1) {
    if (g.hkv <= kMaxHostChunks) {
      int gq = g.g;
      for (int d = g.g - 1; d >= 1; --d)
        if (g.g % d == 0 && g.hkv * (g.g / d) <= kMaxHostChunks) gq = d;
      for (int kv = 0; kv < g.hkv; ++kv)
        for (int j = 0; j < g.g / gq; ++j)
          ch[nch++] = {0, 1, kv * g.g + j * gq, gq, kv, 1, j == 0};
    } else {
      const int per = (g.hkv + kMaxHostChunks - 1) / kMaxHostChunks;
      for (int kv = 0; kv < g.hkv; kv += per) {
        const int n = std::min(per, g.hkv - kv);
        ch[nch++] = {0, 1, kv * g.g, n * g.g, kv, n, true};
      }
    }
  } else {
    const int per = (g.b + kMaxHostChunks - 1) / kMaxHostChunks;
    for (int b = 0; b < g.b; b += per)
      ch[nch++] = {b, std::min(per, g.b - b), 0, g.hq, 0, g.hkv, true};
  }
  const size_t row_q = static_cast<size_t>(g.L) * g.d * 2;   // bytes of one head's rows
  auto at = [](const void *base, size_t off) {
    return const_cast<uint8_t *>(static_cast<const uint8_t *>(base)) + off;
  };
  // the staging buffers may still be in use by earlier work on the caller's stream
  if (cudaEventRecord(hp->start, st) != cudaSuccess ||
      cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return RRA_ERR_CUDA;
  for (int c = 0; c < nch; ++c) {
    const Chunk &k = ch[c];
    rra_params cp = *p;
    cp.batch = k.nb;
    cp.heads_q = k.nh;
    cp.heads_kv = k.nkv;
    cp.shift = (g.shift + k.h0) % g.S;   // the chunk's heads keep their global offsets
    Geometry cg;
    if (resolve(&cp, kNeedsStride | kNeedsHeadDim, &cg) != RRA_OK) return RRA_ERR_INVALID_ARG;
    const WorkspaceLayout cw = rra::workspace_layout(cg, sms);
    // offsets within the [b, H, ...] arrays: batch rows first, then heads
    const size_t qo = row_q * (static_cast<size_t>(k.b0) * g.hq + k.h0);
    const size_t qb = row_q * static_cast<size_t>(k.nb) * k.nh;
    const size_t kvo = row_q * (static_cast<size_t>(k.b0) * g.hkv + k.kv0);
    const size_t kvb = row_q * static_cast<size_t>(k.nb) * k.nkv;
    const int64_t lo = static_cast<int64_t>(k.b0) * g.hq + k.h0;   // first (batch, head) row
    if (cudaMemcpyAsync(at(q_dev, qo), at(q_host, qo), qb, cudaMemcpyHostToDevice, hp->in) !=
            cudaSuccess ||
        (k.copy_kv && (cudaMemcpyAsync(at(k_dev, kvo), at(k_host, kvo), kvb,
                                       cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                       cudaMemcpyAsync(at(v_dev, kvo), at(v_host, kvo), kvb,
                                       cudaMemcpyHostToDevice, hp->in) != cudaSuccess)) ||
        cudaEventRecord(hp->in_done[c], hp->in) != cudaSuccess ||
        cudaStreamWaitEvent(st, hp->in_done[c], 0) != cudaSuccess)
      return RRA_ERR_CUDA;
    s = run_prefill(cg, at(q_dev, qo), at(k_dev, kvo), at(v_dev, kvo), at(out_dev, qo), nullptr,
                    kept_idx + lo * g.tri, kept_cnt + lo * g.nb, workspace, cw, sms, st);
    if (s != RRA_OK) return s;
    if (cudaEventRecord(hp->step_done[c], st) != cudaSuccess ||
        cudaStreamWaitEvent(hp->out, hp->step_done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(at(out_host, qo), at(out_dev, qo), qb, cudaMemcpyDeviceToHost,
                        hp->out) != cudaSuccess)
      return RRA_ERR_CUDA;
  }
  // the call is complete, on the caller's stream, once the last output copy has landed
  if (cudaEventRecord(hp->end, hp->out) != cudaSuccess ||
      cudaStreamWaitEvent(st, hp->end, 0) != cudaSuccess)
    return RRA_ERR_CUDA;
  return RRA_OK;
}

rra_status rra_check_device_status(void *workspace, rra_stream_t stream, uint32_t *raw_word) {
  if (!ptr_ok(workspace)) return RRA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return RRA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RRA_ERR_CUDA;
  if (raw_word) *raw_word = word;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return RRA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return RRA_ERR_CUDA;
  }
  if (word & rra::kErrTimeout) return RRA_ERR_DEVICE_TIMEOUT;
  if (word & rra::kErrBadList) return RRA_ERR_INVALID_ARG;
  return RRA_OK;
}

void rra_set_wait_limit_ns(uint64_t ns) {
  rra::g_wait_limit_ns.store(ns == 0 ? rra::kWaitLimitNs : ns, std::memory_order_relaxed);
}

const char *rra_status_string(rra_status s) {
  switch (s) {
    case RRA_OK: return "ok";
    case RRA_ERR_INVALID_ARG: return "invalid argument";
    case RRA_ERR_UNSUPPORTED: return "unsupported configuration";
    case RRA_ERR_WORKSPACE: return "workspace too small";
    case RRA_ERR_CUDA: return "CUDA error";
    case RRA_ERR_DEVICE_TIMEOUT: return "device barrier wait timed out";
  }
  return "unknown status";
}

const char *rra_version(void) { return "rra 0.1 sm_100a"; }

}  // extern "C"
