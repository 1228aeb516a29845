// Top-tau block selection (RRAttention "adaptive Top-tau selection"; the XAttention review,
// section 3, defines the rule as find_blocks: the smallest set of blocks whose summed
// probability reaches tau). Per (batch, head, block row I) with masses a[0..I]:
//
//   sort J by a descending (ties: smaller J first), keep the shortest prefix whose running
//   sum reaches tau * sum(a) (inclusive), add the diagonal J = I, emit ascending.
//
// One warp per row, no sort. With keys u_J = bits(a_J) (order-preserving for a >= 0) the cut
// value is v* = the largest key with S(v*) = sum_{u_J >= v*} a_J >= tau * total, found by a
// 32-step bisection over the key space with fp64 warp sums. Every block with a larger key is
// in the prefix; of the blocks tied at v*, the first c in ascending J are, with c the smallest
// count that lifts the fp64 running sum to the target. Ballots then compact the kept set in
// ascending order.
#include "common.cuh"
#include "rra_internal.h"

namespace rra {

constexpr int kRegChunks = 32;   // rows up to 32 x 32 = 1024 blocks are held in registers

__device__ __forceinline__ float clamp_mass(float a) { return (a >= 0.f) ? a : 0.f; }  // NaN -> 0

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__global__ void __launch_bounds__(256) topt_select_kernel(const float *__restrict__ mass,
                                                          int32_t *__restrict__ kept_idx,
                                                          int32_t *__restrict__ kept_cnt,
                                                          int64_t rows, int nb, int64_t tri,
                                                          float tau) {
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps_total) {
    const int64_t bh = row / nb;
    const int I = static_cast<int>(row - bh * nb);
    const int n = I + 1;
    const int64_t off = bh * tri + static_cast<int64_t>(I) * (I + 1) / 2;
    const float *a = mass + off;
    int32_t *out = kept_idx + off;
    if (tau >= 1.f) {
      for (int J = lane; J < n; J += 32) out[J] = J;
      if (lane == 0) kept_cnt[row] = n;
      continue;
    }
    const int nchunks = (n + 31) >> 5;
    float reg[kRegChunks];
#pragma unroll
    for (int k = 0; k < kRegChunks; ++k) {
      const int J = k * 32 + lane;
      reg[k] = (k < nchunks && J < n) ? clamp_mass(__ldg(a + J)) : 0.f;
    }
    auto value = [&](int k) -> float {   // chunk k >= kRegChunks of this lane, from memory
      const int J = k * 32 + lane;
      return J < n ? clamp_mass(__ldg(a + J)) : 0.f;
    };
    // ---- row total and target
    double tot = 0.0;
#pragma unroll
    for (int k = 0; k < kRegChunks; ++k)
      if (k < nchunks) tot += static_cast<double>(reg[k]);
    for (int k = kRegChunks; k < nchunks; ++k) tot += static_cast<double>(value(k));
    tot = warp_sum_f64(tot);
    const double target = static_cast<double>(tau) * tot;
    uint32_t vstar;
    if (!(target > 0.0)) {
      // every mass is 0: the first sorted block (the largest key, smallest J among ties)
      // already reaches the target
      uint32_t best = 0;
#pragma unroll
      for (int k = 0; k < kRegChunks; ++k) best = max(best, __float_as_uint(reg[k]));
      for (int k = kRegChunks; k < nchunks; ++k) best = max(best, __float_as_uint(value(k)));
      vstar = __reduce_max_sync(0xffffffffu, best);
    } else {
      // ---- bisection for v*: S(lo) >= target, S(hi) < target
      uint64_t lo = 0, hi = 0x100000000ull;
      while (hi - lo > 1) {
        const uint64_t mid = (lo + hi) >> 1;
        const uint32_t m32 = static_cast<uint32_t>(mid);
        double s = 0.0;
#pragma unroll
        for (int k = 0; k < kRegChunks; ++k)
          if (k < nchunks) s += (__float_as_uint(reg[k]) >= m32) ? static_cast<double>(reg[k]) : 0.0;
        for (int k = kRegChunks; k < nchunks; ++k) {
          const float v = value(k);
          s += (__float_as_uint(v) >= m32) ? static_cast<double>(v) : 0.0;
        }
        s = warp_sum_f64(s);
        if (s >= target) lo = mid; else hi = mid;
      }
      vstar = static_cast<uint32_t>(lo);
    }
    // ---- sum strictly above v*, then the number c of ties at v* to take (ascending J)
    double above = 0.0;
#pragma unroll
    for (int k = 0; k < kRegChunks; ++k)
      if (k < nchunks) above += (__float_as_uint(reg[k]) > vstar) ? static_cast<double>(reg[k]) : 0.0;
    for (int k = kRegChunks; k < nchunks; ++k) {
      const float v = value(k);
      above += (__float_as_uint(v) > vstar) ? static_cast<double>(v) : 0.0;
    }
    above = warp_sum_f64(above);
    const double astar = static_cast<double>(__uint_as_float(vstar));
    int c = 1;
    if (target > 0.0) {
      double x = above + astar;
      while (x < target && c < n) {
        x += astar;
        ++c;
      }
    }
    // ---- compaction in ascending J
    int base = 0, ties_seen = 0;
    auto emit = [&](int k, float v) {
      const int J = k * 32 + lane;
      const uint32_t key = __float_as_uint(v);
      const bool in_row = J < n;
      const bool tie = in_row && key == vstar;
      const uint32_t tie_ballot = __ballot_sync(0xffffffffu, tie);
      const int tie_rank = ties_seen + __popc(tie_ballot & lt_mask);
      const bool keep = in_row && (key > vstar || (tie && tie_rank < c) || J == I);
      const uint32_t kb = __ballot_sync(0xffffffffu, keep);
      if (keep) out[base + __popc(kb & lt_mask)] = J;
      base += __popc(kb);
      ties_seen += __popc(tie_ballot);
    };
#pragma unroll
    for (int k = 0; k < kRegChunks; ++k)
      if (k < nchunks) emit(k, reg[k]);
    for (int k = kRegChunks; k < nchunks; ++k) emit(k, value(k));
    for (int J = base + lane; J < n; J += 32) out[J] = -1;
    if (lane == 0) kept_cnt[row] = base;
  }
}

cudaError_t launch_topt_select(const Geometry &g, const float *mass, int32_t *kept_idx,
                               int32_t *kept_cnt, int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(g.b) * g.hq * g.nb;
  const int threads = 256;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  topt_select_kernel<<<blocks, threads, 0, stream>>>(mass, kept_idx, kept_cnt, rows, g.nb, g.tri,
                                                     g.tau);
  return cudaGetLastError();
}

}  // namespace rra
