// Top-tau block selection (RRAttention "adaptive Top-tau selection"; the XAttention review,
// section 3, defines the rule as find_blocks: the smallest set of blocks whose summed
// probability reaches tau). Per (batch, head, block row I) with masses a[0..I]:
//
//   sort J by a descending (ties: smaller J first), keep the shortest prefix whose running
//   sum reaches tau * sum(a) (inclusive), add the diagonal J = I, emit ascending.
//
// One warp per row, no sort. With keys u_J = bits(a_J) (order-preserving for a >= 0) the cut
// value is v* = the largest key with S(v*) = sum_{u_J >= v*} a_J >= tau * total, found by a
// 32-step bisection over the key space. Every block with a larger key is in the prefix; of the
// blocks tied at v*, the first c in ascending J are, with c the smallest count that lifts the
// fp64 running sum to the target. Ballots then compact the kept set in ascending order.
//
// The decisions are the ones fp64 arithmetic gives: each bisection step first sums in fp32 and
// falls back to an fp64 sum only when the fp32 sum lies within a margin of the target that
// bounds the fp32 rounding error. Rows of up to 1024 blocks are held in registers, in a
// variant specialised to the row's chunk count; longer rows are re-read from memory.
#include "common.cuh"
#include "rra_internal.h"

namespace rra {

__device__ __forceinline__ float clamp_mass(float a) { return (a >= 0.f) ? a : 0.f; }  // NaN -> 0

// Butterfly sums: every lane ends with the same bits (IEEE addition is commutative).
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// One row on one warp. Chunk k of a lane holds J = 32 k + lane; `get(k)` returns its clamped
// mass (0 past the row end). `nch` chunks; NCH > 0 fixes the count at compile time.
template <int NCH, class Get>
__device__ __forceinline__ void select_row(Get get, int nch_rt, int32_t *out, int32_t *cnt_out,
                                           int n, int I, float tau, int lane) {
  const int nch = NCH > 0 ? NCH : nch_rt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  double t4[4] = {0.0, 0.0, 0.0, 0.0};
  float f4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < nch; ++k) {
    const float v = get(k);
    t4[k & 3] += static_cast<double>(v);
    f4[k & 3] += v;
  }
  const double tot = warp_sum_f64((t4[0] + t4[1]) + (t4[2] + t4[3]));
  const float tot32 = warp_sum_f32((f4[0] + f4[1]) + (f4[2] + f4[3]));
  const double target = static_cast<double>(tau) * tot;
  uint32_t vstar;
  if (!(target > 0.0)) {
    // every mass is 0: the first sorted block (largest key, smallest J among ties) reaches it
    uint32_t best = 0;
#pragma unroll
    for (int k = 0; k < nch; ++k) best = max(best, __float_as_uint(get(k)));
    vstar = __reduce_max_sync(0xffffffffu, best);
  } else {
    const float target32 = static_cast<float>(target);
    // |fp32 partial sum - exact| is below (chunks + 5) * 2^-24 * total; 1e-5 * total leaves a
    // wide safety factor for rows up to 1024 blocks
    const float margin = 1e-5f * tot32 + 1e-30f;
    uint64_t lo = 0, hi = 0x100000000ull;
    while (hi - lo > 1) {
      const uint64_t mid = (lo + hi) >> 1;
      const uint32_t m32 = static_cast<uint32_t>(mid);
      bool ge;
      if (NCH > 0) {
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < nch; ++k) {
          const float v = get(k);
          s4[k & 3] += (__float_as_uint(v) >= m32) ? v : 0.f;
        }
        const float s32 = warp_sum_f32((s4[0] + s4[1]) + (s4[2] + s4[3]));
        if (s32 - target32 > margin) {
          ge = true;
        } else if (target32 - s32 > margin) {
          ge = false;
        } else {
          double d4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
          for (int k = 0; k < nch; ++k) {
            const float v = get(k);
            d4[k & 3] += (__float_as_uint(v) >= m32) ? static_cast<double>(v) : 0.0;
          }
          ge = warp_sum_f64((d4[0] + d4[1]) + (d4[2] + d4[3])) >= target;
        }
      } else {   // long rows: straight fp64
        double d4[4] = {0.0, 0.0, 0.0, 0.0};
        for (int k = 0; k < nch; ++k) {
          const float v = get(k);
          d4[k & 3] += (__float_as_uint(v) >= m32) ? static_cast<double>(v) : 0.0;
        }
        ge = warp_sum_f64((d4[0] + d4[1]) + (d4[2] + d4[3])) >= target;
      }
      if (ge) lo = mid; else hi = mid;
    }
    vstar = static_cast<uint32_t>(lo);
  }
  // ---- exact sum strictly above v*, then the number c of ties at v* to take (ascending J)
  double a4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int k = 0; k < nch; ++k) {
    const float v = get(k);
    a4[k & 3] += (__float_as_uint(v) > vstar) ? static_cast<double>(v) : 0.0;
  }
  const double above = warp_sum_f64((a4[0] + a4[1]) + (a4[2] + a4[3]));
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
#pragma unroll
  for (int k = 0; k < nch; ++k) {
    const int J = k * 32 + lane;
    const uint32_t key = __float_as_uint(get(k));
    const bool in_row = J < n;
    const bool tie = in_row && key == vstar;
    const uint32_t tie_ballot = __ballot_sync(0xffffffffu, tie);
    const int tie_rank = ties_seen + __popc(tie_ballot & lt_mask);
    const bool keep = in_row && (key > vstar || (tie && tie_rank < c) || J == I);
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(kb & lt_mask)] = J;
    base += __popc(kb);
    ties_seen += __popc(tie_ballot);
  }
  for (int J = base + lane; J < n; J += 32) out[J] = -1;
  if (lane == 0) *cnt_out = base;
}

template <int NCH>
__device__ __forceinline__ void select_row_regs(const float *a, int32_t *out, int32_t *cnt_out,
                                                int n, int I, float tau, int lane) {
  float v[NCH];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int J = k * 32 + lane;
    v[k] = J < n ? clamp_mass(__ldg(a + J)) : 0.f;
  }
  select_row<NCH>([&](int k) { return v[k]; }, NCH, out, cnt_out, n, I, tau, lane);
}

// Rows longer than 1024 blocks: values re-read from memory (L1 / L2) in every pass.
__device__ __noinline__ void select_row_mem(const float *a, int32_t *out, int32_t *cnt_out,
                                            int n, int I, float tau, int lane) {
  auto get = [&](int k) -> float {
    const int J = k * 32 + lane;
    return J < n ? clamp_mass(__ldg(a + J)) : 0.f;
  };
  select_row<0>(get, (n + 31) >> 5, out, cnt_out, n, I, tau, lane);
}

__global__ void __launch_bounds__(256) topt_select_kernel(const float *__restrict__ mass,
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
    if (tau >= 1.f) {
      for (int J = lane; J < n; J += 32) out[J] = J;
      if (lane == 0) *cnt = n;
      continue;
    }
    const int nch = (n + 31) >> 5;
    if (nch <= 1) select_row_regs<1>(a, out, cnt, n, I, tau, lane);
    else if (nch <= 2) select_row_regs<2>(a, out, cnt, n, I, tau, lane);
    else if (nch <= 4) select_row_regs<4>(a, out, cnt, n, I, tau, lane);
    else if (nch <= 8) select_row_regs<8>(a, out, cnt, n, I, tau, lane);
    else if (nch <= 16) select_row_regs<16>(a, out, cnt, n, I, tau, lane);
    else if (nch <= 32) select_row_regs<32>(a, out, cnt, n, I, tau, lane);
    else select_row_mem(a, out, cnt, n, I, tau, lane);
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
