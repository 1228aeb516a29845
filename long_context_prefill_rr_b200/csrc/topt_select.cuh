// Top-tau selection of one block row by one warp (RRAttention "adaptive Top-tau selection";
// the XAttention review, section 3, defines the rule as find_blocks: the smallest set of
// blocks whose summed probability reaches tau), run by the standalone select kernel on one
// row per warp. With masses a[0..I]:
//
//   sort J by a descending (ties: smaller J first), keep the shortest prefix whose running
//   sum reaches tau * sum(a) (inclusive), add the diagonal J = I, emit ascending.
//
// No sort. With keys u_J = bits(a_J) (order-preserving for a >= 0) the cut value is v* = the
// largest key with S(v*) = sum_{u_J >= v*} a_J >= tau * total, found by a bisection over the
// key space up to the row's largest key, which stops as soon as one key is left in the interval
// (at most 32 steps; about log2 of the row length in practice). Every block with a larger key
// is in the prefix; of the blocks tied at v*, the first c in ascending J are, with c the
// smallest count that lifts the fp64 running sum to the target. Ballots then compact the kept
// set in ascending order.
//
// The decisions are the ones fp64 arithmetic gives: each bisection step first sums in fp32 and
// falls back to an fp64 sum only when the fp32 sum lies within a margin of the target that
// bounds the fp32 rounding error.
#pragma once

#include <stdint.h>

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
  uint32_t kmax = 0;
#pragma unroll
  for (int k = 0; k < nch; ++k) {
    const float v = get(k);
    t4[k & 3] += static_cast<double>(v);
    f4[k & 3] += v;
    kmax = max(kmax, __float_as_uint(v));
  }
  const double tot = warp_sum_f64((t4[0] + t4[1]) + (t4[2] + t4[3]));
  const float tot32 = warp_sum_f32((f4[0] + f4[1]) + (f4[2] + f4[3]));
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const double target = static_cast<double>(tau) * tot;
  uint32_t vstar;
  if (!(target > 0.0)) {
    // every mass is 0: the first sorted block (largest key, smallest J among ties) reaches it
    vstar = kmax;
  } else {
    const float target32 = static_cast<float>(target);
    // |fp32 partial sum - exact| is below (chunks + 5) * 2^-24 * total; 1e-5 * total leaves a
    // wide safety factor for rows up to 1024 blocks
    const float margin = 1e-5f * tot32 + 1e-30f;
    // Invariant: S(lo) >= target > S(hi), with S(v) the sum of the masses whose key is >= v.
    // S changes only at keys that occur, so the answer is the largest key in [lo, hi); once
    // exactly one of the row's 32 * nch slots has its key in [lo, hi), that key is the answer
    // (c_lo, c_hi count the slots with keys >= lo, >= hi; padding slots hold key 0).
    uint64_t lo = 0, hi = static_cast<uint64_t>(kmax) + 1;
    uint32_t c_lo = 32u * static_cast<uint32_t>(nch), c_hi = 0;
    while (hi - lo > 1 && c_lo - c_hi > 1) {
      const uint64_t mid = (lo + hi) >> 1;
      const uint32_t m32 = static_cast<uint32_t>(mid);
      bool ge;
      uint32_t c = 0;
      if (NCH > 0) {
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < nch; ++k) {
          const float v = get(k);
          const bool above = __float_as_uint(v) >= m32;
          s4[k & 3] += above ? v : 0.f;
          c += above ? 1u : 0u;
        }
        c = __reduce_add_sync(0xffffffffu, c);
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
          const bool above = __float_as_uint(v) >= m32;
          d4[k & 3] += above ? static_cast<double>(v) : 0.0;
          c += above ? 1u : 0u;
        }
        c = __reduce_add_sync(0xffffffffu, c);
        ge = warp_sum_f64((d4[0] + d4[1]) + (d4[2] + d4[3])) >= target;
      }
      if (ge) {
        lo = mid;
        c_lo = c;
      } else {
        hi = mid;
        c_hi = c;
      }
    }
    if (hi - lo > 1) {   // one slot left in [lo, hi): its key
      uint32_t best = 0;
#pragma unroll
      for (int k = 0; k < nch; ++k) {
        const uint32_t key = __float_as_uint(get(k));
        if (key >= lo && key < hi) best = max(best, key);
      }
      vstar = __reduce_max_sync(0xffffffffu, best);
    } else {
      vstar = static_cast<uint32_t>(lo);
    }
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

// Selects one row of n = I + 1 masses, read by `load(J)` (the raw fp32 mass of block J), into
// out[0..n) (ascending, -1 padded) and *cnt_out. Rows of up to 1024 blocks are held in
// registers, in a variant specialised to the row's chunk count; longer rows are re-read through
// `load` in every pass. tau >= 1 keeps every block. Whole warp, warp-uniform arguments.
template <int NCH, class Load>
__device__ __forceinline__ void select_row_regs(Load load, int32_t *out, int32_t *cnt_out, int n,
                                                int I, float tau, int lane) {
  float v[NCH];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int J = k * 32 + lane;
    v[k] = J < n ? clamp_mass(load(J)) : 0.f;
  }
  select_row<NCH>([&](int k) { return v[k]; }, NCH, out, cnt_out, n, I, tau, lane);
}

template <class Load>
__device__ __noinline__ void select_row_mem(Load load, int32_t *out, int32_t *cnt_out, int n,
                                            int I, float tau, int lane) {
  auto get = [&](int k) -> float {
    const int J = k * 32 + lane;
    return J < n ? clamp_mass(load(J)) : 0.f;
  };
  select_row<0>(get, (n + 31) >> 5, out, cnt_out, n, I, tau, lane);
}

template <class Load>
__device__ __forceinline__ void select_row_any(Load load, int32_t *out, int32_t *cnt_out, int n,
                                               int I, float tau, int lane) {
  if (tau >= 1.f) {
    for (int J = lane; J < n; J += 32) out[J] = J;
    if (lane == 0) *cnt_out = n;
    return;
  }
  const int nch = (n + 31) >> 5;
  if (nch <= 1) select_row_regs<1>(load, out, cnt_out, n, I, tau, lane);
  else if (nch <= 2) select_row_regs<2>(load, out, cnt_out, n, I, tau, lane);
  else if (nch <= 4) select_row_regs<4>(load, out, cnt_out, n, I, tau, lane);
  else if (nch <= 8) select_row_regs<8>(load, out, cnt_out, n, I, tau, lane);
  else if (nch <= 16) select_row_regs<16>(load, out, cnt_out, n, I, tau, lane);
  else if (nch <= 32) select_row_regs<32>(load, out, cnt_out, n, I, tau, lane);
  else select_row_mem(load, out, cnt_out, n, I, tau, lane);
}

}  // namespace rra
