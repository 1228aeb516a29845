// Round-robin block-importance estimation (RRAttention, abstract and "Summary": one query per
// stride per head at an offset that rotates across heads, stride-pooled keys, stride-level
// softmax, block aggregation).
//
//   K1 pool_keys_kernel   Kbar[kv, j] = sum_{t<S} K[kv, j*S + t]  (fp32 sum, stored as bf16 hi+lo)
//   K2 rr_estimate_kernel z[h, i, j] = scale * Q[h, i*S + o_h] . Kbar[kv(h), j] on tcgen05,
//                         causal (j <= i) stride softmax, block masses
//                         A[h, I, J] = (1/m) sum_{i in I} sum_{j in J} P[h, i, j].
//
// The same kernel, instantiated with XA = true, computes the XAttention antidiagonal estimate
// (XAttention review, sections 2-3): the logit tile is sum_{t<S} Q_t . K_{S-1-t}^T, where Q_t
// holds the queries at in-stride offset t of 128 query strides and K_{S-1-t} the keys at offset
// S-1-t of 128 key strides; the S products accumulate into one TMEM tile (exact bf16 operands,
// no pooling, no hi/lo split), and the epilogue is the same.
//
// K2 is a persistent, warp-specialised kernel. One work item is (batch, head, tile of 128
// sampled queries); the CTA streams the 128-stride key tiles n = 0..t through a 2-stage TMA
// ring, the MMA warp computes each 128x128 logit tile into one of two TMEM accumulators as
// Qhat . Kbar_hi + Qhat . Kbar_lo (bf16 operands, fp32 accumulation, ~16-bit Kbar), and eight
// epilogue warps take the online causal softmax: two sets of one warp per TMEM lane quadrant,
// set a reading accumulator a, so the sets alternate tiles and one set's loads and stores
// overlap the other's exponentials. Because a row's normaliser is known only after its last
// tile, each thread writes its
// per-(row, key block) partial sums with the running maximum they were taken against into the
// CTA's scratch slot. Four more warps then rescale them once the rows are complete and reduce
// the m sampled rows of each block row with warp shuffles, while the epilogue warps go on to the
// next item: the slot holds two buffers, used by alternate items.
#include <math.h>

#include "common.cuh"
#include "rra_internal.h"

namespace rra {

// ---------------------------------------------------------------------------------- K1
template <int S>
__global__ void __launch_bounds__(256) pool_keys_kernel(const uint4 *__restrict__ k,
                                                        uint4 *__restrict__ khi,
                                                        uint4 *__restrict__ klo,
                                                        int64_t out_rows, int vec_per_row) {
  const int64_t total = out_rows * vec_per_row;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / vec_per_row;
    const int v = static_cast<int>(idx - row * vec_per_row);
    const uint4 *src = k + (row * S) * vec_per_row + v;
    uint4 x[S];
#pragma unroll
    for (int t = 0; t < S; ++t) x[t] = __ldg(src + static_cast<int64_t>(t) * vec_per_row);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int t = 0; t < S; ++t) {
      const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&x[t]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    uint4 hi, lo;
    uint32_t *ph = reinterpret_cast<uint32_t *>(&hi);
    uint32_t *pl = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(acc[2 * e] - hf.x, acc[2 * e + 1] - hf.y);
      ph[e] = *reinterpret_cast<const uint32_t *>(&h2);
      pl[e] = *reinterpret_cast<const uint32_t *>(&l2);
    }
    khi[idx] = hi;
    klo[idx] = lo;
  }
}

// ---------------------------------------------------------------------------------- K2
struct EstParams {
  int hq, hkv, g, ns, ntiles, shift, S;
  int n_items;       // b * hq * ntiles
  int bhq;           // b * hq
  float scale_log2;  // softmax scale * log2(e)
  int64_t tri;       // packed entries per (batch, head)
  float *mass;
  float *est_e;
  float *est_ref;
  uint32_t *status;
  uint64_t wait_ns;  // time limit of a barrier wait
};

// Work items in longest-first order: the first b*hq items are the last query tile of every
// head (t = ntiles-1, the most key tiles), then t = ntiles-2, and so on.
__device__ __forceinline__ void est_decode(const EstParams &p, int item, int &bh, int &t) {
  const int level = item / p.bhq;
  bh = item - level * p.bhq;
  t = p.ntiles - 1 - level;
}

// RR: tm_q = 3-D view of Q (box at in-stride offset o_h), tm_khi / tm_klo = pooled keys.
// XA: tm_q = the same 3-D view of Q, tm_khi = 3-D view of K (box at in-stride offset S-1-t).
template <int D, int M, bool XA>
__global__ void __launch_bounds__(512, 1)
    rr_estimate_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_khi,
                       const __grid_constant__ CUtensorMap tm_klo, const EstParams p) {
  constexpr int NCHUNK = D / 64;                  // 64-column (128-byte) chunks per row
  constexpr uint32_t CHUNK_BYTES = 128 * 128;     // 128 rows x 128 bytes
  constexpr uint32_t TILE_BYTES = NCHUNK * CHUNK_BYTES;
  // RR: resident sampled-query tile + 2 stages of (Kbar hi, Kbar lo); XA: 3 stages of (Q_t, K_t)
  constexpr int NSTAGE = XA ? 3 : 2;
  constexpr uint32_t Q_RES = XA ? 0 : TILE_BYTES;
  constexpr int SEG = 64 / M;                     // key blocks per 64-column half tile
  constexpr int SEG_ROW = 128 / M;                // key blocks per 128-stride key tile
  constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;
  uint8_t *sK = smem + Q_RES;                     // stage s at s*2*TILE: (hi, lo) or (Q_t, K_t)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sK + NSTAGE * 2 * TILE_BYTES);
  uint64_t *q_full = bars + 0;
  uint64_t *q_empty = bars + 1;
  uint64_t *kv_full = bars + 2;                   // [NSTAGE]
  uint64_t *kv_empty = kv_full + NSTAGE;          // [NSTAGE]
  uint64_t *acc_full = kv_empty + NSTAGE;         // [2]
  uint64_t *acc_empty = acc_full + 2;             // [2]
  uint64_t *drain = acc_empty + 2;
  uint64_t *fp_full = drain + 2;                  // [2] scratch buffer b holds a complete item
  uint64_t *fp_empty = fp_full + 2;               // [2] scratch buffer b has been reduced
  float *sM = reinterpret_cast<float *>(fp_empty + 2);   // [2][128]
  float *sL = sM + 256;                                  // [2][128]
  float *sRow = sL + 256;     // [2 buffers][2][128]: row max and 1 / row sum of buffer b's item
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sRow + 512);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
  volatile int *s_flag = reinterpret_cast<volatile int *>(s_tmem + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (cta_grid_timed_out(p.status, s_flag)) return;   // the same answer for every thread

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);   // the four epilogue warps of set a
      mbar_init(&fp_full[a], 256);
      mbar_init(&fp_empty[a], 128);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_khi);
    tma_prefetch_desc(&tm_klo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, qph = 0;
      int issued_q = 0;
      int issued[NSTAGE];
      for (int s2 = 0; s2 < NSTAGE; ++s2) issued[s2] = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        int bh, t;
        est_decode(p, item, bh, t);
        const int h = bh % p.hq;
        const int b = bh / p.hq;
        const int kv = h / p.g;
        const int o = ((h + p.shift) % p.S + p.S) % p.S;
        const int krow = (b * p.hkv + kv) * p.ns;
        if constexpr (XA) {
          // per key tile: S stages of (queries at offset tt, keys at offset S-1-tt)
          for (int n = 0; n <= t && ok; ++n)
            for (int tt = 0; tt < p.S; ++tt) {
              if (!mbar_wait(&kv_empty[stage], phase ^ 1, s_abort, p.status, p.wait_ns)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&kv_full[stage], 2 * TILE_BYTES);
              uint8_t *st = sK + stage * 2 * TILE_BYTES;
              for (int c = 0; c < NCHUNK; ++c) {
                tma_load_3d(st + c * CHUNK_BYTES, &tm_q, &kv_full[stage], c * 64, tt,
                            bh * p.ns + t * 128);
                tma_load_3d(st + TILE_BYTES + c * CHUNK_BYTES, &tm_khi, &kv_full[stage],
                            c * 64, p.S - 1 - tt, krow + n * 128);
              }
              ++issued[stage];
              if (++stage == NSTAGE) {
                stage = 0;
                phase ^= 1;
              }
            }
          (void)o;
          continue;
        }
        if (issued_q > 0) {
          if (!mbar_wait(q_empty, qph, s_abort, p.status, p.wait_ns)) break;
          qph ^= 1;
        }
        mbar_arrive_expect_tx(q_full, TILE_BYTES);
        for (int c = 0; c < NCHUNK; ++c)
          tma_load_3d(sQ + c * CHUNK_BYTES, &tm_q, q_full, c * 64, o, bh * p.ns + t * 128);
        ++issued_q;
        for (int n = 0; n <= t; ++n) {
          if (!mbar_wait(&kv_empty[stage], phase ^ 1, s_abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[stage], 2 * TILE_BYTES);
          uint8_t *hi = sK + stage * 2 * TILE_BYTES;
          for (int c = 0; c < NCHUNK; ++c) {
            tma_load_2d(hi + c * CHUNK_BYTES, &tm_khi, &kv_full[stage], c * 64, krow + n * 128);
            tma_load_2d(hi + TILE_BYTES + c * CHUNK_BYTES, &tm_klo, &kv_full[stage], c * 64,
                        krow + n * 128);
          }
          ++issued[stage];
          if (++stage == NSTAGE) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Let every copy already issued land before the CTA exits. Without an abort each of
      // these phases has completed already (the MMA warp consumed it); after one, a copy may
      // still be in flight even though this loop ended normally.
      if (issued_q > 0) mbar_wait_drain(q_full, (issued_q - 1) & 1);
      for (int s = 0; s < NSTAGE; ++s)
        if (issued[s] > 0) mbar_wait_drain(&kv_full[s], (issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, qph = 0;
      // key tile n of an item goes to accumulator n & 1 (so the epilogue set that reads a tile
      // depends on the tile alone, not on the CTA's earlier items); one phase per accumulator
      uint32_t aph[2] = {0, 0};
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        int bh, t;
        est_decode(p, item, bh, t);
        if constexpr (XA) {
          for (int n = 0; n <= t && ok; ++n) {
            const int acc = n & 1;
            if (!mbar_wait(&acc_empty[acc], aph[acc] ^ 1, s_abort, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            const uint32_t d_tmem = tmem + acc * 128;
            for (int tt = 0; tt < p.S; ++tt) {
              if (!mbar_wait(&kv_full[stage], phase, s_abort, p.status, p.wait_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a_base = smem_u32(sK + stage * 2 * TILE_BYTES);
              const uint32_t b_base = a_base + TILE_BYTES;
#pragma unroll
              for (int c = 0; c < NCHUNK; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t a = sdesc_kmajor_sw128(a_base + c * CHUNK_BYTES + kk * 32);
                  const uint64_t bd = sdesc_kmajor_sw128(b_base + c * CHUNK_BYTES + kk * 32);
                  mma_bf16_ss(d_tmem, a, bd, IDESC, (tt | c | kk) != 0);
                }
              mma_commit(&kv_empty[stage]);
              if (++stage == NSTAGE) {
                stage = 0;
                phase ^= 1;
              }
            }
            if (!ok) break;
            mma_commit(&acc_full[acc]);
            aph[acc] ^= 1;
          }
          continue;
        }
        if (!mbar_wait(q_full, qph, s_abort, p.status, p.wait_ns)) break;
        qph ^= 1;
        for (int n = 0; n <= t; ++n) {
          const int acc = n & 1;
          if (!mbar_wait(&acc_empty[acc], aph[acc] ^ 1, s_abort, p.status, p.wait_ns) ||
              !mbar_wait(&kv_full[stage], phase, s_abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + acc * 128;
          const uint32_t k_base = smem_u32(sK + stage * 2 * TILE_BYTES);
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = sdesc_kmajor_sw128(q_base + c * CHUNK_BYTES + kk * 32);
                const uint64_t bd = sdesc_kmajor_sw128(k_base + part * TILE_BYTES +
                                                       c * CHUNK_BYTES + kk * 32);
                mma_bf16_ss(d_tmem, a, bd, IDESC, (part | c | kk) != 0);
              }
          mma_commit(&kv_empty[stage]);
          mma_commit(&acc_full[acc]);
          if (++stage == NSTAGE) {
            stage = 0;
            phase ^= 1;
          }
          aph[acc] ^= 1;
        }
        if (ok) mma_commit(q_empty);
      }
      mma_commit(drain);   // every MMA issued by this thread completes before teardown
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax / mass epilogue
    // Two sets of four warps, one warp per TMEM lane quadrant in each. Set a takes the key tiles
    // n with n & 1 == a, which the MMA warp puts in accumulator a, all 128 columns as two
    // 64-column halves, so one set's TMEM loads and stores overlap the other set's
    // exponentials. The split depends on n alone, so a row's result does not depend on which
    // CTA ran its item.
    const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
    const int set = (warp - 4) >> 2;      // accumulator read by this set
    const int r = quad * 32 + lane;       // row of the 128-row query tile
    const float NEG_INF = -INFINITY;
    uint32_t aph = 0;                     // phase of accumulator `set`
    bool dead = false;
    int kit = 0;   // this CTA's item ordinal; its scratch buffer is kit & 1
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++kit) {
      const int buf = kit & 1;
      // scratch buffer, row-contiguous: partial sum (key tile n, segment s, row r) at
      // e_base[(n * SEG_ROW + s) * 128] and the reference of (n, half) at
      // ref_base[(n * 2 + half) * 128], so each warp access covers one 128-byte line
      float *e_base = p.est_e + (static_cast<size_t>(blockIdx.x) * 2 + buf) * p.ntiles * SEG_ROW *
                                    128 + r;
      float *ref_base =
          p.est_ref + (static_cast<size_t>(blockIdx.x) * 2 + buf) * p.ntiles * 2 * 128 + r;
      // the buffer's previous item (kit - 2) must have been reduced
      if (!dead && kit >= 2)
        dead = !mbar_wait_warp(&fp_empty[buf], ((kit >> 1) - 1) & 1, s_abort, p.status, p.wait_ns);
      int bh, t;
      est_decode(p, item, bh, t);
      const int i = t * 128 + r;          // sampled query (stride) index of this row
      const bool row_ok = i < p.ns;
      float m_run = NEG_INF, l_run = 0.f;
      for (int n = 0; n <= t; ++n) {
        if ((n & 1) != set) continue;   // the other set's tile
        if (!dead) dead = !mbar_wait_warp(&acc_full[set], aph, s_abort, p.status, p.wait_ns);
        aph ^= 1;
        const uint32_t taddr0 = tmem + (static_cast<uint32_t>(quad * 32) << 16) + set * 128;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float e[SEG];
#pragma unroll
          for (int s = 0; s < SEG; ++s) e[s] = 0.f;
          if (!dead) {
            tc_fence_after();
            uint32_t u[64];
            tmem_ld32(taddr0 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tmem_ld32(taddr0 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            tmem_ld_wait();
            if (half == 1) {   // both halves read: the MMA may overwrite the accumulator
              tc_fence_before();
              mbar_arrive(&acc_empty[set]);
            }
            if (row_ok) {
              float *uf = reinterpret_cast<float *>(u);
              if (n == t) {   // diagonal key tile: stride j is visible to query i iff j <= i
                const int j0 = n * 128 + half * 64;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                  if (j0 + c > i) uf[c] = -INFINITY;
              }
              float mx[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
              for (int c = 0; c < 64; c += 8) {
                mx[0] = fmax3(mx[0], uf[c], uf[c + 1]);
                mx[1] = fmax3(mx[1], uf[c + 2], uf[c + 3]);
                mx[2] = fmax3(mx[2], uf[c + 4], uf[c + 5]);
                mx[3] = fmax3(mx[3], uf[c + 6], uf[c + 7]);
              }
              const float tmax = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]) * p.scale_log2;
              if (tmax > m_run) {
                l_run *= fast_exp2(m_run - tmax);    // m_run = -inf: exp2(-inf) = 0
                m_run = tmax;
              }
              if (m_run > NEG_INF) {
                const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
                const uint64_t negm = f2_pack(-m_run, -m_run);
                uint64_t tot = 0;
#pragma unroll
                for (int s = 0; s < SEG; ++s) {
                  uint64_t acc2 = 0;
#pragma unroll
                  for (int c = 0; c < M; c += 2) {
                    const uint64_t xy =
                        ffma2(f2_pack(uf[s * M + c], uf[s * M + c + 1]), sl2, negm);
                    acc2 = fadd2(acc2, f2_pack(fast_exp2(f2_lo(xy)), fast_exp2(f2_hi(xy))));
                  }
                  e[s] = f2_lo(acc2) + f2_hi(acc2);
                  tot = fadd2(tot, acc2);
                }
                l_run += f2_lo(tot) + f2_hi(tot);
              }
            }
          }
          float *dst = e_base + (static_cast<size_t>(n) * SEG_ROW + half * SEG) * 128;
#pragma unroll
          for (int s = 0; s < SEG; ++s) dst[s * 128] = e[s];
          ref_base[(n * 2 + half) * 128] = m_run;
        }
      }
      // ---- combine the two sets' running max / sum of the row
      sM[set * 128 + r] = m_run;
      sL[set * 128 + r] = l_run;
      named_bar_sync(1, 256);
      const float m0 = sM[r], m1 = sM[128 + r];
      const float mx = fmaxf(m0, m1);
      float ltot = 0.f;
      if (m0 > NEG_INF) ltot += sL[r] * fast_exp2(m0 - mx);
      if (m1 > NEG_INF) ltot += sL[128 + r] * fast_exp2(m1 - mx);
      named_bar_sync(1, 256);
      const float inv = (row_ok && ltot > 0.f) ? 1.f / ltot : 0.f;
      if (set == 0) {
        sRow[buf * 256 + r] = mx;
        sRow[buf * 256 + 128 + r] = inv;
      }
      // publishes this thread's partial sums and, for set 0, the row's max and 1 / sum
      mbar_arrive(&fp_full[buf]);
    }
    tc_fence_before();
  } else if (warp >= 12) {
    // ------------------------------------------------------------ partial-sum reduction
    // One thread per row of buffer kit & 1's item: rescale the row's partial sums by
    // 2^(ref - max) / sum and reduce the M sampled rows of each block row (M consecutive lanes).
    const int r = (warp - 12) * 32 + lane;
    const float NEG_INF = -INFINITY;
    int kit = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++kit) {
      const int buf = kit & 1;
      if (!mbar_wait_warp(&fp_full[buf], (kit >> 1) & 1, s_abort, p.status, p.wait_ns)) break;
      const float *e_base = p.est_e + (static_cast<size_t>(blockIdx.x) * 2 + buf) * p.ntiles *
                                          SEG_ROW * 128 + r;
      const float *ref_base =
          p.est_ref + (static_cast<size_t>(blockIdx.x) * 2 + buf) * p.ntiles * 2 * 128 + r;
      int bh, t;
      est_decode(p, item, bh, t);
      const int i = t * 128 + r;
      const bool row_ok = i < p.ns;
      const float mx = sRow[buf * 256 + r];
      const float inv = sRow[buf * 256 + 128 + r];
      const int I = i / M;
      float *mass_row = p.mass + static_cast<int64_t>(bh) * p.tri +
                        static_cast<int64_t>(I) * (I + 1) / 2;
      const bool writer = row_ok && ((lane % M) == 0);
      // PF key tiles per batch: all their loads are issued before any is used, so the loop
      // pays one L2 / DRAM round trip per batch instead of one per tile
      constexpr int PF = (SEG_ROW >= 32) ? 1 : 32 / SEG_ROW;
      for (int n0 = 0; n0 <= t; n0 += PF) {
        float fr[PF][2];
        float e[PF][SEG_ROW];
#pragma unroll
        for (int k = 0; k < PF; ++k) {
          const int n = n0 + k;
          fr[k][0] = fr[k][1] = NEG_INF;
#pragma unroll
          for (int s = 0; s < SEG_ROW; ++s) e[k][s] = 0.f;
          if (n <= t) {
            fr[k][0] = ref_base[(n * 2) * 128];
            fr[k][1] = ref_base[(n * 2 + 1) * 128];
            const float *src = e_base + static_cast<size_t>(n) * SEG_ROW * 128;
#pragma unroll
            for (int s = 0; s < SEG_ROW; ++s) e[k][s] = src[s * 128];
          }
        }
#pragma unroll
        for (int k = 0; k < PF; ++k) {
          const int n = n0 + k;
          float f[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            f[hh] = (inv > 0.f && fr[k][hh] > NEG_INF) ? fast_exp2(fr[k][hh] - mx) * inv : 0.f;
          const int jb0 = (n * 128) / M;
#pragma unroll
          for (int s = 0; s < SEG_ROW; ++s) {
            float v = e[k][s] * f[s / SEG];
#pragma unroll
            for (int off = M / 2; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            const int J = jb0 + s;
            if (writer && J <= I) mass_row[J] = v * (1.f / M);
          }
        }
      }
      // every load of this buffer has returned (its values were used above)
      mbar_arrive(&fp_empty[buf]);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------------- launch
static bool make_map(CUtensorMap *map, void *base, int rank, const cuuint64_t *dims,
                     const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides_bytes, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_pool_keys(const Geometry &g, const void *k, void *khi, void *klo,
                             int num_sms, cudaStream_t stream) {
  const int64_t out_rows = static_cast<int64_t>(g.b) * g.hkv * g.ns;
  const int vec = g.d / 8;
  const int64_t total = out_rows * vec;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint4 *src = static_cast<const uint4 *>(k);
  uint4 *hi = static_cast<uint4 *>(khi), *lo = static_cast<uint4 *>(klo);
  switch (g.S) {
    case 4: pool_keys_kernel<4><<<blocks, threads, 0, stream>>>(src, hi, lo, out_rows, vec); break;
    case 8: pool_keys_kernel<8><<<blocks, threads, 0, stream>>>(src, hi, lo, out_rows, vec); break;
    case 16: pool_keys_kernel<16><<<blocks, threads, 0, stream>>>(src, hi, lo, out_rows, vec); break;
    case 32: pool_keys_kernel<32><<<blocks, threads, 0, stream>>>(src, hi, lo, out_rows, vec); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int D, int M, bool XA>
static cudaError_t launch_est_t(const CUtensorMap &mq, const CUtensorMap &mhi,
                                const CUtensorMap &mlo, const EstParams &ep, int slots,
                                cudaStream_t stream) {
  constexpr size_t TILE = static_cast<size_t>(D / 64) * 128 * 128;
  constexpr int NSTAGE = XA ? 3 : 2;
  const size_t smem = 1024 + TILE * ((XA ? 0 : 1) + 2 * NSTAGE) + (2 + 2 * NSTAGE + 10) * 8 +
                      1024 * 4 + 16;
  auto kern = rr_estimate_kernel<D, M, XA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<slots, 512, smem, stream>>>(mq, mhi, mlo, ep);
  return cudaGetLastError();
}

template <bool XA>
static cudaError_t dispatch_est(const Geometry &g, const CUtensorMap &mq, const CUtensorMap &mhi,
                                const CUtensorMap &mlo, const EstParams &ep, int slots,
                                cudaStream_t stream) {
  if (g.d == 128) {
    switch (g.m) {
      case 4: return launch_est_t<128, 4, XA>(mq, mhi, mlo, ep, slots, stream);
      case 8: return launch_est_t<128, 8, XA>(mq, mhi, mlo, ep, slots, stream);
      case 16: return launch_est_t<128, 16, XA>(mq, mhi, mlo, ep, slots, stream);
      case 32: return launch_est_t<128, 32, XA>(mq, mhi, mlo, ep, slots, stream);
    }
  } else if (g.d == 64) {
    switch (g.m) {
      case 4: return launch_est_t<64, 4, XA>(mq, mhi, mlo, ep, slots, stream);
      case 8: return launch_est_t<64, 8, XA>(mq, mhi, mlo, ep, slots, stream);
      case 16: return launch_est_t<64, 16, XA>(mq, mhi, mlo, ep, slots, stream);
      case 32: return launch_est_t<64, 32, XA>(mq, mhi, mlo, ep, slots, stream);
    }
  }
  return cudaErrorInvalidValue;
}

// 3-D view (d, S, rows / S) of a [rows, d] bf16 tensor: a {64, 1, 128} box at in-stride offset
// o picks 128 rows spaced S apart.
static bool make_strided_map(CUtensorMap *map, const void *base, int64_t rows, int d, int S) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(rows / S)};
  const cuuint64_t str[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(S) * d * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  return make_map(map, const_cast<void *>(base), 3, dims, str, box);
}

static EstParams est_params(const Geometry &g, float *mass, float *est_e, float *est_ref,
                            uint32_t *status) {
  EstParams ep;
  ep.hq = g.hq;
  ep.hkv = g.hkv;
  ep.g = g.g;
  ep.ns = g.ns;
  ep.ntiles = g.ntiles;
  ep.shift = g.shift;
  ep.S = g.S;
  ep.bhq = g.b * g.hq;
  ep.n_items = ep.bhq * g.ntiles;
  ep.scale_log2 = g.scale * 1.4426950408889634f;
  ep.tri = g.tri;
  ep.mass = mass;
  ep.est_e = est_e;
  ep.est_ref = est_ref;
  ep.status = status;
  ep.wait_ns = wait_limit_ns();
  return ep;
}

cudaError_t launch_rr_estimate(const Geometry &g, const void *q, const void *khi,
                               const void *klo, float *mass, float *est_e, float *est_ref,
                               int slots, uint32_t *status, cudaStream_t stream) {
  CUtensorMap mq, mhi, mlo;
  if (!make_strided_map(&mq, q, static_cast<int64_t>(g.b) * g.hq * g.L, g.d, g.S))
    return cudaErrorInvalidValue;
  const cuuint64_t kdims[2] = {static_cast<cuuint64_t>(g.d),
                               static_cast<cuuint64_t>(g.b) * g.hkv * g.ns};
  const cuuint64_t kstr[1] = {static_cast<cuuint64_t>(g.d) * 2};
  const cuuint32_t kbox[2] = {64, 128};
  if (!make_map(&mhi, const_cast<void *>(khi), 2, kdims, kstr, kbox)) return cudaErrorInvalidValue;
  if (!make_map(&mlo, const_cast<void *>(klo), 2, kdims, kstr, kbox)) return cudaErrorInvalidValue;
  const EstParams ep = est_params(g, mass, est_e, est_ref, status);
  if (slots > ep.n_items) slots = ep.n_items;
  return dispatch_est<false>(g, mq, mhi, mlo, ep, slots, stream);
}

cudaError_t launch_xattn_estimate(const Geometry &g, const void *q, const void *k, float *mass,
                                  float *est_e, float *est_ref, int slots, uint32_t *status,
                                  cudaStream_t stream) {
  CUtensorMap mq, mk;
  if (!make_strided_map(&mq, q, static_cast<int64_t>(g.b) * g.hq * g.L, g.d, g.S) ||
      !make_strided_map(&mk, k, static_cast<int64_t>(g.b) * g.hkv * g.L, g.d, g.S))
    return cudaErrorInvalidValue;
  const EstParams ep = est_params(g, mass, est_e, est_ref, status);
  if (slots > ep.n_items) slots = ep.n_items;
  return dispatch_est<true>(g, mq, mk, mk, ep, slots, stream);
}

}  // namespace rra
