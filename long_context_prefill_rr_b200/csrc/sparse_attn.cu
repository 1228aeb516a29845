// Causal block-sparse attention forward over the kept key blocks (RRAttention computes only
// the selected blocks; "regular block-sparse FlashAttention execution" in the RBS-Attention
// digest; online softmax as in FlashAttention / FlashAttention-2), GQA head mapping.
//
// One CTA runs one work item: query block I of one head. Its footprint (256 threads, 256 TMEM
// columns, about 99 KB of shared memory) lets two CTAs share an SM, so the tensor core works on
// one CTA's tile while the other CTA's softmax runs, and one CTA's set-up and epilogue overlap
// the other's work. Grid order is longest-first (I descending), by KV-head chunk when K and V
// exceed L2 (see attn_item). Roles:
//   warp 0       TMA producer: the Q tile, then V(j-1), K(j) through a two-tile ring, in the
//                order the MMA warp consumes them;
//   warp 1       MMA issuer (one thread): O += P(j-1) V(j-1) with P read from TMEM (tcgen05
//                "TS" form; 32 keys at a time, as soon as that quarter of P is written), then
//                S = Q K(j)^T into the same TMEM columns. It counts the
//                item's valid tiles up front, so its issue loop reads no global memory;
//   warp 2       TMEM allocation: S / P (128 columns) | O (d columns);
//   warps 4-7    softmax: one thread per query row reads its 128 logits from TMEM once into
//                registers, masks the diagonal block, keeps a running max (O is rescaled in
//                TMEM, before any P of the tile is published, only when the max grows by more
//                than 2^8, decided per warp) and running sum of the bf16-rounded weights, writes
//                P as bf16 back over S 16 keys at a time (published 32 keys at a time), and at
//                the end normalises O and stores the bf16 row.
// The first warpgroup (warps 0-3) runs with 96 registers a thread and the softmax warpgroup
// with 160 (setmaxnreg), out of the 128 a thread the CTA is launched with; the 160 hold the
// row's 128 logits.
// Because the S / P columns are reused every tile, S(j) completing implies that the previous
// P V product completed (MMAs complete in issue order), so O is stable whenever the softmax
// runs. The kept list is read by every role with the same validity rule (0 <= J <= I, strictly
// ascending); invalid entries are skipped and flagged in the status word by the producer.
#include <math.h>

#include "common.cuh"
#include "rra_internal.h"

namespace rra {

struct AttnParams {
  int hq, hkv, g, L, nb, batch;
  int n_units;       // batch * hq work units (one head each) per query block
  int chunk;         // heads per chunk of the launch order (one KV head's query heads, or all)
  int64_t tri;
  float scale_log2;
  const int32_t *kept_idx;
  const int32_t *kept_cnt;
  __nv_bfloat16 *out;
  uint32_t *status;
  uint64_t wait_ns;  // time limit of a barrier wait
};

// Walks one kept row, yielding the valid entries (0 <= J <= I, strictly ascending). The entry
// after the current one is loaded one call ahead, so its latency overlaps the caller's work.
struct ListCursor {
  const int32_t *lst;
  int cnt, e, prev, I, ahead;
  __device__ void init(const AttnParams &p, int bh, int I_, bool valid) {
    I = I_;
    e = 0;
    prev = -1;
    lst = p.kept_idx + static_cast<int64_t>(bh) * p.tri + static_cast<int64_t>(I) * (I + 1) / 2;
    cnt = 0;
    ahead = -1;
    if (valid) {
      // both loads issued together: the row has I + 1 >= 1 entries, so lst[0] is in bounds
      const int first = lst[0];
      cnt = p.kept_cnt[static_cast<int64_t>(bh) * p.nb + I];
      if (cnt < 0) cnt = 0;
      if (cnt > I + 1) cnt = I + 1;
      ahead = cnt > 0 ? first : -1;
    }
  }
  // next valid block index, or -1; invalid entries are reported through `status` if non-null
  __device__ int next(uint32_t *status) {
    while (e < cnt) {
      const int J = ahead;
      if (++e < cnt) ahead = lst[e];
      if (J > prev && J <= I) {
        prev = J;
        return J;
      }
      if (status) atomicOr(status, kErrBadList);
    }
    return -1;
  }
};

// Number of entries ListCursor::next yields for one row, counted by a whole warp: an entry is
// yielded iff it lies in [0, I] and exceeds every earlier in-range entry (the yielded entries
// are then the strict running maxima of the in-range ones).
__device__ int count_valid_warp(const AttnParams &p, int bh, int I, bool valid, int lane) {
  if (!valid) return 0;
  int cnt = p.kept_cnt[static_cast<int64_t>(bh) * p.nb + I];
  cnt = cnt < 0 ? 0 : (cnt > I + 1 ? I + 1 : cnt);
  const int32_t *lst =
      p.kept_idx + static_cast<int64_t>(bh) * p.tri + static_cast<int64_t>(I) * (I + 1) / 2;
  int carry = -1, n = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int e = base + lane;
    const int J = e < cnt ? lst[e] : -1;
    const int v = (J >= 0 && J <= I) ? J : -1;
    int pm = v;   // inclusive prefix max over the chunk
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, pm, off);
      if (lane >= off) pm = max(pm, o);
    }
    int before = __shfl_up_sync(0xffffffffu, pm, 1);
    before = lane == 0 ? carry : max(before, carry);
    n += __popc(__ballot_sync(0xffffffffu, v >= 0 && v > before));
    carry = max(carry, __shfl_sync(0xffffffffu, pm, 31));
  }
  return n;
}

// Launch order: per batch row, chunks of `chunk` query heads, each chunk's block rows longest
// first (I descending), the chunk's heads innermost. With one chunk per batch row this is plain
// longest-first. With chunks of the query heads of one KV head, the CTAs resident at one time
// read the K/V tiles of one or two KV heads, which fit in L2 even at long lengths, so a tile kept
// by several rows or heads is fetched from DRAM about once.
__device__ __forceinline__ void attn_item(const AttnParams &p, int64_t idx, int &b, int &h,
                                          int &level) {
  const int64_t per_b = static_cast<int64_t>(p.nb) * p.hq;
  b = static_cast<int>(idx / per_b);
  const int64_t r = idx - b * per_b;
  const int C = p.chunk;
  const int nfull = p.hq / C;
  const int64_t full = static_cast<int64_t>(nfull) * p.nb * C;
  if (r < full) {
    const int64_t per_chunk = static_cast<int64_t>(p.nb) * C;
    const int k = static_cast<int>(r / per_chunk);
    const int64_t s = r - k * per_chunk;
    level = static_cast<int>(s / C);
    h = k * C + static_cast<int>(s - static_cast<int64_t>(level) * C);
  } else {   // the last, narrower chunk
    const int crem = p.hq - nfull * C;
    const int64_t s = r - full;
    level = static_cast<int>(s / crem);
    h = nfull * C + static_cast<int>(s - static_cast<int64_t>(level) * crem);
  }
}

template <int D>
__global__ void __launch_bounds__(256, 2)
    bs_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int NCHUNK = D / 64;
  constexpr uint32_t CHUNK_BYTES = 128 * 128;
  constexpr uint32_t TILE_BYTES = NCHUNK * CHUNK_BYTES;   // 128 rows x D bf16
  constexpr int NSTAGE = (D == 128) ? 2 : 4;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, true);
  constexpr float RESCALE_THRESHOLD = 8.0f;               // log2 units

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;
  uint8_t *sRing = sQ + TILE_BYTES;                 // [NSTAGE] tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sRing + NSTAGE * TILE_BYTES);
  uint64_t *q_full = bars + 0;
  uint64_t *kv_full = bars + 1;                     // [NSTAGE]
  uint64_t *kv_empty = kv_full + NSTAGE;            // [NSTAGE]
  uint64_t *s_full = kv_empty + NSTAGE;
  uint64_t *p_q = s_full + 1;                       // [4] P of keys 32q..32q+31 written
  uint64_t *o_final = p_q + 4;
  uint64_t *drain = o_final + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
  volatile int *s_flag = reinterpret_cast<volatile int *>(s_tmem + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int b, h, level;
  attn_item(p, blockIdx.x, b, h, level);
  const int I = p.nb - 1 - level;
  const int bh = b * p.hq + h;
  const int kvrow = (b * p.hkv + h / p.g) * p.L;

  if (cta_grid_timed_out(p.status, s_flag)) return;   // the same answer for every thread
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&p_q[i], 128);
    mbar_init(o_final, 1);
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
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tm_s = tmem;          // S / P: columns 0..127
  const uint32_t tm_o = tmem + 128u;   // O: columns 128..128+D

  if (warp < 4) {
    // Register split between the warpgroups: the producer / MMA / allocator warpgroup gives up
    // registers so that the softmax warpgroup can keep its row slice and more exponentials in
    // flight (96 + 160 = 2 x the 128 the CTA was launched with).
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory");
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int issued[NSTAGE];
        for (int s = 0; s < NSTAGE; ++s) issued[s] = 0;
        bool ok = true;
        auto load = [&](const CUtensorMap *map, int row) -> bool {
          if (!mbar_wait(&kv_empty[stage], phase ^ 1, s_abort, p.status, p.wait_ns)) return false;
          mbar_arrive_expect_tx(&kv_full[stage], TILE_BYTES);
          uint8_t *dst = sRing + stage * TILE_BYTES;
          for (int c = 0; c < NCHUNK; ++c)
            tma_load_2d(dst + c * CHUNK_BYTES, map, &kv_full[stage], c * 64, row);
          ++issued[stage];
          if (++stage == NSTAGE) {
            stage = 0;
            phase ^= 1;
          }
          return true;
        };
        // the Q tile first: its load overlaps the reads of the kept list (a row with no valid
        // entry, rare, loads it for nothing)
        mbar_arrive_expect_tx(q_full, TILE_BYTES);
        for (int c = 0; c < NCHUNK; ++c)
          tma_load_2d(sQ + c * CHUNK_BYTES, &tm_q, q_full, c * 64, bh * p.L + I * 128);
        ListCursor cur;
        cur.init(p, bh, I, true);
        int J = cur.next(p.status), pendV = -1;
        // the MMA warp's order: V(j - 1) for P(j - 1) V(j - 1), then K(j) for S(j)
        while (ok && (pendV >= 0 || J >= 0)) {
          if (pendV >= 0) {
            ok = load(&tm_v, kvrow + pendV * 128);
            pendV = -1;
          }
          if (ok && J >= 0) {
            ok = load(&tm_k, kvrow + J * 128);
            pendV = J;
            J = cur.next(p.status);
          }
        }
        // Let every copy already issued land before the CTA exits (without an abort these
        // phases have completed already: the MMA warp consumed them).
        mbar_wait_drain(q_full, 0);
        for (int s = 0; s < NSTAGE; ++s)
          if (issued[s] > 0) mbar_wait_drain(&kv_full[s], (issued[s] - 1) & 1);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      const int n = count_valid_warp(p, bh, I, true, lane);
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        if (n > 0) ok = mbar_wait(q_full, 0, s_abort, p.status, p.wait_ns);
        const uint32_t ring_base = smem_u32(sRing);
        const uint64_t q_desc = sdesc_kmajor_sw128(smem_u32(sQ));
        const uint64_t k_desc0 = sdesc_kmajor_sw128(ring_base);
        const uint64_t v_desc0 = sdesc_mnmajor_sw128(ring_base, CHUNK_BYTES);
        for (int j = 0; j <= n && ok; ++j) {
          if (j >= 1) {
            // O += P(j-1) V(j-1): 32 keys at a time, as soon as that quarter of P is written
            if (!mbar_wait(&kv_full[stage], phase, s_abort, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            const uint64_t vd = v_desc0 + ((stage * TILE_BYTES) >> 4);
            for (int qq = 0; qq < 4 && ok; ++qq) {
              if (!mbar_wait(&p_q[qq], (j - 1) & 1, s_abort, p.status, p.wait_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kk = 2 * qq; kk < 2 * qq + 2; ++kk)
                mma_bf16_ts(tm_o, tm_s + kk * 8, vd + kk * (2048 >> 4), IDESC_O,
                            (j > 1 || kk > 0) ? 1u : 0u);
            }
            if (!ok) break;
            mma_commit(&kv_empty[stage]);
            if (j == n) mma_commit(o_final);
            if (++stage == NSTAGE) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (j < n) {
            // S = Q K(j)^T into the S / P columns
            if (!mbar_wait(&kv_full[stage], phase, s_abort, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kd = k_desc0 + ((stage * TILE_BYTES) >> 4);
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t off = (c * CHUNK_BYTES + kk * 32) >> 4;
                mma_bf16_ss(tm_s, q_desc + off, kd + off, IDESC_S, (c | kk) != 0);
              }
            mma_commit(&kv_empty[stage]);
            mma_commit(s_full);
            if (++stage == NSTAGE) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 160;\n" ::: "memory");
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_cols = tm_s + lane_off;
    const uint32_t o_cols = tm_o + lane_off;
    const float NEG_INF = -INFINITY;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    float m_run = NEG_INF;
    float lsum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    bool dead = false;
    ListCursor cur;
    cur.init(p, bh, I, true);
    int t = 0;
    for (int J = cur.next(nullptr); J >= 0; J = cur.next(nullptr), ++t) {
      if (!mbar_wait_warp(s_full, t & 1, s_abort, p.status, p.wait_ns)) {
        dead = true;
        break;
      }
      tc_fence_after();
      const bool diag = (J == I);   // diagonal block: key c is visible to query r iff c <= r
      // one read of the 128 logits; they stay in registers for the max and for P
      float u[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(s_cols + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
      tmem_ld_wait();
      if (diag) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) u[c] = NEG_INF;
      }
      float mx[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx[0] = fmax3(mx[0], u[c], u[c + 1]);
        mx[1] = fmax3(mx[1], u[c + 2], u[c + 3]);
        mx[2] = fmax3(mx[2], u[c + 4], u[c + 5]);
        mx[3] = fmax3(mx[3], u[c + 6], u[c + 7]);
      }
      const float tmax = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]) * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (t == 0) {
        m_run = tmax;
      } else if (__any_sync(0xffffffffu, tmax > m_run + RESCALE_THRESHOLD)) {
        const float m_new = fmaxf(m_run, tmax);
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        rescale = true;
#pragma unroll
        for (int c = 0; c < 8; ++c) lsum[c] *= alpha;
      }
      if (rescale) {
        // O is final for the previous tile (S(t) completing implies it); rescaled before any
        // P of this tile is published, 8 columns at a time (the logits hold the registers)
#pragma unroll 1
        for (int c = 0; c < D / 8; ++c) {
          uint32_t o[8];
          tmem_ld8(o_cols + c * 8, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st8(o_cols + c * 8, o);
        }
      }
      // P = 2^(u * scale_log2 - m) in bf16, written over S 16 keys at a time (S is all in
      // registers); each 32 keys are published as soon as they are written
      const uint64_t negm = f2_pack(-m_run, -m_run);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int k = ch * 16 + 2 * q;
          const uint64_t xy = ffma2(f2_pack(u[k], u[k + 1]), sl2x2, negm);
          pk[q] = pack_bf16x2(fast_exp2(f2_lo(xy)), fast_exp2(f2_hi(xy)));
          // the row sum takes the bf16 weights that P V uses, so O / l stays a convex
          // combination of the V rows (one dominant weight is no longer off by its rounding)
          add_bf16x2_to_f32(lsum[(2 * q) & 7], lsum[(2 * q + 1) & 7], pk[q]);
        }
        tmem_st8(s_cols + ch * 8, pk);
        if (ch & 1) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_q[ch >> 1]);
        }
      }
    }
    __nv_bfloat16 *orow = p.out + (static_cast<int64_t>(bh) * p.L + I * 128 + r) * D;
    if (!dead && t > 0 && mbar_wait_warp(o_final, 0, s_abort, p.status, p.wait_ns)) {
      tc_fence_after();
      const float inv = 1.f / (((lsum[0] + lsum[1]) + (lsum[2] + lsum[3])) +
                               ((lsum[4] + lsum[5]) + (lsum[6] + lsum[7])));
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_cols + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[q]) * inv, __uint_as_float(o[q + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[q + 2]) * inv, __uint_as_float(o[q + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[q + 4]) * inv, __uint_as_float(o[q + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[q + 6]) * inv, __uint_as_float(o[q + 7]) * inv);
          *reinterpret_cast<uint4 *>(orow + c * 32 + q) = v;
        }
      }
    } else if (!dead && t == 0) {
#pragma unroll
      for (int c = 0; c < D; c += 8)
        *reinterpret_cast<uint4 *>(orow + c) = make_uint4(0, 0, 0, 0);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
static cudaError_t launch_attn_t(const CUtensorMap &mq, const CUtensorMap &mk,
                                  const CUtensorMap &mv, const AttnParams &ap, int64_t grid,
                                  cudaStream_t stream) {
  constexpr size_t TILE = static_cast<size_t>(D / 64) * 128 * 128;
  constexpr int NSTAGE = (D == 128) ? 2 : 4;
  const size_t smem = 1024 + TILE * (1 + NSTAGE) + (2 * NSTAGE + 8) * 8 + 16;
  auto kern = bs_attn_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(grid), 256, smem, stream>>>(mq, mk, mv, ap);
  return cudaGetLastError();
}

// L2 size of the current device (queried once per device)
static int64_t l2_bytes() {
  static int64_t cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 128ll << 20;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess || v <= 0)
      v = 128 << 20;
    cache[dev] = v;
  }
  return cache[dev];
}

static bool make_map2d(CUtensorMap *map, const void *base, int64_t rows, int d) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t str[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, str, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

cudaError_t launch_sparse_attn(const Geometry &g, const void *q, const void *k, const void *v,
                               const int32_t *kept_idx, const int32_t *kept_cnt, void *out,
                               uint32_t *status, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_map2d(&mq, q, static_cast<int64_t>(g.b) * g.hq * g.L, g.d) ||
      !make_map2d(&mk, k, static_cast<int64_t>(g.b) * g.hkv * g.L, g.d) ||
      !make_map2d(&mv, v, static_cast<int64_t>(g.b) * g.hkv * g.L, g.d))
    return cudaErrorInvalidValue;
  AttnParams ap;
  ap.hq = g.hq;
  ap.hkv = g.hkv;
  ap.g = g.g;
  ap.L = g.L;
  ap.nb = g.nb;
  ap.batch = g.b;
  ap.n_units = g.b * g.hq;
  // KV-head chunks only when K and V of all heads are well beyond L2: then the chunked order
  // keeps re-read tiles in L2. Below that the plain longest-first order balances the tail better.
  const int64_t kv_bytes = static_cast<int64_t>(g.b) * g.hkv * g.L * g.d * 2 * 2;
  ap.chunk = kv_bytes > 2 * l2_bytes() ? g.g : g.hq;
  ap.tri = g.tri;
  ap.scale_log2 = g.scale * 1.4426950408889634f;
  ap.kept_idx = kept_idx;
  ap.kept_cnt = kept_cnt;
  ap.out = static_cast<__nv_bfloat16 *>(out);
  ap.status = status;
  ap.wait_ns = wait_limit_ns();
  const int64_t grid = static_cast<int64_t>(ap.n_units) * g.nb;
  if (g.d == 128) return launch_attn_t<128>(mq, mk, mv, ap, grid, stream);
  if (g.d == 64) return launch_attn_t<64>(mq, mk, mv, ap, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rra
