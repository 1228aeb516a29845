// Causal block-sparse attention forward over the kept key blocks (RRAttention computes only
// the selected blocks; "regular block-sparse FlashAttention execution" in the RBS-Attention
// digest; online softmax as in FlashAttention / FlashAttention-2), GQA head mapping.
//
// One CTA per (batch, head, query block I), launched longest-first (I descending). Roles:
//   warp 0      TMA producer: Q tile once, then K_0, K_1, V_0, K_2, V_1, ... through a 3-stage
//               ring (the order the MMA warp consumes them in);
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into TMEM buffer j%2 (tcgen05, bf16 ->
//               fp32), then O += P_{j-1} V_{j-1} with P from shared memory, so the softmax of
//               tile j overlaps the PV product of tile j-1 and the QK product of tile j+1;
//   warp 2      TMEM allocation (S0 | S1 | O);
//   warps 4-7   softmax: one thread per query row reads its 128 logits from TMEM, applies the
//               causal mask on the diagonal block, keeps a running max (rescaling O in TMEM
//               only when the max grows by more than 2^8) and running sum, writes P as bf16
//               into the 128B-swizzled K-major layout the MMA reads, and finally normalises O
//               and stores the bf16 row.
// The kept list is read by every role with the same validity rule (0 <= J <= I, strictly
// ascending); invalid entries are skipped and flagged in the status word by the producer.
#include <math.h>

#include "common.cuh"
#include "rra_internal.h"

namespace rra {

struct AttnParams {
  int hq, hkv, g, L, nb, bhq;
  int64_t tri;
  float scale_log2;
  const int32_t *kept_idx;
  const int32_t *kept_cnt;
  __nv_bfloat16 *out;
  uint32_t *status;
};

// Clamp the stored count to the row's capacity (I + 1 entries).
__device__ __forceinline__ int row_count(const AttnParams &p, int bh, int I) {
  int cnt = p.kept_cnt[static_cast<int64_t>(bh) * p.nb + I];
  if (cnt < 0) cnt = 0;
  if (cnt > I + 1) cnt = I + 1;
  return cnt;
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    bs_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int NCHUNK = D / 64;
  constexpr uint32_t CHUNK_BYTES = 128 * 128;
  constexpr uint32_t TILE_BYTES = NCHUNK * CHUNK_BYTES;   // 128 rows x D bf16
  constexpr uint32_t P_BYTES = 2 * CHUNK_BYTES;           // 128 rows x 128 keys bf16
  constexpr int NSTAGE = 3;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, true);
  constexpr float RESCALE_THRESHOLD = 8.0f;               // log2 units

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;
  uint8_t *sRing = sQ + TILE_BYTES;
  uint8_t *sP = sRing + NSTAGE * TILE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sP + 2 * P_BYTES);
  uint64_t *q_full = bars + 0;
  uint64_t *kv_full = bars + 1;       // [NSTAGE]
  uint64_t *kv_empty = bars + 4;      // [NSTAGE]
  uint64_t *s_full = bars + 7;        // [2]
  uint64_t *p_full = bars + 9;        // [2]
  uint64_t *o_done = bars + 11;
  uint64_t *o_final = bars + 12;
  uint64_t *drain = bars + 13;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 14);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int level = blockIdx.x / p.bhq;
  const int bh = blockIdx.x - level * p.bhq;
  const int I = p.nb - 1 - level;
  const int h = bh % p.hq;
  const int b = bh / p.hq;
  const int kv = h / p.g;
  const int32_t *lst = p.kept_idx + static_cast<int64_t>(bh) * p.tri +
                       static_cast<int64_t>(I) * (I + 1) / 2;
  const int cnt = row_count(p, bh, I);

  if (grid_timed_out(p.status)) return;   // uniform across the CTA
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(s_tmem, 512);
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
  const uint32_t tmem_o = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[NSTAGE] = {0, 0, 0};
      bool q_issued = false, ok = true;
      const int qrow = bh * p.L + I * 128;
      const int kvrow = (b * p.hkv + kv) * p.L;
      auto load = [&](const CUtensorMap *map, int J) -> bool {
        if (!mbar_wait(&kv_empty[stage], phase ^ 1, s_abort, p.status)) return false;
        mbar_arrive_expect_tx(&kv_full[stage], TILE_BYTES);
        uint8_t *dst = sRing + stage * TILE_BYTES;
        for (int c = 0; c < NCHUNK; ++c)
          tma_load_2d(dst + c * CHUNK_BYTES, map, &kv_full[stage], c * 64, kvrow + J * 128);
        ++issued[stage];
        if (++stage == NSTAGE) {
          stage = 0;
          phase ^= 1;
        }
        return true;
      };
      int prev = -1, last = -1, j = 0;
      for (int e = 0; e < cnt && ok; ++e) {
        const int J = lst[e];
        if (!(J > prev && J <= I)) {
          atomicOr(p.status, kErrBadList);
          continue;
        }
        prev = J;
        if (!q_issued) {
          mbar_arrive_expect_tx(q_full, TILE_BYTES);
          for (int c = 0; c < NCHUNK; ++c)
            tma_load_2d(sQ + c * CHUNK_BYTES, &tm_q, q_full, c * 64, qrow);
          q_issued = true;
        }
        ok = load(&tm_k, J);
        if (ok && j >= 1) ok = load(&tm_v, last);
        last = J;
        ++j;
      }
      if (ok && j >= 1) ok = load(&tm_v, last);
      if (*s_abort) {
        if (q_issued) mbar_wait_drain(q_full, 0);
        for (int s = 0; s < NSTAGE; ++s)
          if (issued[s] > 0) mbar_wait_drain(&kv_full[s], (issued[s] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t p_base = smem_u32(sP);
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(&p_full[jj & 1], (jj >> 1) & 1, s_abort, p.status)) return false;
        if (!mbar_wait(&kv_full[stage], phase, s_abort, p.status)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sRing + stage * TILE_BYTES);
        const uint32_t pb = p_base + (jj & 1) * P_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc_kmajor_sw128(pb + (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32);
          const uint64_t bd = sdesc_mnmajor_sw128(v_base + kk * 2048, CHUNK_BYTES);
          mma_bf16_ss(tmem_o, a, bd, IDESC_O, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[stage]);
        mma_commit(o_done);
        if (++stage == NSTAGE) {
          stage = 0;
          phase ^= 1;
        }
        return true;
      };
      int prev = -1, j = 0;
      for (int e = 0; e < cnt && ok; ++e) {
        const int J = lst[e];
        if (!(J > prev && J <= I)) continue;
        prev = J;
        if (j == 0 && !mbar_wait(q_full, 0, s_abort, p.status)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&kv_full[stage], phase, s_abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_base = smem_u32(sRing + stage * TILE_BYTES);
        const uint32_t s_tm = tmem + (j & 1) * 128;
#pragma unroll
        for (int c = 0; c < NCHUNK; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = sdesc_kmajor_sw128(q_base + c * CHUNK_BYTES + kk * 32);
            const uint64_t bd = sdesc_kmajor_sw128(k_base + c * CHUNK_BYTES + kk * 32);
            mma_bf16_ss(s_tm, a, bd, IDESC_S, (c | kk) != 0);
          }
        mma_commit(&kv_empty[stage]);
        mma_commit(&s_full[j & 1]);
        if (++stage == NSTAGE) {
          stage = 0;
          phase ^= 1;
        }
        if (j >= 1) ok = issue_pv(j - 1);
        ++j;
      }
      if (ok && j >= 1) {
        ok = issue_pv(j - 1);
        if (ok) mma_commit(o_final);
      }
      mma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float NEG_INF = -INFINITY;
    float m_run = NEG_INF, l_run = 0.f;
    int prev = -1, j = 0;
    bool dead = false;
    for (int e = 0; e < cnt && !dead; ++e) {
      const int J = lst[e];
      if (!(J > prev && J <= I)) continue;
      prev = J;
      if (!mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1, s_abort, p.status)) {
        dead = true;
        break;
      }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tmem + lane_off + (j & 1) * 128 + c * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));
      tmem_ld_wait();
      const bool diag = (J == I);
      float tmax = NEG_INF;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = x[c] * p.scale_log2;
        if (diag && c > r) v = NEG_INF;
        x[c] = v;
        tmax = fmaxf(tmax, v);
      }
      if (j == 0) {
        m_run = tmax;
      } else if (__any_sync(0xffffffffu, tmax > m_run + RESCALE_THRESHOLD)) {
        // Warp-uniform: the TMEM accesses below are warp-collective. Lanes whose own max did
        // not move get alpha = 1.
        const float m_new = fmaxf(m_run, tmax);
        const float alpha = fast_exp2(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
        // O must be final for tile j-1 before it is rescaled (the PV of tile j waits for us).
        if (!mbar_wait_warp(o_done, (j - 1) & 1, s_abort, p.status)) {
          dead = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st32(tmem_o + lane_off + c * 32, o);
        }
        tmem_st_wait();
      }
      // P = 2^(x - m) as bf16 into the swizzled K-major tile (two 64-key chunks)
      uint8_t *prow = sP + (j & 1) * P_BYTES + r * 128;
      float lsum = 0.f;
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
        for (int piece = 0; piece < 8; ++piece) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = kc * 64 + piece * 8 + q * 2;
            const float p0 = fast_exp2(x[c] - m_run);
            const float p1 = fast_exp2(x[c + 1] - m_run);
            lsum += p0 + p1;
            w[q] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4 *>(prow + kc * CHUNK_BYTES + ((piece ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      l_run += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
      ++j;
    }
    __nv_bfloat16 *orow = p.out + (static_cast<int64_t>(bh) * p.L + I * 128 + r) * D;
    if (!dead && j > 0 && mbar_wait_warp(o_final, 0, s_abort, p.status)) {
      tc_fence_after();
      const float inv = 1.f / l_run;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + c * 32, o);
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
    } else if (j == 0) {
#pragma unroll
      for (int c = 0; c < D; c += 8)
        *reinterpret_cast<uint4 *>(orow + c) = make_uint4(0, 0, 0, 0);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_attn_t(const CUtensorMap &mq, const CUtensorMap &mk,
                                 const CUtensorMap &mv, const AttnParams &ap, int64_t grid,
                                 cudaStream_t stream) {
  constexpr size_t TILE = static_cast<size_t>(D / 64) * 128 * 128;
  const size_t smem = 1024 + TILE * (1 + 3) + 2 * 2 * 128 * 128 + 14 * 8 + 16;
  auto kern = bs_attn_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(grid), 256, smem, stream>>>(mq, mk, mv, ap);
  return cudaGetLastError();
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
  ap.bhq = g.b * g.hq;
  ap.tri = g.tri;
  ap.scale_log2 = g.scale * 1.4426950408889634f;
  ap.kept_idx = kept_idx;
  ap.kept_cnt = kept_cnt;
  ap.out = static_cast<__nv_bfloat16 *>(out);
  ap.status = status;
  const int64_t grid = static_cast<int64_t>(ap.bhq) * g.nb;
  if (g.d == 128) return launch_attn_t<128>(mq, mk, mv, ap, grid, stream);
  if (g.d == 64) return launch_attn_t<64>(mq, mk, mv, ap, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rra
