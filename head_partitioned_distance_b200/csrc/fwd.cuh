// fwd.cuh -- band-sparse attention forward for sm_100a.
//
// One CTA per unit (b, h, query tile of 128 rows).  The unit walks the
// diagonal strip of 128-key tiles its band needs (sched.cuh), flash style:
//   S = Q K^T         tcgen05.mma, bf16 x bf16 -> fp32 in TMEM (double-buffered)
//   P = exp(S - m)    softmax warps, one thread per row, fp32 online softmax,
//                     per-element distance predicate on edge tiles only
//   O += P V          tcgen05.mma, P as bf16 from 128B-swizzled shared memory
// then O / l -> bf16 through shared memory and a TMA store; lse = m + ln l.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (thread r owns row
// r, which is TMEM lane r), warp 4 TMA producer, warp 5 MMA issuer and TMEM
// owner.  K/V tiles stream through a 2-stage ring; every wait is bounded.
//
// Softmax restricted to a permitted set: "Story of Attention -- Part 4",
// section 1 (Sparse-Attention equation); bands: "Making Every Head Count",
// Figure 1 caption.
#pragma once

#include "common.cuh"

namespace spa {

template <int D>
struct FwdCfg {
  static constexpr int BQ = 128;
  static constexpr int BK = 128;
  static constexpr int NS = 2;         // K/V ring stages
  static constexpr int DB = D / 64;    // 64-column (128-byte) blocks per row
  static constexpr uint32_t Q_BYTES = BQ * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr uint32_t P_BYTES = BQ * BK * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
  // + alignment slack; at least 116 KB so that one CTA (and its 512 TMEM
  // columns) owns an SM even for d = 64
  static constexpr uint32_t SMEM_BYTES =
      (OFF_BAR + 256 + 1024) > 116u * 1024 ? (OFF_BAR + 256 + 1024) : 116u * 1024;
  static constexpr int NTHREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;
  static_assert(D == 64 || D == 128, "head dim");
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, o_done, drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    spa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ AttnParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::OFF_BAR);

  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int64_t N = p.N;
  const int32_t lo = p.lo[h], hi = p.hi[h];
  const int64_t i0 = (int64_t)t * C::BQ;
  const Strip strip = key_strip(N, lo, hi, i0, C::BQ, C::BK);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t rows_here = min64(i0 + C::BQ, N) - i0;

  if (strip.end < strip.begin) {
    // No row of this tile reaches its band: o = 0, lse = -inf.
    zero_rows_bf16(static_cast<uint16_t*>(p.o) + ((int64_t)bh * N + i0) * D, rows_here, D);
    for (int r = threadIdx.x; r < rows_here; r += blockDim.x) p.lse[(int64_t)bh * N + i0 + r] = -INFINITY;
    return;
  }
  const int nkt = strip.end - strip.begin + 1;

  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);
  const uint32_t sP = ptx::smem_u32(smem + C::OFF_P);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->k_full[s], 1);
      ptx::mbar_init(&bars->v_full[s], 1);
      ptx::mbar_init(&bars->kv_empty[s], 1);
      ptx::mbar_init(&bars->s_full[s], 1);
      ptx::mbar_init(&bars->s_free[s], 128);
    }
    ptx::mbar_init(&bars->p_full, 128);
    ptx::mbar_init(&bars->o_done, 1);
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_o);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      for (int c = 0; c < C::DB; ++c)
        ptx::tma_load_3d(smem + C::OFF_Q + c * (C::BQ * 128), &tm_q, &bars->q_full, c * 64, (int)i0, bh);
      int armed[2] = {0, 0};
      for (int it = 0; it < nkt; ++it) {
        const int s = it % C::NS;
        const uint32_t n = it / C::NS;
        if (!bar_wait(&bars->kv_empty[s], (n & 1) ^ 1, abort_flag)) break;
        const int j0 = (strip.begin + it) * C::BK;
        uint8_t* kdst = smem + C::OFF_K + s * C::KV_BYTES;
        uint8_t* vdst = smem + C::OFF_V + s * C::KV_BYTES;
        ptx::mbar_arrive_expect_tx(&bars->k_full[s], C::KV_BYTES);
        for (int c = 0; c < C::DB; ++c)
          ptx::tma_load_3d(kdst + c * (C::BK * 128), &tm_k, &bars->k_full[s], c * 64, j0, bh);
        ptx::mbar_arrive_expect_tx(&bars->v_full[s], C::KV_BYTES);
        for (int c = 0; c < C::DB; ++c)
          ptx::tma_load_3d(vdst + c * (C::BK * 128), &tm_v, &bars->v_full[s], c * 64, j0, bh);
        armed[s]++;
      }
      // Exit path: every load this thread issued has landed before the CTA ends.
      bar_drain(&bars->q_full, 0);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) {
          bar_drain(&bars->k_full[s], (armed[s] - 1) & 1);
          bar_drain(&bars->v_full[s], (armed[s] - 1) & 1);
        }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BK, false, false);
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(128, D, false, true);
      bool ok = bar_wait(&bars->q_full, 0, abort_flag);
      for (int it = 0; ok && it <= nkt; ++it) {
        if (it < nkt) {
          const int s = it % C::NS, sb = it & 1;
          ok = bar_wait(&bars->k_full[s], (it / C::NS) & 1, abort_flag) &&
               bar_wait(&bars->s_free[sb], ((it >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t dS = tmem + (sb ? C::TM_S1 : C::TM_S0);
          const uint32_t kbase = sK + s * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t a = sQ + (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
            const uint32_t bb = kbase + (kk / 4) * (C::BK * 128) + (kk % 4) * 32;
            ptx::mma_bf16(dS, ptx::sdesc_sw128(a, 0, 1024), ptx::sdesc_sw128(bb, 0, 1024), idesc_s,
                          kk > 0);
          }
          ptx::mma_commit(&bars->s_full[sb]);
        }
        if (it >= 1) {
          const int pit = it - 1, s = pit % C::NS;
          ok = bar_wait(&bars->p_full, pit & 1, abort_flag) &&
               bar_wait(&bars->v_full[s], (pit / C::NS) & 1, abort_flag);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t vbase = sV + s * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint32_t a = sP + (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
            const uint32_t bb = vbase + kk * (16 * 128);
            ptx::mma_bf16(tmem + C::TM_O, ptx::sdesc_sw128(a, 0, 1024),
                          ptx::sdesc_sw128(bb, C::BK * 128, 1024), idesc_o, (pit > 0 || kk > 0));
          }
          ptx::mma_commit(&bars->o_done);
          ptx::mma_commit(&bars->kv_empty[s]);
        }
      }
      // Exit path: every MMA this thread issued has completed.
      ptx::mma_commit(&bars->drain);
      bar_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;
    const int64_t i = i0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < nkt; ++it) {
      const int sb = it & 1;
      ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full[sb], (it >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t sr[4][32];
      const uint32_t taddr = tmem + lane_base + (sb ? C::TM_S1 : C::TM_S0);
#pragma unroll
      for (int q = 0; q < 4; ++q) ptx::tmem_ld32(taddr + q * 32, sr[q]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) ptx::reg_fence(sr[q]);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->s_free[sb]);

      const int64_t j0 = (int64_t)(strip.begin + it) * C::BK;
      const bool interior = tile_is_interior(N, lo, hi, i0, C::BQ, j0, C::BK);
      float x[128];
      float tmax = -INFINITY;
      const int64_t dist0 = i - j0;  // distance to the tile's first key
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = __uint_as_float(sr[c / 32][c % 32]) * p.scale_log2;
        if (!interior) {
          const int64_t dd = dist0 - c;
          const bool allowed = (dd >= lo) && (dd < hi) && (j0 + c < N) && (i < N);
          v = allowed ? v : -INFINITY;
        }
        x[c] = v;
        tmax = fmaxf(tmax, v);
      }
      const float m_new = fmaxf(m, tmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ptx::exp2_approx(m - m_use);  // 0 while the row has seen nothing

      if (it > 0) {
        // PV(it-1) must be complete before O is rescaled and P is overwritten.
        ok = __all_sync(0xffffffffu, bar_wait(&bars->o_done, (it - 1) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        const bool need = (m_new > m) && (m != -INFINITY);
        if (__any_sync(0xffffffffu, need)) {
          const float a = need ? alpha : 1.f;
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            ptx::tmem_ld32(tmem + lane_base + C::TM_O + c, o);
            ptx::tmem_wait_ld();
            ptx::reg_fence(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
            ptx::tmem_st32(tmem + lane_base + C::TM_O + c, o);
          }
          ptx::tmem_wait_st();
        }
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        x[c] = ptx::exp2_approx(x[c] - m_use);
        rs += x[c];
      }
      l = l * alpha + rs;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint32_t addr = sP + (ch / 8) * (C::BQ * 128) + ptx::sw128_offset(r, ch % 8);
        ptx::st_shared_v4(addr, ptx::pack_bf16x2(x[8 * ch + 0], x[8 * ch + 1]),
                          ptx::pack_bf16x2(x[8 * ch + 2], x[8 * ch + 3]),
                          ptx::pack_bf16x2(x[8 * ch + 4], x[8 * ch + 5]),
                          ptx::pack_bf16x2(x[8 * ch + 6], x[8 * ch + 7]));
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->p_full);
      m = m_new;
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, bar_wait(&bars->o_done, (nkt - 1) & 1, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        ptx::tmem_ld32(tmem + lane_base + C::TM_O + c, o);
        ptx::tmem_wait_ld();
        ptx::reg_fence(o);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c + q * 8;
          const uint32_t addr = sQ + (col / 64) * (C::BQ * 128) + ptx::sw128_offset(r, (col % 64) / 8);
          const float* f = reinterpret_cast<const float*>(&o[8 * q]);
          ptx::st_shared_v4(addr, ptx::pack_bf16x2(f[0] * inv, f[1] * inv),
                            ptx::pack_bf16x2(f[2] * inv, f[3] * inv),
                            ptx::pack_bf16x2(f[4] * inv, f[5] * inv),
                            ptx::pack_bf16x2(f[6] * inv, f[7] * inv));
        }
      }
      ptx::fence_proxy_async_smem();
    }
    ptx::named_bar_sync(1, 128);
    const bool all_ok = !*abort_flag;
    if (all_ok && threadIdx.x == 0) {
      for (int c = 0; c < C::DB; ++c)
        ptx::tma_store_3d(&tm_o, smem + C::OFF_Q + c * (C::BQ * 128), c * 64, (int)i0, bh);
      ptx::bulk_commit_group();
      ptx::bulk_wait_group_all();
    }
    if (all_ok && i < N)
      p.lse[(int64_t)bh * N + i] = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace spa
