// bwd.cuh -- band-sparse attention backward for sm_100a.
//
// The pages give no backward; these kernels compute the gradient of the
// forward in fwd.cuh.  With L = sum(O * dO), P_ij = exp(scale q_i.k_j - lse_i)
// on the permitted set and 0 elsewhere:
//   D_i   = sum_c dO_ic O_ic                       (spa_bwd_delta_kernel)
//   dV_j  = sum_i P_ij dO_i
//   dK_j  = scale sum_i P_ij (dO_i.v_j - D_i) q_i  (spa_bwd_dkdv_kernel: one CTA
//                                                  per key tile, walking the
//                                                  query tiles its band reaches)
//   dQ_i  = scale sum_j P_ij (dO_i.v_j - D_i) k_j  (spa_bwd_dq_kernel: one CTA per
//                                                  query tile, walking the same
//                                                  key strip as the forward)
// Every output row is written by exactly one CTA, so there are no atomics.
// P is recomputed from lse; every contraction runs on tcgen05 with fp32
// accumulators in TMEM; the same warp roles and bounded waits as fwd.cuh.
#pragma once

#include "common.cuh"

namespace spa {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// D_i = sum_c dO_ic * O_ic (fp32), D/8 threads per row, 16-byte loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int D>
__global__ void __launch_bounds__(256) spa_bwd_delta_kernel(const uint16_t* __restrict__ o,
                                                            const uint16_t* __restrict__ dout,
                                                            float* __restrict__ delta,
                                                            int64_t rows) {
  constexpr int TPR = D / 8;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gid / TPR;
  const int part = (int)(gid % TPR);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + part);
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + part);
    acc = bf16lo(a.x) * bf16lo(g.x) + bf16hi(a.x) * bf16hi(g.x) + bf16lo(a.y) * bf16lo(g.y) +
          bf16hi(a.y) * bf16hi(g.y) + bf16lo(a.z) * bf16lo(g.z) + bf16hi(a.z) * bf16hi(g.z) +
          bf16lo(a.w) * bf16lo(g.w) + bf16hi(a.w) * bf16hi(g.w);
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) delta[row] = acc;
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (key tile of 128, h, b); query tiles of 64.
// ---------------------------------------------------------------------------
template <int D>
struct DkvCfg {
  static constexpr int BK = 128;  // keys per CTA (MMA M)
  static constexpr int BQ = 64;   // queries per step (MMA N of S^T)
  static constexpr int NS = 2;
  static constexpr int DB = D / 64;
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t QT_BYTES = BQ * D * 2;
  static constexpr uint32_t PT_BYTES = BK * BQ * 2;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + KT_BYTES;
  static constexpr uint32_t OFF_Q = OFF_V + KT_BYTES;
  static constexpr uint32_t OFF_DO = OFF_Q + NS * QT_BYTES;
  static constexpr uint32_t OFF_PT = OFF_DO + NS * QT_BYTES;
  static constexpr uint32_t OFF_DST = OFF_PT + PT_BYTES;
  static constexpr uint32_t OFF_VEC = OFF_DST + PT_BYTES;           // [NS][2][BQ] floats
  static constexpr uint32_t OFF_BAR = OFF_VEC + NS * 2 * BQ * 4;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TM_ST = 0, TM_DPT = 64, TM_DV = 128, TM_DK = 128 + D;
  static constexpr uint32_t TMEM_COLS = (128 + 2 * D <= 256) ? 256 : 512;
};

struct DkvBars {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, s_free, p_full, ds_full, dv_done, dk_done, drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    spa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                        const __grid_constant__ AttnParams p) {
  using C = DkvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  DkvBars* bars = reinterpret_cast<DkvBars*>(smem + C::OFF_BAR);
  float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC);

  const int u = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int64_t N = p.N;
  const int32_t lo = p.lo[h], hi = p.hi[h];
  const int64_t j0 = (int64_t)u * C::BK;
  const Strip strip = query_strip(N, lo, hi, j0, C::BK, C::BQ);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t rows_here = min64(j0 + C::BK, N) - j0;

  if (strip.end < strip.begin) {
    // No query reaches these keys: dk = dv = 0.
    zero_rows_bf16(static_cast<uint16_t*>(p.dk) + ((int64_t)bh * N + j0) * D, rows_here, D);
    zero_rows_bf16(static_cast<uint16_t*>(p.dv) + ((int64_t)bh * N + j0) * D, rows_here, D);
    return;
  }
  const int nq = strip.end - strip.begin + 1;

  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);
  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sDO = ptx::smem_u32(smem + C::OFF_DO);
  const uint32_t sPT = ptx::smem_u32(smem + C::OFF_PT);
  const uint32_t sDST = ptx::smem_u32(smem + C::OFF_DST);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->q_full[s], 1);
      ptx::mbar_init(&bars->q_empty[s], 1);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->s_free, 128);
    ptx::mbar_init(&bars->p_full, 128);
    ptx::mbar_init(&bars->ds_full, 128);
    ptx::mbar_init(&bars->dv_done, 1);
    ptx::mbar_init(&bars->dk_done, 1);
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(&bars->kv_full, 2 * C::KT_BYTES);
      for (int c = 0; c < C::DB; ++c) {
        ptx::tma_load_3d(smem + C::OFF_K + c * (C::BK * 128), &tm_k, &bars->kv_full, c * 64, (int)j0, bh);
        ptx::tma_load_3d(smem + C::OFF_V + c * (C::BK * 128), &tm_v, &bars->kv_full, c * 64, (int)j0, bh);
      }
    }
    int armed[2] = {0, 0};
    for (int it = 0; it < nq; ++it) {
      const int s = it % C::NS;
      const bool ok =
          __all_sync(0xffffffffu, bar_wait(&bars->q_empty[s], ((it / C::NS) & 1) ^ 1, abort_flag));
      if (!ok) break;
      const int64_t i0 = (int64_t)(strip.begin + it) * C::BQ;
      // lse (in base-2 units) and D of this step's queries, for the softmax warps
      float* vl = vec + s * 2 * C::BQ;
      float* vd = vl + C::BQ;
      for (int c = lane; c < C::BQ; c += 32) {
        const int64_t i = i0 + c;
        const bool in = i < N;
        vl[c] = in ? p.lse[(int64_t)bh * N + i] * kLog2e : 0.f;
        vd[c] = in ? p.delta[(int64_t)bh * N + i] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::QT_BYTES);
        for (int c = 0; c < C::DB; ++c) {
          ptx::tma_load_3d(smem + C::OFF_Q + s * C::QT_BYTES + c * (C::BQ * 128), &tm_q, &bars->q_full[s],
                           c * 64, (int)i0, bh);
          ptx::tma_load_3d(smem + C::OFF_DO + s * C::QT_BYTES + c * (C::BQ * 128), &tm_do,
                           &bars->q_full[s], c * 64, (int)i0, bh);
        }
      }
      armed[s]++;
    }
    if (lane == 0) {
      bar_drain(&bars->kv_full, 0);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) bar_drain(&bars->q_full[s], (armed[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BQ, false, false);
      constexpr uint32_t idesc_g = ptx::idesc_bf16_f32(128, D, false, true);
      bool ok = bar_wait(&bars->kv_full, 0, abort_flag);
      for (int it = 0; ok && it < nq; ++it) {
        const int s = it % C::NS;
        ok = bar_wait(&bars->q_full[s], (it / C::NS) & 1, abort_flag) &&
             bar_wait(&bars->s_free, (it & 1) ^ 1, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t qb = sQ + s * C::QT_BYTES, dob = sDO + s * C::QT_BYTES;
        // S^T = K Q^T and dP^T = V dO^T (both operands K-major along d)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk / 4) * (C::BK * 128) + (kk % 4) * 32;
          const uint32_t qa = (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
          ptx::mma_bf16(tmem + C::TM_ST, ptx::sdesc_sw128(sK + ka, 0, 1024),
                        ptx::sdesc_sw128(qb + qa, 0, 1024), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk / 4) * (C::BK * 128) + (kk % 4) * 32;
          const uint32_t qa = (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
          ptx::mma_bf16(tmem + C::TM_DPT, ptx::sdesc_sw128(sV + ka, 0, 1024),
                        ptx::sdesc_sw128(dob + qa, 0, 1024), idesc_s, kk > 0);
        }
        ptx::mma_commit(&bars->s_full);
        // dV += P^T dO  (P^T K-major along queries; dO MN-major along d)
        ok = bar_wait(&bars->p_full, it & 1, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          ptx::mma_bf16(tmem + C::TM_DV, ptx::sdesc_sw128(sPT + kk * 32, 0, 1024),
                        ptx::sdesc_sw128(dob + kk * (16 * 128), C::BQ * 128, 1024), idesc_g,
                        (it > 0 || kk > 0));
        ptx::mma_commit(&bars->dv_done);
        // dK += dS^T Q
        ok = bar_wait(&bars->ds_full, it & 1, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          ptx::mma_bf16(tmem + C::TM_DK, ptx::sdesc_sw128(sDST + kk * 32, 0, 1024),
                        ptx::sdesc_sw128(qb + kk * (16 * 128), C::BQ * 128, 1024), idesc_g,
                        (it > 0 || kk > 0));
        ptx::mma_commit(&bars->dk_done);
        ptx::mma_commit(&bars->q_empty[s]);
      }
      ptx::mma_commit(&bars->drain);
      bar_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;  // key row within the tile
    const int64_t j = j0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int it = 0; it < nq; ++it) {
      const int s = it % C::NS;
      ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full, it & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t st[2][32], dpt[2][32];
      ptx::tmem_ld32(tmem + lane_base + C::TM_ST, st[0]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_ST + 32, st[1]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_DPT, dpt[0]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_DPT + 32, dpt[1]);
      ptx::tmem_wait_ld();
      ptx::reg_fence(st[0]);
      ptx::reg_fence(st[1]);
      ptx::reg_fence(dpt[0]);
      ptx::reg_fence(dpt[1]);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->s_free);

      const int64_t i0 = (int64_t)(strip.begin + it) * C::BQ;
      const bool interior = tile_is_interior(N, lo, hi, i0, C::BQ, j0, C::BK);
      const float* vl = vec + s * 2 * C::BQ;
      const float* vd = vl + C::BQ;
      float pt[64];
      const int64_t dist0 = i0 - j;  // distance of the step's first query to this key
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float e = ptx::exp2_approx(__uint_as_float(st[c / 32][c % 32]) * p.scale_log2 - vl[c]);
        bool allowed = true;
        if (!interior) {
          const int64_t dd = dist0 + c;
          allowed = (dd >= lo) && (dd < hi) && (i0 + c < N) && (j < N);
        }
        pt[c] = allowed ? e : 0.f;
      }
      if (it > 0) {
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dv_done, (it - 1) & 1, abort_flag));
        if (!ok) break;
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        ptx::st_shared_v4(sPT + ptx::sw128_offset(r, ch), ptx::pack_bf16x2(pt[8 * ch], pt[8 * ch + 1]),
                          ptx::pack_bf16x2(pt[8 * ch + 2], pt[8 * ch + 3]),
                          ptx::pack_bf16x2(pt[8 * ch + 4], pt[8 * ch + 5]),
                          ptx::pack_bf16x2(pt[8 * ch + 6], pt[8 * ch + 7]));
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->p_full);
#pragma unroll
      for (int c = 0; c < 64; ++c) pt[c] = pt[c] * (__uint_as_float(dpt[c / 32][c % 32]) - vd[c]);
      if (it > 0) {
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dk_done, (it - 1) & 1, abort_flag));
        if (!ok) break;
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        ptx::st_shared_v4(sDST + ptx::sw128_offset(r, ch), ptx::pack_bf16x2(pt[8 * ch], pt[8 * ch + 1]),
                          ptx::pack_bf16x2(pt[8 * ch + 2], pt[8 * ch + 3]),
                          ptx::pack_bf16x2(pt[8 * ch + 4], pt[8 * ch + 5]),
                          ptx::pack_bf16x2(pt[8 * ch + 6], pt[8 * ch + 7]));
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->ds_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, bar_wait(&bars->dk_done, (nq - 1) & 1, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      // dV -> the K tile's smem, scale * dK -> the V tile's smem (both free now)
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_base + (which == 0 ? C::TM_DV : C::TM_DK);
        const uint32_t dst = which == 0 ? sK : sV;
        const float mul = which == 0 ? 1.f : p.scale;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t g[32];
          ptx::tmem_ld32(src + c, g);
          ptx::tmem_wait_ld();
          ptx::reg_fence(g);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = c + q * 8;
            const uint32_t addr = dst + (col / 64) * (C::BK * 128) + ptx::sw128_offset(r, (col % 64) / 8);
            const float* f = reinterpret_cast<const float*>(&g[8 * q]);
            ptx::st_shared_v4(addr, ptx::pack_bf16x2(f[0] * mul, f[1] * mul),
                              ptx::pack_bf16x2(f[2] * mul, f[3] * mul),
                              ptx::pack_bf16x2(f[4] * mul, f[5] * mul),
                              ptx::pack_bf16x2(f[6] * mul, f[7] * mul));
          }
        }
      }
      ptx::fence_proxy_async_smem();
    }
    ptx::named_bar_sync(1, 128);
    if (!*abort_flag && threadIdx.x == 0) {
      for (int c = 0; c < C::DB; ++c) {
        ptx::tma_store_3d(&tm_dv, smem + C::OFF_K + c * (C::BK * 128), c * 64, (int)j0, bh);
        ptx::tma_store_3d(&tm_dk, smem + C::OFF_V + c * (C::BK * 128), c * 64, (int)j0, bh);
      }
      ptx::bulk_commit_group();
      ptx::bulk_wait_group_all();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (query tile of 128, h, b); key tiles of 64.
// ---------------------------------------------------------------------------
template <int D>
struct DqCfg {
  static constexpr int BQ = 128;  // queries per CTA (MMA M)
  static constexpr int BK = 64;   // keys per step
  static constexpr int NS = 2;
  static constexpr int DB = D / 64;
  static constexpr uint32_t QT_BYTES = BQ * D * 2;
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t DS_BYTES = BQ * BK * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_DO = OFF_Q + QT_BYTES;
  static constexpr uint32_t OFF_K = OFF_DO + QT_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KT_BYTES;
  static constexpr uint32_t OFF_DS = OFF_V + NS * KT_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_DS + DS_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 64, TM_DQ = 128;
  static constexpr uint32_t TMEM_COLS = 256;
};

struct DqBars {
  uint64_t qdo_full;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full, s_free, ds_full, dq_done, drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    spa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ AttnParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  DqBars* bars = reinterpret_cast<DqBars*>(smem + C::OFF_BAR);

  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int64_t N = p.N;
  const int32_t lo = p.lo[h], hi = p.hi[h];
  const int64_t i0 = (int64_t)t * C::BQ;
  const Strip strip = key_strip(N, lo, hi, i0, C::BQ, C::BK);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t rows_here = min64(i0 + C::BQ, N) - i0;

  if (strip.end < strip.begin) {
    zero_rows_bf16(static_cast<uint16_t*>(p.dq) + ((int64_t)bh * N + i0) * D, rows_here, D);
    return;
  }
  const int nk = strip.end - strip.begin + 1;

  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sDO = ptx::smem_u32(smem + C::OFF_DO);
  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);
  const uint32_t sDS = ptx::smem_u32(smem + C::OFF_DS);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->qdo_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->kv_full[s], 1);
      ptx::mbar_init(&bars->kv_empty[s], 1);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->s_free, 128);
    ptx::mbar_init(&bars->ds_full, 128);
    ptx::mbar_init(&bars->dq_done, 1);
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(&bars->qdo_full, 2 * C::QT_BYTES);
      for (int c = 0; c < C::DB; ++c) {
        ptx::tma_load_3d(smem + C::OFF_Q + c * (C::BQ * 128), &tm_q, &bars->qdo_full, c * 64, (int)i0, bh);
        ptx::tma_load_3d(smem + C::OFF_DO + c * (C::BQ * 128), &tm_do, &bars->qdo_full, c * 64, (int)i0, bh);
      }
      int armed[2] = {0, 0};
      for (int it = 0; it < nk; ++it) {
        const int s = it % C::NS;
        if (!bar_wait(&bars->kv_empty[s], ((it / C::NS) & 1) ^ 1, abort_flag)) break;
        const int jt = (strip.begin + it) * C::BK;
        ptx::mbar_arrive_expect_tx(&bars->kv_full[s], 2 * C::KT_BYTES);
        for (int c = 0; c < C::DB; ++c) {
          ptx::tma_load_3d(smem + C::OFF_K + s * C::KT_BYTES + c * (C::BK * 128), &tm_k, &bars->kv_full[s],
                           c * 64, jt, bh);
          ptx::tma_load_3d(smem + C::OFF_V + s * C::KT_BYTES + c * (C::BK * 128), &tm_v, &bars->kv_full[s],
                           c * 64, jt, bh);
        }
        armed[s]++;
      }
      bar_drain(&bars->qdo_full, 0);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) bar_drain(&bars->kv_full[s], (armed[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BK, false, false);
      constexpr uint32_t idesc_g = ptx::idesc_bf16_f32(128, D, false, true);
      bool ok = bar_wait(&bars->qdo_full, 0, abort_flag);
      for (int it = 0; ok && it < nk; ++it) {
        const int s = it % C::NS;
        ok = bar_wait(&bars->kv_full[s], (it / C::NS) & 1, abort_flag) &&
             bar_wait(&bars->s_free, (it & 1) ^ 1, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t kb = sK + s * C::KT_BYTES, vb = sV + s * C::KT_BYTES;
        // S = Q K^T and dP = dO V^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qa = (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
          const uint32_t ka = (kk / 4) * (C::BK * 128) + (kk % 4) * 32;
          ptx::mma_bf16(tmem + C::TM_S, ptx::sdesc_sw128(sQ + qa, 0, 1024),
                        ptx::sdesc_sw128(kb + ka, 0, 1024), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qa = (kk / 4) * (C::BQ * 128) + (kk % 4) * 32;
          const uint32_t ka = (kk / 4) * (C::BK * 128) + (kk % 4) * 32;
          ptx::mma_bf16(tmem + C::TM_DP, ptx::sdesc_sw128(sDO + qa, 0, 1024),
                        ptx::sdesc_sw128(vb + ka, 0, 1024), idesc_s, kk > 0);
        }
        ptx::mma_commit(&bars->s_full);
        // dQ += dS K  (dS K-major along keys; K MN-major along d)
        ok = bar_wait(&bars->ds_full, it & 1, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk)
          ptx::mma_bf16(tmem + C::TM_DQ, ptx::sdesc_sw128(sDS + kk * 32, 0, 1024),
                        ptx::sdesc_sw128(kb + kk * (16 * 128), C::BK * 128, 1024), idesc_g,
                        (it > 0 || kk > 0));
        ptx::mma_commit(&bars->dq_done);
        ptx::mma_commit(&bars->kv_empty[s]);
      }
      ptx::mma_commit(&bars->drain);
      bar_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    const int r = threadIdx.x;
    const int64_t i = i0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float lse2 = (i < N) ? p.lse[(int64_t)bh * N + i] * kLog2e : 0.f;
    const float Di = (i < N) ? p.delta[(int64_t)bh * N + i] : 0.f;
    bool ok = true;
    for (int it = 0; it < nk; ++it) {
      ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full, it & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t sv[2][32], dp[2][32];
      ptx::tmem_ld32(tmem + lane_base + C::TM_S, sv[0]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_S + 32, sv[1]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_DP, dp[0]);
      ptx::tmem_ld32(tmem + lane_base + C::TM_DP + 32, dp[1]);
      ptx::tmem_wait_ld();
      ptx::reg_fence(sv[0]);
      ptx::reg_fence(sv[1]);
      ptx::reg_fence(dp[0]);
      ptx::reg_fence(dp[1]);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->s_free);

      const int64_t jt = (int64_t)(strip.begin + it) * C::BK;
      const bool interior = tile_is_interior(N, lo, hi, i0, C::BQ, jt, C::BK);
      const int64_t dist0 = i - jt;
      float ds[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float e = ptx::exp2_approx(__uint_as_float(sv[c / 32][c % 32]) * p.scale_log2 - lse2);
        bool allowed = true;
        if (!interior) {
          const int64_t dd = dist0 - c;
          allowed = (dd >= lo) && (dd < hi) && (jt + c < N) && (i < N);
        }
        const float pv = allowed ? e : 0.f;
        ds[c] = pv * (__uint_as_float(dp[c / 32][c % 32]) - Di);
      }
      if (it > 0) {
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dq_done, (it - 1) & 1, abort_flag));
        if (!ok) break;
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        ptx::st_shared_v4(sDS + ptx::sw128_offset(r, ch), ptx::pack_bf16x2(ds[8 * ch], ds[8 * ch + 1]),
                          ptx::pack_bf16x2(ds[8 * ch + 2], ds[8 * ch + 3]),
                          ptx::pack_bf16x2(ds[8 * ch + 4], ds[8 * ch + 5]),
                          ptx::pack_bf16x2(ds[8 * ch + 6], ds[8 * ch + 7]));
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->ds_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, bar_wait(&bars->dq_done, (nk - 1) & 1, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t g[32];
        ptx::tmem_ld32(tmem + lane_base + C::TM_DQ + c, g);
        ptx::tmem_wait_ld();
        ptx::reg_fence(g);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c + q * 8;
          const uint32_t addr = sQ + (col / 64) * (C::BQ * 128) + ptx::sw128_offset(r, (col % 64) / 8);
          const float* f = reinterpret_cast<const float*>(&g[8 * q]);
          const float mul = p.scale;
          ptx::st_shared_v4(addr, ptx::pack_bf16x2(f[0] * mul, f[1] * mul),
                            ptx::pack_bf16x2(f[2] * mul, f[3] * mul),
                            ptx::pack_bf16x2(f[4] * mul, f[5] * mul),
                            ptx::pack_bf16x2(f[6] * mul, f[7] * mul));
        }
      }
      ptx::fence_proxy_async_smem();
    }
    ptx::named_bar_sync(1, 128);
    if (!*abort_flag && threadIdx.x == 0) {
      for (int c = 0; c < C::DB; ++c)
        ptx::tma_store_3d(&tm_dq, smem + C::OFF_Q + c * (C::BQ * 128), c * 64, (int)i0, bh);
      ptx::bulk_commit_group();
      ptx::bulk_wait_group_all();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace spa
