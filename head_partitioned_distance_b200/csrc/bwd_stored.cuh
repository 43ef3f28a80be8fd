// bwd_stored.cuh -- the dQ pass of the stored-dS backward for sm_100a.
//
// The gradient is the one bwd.cuh computes (the pages give no backward):
//   dS_ij = P_ij (dO_i.v_j - D_i),   dQ_i = scale sum_j dS_ij k_j.
// In the two-pass backward the dQ pass computes S and dP again for every tile
// pair it walks.  In the stored-dS backward the dK/dV pass, which forms
// every tile pair's dS^T for its own dK product, also writes it to a buffer
// (spa_bwd_dkdv_kernel with DS).  This pass then only contracts the stored
// tiles with K:
//   dQ(t) = scale sum_{u in key strip of t} dS(t, u) K(u)
// A stored tile is 32 KB of 8 x 8 core matrices: the 8 queries [8c, 8c + 8)
// of key k are the 16 bytes at (c * 128 + k) * 16, so a tile is, unchanged,
// the A operand dS (queries x keys) in MN-major form without swizzle: core
// matrices 128 bytes apart along the keys (K) and 2048 along the queries
// (M).  The dK/dV pass writes it that way with coalesced stores, and this
// pass copies it whole.
// Persistent grid (one CTA per SM); a unit is (b, h, query tile of 128 rows)
// walking the same key strip as the forward.  Per key tile the copy engine
// brings the stored tile (one 32 KB bulk copy) and the K tile (TMA, the B
// operand, MN-major along d) into a 3-stage ring.  8 SS MMAs of 16 keys add
// into a TMEM accumulator; the accumulator is double-buffered, so one unit's
// epilogue overlaps the next unit's products.
//
// Warp roles (192 threads): warps 0-3 epilogue (thread r = row r = TMEM lane
// r: scale * dQ as bf16 straight to global), warp 4 TMA producer, warp 5 MMA
// issuer (also owns TMEM).  Every wait is bounded (common.cuh).
#pragma once

#include "common.cuh"

namespace spa {

template <int D>
struct DqStoredCfg {
  static constexpr int BQ = 128;  // queries per unit (MMA M)
  static constexpr int BK = 128;  // keys per step
  static constexpr int NS = 3;    // ring stages
  static constexpr int DB = D / 64;
  static constexpr uint32_t DS_BYTES = BQ * BK * 2;  // one dS^T tile
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_DS = 0;
  static constexpr uint32_t OFF_K = OFF_DS + NS * DS_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_K + NS * KT_BYTES;
  static constexpr uint32_t USED_BYTES = OFF_BAR + 256;
  static constexpr uint32_t SMEM_BYTES =
      USED_BYTES + 1024 < kMaxSmemPerBlock ? USED_BYTES + 1024 : kMaxSmemPerBlock;
  static_assert(USED_BYTES <= kMaxSmemPerBlock, "stored-dS dQ tiles exceed shared memory");
  static constexpr int NTHREADS = 192;
  static constexpr uint32_t TMEM_COLS = 2 * D;  // two accumulators of D columns
};

struct DqStoredBars {
  uint64_t full[3], empty[3];
  uint64_t acc_full[2], acc_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    spa_bwd_dq_stored_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ AttnParams p) {
  using C = DqStoredCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if (!smem_fits(smem_raw, smem, C::USED_BYTES)) return;
  DqStoredBars* bars = reinterpret_cast<DqStoredBars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t N = p.N;
  const int num_units = p.B * p.units_per_batch;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bars->acc_full[b], 1);
      ptx::mbar_init(&bars->acc_free[b], 128);
    }
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) ptx::prefetch_tmap(&tm_k);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  // the unit's head, first row and key strip
  auto decode = [&](int u, int& bh, int32_t& lo, int32_t& hi, int64_t& i0, Strip& s) {
    const int b = u / p.units_per_batch;
    const int r = u % p.units_per_batch;
    const int h = head_of(p.unit_start, p.H, r);
    bh = b * p.H + h;
    lo = p.lo[h];
    hi = p.hi[h];
    i0 = (int64_t)(lo / 128 + (r - p.unit_start[h])) * 128;
    s = key_strip(N, lo, hi, i0, 128, 128);
  };

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g = 0, armed[C::NS] = {0, 0, 0};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        int bh;
        int32_t lo, hi;
        int64_t i0;
        Strip s;
        decode(u, bh, lo, hi, i0, s);
        const int t = (int)(i0 / 128);
        for (int kt = s.begin; ok && kt <= s.end; ++kt, ++g) {
          const int st = g % C::NS;
          ok = bar_wait(&bars->empty[st], ((g / C::NS) & 1) ^ 1, abort_flag);
          if (!ok) break;
          const int qa = query_strip(N, lo, hi, (int64_t)kt * 128, 128, 128).begin;
          const int slot = (int)stored_slot(p, bh / p.H, bh % p.H, kt, t, qa);
          ptx::mbar_arrive_expect_tx(&bars->full[st], C::DS_BYTES + C::KT_BYTES);
          ptx::bulk_load_1d(smem + C::OFF_DS + st * C::DS_BYTES,
                            static_cast<const uint8_t*>(p.ds) + (int64_t)slot * C::DS_BYTES, C::DS_BYTES,
                            &bars->full[st]);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_K + st * C::KT_BYTES + c * (C::BK * 128), &tm_k, &bars->full[st],
                             c * 64, kt * 128, bh);
          ++armed[st];
        }
      }
      // Exit path: every load this thread issued has landed before the CTA ends.
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) bar_drain(&bars->full[s], (armed[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // dQ (queries x d) += dS (queries x keys, MN-major core matrices) x K
      // (keys x d, MN-major: head-dim runs of 64 at 16 KB)
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, D, true, true);
      const uint32_t sDS = ptx::smem_u32(smem + C::OFF_DS), sK = ptx::smem_u32(smem + C::OFF_K);
      int g = 0, n = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x, ++n) {
        int bh;
        int32_t lo, hi;
        int64_t i0;
        Strip s;
        decode(u, bh, lo, hi, i0, s);
        const int b = n & 1;
        // the epilogue has read this accumulator's previous unit
        ok = bar_wait(&bars->acc_free[b], ((n >> 1) & 1) ^ 1, abort_flag);
        for (int kt = s.begin; ok && kt <= s.end; ++kt, ++g) {
          const int st = g % C::NS;
          ok = bar_wait(&bars->full[st], (g / C::NS) & 1, abort_flag);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint64_t da = ptx::sdesc_noswz(sDS + st * C::DS_BYTES, 128, 2048);
          const uint64_t db = ptx::sdesc_sw128(sK + st * C::KT_BYTES, C::BK * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)
            ptx::mma_bf16(tmem + (uint32_t)b * D, ptx::sdesc_advance(da, kk * 256),  // 16 keys: 2 core matrices
                          ptx::sdesc_advance(db, kk * (16 * 128)), idesc, (kt > s.begin || kk > 0) ? 1 : 0);
          ptx::mma_commit(&bars->empty[st]);
        }
        if (!ok) break;
        ptx::mma_commit(&bars->acc_full[b]);
      }
      // Exit path: every MMA this thread issued has completed.
      ptx::mma_commit(&bars->drain);
      bar_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int r = threadIdx.x;  // row of the unit = TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int n = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x, ++n) {
      int bh;
      int32_t lo, hi;
      int64_t i0;
      Strip s;
      decode(u, bh, lo, hi, i0, s);
      const int b = n & 1;
      const int64_t i = i0 + r;
      uint16_t* row = static_cast<uint16_t*>(p.dq) + ((int64_t)bh * N + i) * D;
      ok = __all_sync(0xffffffffu, bar_wait(&bars->acc_full[b], (n >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t acc[32];
        ptx::tmem_ld32(tmem + lane_base + (uint32_t)b * D + c, acc);
        ptx::tmem_wait_ld();
        ptx::reg_fence(acc);
        // (rows before the band have an all-zero dS row: dq = 0)
        if (i < N) ptx::store_row32_bf16(row + c, acc, p.scale);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->acc_free[b]);
    }
  }

  // ------------------------------------------------------------ empty blocks
  // Whole 128-row blocks that precede their head's band: dq = 0.
  {
    const int num_fill = p.B * p.fills_per_batch;
    for (int f = blockIdx.x; f < num_fill; f += gridDim.x) {
      const int b = f / p.fills_per_batch;
      const int r = f % p.fills_per_batch;
      const int h = head_of(p.fill_start, p.H, r);
      const int64_t row0 = (int64_t)(b * p.H + h) * N + (int64_t)(r - p.fill_start[h]) * 128;
      zero_rows_bf16(static_cast<uint16_t*>(p.dq) + row0 * D, 128, D);
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
