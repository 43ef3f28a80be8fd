// bwd_fused.cuh -- band-sparse attention backward in one pass over the key
// tiles (sm_100a): dK and dV accumulate in tensor memory as in the dK/dV pass
// of bwd.cuh, and dQ is produced in the same pass, one query tile at a time,
// and summed over the key tiles in an fp32 buffer by reduction operations --
// so S and dP are computed once per tile pair instead of once in each of two
// passes.  The gradient is the one of bwd.cuh:
//   P_ij = exp(scale q_i.k_j - lse_i) on the permitted set, 0 elsewhere,
//   dS_ij = P_ij (dO_i.v_j - D_i),  D_i = sum_c dO_ic O_ic,
//   dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,
//   dQ_i = scale sum_j dS_ij k_j.
// Three launches: spa_bwd_fused_prep_kernel (D, a zeroed fp32 dQ buffer over
// the query tiles some band reaches, zero dq rows before them), the fused
// pass, and spa_bwd_dq_convert_kernel (dq = bf16(scale * buffer)).  The sums
// of dQ are taken in whatever order the reductions arrive, so dq is not
// bit-reproducible from run to run (dk and dv are).
//
// Per unit (b, h, 128 keys), per query tile g of its strip:
//   S^T  = K Q^T      SS MMA -> TMEM [0, 128)              (warp 10)
//   dP^T = V dO^T     SS MMA -> TMEM [128, 256)            (warp 9)
//   element-wise warpgroups: P^T = exp2(S^T c - lse2) (masked on edge
//     tiles), dS^T = P^T (dP^T - D); once both warpgroups hold their dP^T
//     columns in registers, P^T goes as bf16 pairs to TMEM [128, 192) and
//     dS^T as bf16 to shared memory ([2 query halves][128 keys][128 B],
//     128-byte swizzle), which is at once the K-major A operand of dK
//     (rows = keys) and the MN-major A operand of dQ (runs of 64 queries)
//   dQ_p = dS K_p     SS MMA, 64 head dims at a time -> TMEM [192, 256)
//                     (warp 9), drained by the warpgroups into the buffer
//   dV  += P^T dO     TS MMA (A = P^T from TMEM)  -> TMEM [256, 384)  (warp 11)
//   dK  += dS^T Q     SS MMA (A = dS^T from smem) -> TMEM [384, 512)  (warp 9)
// Warp 9 issues, per tile: dQ_0 and dK (for d = 64, whose dQ is one piece,
// dK before dQ_0's commit, so that the piece's completion covers every read
// of dS^T), then -- once the warpgroups hold dQ_0 -- dQ_1 (d = 128), then --
// once dV has read P^T and the last piece is drained -- dP^T of the next
// tile.  The epilogue writes dK and dV exactly as the dK/dV pass does, staged
// in the same shared tile that carries dS^T.
//
// Measured on B200 this pass is slower than the two-pass backward it
// replaces: the reductions of the dQ pieces (per thread, 32 rows x 16 bytes
// per warp instruction) occupy the SM's memory-instruction path long enough
// to delay the barrier arrivals and MMA issues queued behind them.
#pragma once

#include "bwd.cuh"

namespace spa {

template <int D>
struct FusedCfg {
  static constexpr int BK = 128;  // keys per unit (MMA M of S^T, dP^T, dV, dK)
  static constexpr int BQ = 128;  // queries per step (MMA M of dQ)
  static constexpr int NS = 2;    // Q/dO ring stages
  static constexpr int DB = D / 64;
  static constexpr int NPIECE = D / 64;  // 64-column pieces of a dQ tile
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t QT_BYTES = BQ * D * 2;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + KT_BYTES;
  static constexpr uint32_t OFF_Q = OFF_V + KT_BYTES;
  static constexpr uint32_t OFF_DO = OFF_Q + NS * QT_BYTES;
  // dS^T of the current tile; at a unit's end the staging of dV and dK
  static constexpr uint32_t OFF_P = OFF_DO + NS * QT_BYTES;
  static constexpr uint32_t PT_BYTES = BK * 128 * 2;
  static constexpr uint32_t OFF_VEC = OFF_P + PT_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_VEC + 2 * 2 * 128 * 4;
  static constexpr uint32_t USED_BYTES = OFF_BAR + 256;
  static constexpr uint32_t SMEM_BYTES =
      USED_BYTES + 1024 < kMaxSmemPerBlock ? USED_BYTES + 1024 : kMaxSmemPerBlock;
  static_assert(USED_BYTES <= kMaxSmemPerBlock, "fused backward tiles exceed shared memory");
  static constexpr int NTHREADS = 384;
  static constexpr uint32_t LAUNCH_REGS = 168, EW_REGS = 192, CONTROL_REGS = 120;
  static_assert(2 * EW_REGS + CONTROL_REGS <= 3 * LAUNCH_REGS, "register split over budget");
  static constexpr uint32_t TM_ST = 0, TM_B = 128, TM_PT = 128, TM_DQ = 192, TM_DV = 256, TM_DK = 384;
  static constexpr uint32_t TMEM_COLS = 512;
};

struct FusedBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, s_free, dp_full, p_full, ds_full;
  uint64_t pt_read;   // dV of a tile has read its P^T
  uint64_t dq_full;   // a dQ piece is in TMEM
  uint64_t dq_free;   // the warpgroups hold the last dQ piece in registers
  uint64_t ew_sync;   // both warpgroups hold their dP^T columns in registers
  uint64_t vec_full[2], vec_empty[2];
  uint64_t acc_done, acc_free, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void red_add_v4(float* addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

// First row of the query tiles that head (lo) reaches: 128 floor(lo / 128).
__device__ __forceinline__ int64_t reached_row0(int32_t lo) { return (int64_t)(lo / 128) * 128; }

// D_i = dO_i . O_i and a zeroed fp32 dQ buffer row for every row of the query
// tiles some band reaches; dq = 0 for the rows before them (no key tile adds
// to those).  D / 8 threads per row (16 bytes of o and dO each), grid-stride.
template <int D>
__global__ void __launch_bounds__(256) spa_bwd_fused_prep_kernel(const __grid_constant__ AttnParams p) {
  constexpr int TPR = D / 8;
  const int64_t rows = (int64_t)p.B * p.H * p.N;
  const int64_t total = rows * TPR;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride) {
    const int64_t t = base + threadIdx.x;
    const bool valid = t < total;
    const int64_t row = t / TPR;
    const int part = (int)(t % TPR);
    float acc = 0.f;
    bool reached = false;
    if (valid) {
      const int64_t i = row % p.N;
      const int h = (int)((row / p.N) % p.H);
      reached = i >= reached_row0(p.lo[h]);
      if (reached) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.o_in) + row * D) + part);
        const uint4 g = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dout) + row * D) + part);
        acc = bf16lo(a.x) * bf16lo(g.x) + bf16hi(a.x) * bf16hi(g.x) + bf16lo(a.y) * bf16lo(g.y) +
              bf16hi(a.y) * bf16hi(g.y) + bf16lo(a.z) * bf16lo(g.z) + bf16hi(a.z) * bf16hi(g.z) +
              bf16lo(a.w) * bf16lo(g.w) + bf16hi(a.w) * bf16hi(g.w);
        float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D) + 2 * part;
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dq) + row * D)[part] = make_uint4(0, 0, 0, 0);
      }
    }
    // the lanes of one row are in one warp (TPR divides 32) and every lane of
    // the warp takes the same number of rounds
#pragma unroll
    for (int off = TPR / 2; off > 0; off /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (valid && reached && part == 0) p.delta[row] = acc;
  }
}

// dq = bf16(scale * buffer) over the rows of the reached query tiles.
template <int D>
__global__ void __launch_bounds__(256) spa_bwd_dq_convert_kernel(const __grid_constant__ AttnParams p) {
  constexpr int TPR = D / 8;  // 8 values (32 bytes of fp32, 16 of bf16) per thread
  const int64_t rows = (int64_t)p.B * p.H * p.N;
  const int64_t total = rows * TPR;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / TPR;
    const int part = (int)(t % TPR);
    const int64_t i = row % p.N;
    const int h = (int)((row / p.N) % p.H);
    if (i < reached_row0(p.lo[h])) continue;
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc + row * D) + 2 * part;
    const float4 a = __ldcs(src), b = __ldcs(src + 1);
    const float s = p.scale;
    reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dq) + row * D)[part] =
        make_uint4(ptx::pack_bf16x2(a.x * s, a.y * s), ptx::pack_bf16x2(a.z * s, a.w * s),
                   ptx::pack_bf16x2(b.x * s, b.y * s), ptx::pack_bf16x2(b.z * s, b.w * s));
  }
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    spa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                         const __grid_constant__ AttnParams p) {
  using C = FusedCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if (!smem_fits(smem_raw, smem, C::USED_BYTES)) return;
  FusedBars* bars = reinterpret_cast<FusedBars*>(smem + C::OFF_BAR);
  float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t N = p.N;
  const int num_units = p.B * p.units_per_batch;

  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);
  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sDO = ptx::smem_u32(smem + C::OFF_DO);
  const uint32_t sP = ptx::smem_u32(smem + C::OFF_P);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->kv_full, 1);
    ptx::mbar_init(&bars->kv_empty, 2);  // warp 10 (last S^T) and warp 9 (last dQ piece)
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->q_full[s], 1);
      ptx::mbar_init(&bars->q_empty[s], 3);  // one commit from each MMA issuer
      ptx::mbar_init(&bars->vec_full[s], 1);
      ptx::mbar_init(&bars->vec_empty[s], 256);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->s_free, 256);
    ptx::mbar_init(&bars->dp_full, 1);
    ptx::mbar_init(&bars->p_full, 256);
    ptx::mbar_init(&bars->ds_full, 256);
    ptx::mbar_init(&bars->pt_read, 1);
    ptx::mbar_init(&bars->dq_full, 1);
    ptx::mbar_init(&bars->dq_free, 256);
    ptx::mbar_init(&bars->ew_sync, 256);
    ptx::mbar_init(&bars->acc_done, 2);  // dK (warp 9) and dV (warp 11)
    ptx::mbar_init(&bars->acc_free, 256);
    ptx::mbar_init(&bars->drain, 3);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp >= 8) {
    ptx::regs_dec<C::CONTROL_REGS>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer warp
    // Lane 0 issues the tile copies; all lanes load the query tiles' lse and D
    // into the shared vector ring.
    int nkv = 0, gq = 0, armed[2] = {0, 0};
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const DkvUnit U = dkv_decode(u, p);
      ok = __all_sync(0xffffffffu, bar_wait(&bars->kv_empty, (nkv & 1) ^ 1, abort_flag));
      if (!ok) break;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&bars->kv_full, 2 * C::KT_BYTES);
        for (int c = 0; c < C::DB; ++c) {
          ptx::tma_load_3d(smem + C::OFF_K + c * (C::BK * 128), &tm_k, &bars->kv_full, c * 64, (int)U.j0, U.bh);
          ptx::tma_load_3d(smem + C::OFF_V + c * (C::BK * 128), &tm_v, &bars->kv_full, c * 64, (int)U.j0, U.bh);
        }
      }
      ++nkv;
      for (int qt = U.qa; qt <= U.qb; ++qt, ++gq) {
        const int s = gq % C::NS;
        ok = __all_sync(0xffffffffu, bar_wait(&bars->q_empty[s], ((gq / C::NS) & 1) ^ 1, abort_flag));
        if (!ok) break;
        const int64_t i0 = (int64_t)qt * C::BQ;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::QT_BYTES);
          for (int c = 0; c < C::DB; ++c) {
            ptx::tma_load_3d(smem + C::OFF_Q + s * C::QT_BYTES + c * (C::BQ * 128), &tm_q, &bars->q_full[s],
                             c * 64, (int)i0, U.bh);
            ptx::tma_load_3d(smem + C::OFF_DO + s * C::QT_BYTES + c * (C::BQ * 128), &tm_do,
                             &bars->q_full[s], c * 64, (int)i0, U.bh);
          }
        }
        ++armed[s];
        ok = __all_sync(0xffffffffu, bar_wait(&bars->vec_empty[s], ((gq / C::NS) & 1) ^ 1, abort_flag));
        if (!ok) break;
        float* vs = vec + s * 256;
        const float* lrow = p.lse + (int64_t)U.bh * N;
        const float* drow = p.delta + (int64_t)U.bh * N;
        float lv[4], dv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t i = i0 + lane + 32 * e;
          lv[e] = i < N ? lrow[i] : 0.f;
          dv[e] = i < N ? drow[i] : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          vs[lane + 32 * e] = -lv[e] * kLog2e;
          vs[128 + lane + 32 * e] = -dv[e];
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->vec_full[s]);
      }
    }
    if (lane == 0) {
      if (nkv > 0) bar_drain(&bars->kv_full, (nkv - 1) & 1);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) bar_drain(&bars->q_full[s], (armed[s] - 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BQ, false, false);
      constexpr uint32_t idesc_g = ptx::idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc_dk = ptx::idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc_dq = ptx::idesc_bf16_f32(128, 64, true, true);
      int nkv = 0, gq = 0;
      bool ok = true;
      auto qstage = [&](int g) { return g % C::NS; };
      auto qphase = [&](int g) { return (uint32_t)((g / C::NS) & 1); };
      const uint64_t dK = ptx::sdesc_sw128(sK, 0, 1024), dV = ptx::sdesc_sw128(sV, 0, 1024);
      // K-major (B of S^T/dP^T) and MN-major (B of dK/dV) views of both Q/dO stages
      const uint64_t dQk0 = ptx::sdesc_sw128(sQ, 0, 1024), dQk1 = ptx::sdesc_sw128(sQ + C::QT_BYTES, 0, 1024);
      const uint64_t dOk0 = ptx::sdesc_sw128(sDO, 0, 1024), dOk1 = ptx::sdesc_sw128(sDO + C::QT_BYTES, 0, 1024);
      const uint64_t dQm0 = ptx::sdesc_sw128(sQ, C::BQ * 128, 1024);
      const uint64_t dQm1 = ptx::sdesc_sw128(sQ + C::QT_BYTES, C::BQ * 128, 1024);
      const uint64_t dOm0 = ptx::sdesc_sw128(sDO, C::BQ * 128, 1024);
      const uint64_t dOm1 = ptx::sdesc_sw128(sDO + C::QT_BYTES, C::BQ * 128, 1024);
      // dS^T: K-major A of dK (rows = keys, 64-query blocks 16 KB apart) and
      // MN-major A of dQ (runs of 64 queries, the two runs 16 KB apart)
      const uint64_t dSk = ptx::sdesc_sw128(sP, 0, 1024);
      const uint64_t dSm = ptx::sdesc_sw128(sP, C::BK * 128, 1024);
      // K as the MN-major B of dQ: piece p is the 64-column block p
      const uint64_t dKm = ptx::sdesc_sw128(sK, C::BK * 128, 1024);
      auto dQk = [&](int st) { return st ? dQk1 : dQk0; };
      auto dOk = [&](int st) { return st ? dOk1 : dOk0; };
      auto dQm = [&](int st) { return st ? dQm1 : dQm0; };
      auto dOm = [&](int st) { return st ? dOm1 : dOm0; };
      auto issue_nt = [&](uint32_t dst, uint64_t da, uint64_t db) {  // dst = A (keys) x B^T (queries)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_bf16(tmem + dst, ptx::sdesc_advance(da, (kk / 4) * (C::BK * 128) + (kk % 4) * 32),
                        ptx::sdesc_advance(db, (kk / 4) * (C::BQ * 128) + (kk % 4) * 32), idesc_s, kk > 0);
      };
      if (warp == 10) {
        // ---- S^T of each query tile, as soon as the warpgroups hold the last one
        int cf = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DkvUnit U = dkv_decode(u, p);
          const int nq = U.qb - U.qa + 1;
          const int g0 = gq;
          for (int j = 0; ok && j < nq; ++j) {
            const int g = g0 + j;
            if (g > 0) ok = bar_wait(&bars->s_free, (cf++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->kv_full, (nkv++) & 1, abort_flag);
            if (ok) ok = bar_wait(&bars->q_full[qstage(g)], qphase(g), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_nt(C::TM_ST, dK, dQk(qstage(g)));
            ptx::mma_commit(&bars->s_full);
            ptx::mma_commit(&bars->q_empty[qstage(g)]);
            if (j + 1 == nq) ptx::mma_commit(&bars->kv_empty);  // K's last S^T
          }
          gq = g0 + nq;
        }
      } else if (warp == 11) {
        // ---- dV of each query tile, as soon as its P^T is in TMEM
        int cp = 0, cacc = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DkvUnit U = dkv_decode(u, p);
          const int nq = U.qb - U.qa + 1;
          const int g0 = gq;
          for (int j = 0; ok && j < nq; ++j) {
            const int g = g0 + j;
            ok = bar_wait(&bars->p_full, (cp++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->acc_free, ((cacc & 1) ^ 1), abort_flag);
            if (ok) ok = bar_wait(&bars->q_full[qstage(g)], qphase(g), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            // dV += P^T dO: A = P^T, 128 queries as bf16 pairs in 64 columns
#pragma unroll
            for (int kk = 0; kk < C::BQ / 16; ++kk)
              ptx::mma_bf16_ts(tmem + C::TM_DV, tmem + C::TM_PT + kk * 8,
                               ptx::sdesc_advance(dOm(qstage(g)), kk * (16 * 128)), idesc_g, (j > 0 || kk > 0));
            ptx::mma_commit(&bars->pt_read);
            ptx::mma_commit(&bars->q_empty[qstage(g)]);
          }
          if (!ok) break;
          ++cacc;
          ptx::mma_commit(&bars->acc_done);
          gq = g0 + nq;
        }
      } else {
        // ---- dQ pieces and dK of each query tile, dP^T of the next
        int cds = 0, cacc = 0, cpt = 0, cfree = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DkvUnit U = dkv_decode(u, p);
          const int nq = U.qb - U.qa + 1;
          const int g0 = gq;
          // dP^T of tile g overwrites P^T and the last dQ piece of tile g - 1
          ok = bar_wait(&bars->kv_full, (nkv++) & 1, abort_flag) &&
               bar_wait(&bars->q_full[qstage(g0)], qphase(g0), abort_flag) &&
               (g0 == 0 || (bar_wait(&bars->pt_read, (cpt++) & 1, abort_flag) &&
                            bar_wait(&bars->dq_free, (cfree++) & 1, abort_flag)));
          if (!ok) break;
          ptx::tc_fence_after();
          issue_nt(C::TM_B, dV, dOk(qstage(g0)));
          ptx::mma_commit(&bars->dp_full);
          for (int j = 0; j < nq; ++j) {
            const int g = g0 + j;
            ok = bar_wait(&bars->ds_full, (cds++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->acc_free, ((cacc & 1) ^ 1), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            for (int pc = 0; ok && pc < C::NPIECE; ++pc) {
              if (pc > 0) {
                // the piece before is in the warpgroups' registers
                ok = bar_wait(&bars->dq_free, (cfree++) & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
              }
              // dQ_p = dS K_p: A = dS (MN-major), B = K columns [64 p, 64 p + 64) (MN-major)
#pragma unroll
              for (int kk = 0; kk < C::BK / 16; ++kk)
                ptx::mma_bf16(tmem + C::TM_DQ, ptx::sdesc_advance(dSm, kk * (16 * 128)),
                              ptx::sdesc_advance(dKm, pc * (C::BK * 128) + kk * (16 * 128)), idesc_dq, kk > 0);
              // dK += dS^T Q (A = dS^T K-major, B = Q MN-major) right after the
              // first piece; the commit of the last piece then also covers dK,
              // so once the warpgroups hold that piece nothing reads dS^T
              auto issue_dk = [&]() {
#pragma unroll
                for (int kk = 0; kk < C::BQ / 16; ++kk)
                  ptx::mma_bf16(tmem + C::TM_DK, ptx::sdesc_advance(dSk, (kk / 4) * (C::BK * 128) + (kk % 4) * 32),
                                ptx::sdesc_advance(dQm(qstage(g)), kk * (16 * 128)), idesc_dk, (j > 0 || kk > 0));
                ptx::mma_commit(&bars->q_empty[qstage(g)]);
              };
              if (pc == 0 && C::NPIECE == 1) issue_dk();
              ptx::mma_commit(&bars->dq_full);
              if (pc == 0 && C::NPIECE > 1) issue_dk();
            }
            if (!ok) break;
            if (j + 1 < nq) {
              ok = bar_wait(&bars->q_full[qstage(g + 1)], qphase(g + 1), abort_flag) &&
                   bar_wait(&bars->pt_read, (cpt++) & 1, abort_flag) &&
                   bar_wait(&bars->dq_free, (cfree++) & 1, abort_flag);
              if (!ok) break;
              ptx::tc_fence_after();
              issue_nt(C::TM_B, dV, dOk(qstage(g + 1)));  // dP^T of the next tile
              ptx::mma_commit(&bars->dp_full);
            }
          }
          if (!ok) break;
          ++cacc;
          ptx::mma_commit(&bars->acc_done);
          ptx::mma_commit(&bars->kv_empty);  // V's last dP^T and K's last dQ piece
          gq = g0 + nq;
        }
      }
      ptx::mma_commit(&bars->drain);
      bar_drain(&bars->drain, 0);
    }
    __syncwarp();
  }
  } else {
    ptx::regs_inc<C::EW_REGS>();
    // ------------------------------------------------------------ element-wise warpgroups
    const int w = warp / 4;                  // query columns [64w, 64w+64)
    const int wq = warp % 4;
    const int r = threadIdx.x - 128 * w;     // key row (S^T, dP^T) / query row (dQ) = TMEM lane
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::TM_ST + 64 * w;
    const uint32_t tDP = tmem + lane_base + C::TM_B + 64 * w;
    const uint32_t tPT = tmem + lane_base + C::TM_PT + 32 * w;
    const uint32_t tDQ = tmem + lane_base + C::TM_DQ + 32 * w;
    // row r of dS^T block w (128 bytes, 128-byte swizzle)
    const uint32_t ds_row = sP + (uint32_t)w * (C::BK * 128) + (uint32_t)r * 128;
    const float c2 = p.scale_log2;
    int gq = 0, cs = 0, cdp = 0, cdq = 0, cew = 0, cacc = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const DkvUnit U = dkv_decode(u, p);
      const int64_t j = U.j0 + r;
      bool first_step = true;
      for (int qt = U.qa; qt <= U.qb; ++qt, ++gq) {
        const int64_t i0 = (int64_t)qt * C::BQ;
        const bool interior = tile_is_interior(N, U.lo, U.hi, i0, C::BQ, U.j0, C::BK);
        int qlo = 0;
        uint32_t span = 127;
        if (!interior) {
          const int64_t q_first = max64(j + U.lo - i0, 0);
          const int64_t q_last = min64(min64(j + U.hi - 1 - i0, N - 1 - i0), 127);
          if (j >= N || q_last < q_first) {
            qlo = 128;
            span = 0;
          } else {
            qlo = (int)q_first;
            span = (uint32_t)(q_last - q_first);
          }
        }
        const float* vl = vec + (gq % C::NS) * 256 + 64 * w;
        const float* vd = vl + 128;
        const int cb = 64 * w - qlo;
        // ---- P^T = exp2(S^T c - lse2)
        ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full, (cs++) & 1, abort_flag) &&
                                         bar_wait(&bars->vec_full[gq % C::NS], (gq / C::NS) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        float pt[64];
        {
          uint32_t sr[2][32];
          ptx::tmem_ld32(tS, sr[0]);
          ptx::tmem_ld32(tS + 32, sr[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(sr[0]);
          ptx::reg_fence(sr[1]);
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->s_free);
          const float4* nl4 = reinterpret_cast<const float4*>(vl);
          const float2 c2v = make_float2(c2, c2);
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 nl = nl4[q4];
            const int q = 4 * q4;
            const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[q / 32][q % 32]),
                                                     __uint_as_float(sr[q / 32][q % 32 + 1])),
                                         c2v, make_float2(nl.x, nl.y));
            const float2 xb = __ffma2_rn(make_float2(__uint_as_float(sr[q / 32][q % 32 + 2]),
                                                     __uint_as_float(sr[q / 32][q % 32 + 3])),
                                         c2v, make_float2(nl.z, nl.w));
            if (interior) {
              pt[q] = ptx::exp2_approx(xa.x);
              pt[q + 1] = ptx::exp2_approx(xa.y);
              pt[q + 2] = ptx::exp2_approx(xb.x);
              pt[q + 3] = ptx::exp2_approx(xb.y);
            } else {
              pt[q] = (uint32_t)(cb + q) <= span ? ptx::exp2_approx(xa.x) : 0.f;
              pt[q + 1] = (uint32_t)(cb + q + 1) <= span ? ptx::exp2_approx(xa.y) : 0.f;
              pt[q + 2] = (uint32_t)(cb + q + 2) <= span ? ptx::exp2_approx(xb.x) : 0.f;
              pt[q + 3] = (uint32_t)(cb + q + 3) <= span ? ptx::exp2_approx(xb.y) : 0.f;
            }
          }
        }
        // ---- dP^T into registers; P^T and dS^T packed as bf16 pairs
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dp_full, (cdp++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        uint32_t pp[32], pd[32];
        {
          const float4* nd4 = reinterpret_cast<const float4*>(vd);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t dr[32];
            ptx::tmem_ld32(tDP + 32 * half, dr);
            ptx::tmem_wait_ld();
            ptx::reg_fence(dr);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const int q = 32 * half + 4 * q4;
              const float4 nd = nd4[q / 4];
              const float2 da = __fmul2_rn(make_float2(pt[q], pt[q + 1]),
                                           __fadd2_rn(make_float2(__uint_as_float(dr[4 * q4]),
                                                                  __uint_as_float(dr[4 * q4 + 1])),
                                                      make_float2(nd.x, nd.y)));
              const float2 db = __fmul2_rn(make_float2(pt[q + 2], pt[q + 3]),
                                           __fadd2_rn(make_float2(__uint_as_float(dr[4 * q4 + 2]),
                                                                  __uint_as_float(dr[4 * q4 + 3])),
                                                      make_float2(nd.z, nd.w)));
              pp[q / 2] = ptx::pack_bf16x2(pt[q], pt[q + 1]);
              pp[q / 2 + 1] = ptx::pack_bf16x2(pt[q + 2], pt[q + 3]);
              pd[q / 2] = ptx::pack_bf16x2(da.x, da.y);
              pd[q / 2 + 1] = ptx::pack_bf16x2(db.x, db.y);
            }
          }
        }
        // both warpgroups hold their dP^T columns: P^T may overwrite them
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->ew_sync);
        ok = __all_sync(0xffffffffu, bar_wait(&bars->ew_sync, (cew++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        // dS^T row r of block w; at a unit's first tile this warp's bulk
        // stores of the previous epilogue must have read the tile first
        if (first_step) {
          if (lane == 0) ptx::bulk_wait_group_read_all();
          __syncwarp();
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ptx::st_shared_v4(ds_row + ((k ^ (r & 7)) << 4), pd[4 * k], pd[4 * k + 1], pd[4 * k + 2], pd[4 * k + 3]);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars->ds_full);
        ptx::tmem_st32(tPT, pp);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full);
        ptx::mbar_arrive(&bars->vec_empty[gq % C::NS]);
        first_step = false;
        // ---- dQ of this query tile, piece by piece, into the fp32 buffer
        const int64_t iq = i0 + r;  // query row of TMEM lane r
        float* dst = p.dq_acc + ((int64_t)U.bh * N + iq) * D + 32 * w;
#pragma unroll 1
        for (int pc = 0; pc < C::NPIECE; ++pc) {
          ok = __all_sync(0xffffffffu, bar_wait(&bars->dq_full, (cdq++) & 1, abort_flag));
          if (!ok) break;
          ptx::tc_fence_after();
          uint32_t g[32];
          ptx::tmem_ld32(tDQ, g);
          ptx::tmem_wait_ld();
          ptx::reg_fence(g);
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->dq_free);
          if (iq < N) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) red_add_v4(dst + 64 * pc + e, g[e], g[e + 1], g[e + 2], g[e + 3]);
          }
        }
        if (!ok) break;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // As in the dK/dV pass: dV and scale * dK staged per warp as bf16 in the
      // shared tile (now free: the last dK and dQ pieces have read dS^T, which
      // acc_done follows) and written with bulk tensor stores.
      constexpr int NJ = D / 64;
      const int x0 = NJ == 2 ? 64 * w : 0;
      ok = __all_sync(0xffffffffu, bar_wait(&bars->acc_done, (cacc++) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t pk[NJ][32];
#pragma unroll
      for (int t = 0; t < NJ; ++t) {
        const bool is_dk = NJ == 2 ? t == 1 : w == 1;
        const uint32_t src = tmem + lane_base + (is_dk ? C::TM_DK : C::TM_DV) + x0;
        const float mul = is_dk ? p.scale : 1.f;
        uint32_t g[2][32];
        ptx::tmem_ld32(src, g[0]);
        ptx::tmem_ld32(src + 32, g[1]);
        ptx::tmem_wait_ld();
        if (t == NJ - 1) {
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->acc_free);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e)
          pk[t][e] = ptx::pack_bf16x2(__uint_as_float(g[e / 16][(2 * e) % 32]) * mul,
                                      __uint_as_float(g[e / 16][(2 * e) % 32 + 1]) * mul);
      }
      const uint32_t slice = (uint32_t)w * (C::BK * 128) + (uint32_t)wq * (32 * 128);
      const int64_t row0 = U.j0 + 32 * wq;
#pragma unroll
      for (int t = 0; t < NJ; ++t) {
        const bool is_dk = NJ == 2 ? t == 1 : w == 1;
        if (lane == 0) ptx::bulk_wait_group_read_all();
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ptx::st_shared_v4(ds_row + ((k ^ (r & 7)) << 4), pk[t][4 * k], pk[t][4 * k + 1], pk[t][4 * k + 2],
                            pk[t][4 * k + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < N) {
          ptx::tma_store_3d(is_dk ? &tm_dk : &tm_dv, smem + C::OFF_P + slice, x0, (int)row0, U.bh);
          ptx::bulk_commit_group();
        }
      }
    }
    ptx::bulk_wait_group_all();
  }

  // ------------------------------------------------------------ keys no query reaches
  {
    const int num_fill = p.B * p.fills_per_batch;
    for (int f = blockIdx.x; f < num_fill; f += gridDim.x) {
      const int b = f / p.fills_per_batch;
      const int r = f % p.fills_per_batch;
      const int h = head_of(p.fill_start, p.H, r);
      const int64_t kt = dkv_units_of_head(N, p.lo[h]) + (r - p.fill_start[h]);
      const int64_t row0 = (int64_t)(b * p.H + h) * N + kt * 128;
      const int64_t rows = min64(kt * 128 + 128, N) - kt * 128;
      zero_rows_bf16(static_cast<uint16_t*>(p.dk) + row0 * D, rows, D);
      zero_rows_bf16(static_cast<uint16_t*>(p.dv) + row0 * D, rows, D);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace spa
