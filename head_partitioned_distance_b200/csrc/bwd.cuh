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

// The same row sums for the rows the dK/dV pass reads only: rows i >= 128
// floor(lo_h / 128) of every (b, h), the 128-row query tiles its bands reach.
// blockIdx.y walks the (b, h) pairs and blockIdx.x the rows of one, 256 / (D / 8)
// rows per block and round; a round's rows are the same for every lane of a
// warp, so every lane takes part in the row's shuffle.  Rows before the first
// reached tile are neither read nor written.
template <int D>
__global__ void __launch_bounds__(256) spa_bwd_delta_band_kernel(const uint16_t* __restrict__ o,
                                                                 const uint16_t* __restrict__ dout,
                                                                 const __grid_constant__ AttnParams p) {
  constexpr int TPR = D / 8;
  constexpr int RPB = 256 / TPR;  // rows per block and round
  const int part = threadIdx.x % TPR;
  const int BH = p.B * p.H;
  const int64_t N = p.N;
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const int64_t r0 = (int64_t)(p.lo[bh % p.H] / 128) * 128;
    const uint16_t* ob = o + (int64_t)bh * N * D;
    const uint16_t* gb = dout + (int64_t)bh * N * D;
    float* db = p.delta + (int64_t)bh * N;
    for (int64_t base = r0 + (int64_t)blockIdx.x * RPB; base < N; base += (int64_t)gridDim.x * RPB) {
      const int64_t i = base + threadIdx.x / TPR;
      const bool live = i < N;
      float acc = 0.f;
      if (live) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(ob + i * D) + part);
        const uint4 g = __ldg(reinterpret_cast<const uint4*>(gb + i * D) + part);
        acc = bf16lo(a.x) * bf16lo(g.x) + bf16hi(a.x) * bf16hi(g.x) + bf16lo(a.y) * bf16lo(g.y) +
              bf16hi(a.y) * bf16hi(g.y) + bf16lo(a.z) * bf16lo(g.z) + bf16hi(a.z) * bf16hi(g.z) +
              bf16lo(a.w) * bf16lo(g.w) + bf16hi(a.w) * bf16hi(g.w);
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (live && part == 0) db[i] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// dK, dV: persistent grid; a unit is (b, h, key tile of 128 keys), walking
// the 128-query tiles its band reaches.  Per query tile:
//   S^T  = K Q^T      SS MMA -> TMEM [0,128)
//   dP^T = V dO^T     SS MMA -> TMEM [128,256)
//   P^T  = exp2(S^T c - lse2), masked on edge tiles; bf16 over dP^T
//   dS^T = P^T (dP^T - D);                          bf16 over dP^T
//   dV  += P^T dO     TS MMA (A = P^T from TMEM)  -> TMEM [256,384)
//   dK  += dS^T Q     TS MMA (A = dS^T from TMEM) -> TMEM [384,512)
// Two warpgroups share each tile: warpgroup w owns query columns
// [64w, 64w+64) of every key row (thread r = key row r = TMEM lane r).  Once
// it holds its 64 columns of dP^T in registers it writes its P^T pairs to the
// first 32 of them and its dS^T pairs to the other 32, so both gradient
// products read their A operand from TMEM and shared memory carries only the
// tiles the copy engine brings (the SS products of N = 128 need all of its
// bandwidth).  S^T of the next query tile is issued as soon as the
// warpgroups hold this one in registers, so it overlaps their exponentials;
// dP^T of the next tile follows dK.  K and V are released after their last
// S^T/dP^T so the next unit's loads overlap the last step.  Epilogue: bulk
// tensor stores of dV and scale * dK staged through shared memory.
// ---------------------------------------------------------------------------
template <int D>
struct DkvCfg {
  static constexpr int BK = 128;  // keys per unit (MMA M)
  static constexpr int BQ = 128;  // queries per step
  static constexpr int NS = 2;    // Q/dO ring stages
  static constexpr int DB = D / 64;
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t QT_BYTES = BQ * D * 2;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + KT_BYTES;
  static constexpr uint32_t OFF_Q = OFF_V + KT_BYTES;
  static constexpr uint32_t OFF_DO = OFF_Q + NS * QT_BYTES;
  // epilogue staging: dV and dK of the unit as bf16, [keys x 64 head dims]
  // per warpgroup, 128-byte swizzle, for the bulk tensor stores
  static constexpr uint32_t OFF_P = OFF_DO + NS * QT_BYTES;
  static constexpr uint32_t PT_BYTES = BK * 128 * 2;
  // vectors of a query tile, [2 stages][256 floats]: -lse * log2(e) of its
  // 128 queries, then -D of them
  static constexpr uint32_t OFF_VEC = OFF_P + PT_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_VEC + 2 * 2 * 128 * 4;
  static constexpr uint32_t USED_BYTES = OFF_BAR + 256;
  // The tiles want a 1024-byte aligned base; the launch adds that much slack
  // where the per-block limit allows and the kernel checks the rest.
  static constexpr uint32_t SMEM_BYTES =
      USED_BYTES + 1024 < kMaxSmemPerBlock ? USED_BYTES + 1024 : kMaxSmemPerBlock;
  static_assert(USED_BYTES <= kMaxSmemPerBlock, "dK/dV tiles exceed shared memory");
  static constexpr int NTHREADS = 384;
  // register split: 384 threads launch with 168 registers each; the two
  // element-wise warpgroups take 192, the producer/MMA warpgroup 120.
  static constexpr uint32_t LAUNCH_REGS = 168, EW_REGS = 192, CONTROL_REGS = 120;
  static_assert(2 * EW_REGS + CONTROL_REGS <= 3 * LAUNCH_REGS, "register split over budget");
  static constexpr uint32_t TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 384;
  // Once the warpgroups hold dP^T in registers, its columns take P^T and
  // dS^T as bf16 pairs (A operands of dV and dK): warpgroup w's 64 queries
  // at TM_DPT + 64 w + [0, 32) (P^T) and + [32, 64) (dS^T).
  static constexpr uint32_t TM_PT = TM_DPT, TM_DST = TM_DPT + 32;
  static constexpr uint32_t TMEM_COLS = 512;
};

struct DkvBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, s_free, dp_full, p_full, ds_full;
  uint64_t pt_read;  // dV of a query tile has read its P^T (dP^T of the next may overwrite it)
  uint64_t vec_full[2], vec_empty[2];
  uint64_t acc_done, acc_free, drain;
  uint32_t tmem_base;
  int abort;
};

// Key tiles of head h that some query reaches: u <= (N - 1 - lo) / 128.
__device__ __forceinline__ int dkv_units_of_head(int64_t N, int32_t lo) {
  return (int)((N - 1 - lo) / 128) + 1;
}

struct DkvUnit {
  int bh;
  int32_t lo, hi;
  int64_t j0;
  int qa, qb;  // query tiles walked
};

__device__ __forceinline__ DkvUnit dkv_decode(int u, const AttnParams& p) {
  DkvUnit U;
  const int b = u / p.units_per_batch;
  const int r = u % p.units_per_batch;
  const int h = head_of(p.unit_start, p.H, r);
  U.bh = b * p.H + h;
  U.lo = p.lo[h];
  U.hi = p.hi[h];
  U.j0 = (int64_t)(r - p.unit_start[h]) * 128;
  const Strip s = query_strip(p.N, U.lo, U.hi, U.j0, 128, 128);
  U.qa = s.begin;
  U.qb = s.end;
  return U;
}

// ACC: add dk, dv to what the outputs hold (spa_attn_bwd_dkdv_add) and leave
// the keys no query reaches untouched.
// DS: each tile pair's dS^T (bf16, the A operand of dK) also leaves for the
// stored-dS backward's dQ pass, to its tile in p.ds (the layout of
// bwd_stored.cuh: 8 x 8 core matrices).  Once the dK product may read dS^T
// from TMEM, every thread writes its key row's 64 queries as eight 16-byte
// pieces; the 32 rows of a warp make each store instruction 512 contiguous
// bytes.
template <int D, bool ACC = false, bool DS = false>
__global__ void __launch_bounds__(384, 1)
    spa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                        const __grid_constant__ AttnParams p) {
  using C = DkvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if (!smem_fits(smem_raw, smem, C::USED_BYTES)) return;
  DkvBars* bars = reinterpret_cast<DkvBars*>(smem + C::OFF_BAR);
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
    ptx::mbar_init(&bars->kv_empty, 2);  // one commit from each MMA issuer
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
        // -lse * log2(e) and -D of the tile's queries (rows past N: 0)
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
    // Warp 10 issues S^T of every query tile, warp 11 dV, warp 9 dK and dP^T
    // of the next tile.  The issuing thread blocks in each group of MMAs for
    // about as long as the tensor core takes to run it, so a single issuer
    // leaves the tensor core idle while it waits for the warpgroups, and the
    // dK -> dP^T chain would wait behind dV.  Each issuer writes its own
    // TMEM columns (S^T; dV; dK and dP^T); dP^T of the next tile overwrites
    // the P^T that dV reads, so warp 9 issues it only after warp 11's commit
    // on pt_read.  Q/dO stages are released by one commit from each issuer,
    // K/V by one from warps 10 and 9, the accumulators by one from 9 and 11.
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BQ, false, false);
      constexpr uint32_t idesc_g = ptx::idesc_bf16_f32(128, D, false, true);
      int nkv = 0, gq = 0;
      bool ok = true;
      auto qstage = [&](int g) { return g % C::NS; };
      auto qphase = [&](int g) { return (uint32_t)((g / C::NS) & 1); };
      // descriptors of every operand buffer, built once
      const uint64_t dK = ptx::sdesc_sw128(sK, 0, 1024), dV = ptx::sdesc_sw128(sV, 0, 1024);
      // K-major (B of S^T/dP^T) and MN-major (B of dK/dV) views of both Q/dO stages
      const uint64_t dQk0 = ptx::sdesc_sw128(sQ, 0, 1024), dQk1 = ptx::sdesc_sw128(sQ + C::QT_BYTES, 0, 1024);
      const uint64_t dOk0 = ptx::sdesc_sw128(sDO, 0, 1024), dOk1 = ptx::sdesc_sw128(sDO + C::QT_BYTES, 0, 1024);
      const uint64_t dQm0 = ptx::sdesc_sw128(sQ, C::BQ * 128, 1024);
      const uint64_t dQm1 = ptx::sdesc_sw128(sQ + C::QT_BYTES, C::BQ * 128, 1024);
      const uint64_t dOm0 = ptx::sdesc_sw128(sDO, C::BQ * 128, 1024);
      const uint64_t dOm1 = ptx::sdesc_sw128(sDO + C::QT_BYTES, C::BQ * 128, 1024);
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
      auto issue_grad = [&](uint32_t dst, uint32_t a_col, uint64_t db, bool first) {
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          ptx::mma_bf16_ts(tmem + dst, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                           ptx::sdesc_advance(db, kk * (16 * 128)), idesc_g, (!first || kk > 0));
      };
      if (warp == 10) {
        // ---- S^T of each query tile, as soon as the warpgroups hold the last
        // one in registers
        int cf = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DkvUnit U = dkv_decode(u, p);
          const int nq = U.qb - U.qa + 1;
          const int g0 = gq;
          for (int j = 0; ok && j < nq; ++j) {
            const int g = g0 + j;
            // S^T of the previous tile is in registers (for j = 0: the
            // previous unit's last tile, if any)
            if (g > 0) ok = bar_wait(&bars->s_free, (cf++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->kv_full, (nkv++) & 1, abort_flag);
            if (ok) ok = bar_wait(&bars->q_full[qstage(g)], qphase(g), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_nt(C::TM_ST, dK, dQk(qstage(g)));
            ptx::mma_commit(&bars->s_full);
            ptx::mma_commit(&bars->q_empty[qstage(g)]);
            if (j + 1 == nq) ptx::mma_commit(&bars->kv_empty);      // K read for the last time
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
            issue_grad(C::TM_DV, C::TM_PT, dOm(qstage(g)), j == 0);   // dV += P^T dO
            ptx::mma_commit(&bars->pt_read);
            ptx::mma_commit(&bars->q_empty[qstage(g)]);
          }
          if (!ok) break;
          ++cacc;
          ptx::mma_commit(&bars->acc_done);
          gq = g0 + nq;
        }
      } else {
        // ---- dK of each query tile and dP^T of the next
        int cds = 0, cacc = 0, cpt = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DkvUnit U = dkv_decode(u, p);
          const int nq = U.qb - U.qa + 1;
          const int g0 = gq;
          // dP^T of tile g overwrites P^T of tile g - 1: wait for its dV
          ok = bar_wait(&bars->kv_full, (nkv++) & 1, abort_flag) &&
               bar_wait(&bars->q_full[qstage(g0)], qphase(g0), abort_flag) &&
               (g0 == 0 || bar_wait(&bars->pt_read, (cpt++) & 1, abort_flag));
          if (!ok) break;
          ptx::tc_fence_after();
          issue_nt(C::TM_DPT, dV, dOk(qstage(g0)));
          ptx::mma_commit(&bars->dp_full);
          if (nq == 1) ptx::mma_commit(&bars->kv_empty);           // V read for the last time
          for (int j = 0; j < nq; ++j) {
            const int g = g0 + j;
            ok = bar_wait(&bars->ds_full, (cds++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->acc_free, ((cacc & 1) ^ 1), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_grad(C::TM_DK, C::TM_DST, dQm(qstage(g)), j == 0);  // dK += dS^T Q
            ptx::mma_commit(&bars->q_empty[qstage(g)]);
            if (j + 1 < nq) {
              ok = bar_wait(&bars->q_full[qstage(g + 1)], qphase(g + 1), abort_flag) &&
                   bar_wait(&bars->pt_read, (cpt++) & 1, abort_flag);
              if (!ok) break;
              ptx::tc_fence_after();
              issue_nt(C::TM_DPT, dV, dOk(qstage(g + 1)));           // dP^T of the next tile
              ptx::mma_commit(&bars->dp_full);
              if (j + 2 == nq) ptx::mma_commit(&bars->kv_empty);     // V read for the last time
            }
          }
          if (!ok) break;
          ++cacc;
          ptx::mma_commit(&bars->acc_done);
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
    const int w = warp / 4;                          // query columns [64w, 64w+64)
    const int r = threadIdx.x - 128 * w;             // key row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::TM_ST + 64 * w;
    const uint32_t tDP = tmem + lane_base + C::TM_DPT + 64 * w;
    const uint32_t tPT = tmem + lane_base + C::TM_PT + 64 * w;
    const uint32_t tDST = tmem + lane_base + C::TM_DST + 64 * w;
    const float c2 = p.scale_log2;
    int gq = 0, cs = 0, cdp = 0, cacc = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const DkvUnit U = dkv_decode(u, p);
      const int64_t j = U.j0 + r;
      // the unit's dS^T tiles are consecutive, from its first query tile's
      uint8_t* const utile =
          DS ? static_cast<uint8_t*>(p.ds) + stored_slot(p, U.bh / p.H, U.bh % p.H, (int)(U.j0 / 128), U.qa, U.qa) *
                                                 (128 * 128 * 2)
             : nullptr;
      for (int qt = U.qa; qt <= U.qb; ++qt, ++gq) {
        const int64_t i0 = (int64_t)qt * C::BQ;
        const bool interior = tile_is_interior(N, U.lo, U.hi, i0, C::BQ, U.j0, C::BK);
        // Edge tile: query column q (0..127) is permitted for this key iff
        // qlo <= q <= qlo + span.
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
        // this warpgroup's 64 queries in vector stage gq % 2
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
          // S^T is in registers: its columns may take the next tile's S^T
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->s_free);
          // vl holds -lse2 of the 64 queries: x = s * c2 - lse2 in pairs
          const float4* nl4 = reinterpret_cast<const float4*>(vl);
          const float2 c2v = make_float2(c2, c2);
          if (interior) {
            // every query permitted
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
              pt[q] = ptx::exp2_approx(xa.x);
              pt[q + 1] = ptx::exp2_approx(xa.y);
              pt[q + 2] = ptx::exp2_approx(xb.x);
              pt[q + 3] = ptx::exp2_approx(xb.y);
            }
          } else {
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
              pt[q] = (uint32_t)(cb + q) <= span ? ptx::exp2_approx(xa.x) : 0.f;
              pt[q + 1] = (uint32_t)(cb + q + 1) <= span ? ptx::exp2_approx(xa.y) : 0.f;
              pt[q + 2] = (uint32_t)(cb + q + 2) <= span ? ptx::exp2_approx(xb.x) : 0.f;
              pt[q + 3] = (uint32_t)(cb + q + 3) <= span ? ptx::exp2_approx(xb.y) : 0.f;
            }
          }
        }
        // ---- dP^T into registers; its columns take P^T (A of dV), then dS^T
        uint32_t dsk[32];  // dS^T of this key row, bf16 pairs over the warpgroup's 64 queries
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dp_full, (cdp++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        {
          // the first 32 columns of dP^T take P^T: read them first, the
          // other 32 (where dS^T goes) after P^T is written
          uint32_t dr[2][32];
          ptx::tmem_ld32(tDP, dr[0]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(dr[0]);
          {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = ptx::pack_bf16x2(pt[2 * e], pt[2 * e + 1]);
            ptx::tmem_st32(tPT, pk);
            ptx::tmem_wait_st();
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->p_full);
          ptx::tmem_ld32(tDP + 32, dr[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(dr[1]);
          // ---- dS^T = P^T (dP^T - D); vd holds -D of the 64 queries, in pairs
          const float4* nd4 = reinterpret_cast<const float4*>(vd);
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 nd = nd4[q4];
            const int q = 4 * q4;
            const float2 da = __fmul2_rn(make_float2(pt[q], pt[q + 1]),
                                         __fadd2_rn(make_float2(__uint_as_float(dr[q / 32][q % 32]),
                                                                __uint_as_float(dr[q / 32][q % 32 + 1])),
                                                    make_float2(nd.x, nd.y)));
            const float2 db = __fmul2_rn(make_float2(pt[q + 2], pt[q + 3]),
                                         __fadd2_rn(make_float2(__uint_as_float(dr[q / 32][q % 32 + 2]),
                                                                __uint_as_float(dr[q / 32][q % 32 + 3])),
                                                    make_float2(nd.z, nd.w)));
            dsk[2 * q4] = ptx::pack_bf16x2(da.x, da.y);
            dsk[2 * q4 + 1] = ptx::pack_bf16x2(db.x, db.y);
          }
          ptx::tmem_st32(tDST, dsk);
          ptx::tmem_wait_st();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->ds_full);
        ptx::mbar_arrive(&bars->vec_empty[gq % C::NS]);  // last read of this vector stage
        if constexpr (DS) {
          // this key row's 64 queries of dS^T as eight 8-query pieces: piece
          // c of key r at byte (c * 128 + r) * 16 of the tile
          uint8_t* tile = utile + (qt - U.qa) * (128 * 128 * 2);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            ptx::st_global_v4(tile + ((8 * w + k) * 128 + r) * 16, dsk[4 * k], dsk[4 * k + 1], dsk[4 * k + 2],
                              dsk[4 * k + 3]);
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // Warp (w, wq) owns key rows [32 wq, 32 wq + 32) and, for d = 128,
      // head dims [64 w, 64 w + 64) of both dV and dK (for d = 64: all of dV
      // if w = 0, all of dK if w = 1).  It reads them from TMEM (which then
      // goes back to the MMA warp) and stages each as bf16 in its own 4 KB
      // slice of the staging tile (128-byte swizzle)
      // for a bulk tensor store of a 32 x 64 box.  When adding to the
      // outputs, the row's 64 columns of each are read while the last
      // products finish, and added before the rounding.
      constexpr int NJ = D / 64;
      const int x0 = NJ == 2 ? 64 * w : 0;
      uint4 old[ACC ? NJ : 1][8];
      if constexpr (ACC) {
#pragma unroll
        for (int t = 0; t < NJ; ++t) {
          const bool is_dk = NJ == 2 ? t == 1 : w == 1;
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(is_dk ? p.dk : p.dv) +
                                                            ((int64_t)U.bh * N + j) * D + x0);
#pragma unroll
          for (int e = 0; e < 8; ++e)  // rows past N: -0, the identity of the sum
            old[t][e] = j < N ? src[e] : make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
        }
      }
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
        if constexpr (ACC) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 o = ptx::bf16x2_to_float2(ptx::word_of(old[t][e / 4], e % 4));
            pk[t][e] = ptx::pack_bf16x2(fmaf(__uint_as_float(g[e / 16][(2 * e) % 32]), mul, o.x),
                                        fmaf(__uint_as_float(g[e / 16][(2 * e) % 32 + 1]), mul, o.y));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            pk[t][e] = ptx::pack_bf16x2(__uint_as_float(g[e / 16][(2 * e) % 32]) * mul,
                                        __uint_as_float(g[e / 16][(2 * e) % 32 + 1]) * mul);
        }
      }
      const int wq = warp % 4;
      const uint32_t slice = (uint32_t)w * (C::BK * 128) + (uint32_t)wq * (32 * 128);
      const uint32_t srow = sP + (uint32_t)w * (C::BK * 128) + (uint32_t)r * 128;
      const int64_t row0 = U.j0 + 32 * wq;
#pragma unroll
      for (int t = 0; t < NJ; ++t) {
        const bool is_dk = NJ == 2 ? t == 1 : w == 1;
        // the slice is free once this warp's previous bulk store has read it
        if (lane == 0) ptx::bulk_wait_group_read_all();
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ptx::st_shared_v4(srow + ((k ^ (r & 7)) << 4), pk[t][4 * k], pk[t][4 * k + 1], pk[t][4 * k + 2],
                            pk[t][4 * k + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < N) {  // rows past N in the box are clipped
          ptx::tma_store_3d(is_dk ? &tm_dk : &tm_dv, smem + C::OFF_P + slice, x0, (int)row0, U.bh);
          ptx::bulk_commit_group();
        }
      }
    }
    ptx::bulk_wait_group_all();
  }

  // ------------------------------------------------------------ keys no query reaches
  // (left as they are when adding to the output)
  {
    const int num_fill = ACC ? 0 : p.B * p.fills_per_batch;
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

// ---------------------------------------------------------------------------
// dQ: persistent grid; a unit is (b, h, query tile of 128 rows), walking the
// same 128-key strip as the forward.  Q and dO of the unit are fixed, so they
// sit in TMEM as bf16 A operands and the two products of each key tile read
// only K or V from shared memory:
//   S   = Q K^T      TS MMA (A = Q from TMEM [384, 384 + D/2))   -> TMEM [0,128)
//   dP  = dO V^T     TS MMA (A = dO from TMEM [384 + D/2, 512))  -> TMEM [128,256)
//   dS  = P (dP - D), P = exp2(S c - lse2) masked on edge tiles; written as
//                    bf16 over dP
//   dQ += dS K       TS MMA (A = dS from TMEM, B = K MN-major)   -> TMEM [256,384)
// Two warpgroups share each tile: warpgroup w owns key columns [64w, 64w+64)
// of every query row (thread r = row r = TMEM lane r).  S of the next key
// tile is issued as soon as the warpgroups hold this one in registers, so it
// overlaps their exponentials; dP of the next tile follows dQ.  At a unit's
// start warpgroup 0 copies Q and warpgroup 1 copies dO from the staging tiles
// the copy engine filled into TMEM, which frees the staging tiles for the next
// unit.  When the kernel is given o (AttnParams::o_in), the copy engine also
// stages the unit's O tile and warpgroup 1 forms D_i = sum_c dO_ic O_ic from
// the staged rows while it copies dO (fp32, the definition in the backward
// of spa.h), writes D to the workspace for the dK/dV pass and hands it to
// warpgroup 0 through shared memory; otherwise D is read from the workspace.
// Epilogue: scale * dQ straight from TMEM to global, warpgroup w writing head
// dims [D/2 w, D/2 (w+1)).
// ---------------------------------------------------------------------------
template <int D>
struct DqCfg {
  static constexpr int BQ = 128;  // queries per unit (MMA M)
  static constexpr int BK = 128;  // keys per step
  static constexpr int NS = 2;    // K/V ring stages
  static constexpr int DB = D / 64;
  static constexpr uint32_t QT_BYTES = BQ * D * 2;
  static constexpr uint32_t KT_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_DO = OFF_Q + QT_BYTES;
  static constexpr uint32_t OFF_O = OFF_DO + QT_BYTES;    // O staging (D formed in this kernel)
  static constexpr uint32_t OFF_K = OFF_O + QT_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KT_BYTES;
  static constexpr uint32_t OFF_DVEC = OFF_V + NS * KT_BYTES;  // D of the unit's 128 rows
  static constexpr uint32_t OFF_BAR = OFF_DVEC + BQ * 4;
  static constexpr uint32_t SMEM_BYTES =
      (OFF_BAR + 256 + 1024) > 116u * 1024 ? (OFF_BAR + 256 + 1024) : 116u * 1024;
  static constexpr int NTHREADS = 384;
  // register split: 384 threads launch with 168 registers each; the two
  // element-wise warpgroups take 192, the producer/MMA warpgroup 120.
  static constexpr uint32_t LAUNCH_REGS = 168, EW_REGS = 192, CONTROL_REGS = 120;
  static_assert(2 * EW_REGS + CONTROL_REGS <= 3 * LAUNCH_REGS, "register split over budget");
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_QA = 384, TM_DOA = 384 + D / 2;
  static constexpr uint32_t TMEM_COLS = 512;
};

struct DqBars {
  uint64_t q_full, q_empty;  // staging tiles of Q and dO
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t qa_full;          // Q and dO of the unit copied into TMEM
  uint64_t dvec_full;        // D of the unit's rows in shared memory (when formed here)
  uint64_t s_full, s_free, dp_full, ds_full;
  uint64_t acc_done, acc_free, drain;
  uint32_t tmem_base;
  int abort;
};

struct DqUnit {
  int bh;
  int32_t lo, hi;
  int64_t i0;
  int ka, kb;  // key tiles walked
};

__device__ __forceinline__ DqUnit dq_decode(int u, const AttnParams& p) {
  DqUnit U;
  const int b = u / p.units_per_batch;
  const int r = u % p.units_per_batch;
  const int h = head_of(p.unit_start, p.H, r);
  U.bh = b * p.H + h;
  U.lo = p.lo[h];
  U.hi = p.hi[h];
  U.i0 = (int64_t)(p.lo[h] / 128 + (r - p.unit_start[h])) * 128;
  const Strip s = key_strip(p.N, U.lo, U.hi, U.i0, 128, 128);
  U.ka = s.begin;
  U.kb = s.end;
  return U;
}

// ACC: add dq to what the output holds (spa_attn_bwd_dq_add) and leave the
// rows before the band untouched.
template <int D, bool ACC = false>
__global__ void __launch_bounds__(384, 1)
    spa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ AttnParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  DqBars* bars = reinterpret_cast<DqBars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t N = p.N;
  const int num_units = p.B * p.units_per_batch;
  const bool fuse_d = p.o_in != nullptr;  // form D here rather than read it

  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sDO = ptx::smem_u32(smem + C::OFF_DO);
  const uint32_t sO = ptx::smem_u32(smem + C::OFF_O);
  float* dvec = reinterpret_cast<float*>(smem + C::OFF_DVEC);
  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    ptx::mbar_init(&bars->q_empty, 256);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->k_full[s], 1);
      ptx::mbar_init(&bars->v_full[s], 1);
      ptx::mbar_init(&bars->kv_empty[s], 2);  // one commit from each MMA issuer
    }
    ptx::mbar_init(&bars->qa_full, 256);
    ptx::mbar_init(&bars->dvec_full, 128);
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->s_free, 256);
    ptx::mbar_init(&bars->dp_full, 1);
    ptx::mbar_init(&bars->ds_full, 256);
    ptx::mbar_init(&bars->acc_done, 1);
    ptx::mbar_init(&bars->acc_free, 256);
    ptx::mbar_init(&bars->drain, 2);
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
  if (warp >= 11) {
    // idle warps of the control warpgroup
  } else if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int nq = 0, g = 0, armed[2] = {0, 0};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const DqUnit U = dq_decode(u, p);
        // the staging tiles are free once the warpgroups copied the previous
        // unit's Q and dO into TMEM
        ok = bar_wait(&bars->q_empty, (nq & 1) ^ 1, abort_flag);
        if (!ok) break;
        ++nq;
        ptx::mbar_arrive_expect_tx(&bars->q_full, (fuse_d ? 3 : 2) * C::QT_BYTES);
        for (int c = 0; c < C::DB; ++c) {
          ptx::tma_load_3d(smem + C::OFF_Q + c * (C::BQ * 128), &tm_q, &bars->q_full, c * 64, (int)U.i0, U.bh);
          ptx::tma_load_3d(smem + C::OFF_DO + c * (C::BQ * 128), &tm_do, &bars->q_full, c * 64, (int)U.i0, U.bh);
          if (fuse_d)
            ptx::tma_load_3d(smem + C::OFF_O + c * (C::BQ * 128), &tm_o, &bars->q_full, c * 64, (int)U.i0, U.bh);
        }
        for (int kt = U.ka; ok && kt <= U.kb; ++kt, ++g) {
          const int s = g % C::NS;
          ok = bar_wait(&bars->kv_empty[s], ((g / C::NS) & 1) ^ 1, abort_flag);
          if (!ok) break;
          const int j0 = kt * C::BK;
          ptx::mbar_arrive_expect_tx(&bars->k_full[s], C::KT_BYTES);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_K + s * C::KT_BYTES + c * (C::BK * 128), &tm_k, &bars->k_full[s],
                             c * 64, j0, U.bh);
          ptx::mbar_arrive_expect_tx(&bars->v_full[s], C::KT_BYTES);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_V + s * C::KT_BYTES + c * (C::BK * 128), &tm_v, &bars->v_full[s],
                             c * 64, j0, U.bh);
          ++armed[s];
        }
      }
      if (nq > 0) bar_drain(&bars->q_full, (nq - 1) & 1);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) {
          bar_drain(&bars->k_full[s], (armed[s] - 1) & 1);
          bar_drain(&bars->v_full[s], (armed[s] - 1) & 1);
        }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuers
    // Warp 10 issues S of every key tile, warp 9 dQ and dP of the next tile
    // (as in dK/dV: an issuing thread blocks for about the length of each
    // group, so S of the next tile should not queue behind the waits of the
    // dQ chain).  K stages are released by one commit from each.
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BK, false, false);
      constexpr uint32_t idesc_g = ptx::idesc_bf16_f32(128, D, false, true);
      int nq = 0, g = 0;
      bool ok = true;
      // K-major (B of S/dP) and MN-major K (B of dQ) views of both K/V stages
      const uint64_t dKk0 = ptx::sdesc_sw128(sK, 0, 1024), dKk1 = ptx::sdesc_sw128(sK + C::KT_BYTES, 0, 1024);
      const uint64_t dVk0 = ptx::sdesc_sw128(sV, 0, 1024), dVk1 = ptx::sdesc_sw128(sV + C::KT_BYTES, 0, 1024);
      const uint64_t dKm0 = ptx::sdesc_sw128(sK, C::BK * 128, 1024);
      const uint64_t dKm1 = ptx::sdesc_sw128(sK + C::KT_BYTES, C::BK * 128, 1024);
      auto dKk = [&](int st) { return st ? dKk1 : dKk0; };
      auto dVk = [&](int st) { return st ? dVk1 : dVk0; };
      auto dKm = [&](int st) { return st ? dKm1 : dKm0; };
      // dst = A (queries, bf16 pairs in TMEM at a_col) x B^T (keys, K-major in shared memory)
      auto issue_nt = [&](uint32_t dst, uint32_t a_col, uint64_t db) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_bf16_ts(tmem + dst, tmem + a_col + kk * 8,
                           ptx::sdesc_advance(db, (kk / 4) * (C::BK * 128) + (kk % 4) * 32), idesc_s, kk > 0);
      };
      if (warp == 10) {
        // ---- S of each key tile, as soon as the warpgroups hold the last one
        int cf = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DqUnit U = dq_decode(u, p);
          const int nk = U.kb - U.ka + 1;
          const int g0 = g;
          for (int j = 0; ok && j < nk; ++j) {
            const int gj = g0 + j;
            const int st = gj % C::NS;
            if (gj > 0) ok = bar_wait(&bars->s_free, (cf++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->qa_full, (nq++) & 1, abort_flag);
            if (ok) ok = bar_wait(&bars->k_full[st], (uint32_t)((gj / C::NS) & 1), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_nt(C::TM_S, C::TM_QA, dKk(st));
            ptx::mma_commit(&bars->s_full);
            ptx::mma_commit(&bars->kv_empty[st]);
          }
          g = g0 + nk;
        }
      } else {
        // ---- dQ of each key tile and dP of the next
        int cds = 0, cacc = 0;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
          const DqUnit U = dq_decode(u, p);
          const int nk = U.kb - U.ka + 1;
          const int g0 = g;
          auto slot = [&](int jj) { return (g0 + jj) % C::NS; };
          auto par = [&](int jj) { return (uint32_t)(((g0 + jj) / C::NS) & 1); };
          ok = bar_wait(&bars->qa_full, (nq++) & 1, abort_flag) && bar_wait(&bars->v_full[slot(0)], par(0), abort_flag);
          if (!ok) break;
          ptx::tc_fence_after();
          issue_nt(C::TM_DP, C::TM_DOA, dVk(slot(0)));
          ptx::mma_commit(&bars->dp_full);
          for (int j = 0; j < nk; ++j) {
            ok = bar_wait(&bars->ds_full, (cds++) & 1, abort_flag);
            if (ok && j == 0) ok = bar_wait(&bars->acc_free, (cacc & 1) ^ 1, abort_flag);
            if (ok) ok = bar_wait(&bars->k_full[slot(j)], par(j), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            {
              // dQ += dS K: A = dS (bf16 pairs over dP, key halves at +0 / +64),
              // B = K tile MN-major along d
              const uint64_t db = dKm(slot(j));
              const uint32_t abase = tmem + C::TM_DP;
#pragma unroll
              for (int kk = 0; kk < C::BK / 16; ++kk)
                ptx::mma_bf16_ts(tmem + C::TM_DQ, abase + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                                 ptx::sdesc_advance(db, kk * (16 * 128)), idesc_g, (j > 0 || kk > 0));
            }
            ptx::mma_commit(&bars->kv_empty[slot(j)]);
            if (j + 1 < nk) {
              ok = bar_wait(&bars->v_full[slot(j + 1)], par(j + 1), abort_flag);
              if (!ok) break;
              ptx::tc_fence_after();
              issue_nt(C::TM_DP, C::TM_DOA, dVk(slot(j + 1)));  // dP of the next key tile
              ptx::mma_commit(&bars->dp_full);
            }
          }
          if (!ok) break;
          ++cacc;
          ptx::mma_commit(&bars->acc_done);
          g = g0 + nk;
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
    const int w = warp / 4;                      // key columns [64w, 64w+64)
    const int r = threadIdx.x - 128 * w;         // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::TM_S + 64 * w;
    const uint32_t tDP = tmem + lane_base + C::TM_DP + 64 * w;
    const float c2 = p.scale_log2;
    int cq = 0, cs = 0, cdp = 0, cacc = 0;
    bool ok = true;
    // Row r of the staged Q (warpgroup 0) or dO (warpgroup 1), 128-byte
    // swizzled, into the warpgroup's TMEM operand as bf16 pairs along d.
    // The unit and the raw lse, D of row r; the loads land while other work
    // runs (D only when it is not formed here).
    DqUnit U{};
    float lraw = 0.f, draw = 0.f;
    auto fetch_unit = [&](int uu) {
      U = dq_decode(uu, p);
      const int64_t i = U.i0 + r;
      lraw = 0.f;
      draw = 0.f;
      if (i < N) {
        lraw = p.lse[(int64_t)U.bh * N + i];
        if (!fuse_d) draw = p.delta[(int64_t)U.bh * N + i];
      }
    };
    // Row r of the staged Q (warpgroup 0) or dO (warpgroup 1), 128-byte
    // swizzled, into the warpgroup's TMEM operand as bf16 pairs along d;
    // the staging tiles are then free.  With fuse_d, warpgroup 1 also forms
    // D_r from the staged dO and O rows of unit U (decoded just before).
    auto stage_operands = [&]() -> bool {
      if (!__all_sync(0xffffffffu, bar_wait(&bars->q_full, (cq++) & 1, abort_flag))) return false;
      const uint32_t src = (w == 0 ? sQ : sDO) + (uint32_t)r * 128;
      const uint32_t dst = tmem + lane_base + (w == 0 ? C::TM_QA : C::TM_DOA);
      const bool form_d = fuse_d && w == 1;
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < C::DB; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ptx::ld_shared_v4(src + c * (C::BQ * 128) + ((k ^ (r & 7)) << 4), v[4 * k], v[4 * k + 1],
                            v[4 * k + 2], v[4 * k + 3]);
        ptx::tmem_st32(dst + 32 * c, v);
        if (form_d) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t o4[4];
            ptx::ld_shared_v4(sO + (uint32_t)r * 128 + c * (C::BQ * 128) + ((k ^ (r & 7)) << 4), o4[0], o4[1],
                              o4[2], o4[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              acc = __ffma2_rn(ptx::bf16x2_to_float2(v[4 * k + e]), ptx::bf16x2_to_float2(o4[e]), acc);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->q_empty);
      ptx::mbar_arrive(&bars->qa_full);
      if (fuse_d) {
        if (w == 1) {
          draw = acc.x + acc.y;
          dvec[r] = draw;
          ptx::mbar_arrive(&bars->dvec_full);
          const int64_t i = U.i0 + r;
          if (i < N) p.delta[(int64_t)U.bh * N + i] = draw;
        } else {
          // this unit's D from warpgroup 1 (it rewrites the array only after
          // every step of the unit, each of which waits for both warpgroups)
          if (!__all_sync(0xffffffffu, bar_wait(&bars->dvec_full, (cq - 1) & 1, abort_flag))) return false;
          draw = dvec[r];
        }
      }
      return true;
    };
    int u = blockIdx.x;
    if (u < num_units) {
      fetch_unit(u);
      ok = stage_operands();
    }
    for (; ok && u < num_units; u += gridDim.x) {
      const int64_t i = U.i0 + r;
      const bool in = i < N;
      const float nlse2 = -lraw * kLog2e;
      const float Di = draw;
      for (int kt = U.ka; kt <= U.kb; ++kt) {
        const int64_t j0 = (int64_t)kt * C::BK;
        const bool interior = tile_is_interior(N, U.lo, U.hi, U.i0, C::BQ, j0, C::BK);
        int clo = 0;
        uint32_t span = 127;
        if (!interior) {
          const int64_t c_first = max64(i - U.hi + 1 - j0, 0);
          const int64_t c_last = min64(min64(i - U.lo - j0, N - 1 - j0), 127);
          if (!in || c_last < c_first) {
            clo = 128;
            span = 0;
          } else {
            clo = (int)c_first;
            span = (uint32_t)(c_last - c_first);
          }
        }
        const int cb = 64 * w - clo;
        ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full, (cs++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        float pv[64];
        {
          uint32_t sr[2][32];
          ptx::tmem_ld32(tS, sr[0]);
          ptx::tmem_ld32(tS + 32, sr[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(sr[0]);
          ptx::reg_fence(sr[1]);
          // S is in registers: its columns may take the next key tile's S
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->s_free);
          // x = s * c2 - lse2 in pairs
          const float2 c2v = make_float2(c2, c2);
          const float2 nlv = make_float2(nlse2, nlse2);
          if (interior) {
            // every key permitted
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[e / 32][e % 32]),
                                                      __uint_as_float(sr[e / 32][e % 32 + 1])),
                                          c2v, nlv);
              pv[e] = ptx::exp2_approx(x.x);
              pv[e + 1] = ptx::exp2_approx(x.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[e / 32][e % 32]),
                                                      __uint_as_float(sr[e / 32][e % 32 + 1])),
                                          c2v, nlv);
              pv[e] = (uint32_t)(cb + e) <= span ? ptx::exp2_approx(x.x) : 0.f;
              pv[e + 1] = (uint32_t)(cb + e + 1) <= span ? ptx::exp2_approx(x.y) : 0.f;
            }
          }
        }
        ok = __all_sync(0xffffffffu, bar_wait(&bars->dp_full, (cdp++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        {
          uint32_t dr[2][32];
          ptx::tmem_ld32(tDP, dr[0]);
          ptx::tmem_ld32(tDP + 32, dr[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(dr[0]);
          ptx::reg_fence(dr[1]);
          // dS = P (dP - D) in pairs, bf16 over the first half of the columns read
          const float2 ndv = make_float2(-Di, -Di);
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 d = __fmul2_rn(make_float2(pv[2 * e], pv[2 * e + 1]),
                                        __fadd2_rn(make_float2(__uint_as_float(dr[e / 16][(2 * e) % 32]),
                                                               __uint_as_float(dr[e / 16][(2 * e) % 32 + 1])),
                                                   ndv));
            pk[e] = ptx::pack_bf16x2(d.x, d.y);
          }
          ptx::tmem_st32(tDP, pk);
          ptx::tmem_wait_st();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->ds_full);
      }
      if (!ok) break;
      const int bh = U.bh;
      // the next unit's Q and dO go into TMEM while the last dQ products run
      // (S and dP of this unit, their last readers, have completed)
      if (u + (int)gridDim.x < num_units) {
        fetch_unit(u + gridDim.x);
        ok = stage_operands();
        if (!ok) break;
      }
      // ---------------------------------------------------------- epilogue
      uint16_t* grow = static_cast<uint16_t*>(p.dq) + ((int64_t)bh * N + i) * D;
      const float mul = p.scale;
      if constexpr (ACC) {
        // the half row already in the output is read while the last products
        // finish
        uint4 old[D / 16];
        if (in) {
#pragma unroll
          for (int e = 0; e < D / 16; ++e) old[e] = reinterpret_cast<const uint4*>(grow + w * (D / 2))[e];
        }
        ok = __all_sync(0xffffffffu, bar_wait(&bars->acc_done, (cacc++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          const int c = w * (D / 2) + 32 * cc;
          uint32_t g[32];
          ptx::tmem_ld32(tmem + lane_base + C::TM_DQ + c, g);
          ptx::tmem_wait_ld();
          ptx::reg_fence(g);
          if (in) ptx::store_row32_bf16_add(grow + c, g, mul, old + 4 * cc);
        }
      } else {
        ok = __all_sync(0xffffffffu, bar_wait(&bars->acc_done, (cacc++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll 1
        for (int c = w * (D / 2); c < (w + 1) * (D / 2); c += 32) {
          uint32_t g[32];
          ptx::tmem_ld32(tmem + lane_base + C::TM_DQ + c, g);
          ptx::tmem_wait_ld();
          ptx::reg_fence(g);
          if (in) ptx::store_row32_bf16(grow + c, g, mul);
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->acc_free);
    }
  }

  // ------------------------------------------------------------ rows before their band
  // (left as they are when adding to the output)
  {
    const int num_fill = ACC ? 0 : p.B * p.fills_per_batch;
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
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace spa
