// fwd.cuh -- band-sparse attention forward for sm_100a.
//
// Persistent grid (one CTA per SM).  A unit is (b, h, 256 query rows), split
// into two 128-row Q tiles that two softmax warpgroups process in ping-pong:
// while one warpgroup turns its scores into probabilities, the tensor core
// works on the other tile.  Each tile walks the diagonal strip of 128-key
// tiles its band needs (sched.cuh); the unit streams the union of the two
// strips through a 2-stage K/V ring:
//   S_t = Q_t K^T   tcgen05.mma, both operands from 128B-swizzled smem, fp32 in TMEM
//   P_t = exp2(S_t - m)   softmax warpgroup t, one thread per row; the
//                   distance predicate only on edge tiles; P_t written back
//                   as bf16 over the first half of S_t in TMEM
//   O_t += P_t V    tcgen05.mma with A = P_t read from TMEM, B = V from smem
// The running max is only moved (and O_t rescaled) when it grows by more than
// 2^8, so probabilities stay <= 256 and most tiles skip the rescale.  O and
// lse are written straight from registers; rows that precede their band get
// o = 0 and lse = -inf.
//
// Warp roles (384 threads): warps 0-3 tile 0, warps 4-7 tile 1 (thread r of a
// warpgroup owns row r = TMEM lane r), warp 8 TMA producer, warps 9 and 10
// MMA issuers of tile 0 and tile 1 (warp 9 also owns TMEM), warp 11 idle; the
// softmax warpgroups take most of the register file (setmaxnreg).  Every wait
// is bounded (common.cuh).
//
// Softmax restricted to a permitted set: "Story of Attention -- Part 4",
// section 1 (Sparse-Attention equation); bands: "Making Every Head Count",
// Figure 1 caption.
#pragma once

#include "common.cuh"

namespace spa {

template <int D>
struct FwdCfg {
  static constexpr int BQ = 128;        // rows per Q tile (one warpgroup)
  static constexpr int TILES = 2;       // Q tiles per unit
  static constexpr int BU = BQ * TILES; // rows per unit
  static constexpr int BK = 128;        // keys per K/V tile
  static constexpr int NS = 2;          // K/V ring stages
  static constexpr int DB = D / 64;     // 64-column (128-byte) blocks per row
  static constexpr uint32_t Q_BYTES = BQ * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + TILES * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * KV_BYTES;
  // + alignment slack; at least 116 KB so that one CTA (and its 512 TMEM
  // columns) owns an SM even for d = 64
  static constexpr uint32_t SMEM_BYTES =
      (OFF_BAR + 256 + 1024) > 116u * 1024 ? (OFF_BAR + 256 + 1024) : 116u * 1024;
  static constexpr int NTHREADS = 384;
  // register split: 384 threads launch with 168 registers each (64512); the
  // two softmax warpgroups take 200, the producer/MMA warpgroup 104.
  static constexpr uint32_t LAUNCH_REGS = 168, SOFTMAX_REGS = 200, CONTROL_REGS = 104;
  static_assert(2 * SOFTMAX_REGS + CONTROL_REGS <= 3 * LAUNCH_REGS, "register split over budget");
  static constexpr uint32_t TMEM_COLS = 512;
  // tile t: S_t (and P_t over its first 64 columns) at t*256, O_t at t*256 + 128
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return (uint32_t)t * 256u; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return (uint32_t)t * 256u + 128u; }
  static_assert(D == 64 || D == 128, "head dim");
};

struct FwdBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2];
  uint64_t turn[2];  // turn[t]: softmax warpgroup t may start its next step
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

// One unit of the forward: rows [i0, i0 + 256) of head (b, h).
struct FwdUnit {
  int bh;
  int32_t lo, hi;
  int64_t i0;
  int a[2], b[2];     // key-tile strip of each Q tile (b < a: tile inactive)
  bool act[2];
  int u0, u1;         // union of the active strips
};

template <int D>
__device__ __forceinline__ FwdUnit fwd_decode(int u, const AttnParams& p) {
  using C = FwdCfg<D>;
  FwdUnit U;
  const int b = u / p.units_per_batch;
  const int r = u % p.units_per_batch;
  const int h = head_of(p.unit_start, p.H, r);
  U.bh = b * p.H + h;
  U.lo = p.lo[h];
  U.hi = p.hi[h];
  U.i0 = (int64_t)(p.lo[h] / C::BU + (r - p.unit_start[h])) * C::BU;
  U.u0 = 1 << 30;
  U.u1 = -1;
  for (int t = 0; t < 2; ++t) {
    const int64_t it0 = U.i0 + (int64_t)t * C::BQ;
    Strip s{0, -1};
    if (it0 < p.N) s = key_strip(p.N, U.lo, U.hi, it0, C::BQ, C::BK);
    U.a[t] = s.begin;
    U.b[t] = s.end;
    U.act[t] = s.end >= s.begin;
    if (U.act[t]) {
      U.u0 = min(U.u0, s.begin);
      U.u1 = max(U.u1, s.end);
    }
  }
  return U;
}

// MERGE: o and lse hold, on entry, a softmax over another set of keys,
// disjoint from this kernel's bands (spa_attn_fwd_merge); each row is
// combined with it through the two lse values, and rows this kernel's bands
// do not reach are left as they are.
// TURN: the two softmax warpgroups take turns (below).  That pays when the
// key strips are long; with short strips (narrow bands) the turn order also
// serialises the pipeline's refill at every unit boundary, and the two
// warpgroups run freely instead.  The host picks from the band widths.
template <int D, bool MERGE = false, bool TURN = true>
__global__ void __launch_bounds__(384, 1)
    spa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t N = p.N;
  const int num_units = p.B * p.units_per_batch;

  const uint32_t sQ = ptx::smem_u32(smem + C::OFF_Q);
  const uint32_t sK = ptx::smem_u32(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_u32(smem + C::OFF_V);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->q_full[i], 1);
      ptx::mbar_init(&bars->q_empty[i], 1);
      ptx::mbar_init(&bars->k_full[i], 1);
      ptx::mbar_init(&bars->v_full[i], 1);
      ptx::mbar_init(&bars->kv_empty[i], 2);  // one release per MMA issuer
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
      ptx::mbar_init(&bars->o_done[i], 1);
      ptx::mbar_init(&bars->o_free[i], 128);
      ptx::mbar_init(&bars->turn[i], 128);
    }
    ptx::mbar_init(&bars->drain[0], 1);
    ptx::mbar_init(&bars->drain[1], 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  if (warp >= 8) {
    ptx::regs_dec<C::CONTROL_REGS>();
  if (warp == 11) {
    // idle warp of the control warpgroup
  } else if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int nq[2] = {0, 0}, armed[2] = {0, 0};
      int g = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const FwdUnit U = fwd_decode<D>(u, p);
        for (int t = 0; t < 2 && ok; ++t) {
          if (!U.act[t]) continue;
          ok = bar_wait(&bars->q_empty[t], (nq[t] & 1) ^ 1, abort_flag);
          if (!ok) break;
          ++nq[t];
          ptx::mbar_arrive_expect_tx(&bars->q_full[t], C::Q_BYTES);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + c * (C::BQ * 128), &tm_q, &bars->q_full[t],
                             c * 64, (int)(U.i0 + t * C::BQ), U.bh);
        }
        for (int it = U.u0; ok && it <= U.u1; ++it, ++g) {
          const int s = g % C::NS;
          ok = bar_wait(&bars->kv_empty[s], ((g / C::NS) & 1) ^ 1, abort_flag);
          if (!ok) break;
          const int j0 = it * C::BK;
          ptx::mbar_arrive_expect_tx(&bars->k_full[s], C::KV_BYTES);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_K + s * C::KV_BYTES + c * (C::BK * 128), &tm_k, &bars->k_full[s],
                             c * 64, j0, U.bh);
          ptx::mbar_arrive_expect_tx(&bars->v_full[s], C::KV_BYTES);
          for (int c = 0; c < C::DB; ++c)
            ptx::tma_load_3d(smem + C::OFF_V + s * C::KV_BYTES + c * (C::BK * 128), &tm_v, &bars->v_full[s],
                             c * 64, j0, U.bh);
          ++armed[s];
        }
      }
      // Exit path: every load this thread issued has landed before the CTA ends.
      for (int t = 0; t < 2; ++t)
        if (nq[t] > 0) bar_drain(&bars->q_full[t], (nq[t] - 1) & 1);
      for (int s = 0; s < C::NS; ++s)
        if (armed[s] > 0) {
          bar_drain(&bars->k_full[s], (armed[s] - 1) & 1);
          bar_drain(&bars->v_full[s], (armed[s] - 1) & 1);
        }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuers
    // warp 9 issues every MMA of Q tile 0, warp 10 those of Q tile 1; both
    // walk the unit's whole key range in the same order, so they agree on the
    // K/V ring, and each releases a K/V stage once (kv_empty counts two).
    const int t = warp - 9;
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, C::BK, false, false);
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(128, D, false, true);
      // descriptors of every operand buffer, built once; a K-step only adds
      // a constant offset to the start address
      const uint64_t dq = ptx::sdesc_sw128(sQ + t * C::Q_BYTES, 0, 1024);
      const uint64_t dk0 = ptx::sdesc_sw128(sK, 0, 1024), dk1 = ptx::sdesc_sw128(sK + C::KV_BYTES, 0, 1024);
      const uint64_t dv0 = ptx::sdesc_sw128(sV, C::BK * 128, 1024);
      const uint64_t dv1 = ptx::sdesc_sw128(sV + C::KV_BYTES, C::BK * 128, 1024);
      const uint32_t tS = tmem + C::tm_s(t), tO = tmem + C::tm_o(t);
      uint64_t* s_full = &bars->s_full[t];
      uint64_t* p_full = &bars->p_full[t];
      int cq = 0, cp = 0, co = 0;
      int g = 0;
      bool ok = true;
      auto issue_s = [&](int slot) {
        const uint64_t db = slot ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_bf16(tS, ptx::sdesc_advance(dq, (kk / 4) * (C::BQ * 128) + (kk % 4) * 32),
                        ptx::sdesc_advance(db, (kk / 4) * (C::BK * 128) + (kk % 4) * 32), idesc_s, kk > 0);
        ptx::mma_commit(s_full);
      };
      auto issue_pv = [&](int slot, bool first) {
        const uint64_t db = slot ? dv1 : dv0;
        ptx::mma_bf16_ts(tO, tS, db, idesc_o, !first);
#pragma unroll
        for (int kk = 1; kk < C::BK / 16; ++kk)
          ptx::mma_bf16_ts(tO, tS + kk * 8, ptx::sdesc_advance(db, kk * (16 * 128)), idesc_o, 1);
      };
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const FwdUnit U = fwd_decode<D>(u, p);
        if (U.u1 < U.u0) continue;
        const bool act_t = t ? U.act[1] : U.act[0];
        const int a_t = t ? U.a[1] : U.a[0];
        const int b_t = t ? U.b[1] : U.b[0];
        auto act = [&](int it) { return act_t && it >= a_t && it <= b_t; };
        const int g0 = g;
        auto slot = [&](int it) { return (g0 + it - U.u0) % C::NS; };
        auto ring_par = [&](int it) { return (uint32_t)(((g0 + it - U.u0) / C::NS) & 1); };
        if (act_t) ok = bar_wait(&bars->q_full[t], (cq++) & 1, abort_flag);
        bool first = true;
        ok = ok && bar_wait(&bars->k_full[slot(U.u0)], ring_par(U.u0), abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
        if (act(U.u0)) {
          issue_s(slot(U.u0));
          if (U.u0 == b_t) ptx::mma_commit(&bars->q_empty[t]);
        }
        for (int it = U.u0; ok && it <= U.u1; ++it) {
          const int s = slot(it);
          ok = bar_wait(&bars->v_full[s], ring_par(it), abort_flag);
          if (!ok) break;
          if (act(it)) {
            // O_t += P_t V, then release the stage (this tile's reads of it are issued)
            ok = bar_wait(p_full, (cp++) & 1, abort_flag);
            if (ok && first) ok = bar_wait(&bars->o_free[t], ((co++) & 1) ^ 1, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_pv(s, first);
            first = false;
            if (it == b_t) ptx::mma_commit(&bars->o_done[t]);
            ptx::mma_commit(&bars->kv_empty[s]);
          } else {
            ptx::mbar_arrive(&bars->kv_empty[s]);  // this tile does not use the stage
          }
          if (it + 1 <= U.u1) {
            // S_t of the next key tile
            ok = bar_wait(&bars->k_full[slot(it + 1)], ring_par(it + 1), abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            if (act(it + 1)) {
              issue_s(slot(it + 1));
              if (it + 1 == b_t) ptx::mma_commit(&bars->q_empty[t]);
            }
          }
        }
        g = g0 + (U.u1 - U.u0 + 1);
      }
      // Exit path: every MMA this thread issued has completed.
      ptx::mma_commit(&bars->drain[t]);
      bar_drain(&bars->drain[t], 0);
    }
    __syncwarp();
  }
  } else {
    ptx::regs_inc<C::SOFTMAX_REGS>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp / 4;                    // Q tile of this warpgroup
    const int r = threadIdx.x - 128 * t;       // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::tm_s(t);
    const uint32_t tO = tmem + lane_base + C::tm_o(t);
    int cs = 0, cd = 0;
    bool ok = true;
    // The two warpgroups take turns: within a unit their softmax steps run
    // one at a time in the order (key tile it, tile 0), (it, tile 1),
    // (it + 1, tile 0), ... so each one's special-function work overlaps the
    // tensor core's work on the other tile instead of both competing at
    // once.  At every change of owner the finishing warpgroup arrives on the
    // other's turn barrier.  Across units the order is not kept: each
    // warpgroup starts its next unit as soon as it can (1-2 % faster than
    // one order through the whole launch at band widths 768-1024).
    int turns = 0;        // waits on this warpgroup's turn barrier so far
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const FwdUnit U = fwd_decode<D>(u, p);
      auto actv = [&](int tt, int it) {
        return tt ? (U.act[1] && it >= U.a[1] && it <= U.b[1]) : (U.act[0] && it >= U.a[0] && it <= U.b[0]);
      };
      const int64_t it0 = U.i0 + (int64_t)t * C::BQ;
      const int64_t i = it0 + r;
      const bool act_t = t ? U.act[1] : U.act[0];
      const int a_t = t ? U.a[1] : U.a[0];
      const int b_t = t ? U.b[1] : U.b[0];
      uint16_t* orow = static_cast<uint16_t*>(p.o) + ((int64_t)U.bh * N + i) * D;
      if (!act_t) {
        // rows of this tile precede their band (or lie past N)
        if (!MERGE && i < N) {
          for (int c = 0; c < D; c += 8) ptx::st_global_v4(orow + c, 0u, 0u, 0u, 0u);
          p.lse[(int64_t)U.bh * N + i] = -INFINITY;
        }
        continue;
      }
      float m_ref = -INFINITY, l = 0.f;  // running max (base-2 units) and sum
      for (int it = a_t; it <= b_t; ++it) {
        int prev;
        if (t == 1 && actv(0, it)) prev = 0;
        else if (actv(1, it - 1)) prev = 1;
        else if (actv(0, it - 1)) prev = 0;
        else prev = -1;  // a unit's first step waits for no turn
        const int64_t j0 = (int64_t)it * C::BK;
        const bool interior = tile_is_interior(N, U.lo, U.hi, it0, C::BQ, j0, C::BK);
        // Edge tile: the permitted keys of this row are the columns c with
        // clo <= c <= clo + span (distance in [lo, hi), key and row inside N).
        int clo = 0;
        uint32_t span = 127;
        if (!interior) {
          const int64_t c_first = max64(i - U.hi + 1 - j0, 0);
          const int64_t c_last = min64(min64(i - U.lo - j0, N - 1 - j0), 127);
          if (i >= N || c_last < c_first) {
            clo = 128;
            span = 0;
          } else {
            clo = (int)c_first;
            span = (uint32_t)(c_last - c_first);
          }
        }
        // owner of the next step in this CTA's order
        int nxt = -1;
        if (t == 0 && actv(1, it)) nxt = 1;
        else if (actv(0, it + 1)) nxt = 0;
        else if (actv(1, it + 1)) nxt = 1;  // and a unit's last step passes none
        const bool pass_turn = nxt == 1 - t;
        const bool fast = __all_sync(0xffffffffu, m_ref != -INFINITY);
        ok = __all_sync(0xffffffffu, bar_wait(&bars->s_full[t], (cs++) & 1, abort_flag));
        if (!ok) break;
        if (TURN && prev == 1 - t)
          ok = __all_sync(0xffffffffu, bar_wait(&bars->turn[t], (turns++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        // Hand the turn over as soon as this step's exponentials are done
        // (before P is stored) if the next step belongs to the other tile.
        auto hand_turn = [&]() {
          if (TURN && pass_turn) ptx::mbar_arrive(&bars->turn[1 - t]);
        };
        // Fast path, for every tile after a row's first: exponentiate against
        // the current reference max while tracking this tile's max, keeping P
        // packed in registers.  Only if some row's max rose past the reference
        // by more than 2^8 is the tile redone by the two-pass path below (S is
        // still intact then: nothing has been stored over it).
        bool done = false;
        if (fast) {
          const float2 c2v = make_float2(p.scale_log2, p.scale_log2);
          const float2 mnv = make_float2(-m_ref, -m_ref);
          float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
          float mx0 = -INFINITY, mx1 = -INFINITY;
          uint32_t pk[2][32];
          uint32_t sr[2][32];
          ptx::tmem_ld32(tS, sr[0]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(sr[0]);
          // chunk q of the row: masked scores become -inf on edge tiles
#define SPA_FWD_FAST_CHUNKS(INTERIOR)                                                              \
  _Pragma("unroll") for (int q = 0; q < 4; ++q) {                                                  \
    if (q < 3) ptx::tmem_ld32(tS + (q + 1) * 32, sr[(q + 1) & 1]); /* next chunk in flight */      \
    const uint32_t* cur = sr[q & 1];                                                               \
    const int cb = q * 32 - clo;                                                                   \
    _Pragma("unroll") for (int e = 0; e < 32; e += 4) {                                            \
      float s0 = __uint_as_float(cur[e]), s1 = __uint_as_float(cur[e + 1]);                        \
      float s2 = __uint_as_float(cur[e + 2]), s3 = __uint_as_float(cur[e + 3]);                    \
      if (!(INTERIOR)) {                                                                           \
        s0 = (uint32_t)(cb + e) <= span ? s0 : -INFINITY;                                          \
        s1 = (uint32_t)(cb + e + 1) <= span ? s1 : -INFINITY;                                      \
        s2 = (uint32_t)(cb + e + 2) <= span ? s2 : -INFINITY;                                      \
        s3 = (uint32_t)(cb + e + 3) <= span ? s3 : -INFINITY;                                      \
      }                                                                                            \
      mx0 = ptx::fmax3(mx0, s0, s1);                                                               \
      mx1 = ptx::fmax3(mx1, s2, s3);                                                               \
      const float2 x01 = __ffma2_rn(make_float2(s0, s1), c2v, mnv);                                \
      const float2 x23 = __ffma2_rn(make_float2(s2, s3), c2v, mnv);                                \
      const float2 p01 = make_float2(ptx::exp2_approx(x01.x), ptx::exp2_approx(x01.y));            \
      const float2 p23 = make_float2(ptx::exp2_approx(x23.x), ptx::exp2_approx(x23.y));            \
      sa = __fadd2_rn(sa, p01);                                                                    \
      sb = __fadd2_rn(sb, p23);                                                                    \
      pk[q / 2][(q % 2) * 16 + e / 2] = ptx::pack_bf16x2(p01.x, p01.y);                            \
      pk[q / 2][(q % 2) * 16 + e / 2 + 1] = ptx::pack_bf16x2(p23.x, p23.y);                        \
    }                                                                                              \
    if (q < 3) {                                                                                   \
      ptx::tmem_wait_ld();                                                                         \
      ptx::reg_fence(sr[(q + 1) & 1]);                                                             \
    }                                                                                              \
  }
          if (interior) {
            SPA_FWD_FAST_CHUNKS(true)
          } else {
            SPA_FWD_FAST_CHUNKS(false)
          }
#undef SPA_FWD_FAST_CHUNKS
          const float c2 = p.scale_log2;
          const float sm0 = sa.x, sm1 = sa.y, sm2 = sb.x, sm3 = sb.y;
          const bool over = fmaxf(mx0, mx1) * c2 > m_ref + 8.f;
          if (!__any_sync(0xffffffffu, over)) {
            hand_turn();
            ptx::tmem_st32(tS, pk[0]);
            ptx::tmem_st32(tS + 32, pk[1]);
            l += (sm0 + sm1) + (sm2 + sm3);
            done = true;
          }
        }
        if (!done) {
          // pass 1: row max of the raw scores (scale > 0 commutes with max)
          float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
  #pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint32_t sr[32];
            ptx::tmem_ld32(tS + q * 32, sr);
            ptx::tmem_wait_ld();
            ptx::reg_fence(sr);
            if (interior) {
  #pragma unroll
              for (int e = 0; e < 32; e += 4) {
                mx0 = fmaxf(mx0, __uint_as_float(sr[e]));
                mx1 = fmaxf(mx1, __uint_as_float(sr[e + 1]));
                mx2 = fmaxf(mx2, __uint_as_float(sr[e + 2]));
                mx3 = fmaxf(mx3, __uint_as_float(sr[e + 3]));
              }
            } else {
              const int cb = q * 32 - clo;
  #pragma unroll
              for (int e = 0; e < 32; e += 4) {
                mx0 = fmaxf(mx0, (uint32_t)(cb + e) <= span ? __uint_as_float(sr[e]) : -INFINITY);
                mx1 = fmaxf(mx1, (uint32_t)(cb + e + 1) <= span ? __uint_as_float(sr[e + 1]) : -INFINITY);
                mx2 = fmaxf(mx2, (uint32_t)(cb + e + 2) <= span ? __uint_as_float(sr[e + 2]) : -INFINITY);
                mx3 = fmaxf(mx3, (uint32_t)(cb + e + 3) <= span ? __uint_as_float(sr[e + 3]) : -INFINITY);
              }
            }
          }
          const float m_new = fmaxf(m_ref, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * p.scale_log2);
          const bool need = m_new > m_ref + 8.f;   // also true for a row's first finite max
          const bool need_o = need && (m_ref != -INFINITY);
          float alpha = 1.f;
          if (need) {
            alpha = ptx::exp2_approx(m_ref - m_new);  // 0 while the row had seen nothing
            l *= alpha;
            m_ref = m_new;
          }
          if (__any_sync(0xffffffffu, need_o)) {
            // O_t is stable: the PV of the previous key tile completed before S_t did
            const float a = need_o ? alpha : 1.f;
  #pragma unroll 1
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              ptx::tmem_ld32(tO + c, o);
              ptx::tmem_wait_ld();
              ptx::reg_fence(o);
  #pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
              ptx::tmem_st32(tO + c, o);
            }
          }
          // pass 2: p = exp2(s * scale_log2 - m), bf16 pairs over the first half
          // of S_t (chunk q of P covers columns [16q, 16q+16), already read)
          const float c2 = p.scale_log2;
          const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
          float sm0 = 0.f, sm1 = 0.f, sm2 = 0.f, sm3 = 0.f;
  #pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint32_t sr[32];
            ptx::tmem_ld32(tS + q * 32, sr);
            ptx::tmem_wait_ld();
            ptx::reg_fence(sr);
            uint32_t pk[16];
            if (interior) {
              // every key permitted
  #pragma unroll
              for (int e = 0; e < 32; e += 4) {
                const float p0 = ptx::exp2_approx(fmaf(__uint_as_float(sr[e]), c2, mneg));
                const float p1 = ptx::exp2_approx(fmaf(__uint_as_float(sr[e + 1]), c2, mneg));
                const float p2 = ptx::exp2_approx(fmaf(__uint_as_float(sr[e + 2]), c2, mneg));
                const float p3 = ptx::exp2_approx(fmaf(__uint_as_float(sr[e + 3]), c2, mneg));
                sm0 += p0;
                sm1 += p1;
                sm2 += p2;
                sm3 += p3;
                pk[e / 2] = ptx::pack_bf16x2(p0, p1);
                pk[e / 2 + 1] = ptx::pack_bf16x2(p2, p3);
              }
            } else {
              const int cb = q * 32 - clo;
  #pragma unroll
              for (int e = 0; e < 32; e += 4) {
                float x0 = fmaf(__uint_as_float(sr[e]), c2, mneg);
                float x1 = fmaf(__uint_as_float(sr[e + 1]), c2, mneg);
                float x2 = fmaf(__uint_as_float(sr[e + 2]), c2, mneg);
                float x3 = fmaf(__uint_as_float(sr[e + 3]), c2, mneg);
                x0 = (uint32_t)(cb + e) <= span ? x0 : -INFINITY;
                x1 = (uint32_t)(cb + e + 1) <= span ? x1 : -INFINITY;
                x2 = (uint32_t)(cb + e + 2) <= span ? x2 : -INFINITY;
                x3 = (uint32_t)(cb + e + 3) <= span ? x3 : -INFINITY;
                const float p0 = ptx::exp2_approx(x0), p1 = ptx::exp2_approx(x1);
                const float p2 = ptx::exp2_approx(x2), p3 = ptx::exp2_approx(x3);
                sm0 += p0;
                sm1 += p1;
                sm2 += p2;
                sm3 += p3;
                pk[e / 2] = ptx::pack_bf16x2(p0, p1);
                pk[e / 2 + 1] = ptx::pack_bf16x2(p2, p3);
              }
            }
            ptx::tmem_st16(tS + q * 16, pk);
          }
          l += (sm0 + sm1) + (sm2 + sm3);
          hand_turn();
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full[t]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if constexpr (MERGE) {
        // The row already in o (lse1, o1) is combined with this part's.  In
        // base 2, with a = lse1 log2(e) and b = m + log2(l) this
        // part's lse: L = log2(2^a + 2^b), o = 2^(a - L) o1 + 2^(b - L) O / l.
        // A row this part leaves empty (l = 0) keeps o1 and lse1 unchanged.
        const float lse1 = i < N ? p.lse[(int64_t)U.bh * N + i] : -INFINITY;
        ok = __all_sync(0xffffffffu, bar_wait(&bars->o_done[t], (cd++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        const float a = lse1 * 1.4426950408889634f;
        const float b = (l > 0.f) ? m_ref + log2f(l) : -INFINITY;
        const bool write = i < N && b != -INFINITY;
        const float mx = fmaxf(a, b);
        const float L = write ? mx + ptx::log2_approx(ptx::exp2_approx(a - mx) + ptx::exp2_approx(b - mx)) : 0.f;
        const float w1 = write ? ptx::exp2_approx(a - L) : 0.f;
        const float w2 = write ? ptx::exp2_approx(b - L) / l : 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + c, o);
          ptx::tmem_wait_ld();
          ptx::reg_fence(o);
          if (write) {
            uint4 o1[4];  // part 1's 32 columns
#pragma unroll
            for (int e = 0; e < 4; ++e) o1[e] = reinterpret_cast<const uint4*>(orow + c)[e];
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 f1 = ptx::bf16x2_to_float2(ptx::word_of(o1[e / 4], e % 4));
              pk[e] = ptx::pack_bf16x2(fmaf(__uint_as_float(o[2 * e]), w2, w1 * f1.x),
                                       fmaf(__uint_as_float(o[2 * e + 1]), w2, w1 * f1.y));
            }
            ptx::st_global_v8(orow + c, pk);
            ptx::st_global_v8(orow + c + 16, pk + 8);
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->o_free[t]);
        if (write) p.lse[(int64_t)U.bh * N + i] = L * 0.69314718055994531f;
      } else {
        ok = __all_sync(0xffffffffu, bar_wait(&bars->o_done[t], (cd++) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + c, o);
          ptx::tmem_wait_ld();
          ptx::reg_fence(o);
          if (i < N) ptx::store_row32_bf16(orow + c, o, inv);
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->o_free[t]);
        if (i < N)
          p.lse[(int64_t)U.bh * N + i] = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  // ------------------------------------------------------------ empty blocks
  // Whole 256-row blocks that precede their head's band: o = 0, lse = -inf
  // (left as they are when merging).
  {
    const int num_fill = MERGE ? 0 : p.B * p.fills_per_batch;
    for (int f = blockIdx.x; f < num_fill; f += gridDim.x) {
      const int b = f / p.fills_per_batch;
      const int r = f % p.fills_per_batch;
      const int h = head_of(p.fill_start, p.H, r);
      const int64_t row0 = (int64_t)(b * p.H + h) * N + (int64_t)(r - p.fill_start[h]) * C::BU;
      zero_rows_bf16(static_cast<uint16_t*>(p.o) + row0 * D, C::BU, D);
      for (int e = threadIdx.x; e < C::BU; e += blockDim.x) p.lse[row0 + e] = -INFINITY;
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
