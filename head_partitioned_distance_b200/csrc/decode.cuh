// decode.cuh -- band-sparse attention for one new token per sequence (the
// inference step of the method: a query at position t of head h needs only
// the keys j with lo_h <= t - j < hi_h, i.e. at most the band's width of the
// cache; "Making Every Head Count", abstract and Figure 1 caption; softmax
// over the permitted set: "Story of Attention -- Part 4", section 1).
//
// Memory-bound: every key and value of the band is read once.  Split over
// the keys: spa_decode_chunk_kernel gives each (b, h, chunk of 256 keys) a
// CTA of four warps; four lanes share a key (a quarter of d each) for the
// scores, then each lane accumulates d/32 output columns over the warp's
// keys with an online max and sum.  The warps' partials merge in shared
// memory into one (m, l, o[d]) per chunk; spa_decode_merge_kernel merges the
// chunks of each (b, h) into o (bf16) and lse (natural log); it is launched
// as a programmatic dependent of the chunk kernel, so its launch overlaps the
// chunk kernel's last CTAs and it waits for that grid before reading.
#pragma once

#include "common.cuh"

namespace spa {

constexpr int kDecodeChunk = 256;  // keys per CTA
constexpr int kDecodeWarps = 4;    // 64 keys per warp, 8 at a time

struct DecodeParams {
  int B, H;
  int64_t N;
  int d;
  float scale_log2;
  int nchunk;  // chunks per (b, h) in the workspace
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* pos;
  uint16_t* o;
  float* lse;
  float* part;  // [B][H][nchunk][d + 2]: o partial, then m (base 2), l
  int32_t lo[kMaxHeads];
  int32_t hi[kMaxHeads];
};

// The band of keys that the query at position t of head h reads:
// j in [jlo, jhi]; empty when jhi < jlo (t outside [0, N) counts as empty).
__device__ __forceinline__ void decode_band(const DecodeParams& p, int h, int64_t t, int64_t* jlo, int64_t* jhi) {
  if (t < 0 || t >= p.N) {
    *jlo = 0;
    *jhi = -1;
    return;
  }
  *jlo = max64(0, t - (int64_t)p.hi[h] + 1);
  *jhi = t - (int64_t)p.lo[h];
}

template <int D>
__global__ void __launch_bounds__(128) spa_decode_chunk_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int QD = D / 4;    // dims per lane in the score (a quarter of d)
  constexpr int OD = D / 32;   // output dims per lane
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t bh = (int64_t)b * p.H + h;
  int64_t jlo, jhi;
  decode_band(p, h, (int64_t)p.pos[b], &jlo, &jhi);
  const int64_t c0 = jlo + (int64_t)c * kDecodeChunk;
  const int64_t c1 = min64(c0 + kDecodeChunk - 1, jhi);  // chunk keys [c0, c1]

  __shared__ float s_m[kDecodeWarps], s_l[kDecodeWarps];
  __shared__ float s_o[kDecodeWarps][D];

  // this lane's quarter of q, as floats
  float qv[QD];
  {
    const uint4* qp = reinterpret_cast<const uint4*>(p.q + bh * D + (lane % 4) * QD);
#pragma unroll
    for (int x = 0; x < QD / 8; ++x) {
      const uint4 u = qp[x];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const float2 f = ptx::bf16x2_to_float2(w4[y]);
        qv[8 * x + 2 * y] = f.x;
        qv[8 * x + 2 * y + 1] = f.y;
      }
    }
  }
  float m = -INFINITY, l = 0.f;  // base-2 running max and sum of this warp
  float acc[OD];
#pragma unroll
  for (int e = 0; e < OD; ++e) acc[e] = 0.f;

  const uint16_t* kh = p.k + bh * p.N * D;
  const uint16_t* vh = p.v + bh * p.N * D;
  const int64_t w0 = c0 + (int64_t)warp * (kDecodeChunk / kDecodeWarps);
#pragma unroll 1
  for (int g8 = 0; g8 < kDecodeChunk / kDecodeWarps; g8 += 8) {
    const int64_t kb = w0 + g8;  // keys kb .. kb + 7 of this group
    if (kb > c1) break;
    // every load of the group first (keys past c1 read as zero), so one
    // memory latency covers both the scores and the values
    const int64_t j = kb + lane / 4;  // this lane's key for the score
    uint4 kq[QD / 8];
#pragma unroll
    for (int x = 0; x < QD / 8; ++x) kq[x] = make_uint4(0u, 0u, 0u, 0u);
    if (j <= c1) {
      const uint4* kp = reinterpret_cast<const uint4*>(kh + j * D + (lane % 4) * QD);
#pragma unroll
      for (int x = 0; x < QD / 8; ++x) kq[x] = kp[x];
    }
    uint32_t vw[8][OD / 2];  // this lane's OD value columns of the group's 8 keys
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int e = 0; e < OD / 2; ++e) vw[kk][e] = 0u;
      if (kb + kk <= c1) {
        const uint16_t* vr = vh + (kb + kk) * D + OD * lane;
        if (OD == 4) {
          const uint2 u = *reinterpret_cast<const uint2*>(vr);
          vw[kk][0] = u.x;
          vw[kk][1 % (OD / 2)] = u.y;
        } else {
          vw[kk][0] = *reinterpret_cast<const uint32_t*>(vr);
        }
      }
    }
    // score of key j (masked past c1)
    float s = -INFINITY;
    if (j <= c1) {
      float2 a = make_float2(0.f, 0.f);
#pragma unroll
      for (int x = 0; x < QD / 8; ++x) {
        const uint32_t w4[4] = {kq[x].x, kq[x].y, kq[x].z, kq[x].w};
#pragma unroll
        for (int y = 0; y < 4; ++y)
          a = __ffma2_rn(ptx::bf16x2_to_float2(w4[y]), make_float2(qv[8 * x + 2 * y], qv[8 * x + 2 * y + 1]), a);
      }
      s = a.x + a.y;
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s = (s == -INFINITY) ? s : s * p.scale_log2;  // base-2 units
    // group max, then the running reference
    float gm = s;
    gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 4));
    gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 8));
    gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 16));
    const float m_new = fmaxf(m, gm);
    const float alpha = (m == -INFINITY) ? 0.f : ptx::exp2_approx(m - m_new);
    m = m_new;
    l *= alpha;
#pragma unroll
    for (int e = 0; e < OD; ++e) acc[e] *= alpha;
    const float pj = (s == -INFINITY) ? 0.f : ptx::exp2_approx(s - m);
    // sum of the group's 8 probabilities (one copy per key's four lanes)
    float ps = (lane % 4 == 0) ? pj : 0.f;
    ps += __shfl_xor_sync(0xffffffffu, ps, 4);
    ps += __shfl_xor_sync(0xffffffffu, ps, 8);
    ps += __shfl_xor_sync(0xffffffffu, ps, 16);
    l += ps;
    // o += p_j v_j over the group's keys; lane owns dims [OD lane, OD lane + OD)
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, pj, 4 * kk);  // 0 past c1
#pragma unroll
      for (int e = 0; e < OD / 2; ++e) {
        const float2 f = ptx::bf16x2_to_float2(vw[kk][e]);
        acc[2 * e] = fmaf(pk, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(pk, f.y, acc[2 * e + 1]);
      }
    }
  }
  // the merge kernel (launched as this grid's programmatic dependent) may
  // start its launch now; it reads nothing before this grid has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // merge the four warps
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < OD; ++e) s_o[warp][OD * lane + e] = acc[e];
  __syncthreads();
  float* out = p.part + ((bh * p.nchunk) + c) * (D + 2);
  float M = -INFINITY;
#pragma unroll
  for (int x = 0; x < kDecodeWarps; ++x) M = fmaxf(M, s_m[x]);
  float a[kDecodeWarps];
#pragma unroll
  for (int x = 0; x < kDecodeWarps; ++x) a[x] = (s_m[x] == -INFINITY) ? 0.f : ptx::exp2_approx(s_m[x] - M);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int x = 0; x < kDecodeWarps; ++x) o = fmaf(a[x], s_o[x][e], o);
    out[e] = o;
  }
  if (threadIdx.x == 0) {
    float L = 0.f;
#pragma unroll
    for (int x = 0; x < kDecodeWarps; ++x) L = fmaf(a[x], s_l[x], L);
    out[D] = M;
    out[D + 1] = L;
  }
}

// Merge the chunks of each (b, h): o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
template <int D>
__global__ void __launch_bounds__(128) spa_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  // launched as the chunk kernel's programmatic dependent: wait until that
  // grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t bh = (int64_t)b * p.H + h;
  int64_t jlo, jhi;
  decode_band(p, h, (int64_t)p.pos[b], &jlo, &jhi);
  const int used = jhi < jlo ? 0 : (int)((jhi - jlo) / kDecodeChunk) + 1;  // chunks written
  const float* part = p.part + bh * p.nchunk * (D + 2);
  float M = -INFINITY;
  for (int c = 0; c < used; ++c) M = fmaxf(M, part[c * (D + 2) + D]);
  float L = 0.f;
  for (int c = 0; c < used; ++c) {
    const float mc = part[c * (D + 2) + D];
    if (mc != -INFINITY) L = fmaf(ptx::exp2_approx(mc - M), part[c * (D + 2) + D + 1], L);
  }
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
    for (int c = 0; c < used; ++c) {
      const float mc = part[c * (D + 2) + D];
      if (mc != -INFINITY) o = fmaf(ptx::exp2_approx(mc - M), part[c * (D + 2) + e], o);
    }
    const float val = o * inv;
    p.o[bh * D + e] = (uint16_t)(ptx::pack_bf16x2(val, 0.f) & 0xffffu);
  }
  if (threadIdx.x == 0) p.lse[bh] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace spa
