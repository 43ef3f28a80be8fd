// union.cuh -- attention over a head's band plus a local window shared by
// every head, composed from two band passes.
//
// In "Making Every Head Count", Figure 2(b), the EBALL ablation is the
// exclusive bands with local sharing taken out, which suggests that the full
// method may add distances [0, w) that every head attends to.  The pages
// define nothing more, so the permitted set read here is
//   S_i^h = { j <= i : i - j < w  or  lo_h <= i - j < hi_h }.
// The host splits each head's set into two disjoint, non-empty distance
// intervals (the window and the band when they do not touch, else the two
// halves of their union) and runs the band kernels once per part:
//  - forward: part 1 writes (o, lse), part 2 writes (o2, lse2); the merge
//    kernel forms softmax over the union from the two partial softmaxes,
//      L = log(e^lse + e^lse2),  o = e^(lse - L) o + e^(lse2 - L) o2;
//  - backward: P_ij = exp(s_ij - L_i) and D_i = dO_i . o_i are the same for
//    every key of the union, so each part's dq/dk/dv passes run with the
//    joint L and D and the two sets of gradients add (the add kernel).
#pragma once

#include "common.cuh"

namespace spa {

__device__ __forceinline__ void unpack8_bf16(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&f)[8]) {
  return make_uint4(ptx::pack_bf16x2(f[0], f[1]), ptx::pack_bf16x2(f[2], f[3]), ptx::pack_bf16x2(f[4], f[5]),
                    ptx::pack_bf16x2(f[6], f[7]));
}

// (o, lse) <- merge of (o, lse) and (o2, lse2), row by row; D / 8 threads per
// row (16 bytes each), rows of a warp never split across warps; grid-stride
// over the rows, every lane of a warp taking the same number of rounds.  A row
// with both parts empty stays o = 0, lse = -inf.
template <int D>
__global__ void __launch_bounds__(256) spa_union_merge_kernel(uint16_t* __restrict__ o, float* __restrict__ lse,
                                                              const uint16_t* __restrict__ o2,
                                                              const float* __restrict__ lse2, int64_t rows) {
  constexpr int TPR = D / 8;
  const int64_t total = rows * TPR;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride) {
    const int64_t t = base + threadIdx.x;
    const int64_t row = t / TPR;
    const int c = (int)(t % TPR);
    const bool valid = t < total;
    const float l1 = valid ? lse[row] : -INFINITY, l2 = valid ? lse2[row] : -INFINITY;
    // every lane of the row has read lse[row] before lane c = 0 rewrites it
    __syncwarp();
    if (!valid) continue;
    const float m = fmaxf(l1, l2);
    float L = -INFINITY, w1 = 0.f, w2 = 0.f;
    if (m != -INFINITY) {
      const float e1 = expf(l1 - m), e2 = expf(l2 - m);
      const float s = e1 + e2;
      L = m + logf(s);
      w1 = e1 / s;
      w2 = e2 / s;
    }
    uint4* po = reinterpret_cast<uint4*>(o + row * D) + c;
    const uint4 a = *po;
    const uint4 b = reinterpret_cast<const uint4*>(o2 + row * D)[c];
    float fa[8], fb[8];
    unpack8_bf16(a, fa);
    unpack8_bf16(b, fb);
#pragma unroll
    for (int e = 0; e < 8; ++e) fa[e] = w1 * fa[e] + w2 * fb[e];
    *po = pack8_bf16(fa);
    if (c == 0) lse[row] = L;
  }
}

// dst_t += src_t (bf16, summed in fp32, rounded once) for three tensors of
// n16 16-byte chunks each; grid-stride over 3 * n16 chunks.
__global__ void __launch_bounds__(256) spa_add3_bf16_kernel(uint16_t* __restrict__ d0, uint16_t* __restrict__ d1,
                                                            uint16_t* __restrict__ d2,
                                                            const uint16_t* __restrict__ s0,
                                                            const uint16_t* __restrict__ s1,
                                                            const uint16_t* __restrict__ s2, int64_t n16) {
  const int64_t total = 3 * n16;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int which = (int)(t / n16);
    const int64_t i = t - (int64_t)which * n16;
    uint16_t* d = which == 0 ? d0 : (which == 1 ? d1 : d2);
    const uint16_t* s = which == 0 ? s0 : (which == 1 ? s1 : s2);
    uint4* pd = reinterpret_cast<uint4*>(d) + i;
    float fa[8], fb[8];
    unpack8_bf16(*pd, fa);
    unpack8_bf16(reinterpret_cast<const uint4*>(s)[i], fb);
#pragma unroll
    for (int e = 0; e < 8; ++e) fa[e] += fb[e];
    *pd = pack8_bf16(fa);
  }
}

}  // namespace spa
