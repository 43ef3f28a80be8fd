// common.cuh -- pieces shared by the kernels: launch parameters, the device
// error word, and bounded mbarrier waits.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "ptx.cuh"
#include "sched.cuh"

namespace spa {

constexpr int kMaxHeads = 256;

// Status codes mirrored from spa.h (kept numerically identical).
constexpr int kStatusOk = 0;
constexpr int kStatusUnsupported = 2;
constexpr int kStatusTimeout = 4;

// Opt-in dynamic shared memory per block on sm_100 (227 KB).
constexpr uint32_t kMaxSmemPerBlock = 232448;

// Longest a thread waits on one mbarrier phase before the kernel gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Longest the exit path waits for its own copies and MMAs in flight.
constexpr uint64_t kDrainLimitNs = 200000000ull;

struct AttnParams {
  int B;
  int H;
  int64_t N;
  float scale;        // multiplies q.k
  float scale_log2;   // scale * log2(e): scores in base-2 units
  // Work list of a persistent grid, per batch: the kernel's units (tiles it
  // computes) and fills (tiles it only zeroes), head by head.  The units of
  // head h are numbers [unit_start[h], unit_start[h + 1]) of the batch, the
  // fills [fill_start[h], fill_start[h + 1]); unit_start[H] = units_per_batch.
  int units_per_batch;
  int fills_per_batch;
  // forward: lse is written; backward: lse (read) and delta (workspace)
  float* lse;
  float* delta;
  // raw pointers, for the rows that empty units write directly
  void* o;
  void* dq;
  void* dk;
  void* dv;
  const void* o_in;
  const void* dout;
  float* dq_acc;      // fused backward: fp32 dQ sums, [B, H, N, d]
  // stored-dS backward: the dS^T buffer's tiles of head h start at tile
  // ds_base[h]; each of its B x (key tiles some query reaches) key tiles owns
  // ds_len[h] consecutive tiles (stored_slot)
  int64_t ds_base[kMaxHeads];
  int32_t ds_len[kMaxHeads];
  void* ds;  // the dS^T tiles (layout in bwd_stored.cuh)
  int32_t lo[kMaxHeads];
  int32_t hi[kMaxHeads];
  int32_t unit_start[kMaxHeads + 1];
  int32_t fill_start[kMaxHeads + 1];
};

// Index of the 128 x 128 dS^T tile of (b, h, key tile u, query tile t) in
// the stored-dS backward's buffer.  Head h's key tiles 0 .. reached - 1 of
// batch b own ds_len[h] consecutive tiles each, one per query tile of the
// key tile's strip from its first, qa.
__host__ __device__ __forceinline__ int64_t stored_slot(const AttnParams& p, int b, int h, int u, int t, int qa) {
  const int64_t reached = (p.N - 1 - p.lo[h]) / 128 + 1;
  return p.ds_base[h] + ((int64_t)b * reached + u) * p.ds_len[h] + (t - qa);
}

// Head whose range [start[h], start[h + 1]) holds r, for 0 <= r < start[H]:
// the number of k in [1, H] with start[k] <= r (start is non-decreasing).
// Eight independent parameter loads per round rather than a dependent chain
// of one load per head.
__device__ __forceinline__ int head_of(const int32_t* start, int H, int r) {
  int h = 0;
#pragma unroll 1
  for (int base = 1; base <= H; base += 8) {
    int n = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) n += start[min(base + k, H)] <= r ? 1 : 0;
    h += n;
    if (n < 8) break;
  }
  return h;
}

// The library's device error word: a kernel that times out on a wait stores
// kStatusTimeout here; spa_device_status() reads and clears it.
__device__ int g_spa_status;

// Bounded wait on one mbarrier phase.  Returns false when the CTA aborted:
// either this wait ran past kWaitLimitNs (it then raises the CTA's abort flag
// and the device error word) or another thread already raised the flag.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t a = ptx::smem_u32(bar);
  if (ptx::mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int n = 0; n < 32; ++n)
      if (ptx::mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicExch(&g_spa_status, kStatusTimeout);
      return false;
    }
  }
}

// Wait used on the exit path only: gives up silently after kDrainLimitNs.
__device__ __forceinline__ bool bar_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t a = ptx::smem_u32(bar);
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(a, parity)) {
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) {
      atomicExch(&g_spa_status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// True when `used` bytes from the aligned base stay inside the launch's
// dynamic shared memory.  Otherwise the device error word becomes
// kStatusUnsupported and the caller returns before touching shared memory
// (the condition is the same for every thread of the block).
__device__ __forceinline__ bool smem_fits(const uint8_t* raw, const uint8_t* aligned, uint32_t used) {
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const bool fits = (uint32_t)(aligned - raw) + used <= dyn;
  if (!fits && threadIdx.x == 0) atomicExch(&g_spa_status, kStatusUnsupported);
  return fits;
}

// Zero `rows` rows of a [.., d] bf16 matrix starting at `base` (16-byte
// stores, all threads of the CTA cooperating).
__device__ __forceinline__ void zero_rows_bf16(void* base, int64_t rows, int d) {
  uint4* p = reinterpret_cast<uint4*>(base);
  const int64_t n16 = rows * d / 8;
  for (int64_t e = threadIdx.x; e < n16; e += blockDim.x) p[e] = make_uint4(0, 0, 0, 0);
}

}  // namespace spa
