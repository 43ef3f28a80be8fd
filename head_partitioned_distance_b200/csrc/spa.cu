// spa.cu -- the C ABI of libspa.so (declared in include/spa.h): argument
// checks, TMA tensor maps, and kernel launches.  One translation unit so the
// device error word is shared by every kernel without relocatable code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "spa.h"

#include "bwd.cuh"
#include "bwd_fused.cuh"
#include "bwd_stored.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "fwd.cuh"
#include "sched.cuh"
#include "union.cuh"

namespace {

using spa::AttnParams;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*H][N][d] bf16 tensor viewed as 3-D (d, N, B*H); box = 64 columns x rows x 1,
// 128-byte swizzle (matches the kernels' shared-memory layout), zero fill
// outside the tensor.
int make_map(CUtensorMap* m, const void* ptr, int64_t N, int64_t BH, int d, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return SPA_ERR_CUDA;
  // The encoder is a driver call and needs a current context; a thread that
  // has made no runtime call yet (an autograd worker, say) has none.
  // cudaSetDevice makes the device's primary context current for the thread.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return SPA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * (cuuint64_t)d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SPA_OK : SPA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int B, int H, int64_t N, int d) {
  if (B < 1 || H < 1 || N < 1) return SPA_ERR_INVAL;
  if (N > 2147483647LL) return SPA_ERR_INVAL;
  if (B > 65535 || H > spa::kMaxHeads) return SPA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return SPA_ERR_UNSUPPORTED;
  return SPA_OK;
}

// Fill p.lo/p.hi from explicit bands (lo/hi non-null) or from Balanced
// Distance Partitioning.
int fill_bands(AttnParams& p, int H, int64_t N, const int32_t* lo, const int32_t* hi) {
  if ((lo == nullptr) != (hi == nullptr)) return SPA_ERR_INVAL;
  if (lo == nullptr) {
    if (H > N) return SPA_ERR_INVAL;
    for (int h = 0; h < H; ++h) spa::band_of_head(N, H, h, &p.lo[h], &p.hi[h]);
    return SPA_OK;
  }
  for (int h = 0; h < H; ++h) {
    if (lo[h] < 0 || lo[h] >= hi[h] || (int64_t)hi[h] > N) return SPA_ERR_INVAL;
    p.lo[h] = lo[h];
    p.hi[h] = hi[h];
  }
  return SPA_OK;
}

// Opt a kernel into its dynamic shared memory once per device.
template <typename K>
int prepare_kernel(K kernel, uint32_t smem_bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPA_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_acquire) & bit) return SPA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes) !=
      cudaSuccess)
    return SPA_ERR_CUDA;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return SPA_OK;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? SPA_OK : SPA_ERR_CUDA; }

// A kernel that re-splits its registers between warpgroups (setmaxnreg) must
// have been compiled to exactly the per-thread count the split was budgeted
// for; otherwise an increase could wait for registers that never come.
template <typename K>
int check_regs(K kernel, int want, std::atomic<int>& verdict) {
  int v = verdict.load(std::memory_order_acquire);
  if (v == 0) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return SPA_ERR_CUDA;
    v = (a.numRegs == want) ? 1 : 2;
    verdict.store(v, std::memory_order_release);
  }
  return v == 1 ? SPA_OK : SPA_ERR_UNSUPPORTED;
}

int sm_count(int* n) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPA_ERR_CUDA;
  const int slot = dev & 63;
  int v = cache[slot].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return SPA_ERR_CUDA;
    cache[slot].store(v, std::memory_order_relaxed);
  }
  *n = v;
  return SPA_OK;
}

// Per-head work lists of a persistent grid: unit and fill counts of head h
// from units_of(h) and fills_of(h), stored as prefix sums in p.
template <class Units, class Fills>
int set_work_lists(AttnParams& p, Units units_of, Fills fills_of) {
  int64_t u = 0, f = 0;
  for (int h = 0; h < p.H; ++h) {
    p.unit_start[h] = (int32_t)u;
    p.fill_start[h] = (int32_t)f;
    u += units_of(h);
    f += fills_of(h);
    if (u > 2147483647LL || f > 2147483647LL) return SPA_ERR_UNSUPPORTED;
  }
  if ((int64_t)p.B * u > 2147483647LL || (int64_t)p.B * f > 2147483647LL) return SPA_ERR_UNSUPPORTED;
  p.unit_start[p.H] = (int32_t)u;
  p.fill_start[p.H] = (int32_t)f;
  p.units_per_batch = (int)u;
  p.fills_per_batch = (int)f;
  return SPA_OK;
}

// mean band width from which the forward's softmax warpgroups take turns
constexpr int64_t kFwdTurnMinWidth = 768;

template <int D>
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, AttnParams& p,
             cudaStream_t stream, bool merge) {
  using C = spa::FwdCfg<D>;
  // one (prepared, register check) pair per kernel instantiation:
  // [merging][turns]
  static std::atomic<uint64_t> prepared[2][2];
  static std::atomic<int> regs_ok[2][2];
  // The softmax warpgroups take turns when the bands are wide on average:
  // measured on B1 H32 N32768 d128 (forward, turns / no turns): width 768
  // 0.351 / 0.359 ms, 1024 0.415 / 0.440, 2048 0.683 / 0.769; at 512 turns
  // kept through the whole launch were 6 % slower (0.292 / 0.276).
  int64_t width_sum = 0;
  for (int h = 0; h < p.H; ++h) width_sum += (int64_t)(p.hi[h] - p.lo[h]);
  const bool turn = width_sum >= kFwdTurnMinWidth * (int64_t)p.H;
  auto* kernel = merge ? (turn ? spa::spa_fwd_kernel<D, true, true> : spa::spa_fwd_kernel<D, true, false>)
                       : (turn ? spa::spa_fwd_kernel<D, false, true> : spa::spa_fwd_kernel<D, false, false>);
  const int64_t BH = (int64_t)p.B * p.H;
  CUtensorMap mq, mk, mv;
  int st;
  if ((st = make_map(&mq, q, p.N, BH, D, C::BQ)) || (st = make_map(&mk, k, p.N, BH, D, C::BK)) ||
      (st = make_map(&mv, v, p.N, BH, D, C::BK)))
    return st;
  if ((st = prepare_kernel(kernel, C::SMEM_BYTES, prepared[merge][turn]))) return st;
  if ((st = check_regs(kernel, (int)C::LAUNCH_REGS, regs_ok[merge][turn]))) return st;
  // Work list of the persistent grid: per batch, every 256-row block of every
  // head from the one holding lo_h on (units), and the blocks before it (fills).
  const int64_t nblk = (p.N + C::BU - 1) / C::BU;
  if ((st = set_work_lists(
           p, [&](int h) { return nblk - p.lo[h] / C::BU; }, [&](int h) { return (int64_t)(p.lo[h] / C::BU); })))
    return st;
  const int64_t upb = p.units_per_batch;
  p.lse = lse;
  p.o = o;
  int sms = 0;
  if ((st = sm_count(&sms))) return st;
  const int64_t units = (int64_t)p.B * upb;
  const unsigned grid = (unsigned)(units < sms ? units : sms);
  kernel<<<grid, C::NTHREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  return launch_status();
}

// Backward steps.  The full backward runs the dQ pass first, forming D there
// (kStepDqDelta), then the dK/dV pass reading it; the separate D kernel
// serves the three-step entry points.  kStepAccumulate makes the dQ and dK/dV
// passes add to their outputs (the second part of the band-plus-window
// backward).
// The stored-dS backward runs D, then the dK/dV pass writing every tile
// pair's dS^T to `ds` (the layout of stored_layout), then kStepDqStored.
enum BwdStep {
  kStepDelta = 1,
  kStepDkDv = 2,
  kStepDq = 4,
  kStepDqDelta = 8,
  kStepAccumulate = 16,
  kStepDqStored = 32,
  kStepDeltaBand = 64,  // D of the rows the dK/dV pass reads only
  kStepAll = kStepDqDelta | kStepDkDv,
  kStepStored = kStepDeltaBand | kStepDkDv | kStepDqStored
};

// The stored-dS backward's workspace: D (fp32 [B H N], padded to 1024
// bytes), then the dS^T tiles, 128 x 128 bf16 each.  Head h owns, for each
// batch and each key tile some query reaches, ds_len[h] consecutive tiles:
// a key tile's query strip starts at tile u + lo / 128 and ends at most at
// u + (hi + 126) / 128, so it has at most (hi + 126) / 128 - lo / 128 + 1
// tiles.  Fills p.ds_base / p.ds_len (bands already in p) and returns the
// number of tiles, or -1 when it does not fit the kernels' 32-bit tile index.
constexpr size_t kStoredTileBytes = 128 * 128 * 2;
size_t stored_delta_bytes(int64_t rows) { return (size_t)((rows * 4 + 1023) & ~int64_t(1023)); }
int64_t stored_layout(AttnParams& p) {
  int64_t n = 0;
  for (int h = 0; h < p.H; ++h) {
    p.ds_base[h] = n;
    p.ds_len[h] = (int32_t)((p.hi[h] + 126LL) / 128 - p.lo[h] / 128 + 1);
    n += (int64_t)p.B * ((p.N - 1 - p.lo[h]) / 128 + 1) * p.ds_len[h];
    if (n > 2147483647LL) return -1;
  }
  return n;
}

template <int D>
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, float* delta, AttnParams& p,
             cudaStream_t stream, int steps, void* ds = nullptr) {
  using KC = spa::DkvCfg<D>;
  using QC = spa::DqCfg<D>;
  // one (prepared, register check) pair per kernel instantiation: [adding],
  // and the dK/dV pass that also stores dS^T
  static std::atomic<uint64_t> prepared_kv[2], prepared_q[2], prepared_kvs, prepared_qs;
  static std::atomic<int> regs_kv[2], regs_q[2], regs_kvs;
  const bool acc = (steps & kStepAccumulate) != 0;
  const int64_t BH = (int64_t)p.B * p.H;
  int st;
  p.lse = const_cast<float*>(lse);
  p.delta = delta;
  p.ds = ds;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  if (steps & kStepDelta) {
    const int64_t rows = BH * p.N;
    const int64_t threads = rows * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 2147483647LL) return SPA_ERR_UNSUPPORTED;
    spa::spa_bwd_delta_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), delta, rows);
    if ((st = launch_status())) return st;
  }
  if (steps & kStepDeltaBand) {
    // about eight blocks per SM: the (b, h) pairs on y, each pair's rows on x
    int sms = 0;
    if ((st = sm_count(&sms))) return st;
    const int64_t target = (int64_t)sms * 8;
    const unsigned gy = (unsigned)(BH < 65535 ? BH : 65535);
    const int64_t rows_blocks = (p.N + (256 / (D / 8)) - 1) / (256 / (D / 8));
    int64_t gx = (target + gy - 1) / gy;
    gx = gx < rows_blocks ? gx : rows_blocks;
    spa::spa_bwd_delta_band_kernel<D><<<dim3((unsigned)gx, gy), 256, 0, stream>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), p);
    if ((st = launch_status())) return st;
  }
  if (steps & (kStepDq | kStepDqDelta)) {
    // persistent grid over query tiles of 128 with a row inside its band; the
    // whole tiles before the band only get zero rows.  With kStepDqDelta the
    // kernel also forms D (from o and dout) and writes it to the workspace.
    const bool fuse_d = (steps & kStepDqDelta) != 0;
    CUtensorMap qq, qk, qv, qdo, qo;
    if ((st = make_map(&qq, q, p.N, BH, D, QC::BQ)) || (st = make_map(&qk, k, p.N, BH, D, QC::BK)) ||
        (st = make_map(&qv, v, p.N, BH, D, QC::BK)) || (st = make_map(&qdo, dout, p.N, BH, D, QC::BQ)) ||
        (st = make_map(&qo, fuse_d ? o : dout, p.N, BH, D, QC::BQ)))
      return st;
    p.o_in = fuse_d ? o : nullptr;
    auto* kernel_q = acc ? spa::spa_bwd_dq_kernel<D, true> : spa::spa_bwd_dq_kernel<D, false>;
    if ((st = prepare_kernel(kernel_q, QC::SMEM_BYTES, prepared_q[acc]))) return st;
    if ((st = check_regs(kernel_q, (int)QC::LAUNCH_REGS, regs_q[acc]))) return st;
    const int64_t nqt = (p.N + 127) / 128;
    if ((int64_t)p.B * p.H * nqt > 2147483647LL) return SPA_ERR_UNSUPPORTED;
    if ((st = set_work_lists(
             p, [&](int h) { return nqt - p.lo[h] / 128; }, [&](int h) { return (int64_t)(p.lo[h] / 128); })))
      return st;
    const int64_t upb = p.units_per_batch;
    int sms = 0;
    if ((st = sm_count(&sms))) return st;
    const int64_t units = (int64_t)p.B * upb;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    kernel_q<<<grid, QC::NTHREADS, QC::SMEM_BYTES, stream>>>(qq, qk, qv, qdo, qo, p);
    if ((st = launch_status())) return st;
  }
  if (steps & kStepDkDv) {
    // persistent grid over key tiles of 128 that some query reaches; the
    // other key tiles only get zero rows
    // dk and dv leave through bulk tensor stores of 32-row boxes
    CUtensorMap kq, kk, kv, kdo, kdk, kdv;
    if ((st = make_map(&kq, q, p.N, BH, D, KC::BQ)) || (st = make_map(&kk, k, p.N, BH, D, KC::BK)) ||
        (st = make_map(&kv, v, p.N, BH, D, KC::BK)) || (st = make_map(&kdo, dout, p.N, BH, D, KC::BQ)) ||
        (st = make_map(&kdk, dk, p.N, BH, D, 32)) || (st = make_map(&kdv, dv, p.N, BH, D, 32)))
      return st;
    const int64_t nkt = (p.N + 127) / 128;
    auto* kernel_kv = ds ? spa::spa_bwd_dkdv_kernel<D, false, true>
                         : (acc ? spa::spa_bwd_dkdv_kernel<D, true> : spa::spa_bwd_dkdv_kernel<D, false>);
    if ((st = prepare_kernel(kernel_kv, KC::SMEM_BYTES, ds ? prepared_kvs : prepared_kv[acc]))) return st;
    if ((st = check_regs(kernel_kv, (int)KC::LAUNCH_REGS, ds ? regs_kvs : regs_kv[acc]))) return st;
    if ((int64_t)p.B * p.H * nkt > 2147483647LL) return SPA_ERR_UNSUPPORTED;
    if ((st = set_work_lists(
             p, [&](int h) { return (p.N - 1 - p.lo[h]) / 128 + 1; },
             [&](int h) { return nkt - ((p.N - 1 - p.lo[h]) / 128 + 1); })))
      return st;
    const int64_t upb = p.units_per_batch;
    int sms = 0;
    if ((st = sm_count(&sms))) return st;
    const int64_t units = (int64_t)p.B * upb;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    kernel_kv<<<grid, KC::NTHREADS, KC::SMEM_BYTES, stream>>>(kq, kk, kv, kdo, kdk, kdv, p);
    if ((st = launch_status())) return st;
  }
  if (steps & kStepDqStored) {
    // persistent grid over query tiles of 128 with a row inside its band,
    // contracting the stored dS tiles with K; whole tiles before the band
    // only get zero rows
    using SC = spa::DqStoredCfg<D>;
    if (!ds) return SPA_ERR_INVAL;
    const int64_t nqt = (p.N + 127) / 128;
    CUtensorMap mk;
    if ((st = make_map(&mk, k, p.N, BH, D, SC::BK))) return st;
    auto* kernel_qs = spa::spa_bwd_dq_stored_kernel<D>;
    if ((st = prepare_kernel(kernel_qs, SC::SMEM_BYTES, prepared_qs))) return st;
    if ((int64_t)p.B * p.H * nqt > 2147483647LL) return SPA_ERR_UNSUPPORTED;
    if ((st = set_work_lists(
             p, [&](int h) { return nqt - p.lo[h] / 128; }, [&](int h) { return (int64_t)(p.lo[h] / 128); })))
      return st;
    int sms = 0;
    if ((st = sm_count(&sms))) return st;
    const int64_t units = (int64_t)p.B * p.units_per_batch;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    kernel_qs<<<grid, SC::NTHREADS, SC::SMEM_BYTES, stream>>>(mk, p);
    if ((st = launch_status())) return st;
  }
  return SPA_OK;
}



// Bytes of the fused backward's workspace: D (fp32 [B H N], padded to 256
// bytes) then the fp32 dQ sums [B H N d].
size_t fused_delta_bytes(int64_t rows) { return (size_t)((rows * 4 + 255) & ~int64_t(255)); }

// The fused backward: D and the zeroed dQ sums (prep kernel), the one pass
// over key tiles (dK, dV and the dQ sums), dq from the sums (convert kernel).
enum FusedStep { kFusedPrep = 1, kFusedPass = 2, kFusedConvert = 4, kFusedAll = 7 };

template <int D>
int fused_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, void* workspace, AttnParams& p, cudaStream_t stream, int steps) {
  using C = spa::FusedCfg<D>;
  static std::atomic<uint64_t> prepared;
  static std::atomic<int> regs_ok;
  const int64_t BH = (int64_t)p.B * p.H;
  const int64_t rows = BH * p.N;
  int st;
  p.lse = const_cast<float*>(lse);
  p.delta = static_cast<float*>(workspace);
  p.dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + fused_delta_bytes(rows));
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.o_in = o;
  p.dout = dout;
  int sms = 0;
  if ((st = sm_count(&sms))) return st;
  const int64_t cap = (int64_t)sms * 8;
  const int64_t want = (rows * (D / 8) + 255) / 256;
  const unsigned eblocks = (unsigned)(want < cap ? want : cap);
  if (steps & kFusedPrep) {
    spa::spa_bwd_fused_prep_kernel<D><<<eblocks, 256, 0, stream>>>(p);
    if ((st = launch_status())) return st;
  }
  if (steps & kFusedPass) {
  CUtensorMap kq, kk, kv, kdo, kdk, kdv;
  if ((st = make_map(&kq, q, p.N, BH, D, C::BQ)) || (st = make_map(&kk, k, p.N, BH, D, C::BK)) ||
      (st = make_map(&kv, v, p.N, BH, D, C::BK)) || (st = make_map(&kdo, dout, p.N, BH, D, C::BQ)) ||
      (st = make_map(&kdk, dk, p.N, BH, D, 32)) || (st = make_map(&kdv, dv, p.N, BH, D, 32)))
    return st;
  auto* kernel = spa::spa_bwd_fused_kernel<D>;
  if ((st = prepare_kernel(kernel, C::SMEM_BYTES, prepared))) return st;
  if ((st = check_regs(kernel, (int)C::LAUNCH_REGS, regs_ok))) return st;
  const int64_t nkt = (p.N + 127) / 128;
  if (BH * nkt > 2147483647LL) return SPA_ERR_UNSUPPORTED;
  if ((st = set_work_lists(
           p, [&](int h) { return (p.N - 1 - p.lo[h]) / 128 + 1; },
           [&](int h) { return nkt - ((p.N - 1 - p.lo[h]) / 128 + 1); })))
    return st;
  const int64_t units = (int64_t)p.B * p.units_per_batch;
  const unsigned grid = (unsigned)(units < sms ? units : sms);
  kernel<<<grid, C::NTHREADS, C::SMEM_BYTES, stream>>>(kq, kk, kv, kdo, kdk, kdv, p);
  if ((st = launch_status())) return st;
  }
  if (steps & kFusedConvert) {
    spa::spa_bwd_dq_convert_kernel<D><<<eblocks, 256, 0, stream>>>(p);
    if ((st = launch_status())) return st;
  }
  return SPA_OK;
}

int fwd_entry(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
              int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi, void* stream,
              bool merge = false) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!q || !k || !v || !o || !lse) return SPA_ERR_INVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SPA_ERR_INVAL;
  // o leaves in 32-byte stores
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 32) || !aligned(lse, 4))
    return SPA_ERR_UNSUPPORTED;
  static AttnParams zero{};
  AttnParams p = zero;
  p.B = B;
  p.H = H;
  p.N = N;
  p.scale = scale;
  p.scale_log2 = scale * spa::kLog2e;
  if ((st = fill_bands(p, H, N, lo, hi))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? fwd_impl<64>(q, k, v, o, lse, p, s, merge) : fwd_impl<128>(q, k, v, o, lse, p, s, merge);
}

int bwd_entry(const void* q, const void* k, const void* v, const void* o, const void* dout,
              const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H, int64_t N,
              int d, float scale, const int32_t* lo, const int32_t* hi, void* stream, int steps) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  // every step reads the workspace (D); each checks the tensors it touches
  if (!workspace) return SPA_ERR_INVAL;
  if ((steps & (kStepDelta | kStepDqDelta)) && (!o || !dout)) return SPA_ERR_INVAL;
  if ((steps & (kStepDkDv | kStepDq | kStepDqDelta)) && (!q || !k || !v || !dout || !lse)) return SPA_ERR_INVAL;
  if ((steps & kStepDkDv) && (!dk || !dv)) return SPA_ERR_INVAL;
  if ((steps & (kStepDq | kStepDqDelta)) && !dq) return SPA_ERR_INVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SPA_ERR_INVAL;
  for (const void* t : {q, k, v, o, dout})
    if (t && !aligned(t, 16)) return SPA_ERR_UNSUPPORTED;
  // the gradients leave in 32-byte stores
  for (const void* t : {(const void*)dq, (const void*)dk, (const void*)dv})
    if (t && !aligned(t, 32)) return SPA_ERR_UNSUPPORTED;
  if ((lse && !aligned(lse, 4)) || !aligned(workspace, 4)) return SPA_ERR_UNSUPPORTED;
  static AttnParams zero{};
  AttnParams p = zero;
  p.B = B;
  p.H = H;
  p.N = N;
  p.scale = scale;
  p.scale_log2 = scale * spa::kLog2e;
  if ((st = fill_bands(p, H, N, lo, hi))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* delta = static_cast<float*>(workspace);
  return d == 64 ? bwd_impl<64>(q, k, v, o, dout, lse, dq, dk, dv, delta, p, s, steps)
                 : bwd_impl<128>(q, k, v, o, dout, lse, dq, dk, dv, delta, p, s, steps);
}

// ---------------------------------------------------------------------------
// Band plus shared window (union.cuh): each head's permitted distances
// [0, w) u [lo_h, hi_h) as two disjoint, non-empty parts [a1, b1), [a2, b2):
// the window and the band when they do not touch, else the two halves of
// [0, max(w, hi_h)).
struct UnionParts {
  int32_t a1[spa::kMaxHeads], b1[spa::kMaxHeads], a2[spa::kMaxHeads], b2[spa::kMaxHeads];
};

int union_parts(int H, int64_t N, int64_t window, const int32_t* lo, const int32_t* hi, UnionParts& u) {
  if (window < 1 || window > N) return SPA_ERR_INVAL;
  static AttnParams zero{};
  AttnParams p = zero;
  int st = fill_bands(p, H, N, lo, hi);
  if (st) return st;
  for (int h = 0; h < H; ++h) {
    if (window < p.lo[h]) {
      u.a1[h] = 0;
      u.b1[h] = (int32_t)window;
      u.a2[h] = p.lo[h];
      u.b2[h] = p.hi[h];
    } else {
      const int64_t len = window > p.hi[h] ? window : p.hi[h];
      if (len < 2) return SPA_ERR_UNSUPPORTED;  // one distance cannot be split
      const int64_t m = (len + 1) / 2;
      u.a1[h] = 0;
      u.b1[h] = (int32_t)m;
      u.a2[h] = (int32_t)m;
      u.b2[h] = (int32_t)len;
    }
  }
  return SPA_OK;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Workspace of the union calls: the backward's row sums D, fp32 [B H N]
// (the forward merges in place and needs none).

int union_launch_status() { return cudaGetLastError() == cudaSuccess ? SPA_OK : SPA_ERR_CUDA; }

int union_merge(void* o, float* lse, const void* o2, const float* lse2, int B, int H, int64_t N, int d,
                void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!o || !lse || !o2 || !lse2) return SPA_ERR_INVAL;
  if (!aligned(o, 16) || !aligned(o2, 16) || !aligned(lse, 4) || !aligned(lse2, 4)) return SPA_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)B * H * N;
  const int64_t threads = rows * (d / 8);
  // a grid-stride kernel: at most eight blocks per SM
  int sms = 0;
  if ((st = sm_count(&sms))) return st;
  const int64_t want = (threads + 255) / 256;
  const unsigned blocks = (unsigned)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64)
    spa::spa_union_merge_kernel<64><<<blocks, 256, 0, s>>>(static_cast<uint16_t*>(o), lse,
                                                           static_cast<const uint16_t*>(o2), lse2, rows);
  else
    spa::spa_union_merge_kernel<128><<<blocks, 256, 0, s>>>(static_cast<uint16_t*>(o), lse,
                                                            static_cast<const uint16_t*>(o2), lse2, rows);
  return union_launch_status();
}

int union_add_grads(void* dq, void* dk, void* dv, const void* dq2, const void* dk2, const void* dv2, int B, int H,
                    int64_t N, int d, void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  for (const void* t : {(const void*)dq, (const void*)dk, (const void*)dv, dq2, dk2, dv2}) {
    if (!t) return SPA_ERR_INVAL;
    if (!aligned(t, 16)) return SPA_ERR_UNSUPPORTED;
  }
  int sms = 0;
  if ((st = sm_count(&sms))) return st;
  const int64_t n16 = (int64_t)B * H * N * d / 8;
  const int64_t want = (3 * n16 + 255) / 256;
  const unsigned blocks = (unsigned)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  spa::spa_add3_bf16_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t*>(dq), static_cast<uint16_t*>(dk), static_cast<uint16_t*>(dv),
      static_cast<const uint16_t*>(dq2), static_cast<const uint16_t*>(dk2), static_cast<const uint16_t*>(dv2), n16);
  return union_launch_status();
}

struct BandArgs {
  int32_t lo[spa::kMaxHeads];
  int32_t hi[spa::kMaxHeads];
};

__global__ void tile_class_kernel(int64_t N, int H, int Bq, int Bk, int nqt, int nkt,
                                  const __grid_constant__ BandArgs bands, uint8_t* out) {
  const int64_t total = (int64_t)H * nqt * nkt;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int u = (int)(e % nkt);
    const int t = (int)((e / nkt) % nqt);
    const int h = (int)(e / ((int64_t)nkt * nqt));
    out[e] = spa::tile_class(N, bands.lo[h], bands.hi[h], t, Bq, u, Bk);
  }
}

// One warp waits on an mbarrier that nothing ever arrives on, with the given
// limit: the bounded-wait path every kernel uses, exercised on purpose.
__global__ void wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    spa::ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    spa::ptx::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = spa::bar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0 && ok) atomicExch(&spa::g_spa_status, -1);  // cannot happen: nothing arrives
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for spa_attn_bwd_noalloc: the fp32 row sums D_i of the backward, in
// a file-scope device array so that the call allocates nothing.  Every GPU
// that loads this library holds these SPA_NOALLOC_MAX_ROWS * 4 bytes (4 MiB)
// until the process exits.  Host code cannot use the array's name as a device
// address; noalloc_scratch() looks the address up once per device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) float g_spa_noalloc_delta[SPA_NOALLOC_MAX_ROWS];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocSlot {
  unsigned long long ctx_id;  // unique id of the context the address belongs to
  void* ptr;
};
NoallocSlot g_noalloc[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the context current on this thread (ids are never reused
// within a process, unlike context handles); 0 when it cannot be had.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_spa_noalloc_delta on the current device.  The first
// call on a device (with that device current) resolves it with
// cudaGetSymbolAddress and caches it together with the id of the context it
// belongs to; later calls in the same context only read the cache.  After a
// device reset the primary context, and with it the module and its arrays, is
// new: its id differs, so the address is resolved again.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SPA_ERR_UNSUPPORTED;
  // make the device's primary context current on this thread (a thread that
  // has made no runtime call yet has none)
  if (cudaSetDevice(dev) != cudaSuccess) return SPA_ERR_CUDA;
  const unsigned long long id = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  if (slot.ptr == nullptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_spa_noalloc_delta) != cudaSuccess || p == nullptr) return SPA_ERR_CUDA;
    slot.ptr = p;
    slot.ctx_id = id;
  }
  *out = slot.ptr;
  return SPA_OK;
}

}  // namespace

extern "C" {

const char* spa_status_string(int status) {
  switch (status) {
    case SPA_OK: return "SPA_OK";
    case SPA_ERR_INVAL: return "SPA_ERR_INVAL: invalid argument";
    case SPA_ERR_UNSUPPORTED: return "SPA_ERR_UNSUPPORTED: shape or alignment not supported";
    case SPA_ERR_CUDA: return "SPA_ERR_CUDA: CUDA call or kernel launch failed";
    case SPA_ERR_TIMEOUT: return "SPA_ERR_TIMEOUT: a device-side wait ran out of time";
    default: return "unknown spa status";
  }
}

int spa_version(void) { return 100; }

int spa_band_bounds(int64_t N, int H, int32_t* lo, int32_t* hi) {
  if (!lo || !hi || H < 1 || N < 1 || (int64_t)H > N || N > 2147483647LL) return SPA_ERR_INVAL;
  for (int h = 0; h < H; ++h) spa::band_of_head(N, H, h, &lo[h], &hi[h]);
  return SPA_OK;
}

int spa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int64_t N, int d, float scale, void* stream) {
  return fwd_entry(q, k, v, o, lse, B, H, N, d, scale, nullptr, nullptr, stream);
}

int spa_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  if (!lo || !hi) return SPA_ERR_INVAL;
  return fwd_entry(q, k, v, o, lse, B, H, N, d, scale, lo, hi, stream);
}

size_t spa_attn_bwd_workspace_bytes(int B, int H, int64_t N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return (size_t)B * (size_t)H * (size_t)N * sizeof(float);
}

int spa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H,
                 int64_t N, int d, float scale, void* stream) {
  return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, d, scale, nullptr, nullptr,
                   stream, kStepAll);
}

int spa_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H,
                    int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi,
                    void* stream) {
  if (!lo || !hi) return SPA_ERR_INVAL;
  return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, d, scale, lo, hi, stream,
                   kStepAll);
}

int spa_attn_bwd_preprocess(const void* o, const void* dout, void* workspace, int B, int H, int64_t N,
                            int d, void* stream) {
  return bwd_entry(nullptr, nullptr, nullptr, o, dout, nullptr, nullptr, nullptr, nullptr, workspace, B,
                   H, N, d, 1.0f, nullptr, nullptr, stream, kStepDelta);
}

int spa_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                      const void* workspace, void* dk, void* dv, int B, int H, int64_t N, int d,
                      float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return bwd_entry(q, k, v, nullptr, dout, lse, nullptr, dk, dv, const_cast<void*>(workspace), B, H, N,
                   d, scale, lo, hi, stream, kStepDkDv);
}

int spa_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                    const void* workspace, void* dq, int B, int H, int64_t N, int d, float scale,
                    const int32_t* lo, const int32_t* hi, void* stream) {
  return bwd_entry(q, k, v, nullptr, dout, lse, dq, nullptr, nullptr, const_cast<void*>(workspace), B, H,
                   N, d, scale, lo, hi, stream, kStepDq);
}

int spa_attn_bwd_dkdv_add(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                          const void* workspace, void* dk, void* dv, int B, int H, int64_t N, int d,
                          float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return bwd_entry(q, k, v, nullptr, dout, lse, nullptr, dk, dv, const_cast<void*>(workspace), B, H, N,
                   d, scale, lo, hi, stream, kStepDkDv | kStepAccumulate);
}

int spa_attn_bwd_dq_add(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                        const void* workspace, void* dq, int B, int H, int64_t N, int d, float scale,
                        const int32_t* lo, const int32_t* hi, void* stream) {
  return bwd_entry(q, k, v, nullptr, dout, lse, dq, nullptr, nullptr, const_cast<void*>(workspace), B, H,
                   N, d, scale, lo, hi, stream, kStepDq | kStepAccumulate);
}

int spa_attn_bwd_dq_delta(const void* q, const void* k, const void* v, const void* o, const void* dout,
                          const float* lse, void* workspace, void* dq, int B, int H, int64_t N, int d,
                          float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return bwd_entry(q, k, v, o, dout, lse, dq, nullptr, nullptr, workspace, B, H, N, d, scale, lo, hi, stream,
                   kStepDqDelta);
}

size_t spa_attn_bwd_stored_workspace_bytes(int B, int H, int64_t N, int d, const int32_t* lo,
                                           const int32_t* hi) {
  if (check_shape(B, H, N, d)) return 0;
  static AttnParams zero{};
  AttnParams p = zero;
  p.B = B;
  p.H = H;
  p.N = N;
  if (fill_bands(p, H, N, lo, hi)) return 0;
  const int64_t tiles = stored_layout(p);
  if (tiles < 0) return 0;
  return stored_delta_bytes((int64_t)B * H * N) + (size_t)tiles * kStoredTileBytes;
}

int spa_attn_bwd_stored(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H, int64_t N,
                        int d, float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return spa_attn_bwd_stored_steps(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, d, scale, lo, hi, stream,
                                   7);
}

int spa_attn_bwd_stored_steps(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H,
                              int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi, void* stream,
                              int steps) {
  if (steps < 1 || steps > 7) return SPA_ERR_INVAL;
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return SPA_ERR_INVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SPA_ERR_INVAL;
  for (const void* t : {q, k, v, o, dout})
    if (!aligned(t, 16)) return SPA_ERR_UNSUPPORTED;
  // the gradients leave in 32-byte stores; the dS^T tiles are copied by TMA
  if (!aligned(dq, 32) || !aligned(dk, 32) || !aligned(dv, 32) || !aligned(lse, 4) || !aligned(workspace, 256))
    return SPA_ERR_UNSUPPORTED;
  static AttnParams zero{};
  AttnParams p = zero;
  p.B = B;
  p.H = H;
  p.N = N;
  p.scale = scale;
  p.scale_log2 = scale * spa::kLog2e;
  if ((st = fill_bands(p, H, N, lo, hi))) return st;
  if (stored_layout(p) < 0) return SPA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* delta = static_cast<float*>(workspace);
  void* ds = static_cast<uint8_t*>(workspace) + stored_delta_bytes((int64_t)B * H * N);
  const int bits = ((steps & 1) ? kStepDeltaBand : 0) | ((steps & 2) ? kStepDkDv : 0) | ((steps & 4) ? kStepDqStored : 0);
  return d == 64 ? bwd_impl<64>(q, k, v, o, dout, lse, dq, dk, dv, delta, p, s, bits, ds)
                 : bwd_impl<128>(q, k, v, o, dout, lse, dq, dk, dv, delta, p, s, bits, ds);
}

size_t spa_attn_bwd_fused_workspace_bytes(int B, int H, int64_t N, int d) {
  if (check_shape(B, H, N, d)) return 0;
  const int64_t rows = (int64_t)B * H * N;
  return fused_delta_bytes(rows) + (size_t)rows * (size_t)d * sizeof(float);
}

int spa_attn_bwd_fused(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H, int64_t N,
                       int d, float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return spa_attn_bwd_fused_steps(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, d, scale, lo, hi, stream,
                                  kFusedAll);
}

int spa_attn_bwd_fused_steps(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H,
                             int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi, void* stream,
                             int steps) {
  if (steps < 1 || steps > kFusedAll) return SPA_ERR_INVAL;
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return SPA_ERR_INVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SPA_ERR_INVAL;
  for (const void* t : {q, k, v, o, dout, (const void*)dq})
    if (!aligned(t, 16)) return SPA_ERR_UNSUPPORTED;
  // dk and dv leave in 32-byte stores, the workspace in 16-byte reductions
  if (!aligned(dk, 32) || !aligned(dv, 32) || !aligned(lse, 4) || !aligned(workspace, 256))
    return SPA_ERR_UNSUPPORTED;
  static AttnParams zero{};
  AttnParams p = zero;
  p.B = B;
  p.H = H;
  p.N = N;
  p.scale = scale;
  p.scale_log2 = scale * spa::kLog2e;
  if ((st = fill_bands(p, H, N, lo, hi))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? fused_impl<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, p, s, steps)
                 : fused_impl<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, p, s, steps);
}

int spa_tile_schedule(int64_t N, int H, const int32_t* lo, const int32_t* hi, int Bq, int Bk,
                      int32_t* kt_begin, int32_t* kt_end, uint8_t* tile_class, int32_t* qt_begin,
                      int32_t* qt_end) {
  if (N < 1 || N > 2147483647LL || H < 1 || H > spa::kMaxHeads || Bq < 1 || Bk < 1 || Bq > 4096 ||
      Bk > 4096)
    return SPA_ERR_INVAL;
  AttnParams p{};
  int st = fill_bands(p, H, N, lo, hi);
  if (st) return st;
  const int nqt = (int)((N + Bq - 1) / Bq), nkt = (int)((N + Bk - 1) / Bk);
  for (int h = 0; h < H; ++h) {
    for (int t = 0; t < nqt; ++t) {
      const spa::Strip s = spa::key_strip(N, p.lo[h], p.hi[h], (int64_t)t * Bq, Bq, Bk);
      if (kt_begin) kt_begin[(int64_t)h * nqt + t] = s.end < s.begin ? 0 : s.begin;
      if (kt_end) kt_end[(int64_t)h * nqt + t] = s.end < s.begin ? -1 : s.end;
      if (tile_class)
        for (int u = 0; u < nkt; ++u)
          tile_class[((int64_t)h * nqt + t) * nkt + u] = spa::tile_class(N, p.lo[h], p.hi[h], t, Bq, u, Bk);
    }
    for (int u = 0; u < nkt; ++u) {
      const spa::Strip s = spa::query_strip(N, p.lo[h], p.hi[h], (int64_t)u * Bk, Bk, Bq);
      if (qt_begin) qt_begin[(int64_t)h * nkt + u] = s.end < s.begin ? 0 : s.begin;
      if (qt_end) qt_end[(int64_t)h * nkt + u] = s.end < s.begin ? -1 : s.end;
    }
  }
  return SPA_OK;
}

int spa_tile_classes_device(int64_t N, int H, const int32_t* lo, const int32_t* hi, int Bq, int Bk,
                            uint8_t* tile_class_dev, void* stream) {
  if (N < 1 || N > 2147483647LL || H < 1 || H > spa::kMaxHeads || Bq < 1 || Bk < 1 || Bq > 4096 ||
      Bk > 4096 || !tile_class_dev)
    return SPA_ERR_INVAL;
  AttnParams p{};
  int st = fill_bands(p, H, N, lo, hi);
  if (st) return st;
  BandArgs bands{};
  std::memcpy(bands.lo, p.lo, sizeof(bands.lo));
  std::memcpy(bands.hi, p.hi, sizeof(bands.hi));
  const int nqt = (int)((N + Bq - 1) / Bq), nkt = (int)((N + Bk - 1) / Bk);
  tile_class_kernel<<<148 * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(N, H, Bq, Bk, nqt, nkt, bands,
                                                                            tile_class_dev);
  return launch_status();
}

int spa_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int64_t N, int d, float scale, void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if ((int64_t)B * H * N > (int64_t)SPA_NOALLOC_MAX_ROWS) return SPA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  // The dQ pass forms D and writes it for every row of the 128-row query
  // blocks that some band reaches, before the dK/dV pass reads it; the dK/dV
  // pass reads D only for those rows, so whatever an earlier call left in the
  // scratch is never read and the array needs no clearing between calls.
  return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, scratch, B, H, N, d, scale, nullptr, nullptr,
                   stream, kStepAll);
}

int spa_debug_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000LL) return SPA_ERR_INVAL;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ns);
  return launch_status();
}

// Chunks of kDecodeChunk keys that the widest band needs.
int64_t decode_chunks(const AttnParams& p, int H) {
  int64_t w = 1;
  for (int h = 0; h < H; ++h) w = std::max<int64_t>(w, (int64_t)p.hi[h] - p.lo[h]);
  return (w + spa::kDecodeChunk - 1) / spa::kDecodeChunk;
}

size_t spa_attn_decode_workspace_bytes(int B, int H, int64_t N, int d, const int32_t* lo, const int32_t* hi) {
  if (check_shape(B, H, N, d)) return 0;
  static AttnParams zero{};
  AttnParams p = zero;
  if (fill_bands(p, H, N, lo, hi)) return 0;
  return (size_t)B * H * decode_chunks(p, H) * (d + 2) * sizeof(float);
}

int spa_attn_decode(const void* q, const void* k, const void* v, const int32_t* pos, void* o, float* lse,
                    void* workspace, int B, int H, int64_t N, int d, float scale, const int32_t* lo,
                    const int32_t* hi, void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!q || !k || !v || !pos || !o || !lse || !workspace) return SPA_ERR_INVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SPA_ERR_INVAL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(pos, 4) || !aligned(workspace, 4))
    return SPA_ERR_UNSUPPORTED;
  static AttnParams zero{};
  AttnParams bands = zero;
  if ((st = fill_bands(bands, H, N, lo, hi))) return st;
  static spa::DecodeParams dzero{};
  spa::DecodeParams p = dzero;
  p.B = B;
  p.H = H;
  p.N = N;
  p.d = d;
  p.scale_log2 = scale * spa::kLog2e;
  const int64_t nchunk = decode_chunks(bands, H);
  if (nchunk > 2147483647LL) return SPA_ERR_UNSUPPORTED;
  p.nchunk = (int)nchunk;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.pos = pos;
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.part = static_cast<float*>(workspace);
  std::memcpy(p.lo, bands.lo, sizeof(p.lo));
  std::memcpy(p.hi, bands.hi, sizeof(p.hi));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid_c((unsigned)nchunk, (unsigned)H, (unsigned)B), grid_m((unsigned)H, (unsigned)B);
  // the merge kernel is the chunk kernel's programmatic dependent: its launch
  // may begin once every chunk CTA has finished its keys, and it waits for
  // the chunk grid (griddepcontrol.wait) before reading the partials
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid_m;
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (d == 64) {
    spa::spa_decode_chunk_kernel<64><<<grid_c, 128, 0, s>>>(p);
    if ((st = launch_status())) return st;
    if (cudaLaunchKernelEx(&cfg, spa::spa_decode_merge_kernel<64>, p) != cudaSuccess) return SPA_ERR_CUDA;
  } else {
    spa::spa_decode_chunk_kernel<128><<<grid_c, 128, 0, s>>>(p);
    if ((st = launch_status())) return st;
    if (cudaLaunchKernelEx(&cfg, spa::spa_decode_merge_kernel<128>, p) != cudaSuccess) return SPA_ERR_CUDA;
  }
  return launch_status();
}

int spa_union_parts(int64_t N, int H, int64_t window, const int32_t* lo, const int32_t* hi, int32_t* a1,
                    int32_t* b1, int32_t* a2, int32_t* b2) {
  if (H < 1 || H > spa::kMaxHeads || N < 1 || N > 2147483647LL) return SPA_ERR_INVAL;
  if (!a1 || !b1 || !a2 || !b2) return SPA_ERR_INVAL;
  static UnionParts zero{};
  UnionParts u = zero;
  const int st = union_parts(H, N, window, lo, hi, u);
  if (st) return st;
  for (int h = 0; h < H; ++h) {
    a1[h] = u.a1[h];
    b1[h] = u.b1[h];
    a2[h] = u.a2[h];
    b2[h] = u.b2[h];
  }
  return SPA_OK;
}

size_t spa_attn_union_workspace_bytes(int B, int H, int64_t N, int d) {
  if (check_shape(B, H, N, d)) return 0;
  const size_t rows = (size_t)B * H * N;
  return align256(rows * 4);
}

int spa_attn_fwd_union(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                       int64_t N, int d, float scale, int64_t window, const int32_t* lo, const int32_t* hi,
                       void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  static UnionParts zero{};
  UnionParts u = zero;
  if ((st = union_parts(H, N, window, lo, hi, u))) return st;
  // part 2's forward merges into part 1's o and lse in its epilogue
  if ((st = fwd_entry(q, k, v, o, lse, B, H, N, d, scale, u.a1, u.b1, stream))) return st;
  return fwd_entry(q, k, v, o, lse, B, H, N, d, scale, u.a2, u.b2, stream, true);
}

int spa_attn_bwd_union(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int H, int64_t N,
                       int d, float scale, int64_t window, const int32_t* lo, const int32_t* hi, void* stream) {
  int st = check_shape(B, H, N, d);
  if (st) return st;
  if (!workspace || !dq || !dk || !dv) return SPA_ERR_INVAL;
  if (!aligned(workspace, 32)) return SPA_ERR_UNSUPPORTED;
  static UnionParts zero{};
  UnionParts u = zero;
  if ((st = union_parts(H, N, window, lo, hi, u))) return st;
  float* D_ = static_cast<float*>(workspace);
  // part 1 starts at distance 0, so its dQ pass forms D for every row; part
  // 2's passes add their gradients to part 1's in their epilogues
  if ((st = bwd_entry(q, k, v, o, dout, lse, dq, nullptr, nullptr, D_, B, H, N, d, scale, u.a1, u.b1,
                      stream, kStepDqDelta)) ||
      (st = bwd_entry(q, k, v, o, dout, lse, nullptr, dk, dv, D_, B, H, N, d, scale, u.a1, u.b1, stream,
                      kStepDkDv)) ||
      (st = bwd_entry(q, k, v, o, dout, lse, dq, nullptr, nullptr, D_, B, H, N, d, scale, u.a2, u.b2,
                      stream, kStepDq | kStepAccumulate)) ||
      (st = bwd_entry(q, k, v, o, dout, lse, nullptr, dk, dv, D_, B, H, N, d, scale, u.a2, u.b2, stream,
                      kStepDkDv | kStepAccumulate)))
    return st;
  return SPA_OK;
}

int spa_attn_fwd_merge(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int64_t N,
                       int d, float scale, const int32_t* lo, const int32_t* hi, void* stream) {
  return fwd_entry(q, k, v, o, lse, B, H, N, d, scale, lo, hi, stream, true);
}

int spa_attn_union_merge(void* o, float* lse, const void* o2, const float* lse2, int B, int H, int64_t N, int d,
                         void* stream) {
  return union_merge(o, lse, o2, lse2, B, H, N, d, stream);
}

int spa_attn_union_add_grads(void* dq, void* dk, void* dv, const void* dq2, const void* dk2, const void* dv2,
                             int B, int H, int64_t N, int d, void* stream) {
  return union_add_grads(dq, dk, dv, dq2, dk2, dv2, B, H, N, d, stream);
}

int spa_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SPA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, spa::g_spa_status, sizeof(int)) != cudaSuccess) return SPA_ERR_CUDA;
  if (v != 0) {
    const int z = 0;
    if (cudaMemcpyToSymbol(spa::g_spa_status, &z, sizeof(int)) != cudaSuccess) return SPA_ERR_CUDA;
  }
  if (v == 0) return SPA_OK;
  return v == spa::kStatusUnsupported ? SPA_ERR_UNSUPPORTED : SPA_ERR_TIMEOUT;
}

}  // extern "C"
