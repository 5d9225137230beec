// Device-side helpers shared by the PQ-HSA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pqhsa.h"

namespace pqhsa {

constexpr int kD = 128;        // head dim
constexpr int kM = 16;         // PQ subspaces
constexpr int kDsub = 8;       // dims per subspace
constexpr int kNcode = 256;    // codewords per subspace
constexpr int kNB = 2048;      // selection-score histogram bins
constexpr int kBgClusters = 64;  // clusters per background CTA
constexpr int kMaxSplits = 64;   // exact/dense split-K chunks per unit (upper bound)
constexpr int kTile = 32;        // tokens per attention tile (one per lane)
constexpr float kLog2e = 1.4426950408889634f;

// Workspace error word lives at offset 0 of every workspace.
struct WsHeader {
  int32_t err;
  int32_t pad[63];
};

__device__ __forceinline__ void record_error(int32_t* err, int32_t bit) {
  if (err) atomicOr(err, bit);
}

// ---------------------------------------------------------------------------
// shared-memory / async-proxy primitives
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false (and records a timeout) when
// the phase has not completed after a fixed number of polls.
constexpr uint32_t kSpinLimit = 1u << 24;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  record_error(err, HSA_DEVERR_TIMEOUT);
  return false;
}

// 2-D tiled TMA load, completion signalled on `bar` (transaction bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(tmap), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk copy global -> shared (both 16-byte aligned, bytes a multiple of 16),
// completion signalled on `bar` (transaction bytes).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Programmatic dependent launch: wait for the producer grid / let dependents start.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Monotone map float -> uint32 (larger float -> larger key; -0 and +0 equal).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Histogram bin of a selection score; identical arithmetic wherever it is used.
__device__ __forceinline__ int score_bin(float sigma, float lo, float inv_w) {
  float t = __fmul_rn(__fsub_rn(sigma, lo), inv_w);
  int b = (t >= 0.f) ? static_cast<int>(t) : 0;   // NaN/negatives -> bin 0
  return b > kNB - 1 ? kNB - 1 : b;
}

// k = floor(budget * N) in double, clipped; identical to the host computation.
__host__ __device__ __forceinline__ int decode_k(double budget, int32_t k_override, int n) {
  if (n <= 0) return 0;
  if (k_override >= 0) return k_override < n ? k_override : n;
  double f = budget * static_cast<double>(n);
  long long k = (f <= 0.0) ? 0 : static_cast<long long>(f);  // floor for f >= 0
  if (k > n) k = n;
  return static_cast<int>(k);
}

// Raise a kernel's dynamic shared-memory limit once per device (never inside a
// stream capture after the first call on that device).
// The cache is per kernel (template on the function itself, not its type).
template <auto Kern>
inline cudaError_t ensure_dyn_smem(size_t bytes) {
  static int set_bytes[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (set_bytes[dev] >= static_cast<int>(bytes)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) set_bytes[dev] = static_cast<int>(bytes);
  return e;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Workspace layout of hsa_decode (computed identically on host and device).
// ---------------------------------------------------------------------------
struct UnitState {          // per unit bookkeeping written by the top-k kernels
  int32_t bstar;            // threshold bin
  int32_t above;            // tokens in bins above bstar
  int32_t ncand;            // tokens in bin bstar (candidates)
  int32_t nsel;             // selected count written by finalize
  int32_t pad[4];
};

struct DecodeLayout {
  // sizes
  int U, G, GP, C, cap, nq, nsplit_max, nbg, bitmap_words;
  // byte offsets from the workspace base
  size_t off_units, off_bounds, off_lut, off_qc, off_w, off_hist, off_sigma, off_bitmap, off_cand,
      off_sel, off_pm, off_pl, off_pacc, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline DecodeLayout make_decode_layout(int U, int G, int C, int cap, int nsplit_max) {
  DecodeLayout L;
  L.U = U;
  L.G = G;
  L.GP = (G + 3) / 4;
  L.C = C;
  L.cap = cap;
  L.nq = (C + 127) / 128;  // qc slices per unit in the table builder
  L.nsplit_max = nsplit_max;
  L.nbg = (C + kBgClusters - 1) / kBgClusters;
  L.bitmap_words = static_cast<int>(align_up(static_cast<size_t>((cap + 31) / 32), 8));
  size_t o = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    o = align_up(o, 256);
    size_t r = o;
    o += bytes;
    return r;
  };
  const size_t u = static_cast<size_t>(U);
  L.off_units = take(u * sizeof(UnitState));
  L.off_bounds = take(u * (1 + L.nq) * 2 * 4 * L.GP * sizeof(float));
  L.off_lut = take(u * L.GP * kNcode * kM * 4 * sizeof(float));
  L.off_qc = take(u * L.GP * C * 4 * sizeof(float));
  L.off_w = take(u * G * C * sizeof(float));
  L.off_hist = take(u * kNB * sizeof(uint32_t));
  L.off_sigma = take(u * cap * sizeof(float));
  L.off_bitmap = take(u * L.bitmap_words * sizeof(uint32_t));
  L.off_cand = take(u * cap * sizeof(uint64_t));
  L.off_sel = take(u * cap * sizeof(int32_t));
  const size_t parts = u * (nsplit_max + L.nbg) * G;
  L.off_pm = take(parts * sizeof(float));
  L.off_pl = take(parts * sizeof(float));
  L.off_pacc = take(parts * kD * sizeof(float));
  L.total = align_up(o, 256);
  return L;
}

}  // namespace pqhsa
