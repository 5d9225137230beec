// Device-side helpers shared by the PQ-HSA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
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
constexpr int kCandWeights = 1024;  // threshold-bin candidates whose head weights the filter precomputes
constexpr int kMaxSplits = 64;   // exact/dense split-K chunks per unit (upper bound)
constexpr int kMaxClusters = 4096;                        // IVF clusters per unit (upper bound)
constexpr int kMaxBgChunks = kMaxClusters / kBgClusters;  // background partials per unit
constexpr int kTile = 32;        // tokens per attention tile (one per lane)
constexpr int kLutParts = 8;     // table-builder CTAs per unit for the LUT (2 subspaces each)
constexpr int kQcSlice = 64;     // clusters per table-builder CTA for the centroid terms
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase: gives up after kWaitLimitNs of wall time,
// records a timeout and returns false. Lanes may leave at different polls, so a
// warp must reconverge (e.g. one polling lane + __shfl_sync) before any
// .aligned warp-collective instruction.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  record_error(err, HSA_DEVERR_TIMEOUT);
  return false;
}

// Warp-uniform wait: lane 0 polls, the outcome is broadcast (and the warp reconverged).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int32_t* err) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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

// Two fp32 additions in one instruction (sm_100 packed f32x2), each rounded to nearest
// like __fadd_rn; a and b hold (lo, hi) = (first, second) float.
__device__ __forceinline__ unsigned long long fadd2_rn(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Two fp32 fused multiply-adds in one instruction (sm_100 packed f32x2), each rounded once.
__device__ __forceinline__ unsigned long long ffma2_rn(unsigned long long a, unsigned long long b,
                                                       unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long pack_f2(float lo, float hi) {
  return static_cast<unsigned long long>(__float_as_uint(lo)) |
         (static_cast<unsigned long long>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo_f(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// LSU asynchronous copies (16 or 4 bytes per thread): for small gathers, where one
// bulk copy per few hundred bytes would be limited by the copy engine's per-operation
// cost. Completion is tracked per thread by commit groups, or signalled on an mbarrier.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed; the
// arrival counts toward the barrier's expected count (initialise it accordingly).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
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
// tensor-core fragments (mma.sync m16n8k16, bf16 in, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                              uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// x = hi + lo with hi, lo bf16 (round to nearest): |x - hi - lo| <= 2^-16 |x| roughly.
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
  hi = __bfloat16_as_ushort(h);
  lo = __bfloat16_as_ushort(l);
}
// Two values packed as bf16x2 (x0 in the low half), split into hi and lo parts.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  uint16_t h0, l0, h1, l1;
  split_bf16(x0, h0, l0);
  split_bf16(x1, h1, l1);
  hi = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
  lo = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
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
// Largest value over the full warp in one instruction (sm_100a redux of f32).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
// Smallest value over the full warp in one instruction (sm_100a redux of f32).
__device__ __forceinline__ float warp_min_f32(float v) {
  float r;
  asm("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// List slots an index of cap tokens and C clusters needs: every cluster's last chunk
// of 32 slots may be partly empty.
__host__ __device__ inline long long list_slots_needed(int cap, int C) {
  return 32LL * ((static_cast<long long>(cap) + 31) / 32 + C);
}

// Workspace layout of hsa_decode (computed identically on host and device).
// ---------------------------------------------------------------------------
// Per unit bookkeeping of the scan and selection (zeroed by the tables). Every counter
// that CTAs poll while others update it sits on a 128-byte line of its own (the attention
// CTAs poll the ready flag, the selection's parts poll the phase counters), so polling
// never slows the atomics on the other lines.
struct alignas(128) UnitState {
  int32_t bstar;            // threshold bin
  int32_t above;            // tokens in bins above bstar
  int32_t ncand;            // tokens in bin bstar (candidates)
  int32_t ndef;             // tokens above the threshold bin whose rows are written (definite)
  int32_t pad0[28];
  int32_t scan_done;        // chunks of the unit scanned (histogram, weights and scores written)
  int32_t pad1[31];
  int32_t filt_done;        // chunks of the unit whose selections and candidates are written
  int32_t pad2[31];
  int32_t pad3[32];
  int32_t ready;            // set (release) once the unit's selection and weight fix-up are final
  int32_t pad4[31];
};
static_assert(sizeof(UnitState) == 640, "five 128-byte lines per unit");

// Bounded wait (acquire) for a flag another running grid publishes; a timeout is
// recorded and returns false. Callers only wait on CTAs that are already resident.
// Call it from one thread and share the outcome through a barrier (the flag's line is
// also written by the publisher: many pollers would slow it down).
__device__ __forceinline__ bool wait_flag(const int32_t* flag, int32_t* err) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  if (v) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    __nanosleep(256);
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v) return true;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  record_error(err, HSA_DEVERR_TIMEOUT);
  return false;
}

// Bounded wait (acquire) until a counter that other resident CTAs of this grid advance
// reaches `target`; a timeout is recorded and returns false. One thread calls it.
__device__ __forceinline__ bool wait_count(const int32_t* ctr, int32_t target, int32_t* err) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
  if (v >= target) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    __nanosleep(64);
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  record_error(err, HSA_DEVERR_TIMEOUT);
  return false;
}

struct DecodeLayout {
  // sizes
  int U, G, GP, C, cap, nq, nsplit_max, nbg, bitmap_words;
  // byte offsets from the workspace base
  size_t off_units, off_bounds, off_fbounds, off_lut, off_qc, off_w, off_hist, off_sigma, off_cmax, off_bitmap,
      off_cand,
      off_candw, off_candc, off_candr, off_sel, off_pm, off_pl, off_pacc, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline DecodeLayout make_decode_layout(int U, int G, int C, int cap, int list_slots,
                                                           int nsplit_max) {
  DecodeLayout L;
  L.U = U;
  L.G = G;
  L.GP = (G + 3) / 4;
  L.C = C;
  L.cap = cap;
  L.nq = (C + kQcSlice - 1) / kQcSlice;  // qc slices per unit in the table builder
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
  L.off_bounds = take(u * (kLutParts + L.nq) * 2 * 4 * L.GP * sizeof(float));
  L.off_fbounds = take(u * 2 * G * sizeof(float));
  L.off_lut = take(u * L.GP * kNcode * kM * 4 * sizeof(float));
  L.off_qc = take(u * L.GP * C * 4 * sizeof(float));
  L.off_w = take(u * G * C * sizeof(float));
  L.off_hist = take(u * kNB * sizeof(uint32_t));
  L.off_sigma = take(u * list_slots * sizeof(float));   // one score per list slot
  L.off_cmax = take(u * (list_slots / 32) * sizeof(float));   // largest score per chunk
  L.off_bitmap = take(u * L.bitmap_words * sizeof(uint32_t));
  L.off_cand = take(u * cap * sizeof(uint64_t));
  L.off_candw = take(u * kCandWeights * G * sizeof(float));
  L.off_candc = take(u * kCandWeights * sizeof(int32_t));
  L.off_candr = take(u * cap * sizeof(int32_t));   // KV-pool row of each candidate
  L.off_sel = take(u * cap * sizeof(int32_t));
  const size_t parts = u * (nsplit_max + L.nbg) * G;
  L.off_pm = take(parts * sizeof(float));
  L.off_pl = take(parts * sizeof(float));
  L.off_pacc = take(parts * kD * sizeof(float));
  L.total = align_up(o, 256);
  return L;
}

}  // namespace pqhsa
