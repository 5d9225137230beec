// Nearest-centroid assignment of the training keys on the 5th-generation tensor cores.
//
// The coarse Lloyd step assigns every training key x to argmin_c |x - c|^2. Over all
// keys of a (sequence, KV head) unit and all C centroids this is one dense contraction:
// argmin_c (|c|^2 - 2 x.c), with x.c the [n x 128] x [128 x C] product. Keys are bf16
// already; each fp32 centroid is carried as three bf16 terms (hi + mid + lo, together
// about 24 significant bits), so the product sum over the three terms reproduces the
// fp32 dot product to fp32 accuracy while the tensor cores accumulate in fp32.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0  TMA producer: key tile (128 keys = 16 page-row groups of 8, starting at the
//           8-aligned position at or before the unit's first key) into one of two
//           A buffers, then per 256-centroid tile, term and 64-column half a 32 KB operand
//           stage (four stages in flight);
//   warp 1  allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and issues the
//           tcgen05.mma instructions (one elected lane);
//   warps 2-5 epilogue: tcgen05.ld of the accumulator rows (TMEM lane = key), running
//           argmin of |c|^2 - 2 x.c (ties to the lower centroid index), one key per thread.
// Every wait is bounded; a wait that gives up flags HSA_DEVERR_TIMEOUT and the CTA drains
// its copies and MMAs (bounded) and frees TMEM before returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pqhsa.h"
#include "common.cuh"
#include "kernels.h"

namespace pqhsa {
namespace {

constexpr int kAsM = 128;                 // keys per tile (MMA M)
constexpr int kAsN = 256;                 // centroids per tile (MMA N)
constexpr int kAsK = 16;                  // K of one bf16 MMA
constexpr int kAsRows = 8;                // rows per key-tile TMA box (one page-row group)
constexpr uint32_t kAHalf = kAsM * 128;   // one 64-column half of the key tile (16 KB)
constexpr uint32_t kBHalf = kAsN * 128;   // one 64-column half of a centroid stage (32 KB)
constexpr uint32_t kATile = 2 * kAHalf;
constexpr int kBStages = 4;               // centroid operand stages (one term, one 64-column half each)
constexpr int kAsThreads = 192;
constexpr uint32_t kTmemCols = 2 * kAsN;

struct AsSmem {
  static constexpr uint32_t a = 0;                         // 2 x 32 KB key tiles
  static constexpr uint32_t b = 2 * kATile;                // 4 x 32 KB centroid stages
  static constexpr uint32_t bars = b + kBStages * kBHalf;  // mbarriers
  static constexpr uint32_t total = bars + 24 * 8 + 16;
};
constexpr size_t kAsSmemBytes = AsSmem::total + 1024;   // + alignment slack (1024-byte swizzle atoms)

// tcgen05 instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t kAsIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kAsN >> 3) << 17) |
                              (static_cast<uint32_t>(kAsM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major operand in 128-byte swizzle atoms
// (8 rows x 128 B, atoms 1024 B apart): start address, leading offset 16 B (unused for
// swizzled K-major), stride offset 1024 B, descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(kAsIdesc), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (completion: tmem_wait_ld).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Split every centroid into three bf16 terms (rows >= C are zero) and write |c|^2
// (+inf for the padding rows, so they never win). One warp per centroid row.
__global__ void __launch_bounds__(256) centroid_terms_kernel(TrainParams p) {
  const int u = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.y * 8 + warp;
  if (c >= p.Cpad) return;
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c < p.C) x = reinterpret_cast<const float4*>(p.centroids + (static_cast<size_t>(u) * p.C + c) * kD)[lane];
  const float xs[4] = {x.x, x.y, x.z, x.w};
  uint16_t t[3][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float r = xs[i];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const __nv_bfloat16 hb = __float2bfloat16_rn(r);
      t[k][i] = __bfloat16_as_ushort(hb);
      r = __fsub_rn(r, __bfloat162float(hb));
    }
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    uint2 w;
    w.x = static_cast<uint32_t>(t[k][0]) | (static_cast<uint32_t>(t[k][1]) << 16);
    w.y = static_cast<uint32_t>(t[k][2]) | (static_cast<uint32_t>(t[k][3]) << 16);
    reinterpret_cast<uint2*>(p.terms + ((static_cast<size_t>(u) * 3 + k) * p.Cpad + c) * kD)[lane] = w;
  }
  float s = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
  s = warp_sum(s);
  if (lane == 0) p.cnorm[static_cast<size_t>(u) * p.Cpad + c] = c < p.C ? s : INFINITY;
}

__global__ void __launch_bounds__(kAsThreads, 1)
    assign_mma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmb,
                      TrainParams p) {
  extern __shared__ uint8_t as_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(as_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + AsSmem::bars);
  uint64_t* a_full = bars + 0;     // [2]
  uint64_t* a_empty = bars + 2;    // [2]
  uint64_t* b_full = bars + 4;     // [kBStages]
  uint64_t* b_empty = bars + 8;    // [kBStages]
  uint64_t* acc_full = bars + 12;  // [2]
  uint64_t* acc_empty = bars + 14; // [2]
  uint64_t* mma_done = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(a_full + i, 1);
      mbar_init(a_empty + i, 1);
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
    }
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(b_full + i, 1);
      mbar_init(b_empty + i, 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = p.Cpad / kAsN;
  if (warp == 0) {
    // The whole warp produces: lanes 0-15 each load one 8-row group of the key tile (its
    // page looked up one item ahead, so the block-table reads overlap the previous
    // item's operand stream); lane 0 arms the barriers and loads the centroid stages.
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmb);
    }
    auto group_row = [&](int it) -> int {
      if (it >= p.items || lane >= kAsM / kAsRows) return 0;
      const int u = it / p.tiles_per_unit, t = it % p.tiles_per_unit;
      const int b = u / p.Hkv, h = u % p.Hkv;
      const int first = p.n_sink + (p.slot0 ? p.slot0[b] : 0);   // position of key 0
      const int pos = (first & ~(kAsRows - 1)) + t * kAsM + lane * kAsRows;
      const int lp = pos / p.page_size;
      int page = lp < p.max_pages ? p.block_table[static_cast<size_t>(b) * p.max_pages + lp] : -1;
      if (page < 0 || page >= p.num_pages) {
        if (pos + kAsRows > first && pos < first + p.n_train) record_error(p.err, HSA_DEVERR_PAGE);
        page = 0;   // rows outside the key range are loaded but never assigned
      }
      return (page * p.Hkv + h) * p.page_size + (pos % p.page_size);
    };
    uint32_t armed[2 + kBStages] = {};   // arms of a_full[], b_full[] (lane 0)
    int li = 0, sb = 0;
    bool ok = true;
    int row = group_row(blockIdx.x);
    for (int it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++li) {
      const int u = it / p.tiles_per_unit;
      const int ia = li & 1;
      if (!mbar_wait_warp(a_empty + ia, ((li >> 1) & 1) ^ 1, p.err)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(a_full + ia, kATile);
        ++armed[ia];
      }
      __syncwarp();
      uint8_t* A = sm + AsSmem::a + ia * kATile;
      if (lane < kAsM / kAsRows) {
        tma_load_2d(A + lane * kAsRows * 128, &tmk, a_full + ia, 0, row);
        tma_load_2d(A + kAHalf + lane * kAsRows * 128, &tmk, a_full + ia, 64, row);
      }
      row = group_row(it + gridDim.x);
      for (int n = 0; ok && n < n_tiles; ++n) {
        for (int k = 0; ok && k < 3; ++k) {
          for (int kh = 0; kh < 2; ++kh, ++sb) {
            const int ib = sb % kBStages;
            if (!mbar_wait_warp(b_empty + ib, ((sb / kBStages) & 1) ^ 1, p.err)) { ok = false; break; }
            if (lane == 0) {
              mbar_arrive_expect_tx(b_full + ib, kBHalf);
              ++armed[2 + ib];
              tma_load_2d(sm + AsSmem::b + ib * kBHalf, &tmb, b_full + ib, kh * 64, (u * 3 + k) * p.Cpad + n * kAsN);
            }
            __syncwarp();
          }
        }
      }
    }
    // copies still in flight land before the CTA leaves (bounded; immediate when the
    // MMA warp consumed them all)
    if (lane == 0) {
      for (int i = 0; i < 2; ++i)
        if (armed[i]) mbar_wait(a_full + i, (armed[i] - 1) & 1, p.err);
      for (int i = 0; i < kBStages; ++i)
        if (armed[2 + i]) mbar_wait(b_full + i, (armed[2 + i] - 1) & 1, p.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int li = 0, sb = 0, sa = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++li) {
        const int ia = li & 1;
        if (!mbar_wait(a_full + ia, (li >> 1) & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t A = smem_addr(sm + AsSmem::a + ia * kATile);
        for (int n = 0; ok && n < n_tiles; ++n, ++sa) {
          const int buf = sa & 1;
          if (!mbar_wait(acc_empty + buf, ((sa >> 1) & 1) ^ 1, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * kAsN;
          for (int k = 0; ok && k < 3; ++k) {
            for (int kh = 0; kh < 2; ++kh, ++sb) {
              const int ib = sb % kBStages;
              if (!mbar_wait(b_full + ib, (sb / kBStages) & 1, p.err)) { ok = false; break; }
              tc_fence_after();
              const uint32_t B = smem_addr(sm + AsSmem::b + ib * kBHalf);
#pragma unroll
              for (int kk = 0; kk < 64 / kAsK; ++kk) {
                const uint32_t off = kk * (kAsK * 2);   // K step inside the 128-byte atom row
                const uint64_t ad = sw128_desc(A + kh * kAHalf + off);
                const uint64_t bd = sw128_desc(B + off);
                tc_mma(d, ad, bd, (k > 0 || kh > 0 || kk > 0) ? 1u : 0u);
              }
              tc_commit(b_empty + ib);   // the stage is free once these MMAs have read it
            }
          }
          if (ok) tc_commit(acc_full + buf);
        }
        tc_commit(a_empty + ia);
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, p.err);   // nothing of ours still writes TMEM
    }
    __syncwarp();
  } else {
    // epilogue: TMEM lanes [32 * (warp % 4), +32) are this warp's keys
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int sa = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.items; it += gridDim.x) {
      const int u = it / p.tiles_per_unit, t = it % p.tiles_per_unit;
      const float* cn = p.cnorm + static_cast<size_t>(u) * p.Cpad;
      float best = INFINITY;
      int besti = 0;
      for (int n = 0; n < n_tiles; ++n, ++sa) {
        const int buf = sa & 1;
        if (!mbar_wait_warp(acc_full + buf, (sa >> 1) & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int ch = 0; ch < kAsN / 64; ++ch) {
          uint32_t v[64];
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * kAsN + ch * 64;
          tmem_ld32(ta, v);
          tmem_ld32(ta + 32, v + 32);
          tmem_wait_ld();
          const int c0 = n * kAsN + ch * 64;
#pragma unroll
          for (int i = 0; i < 64; i += 4) {
            const float4 nn = __ldg(reinterpret_cast<const float4*>(cn + c0 + i));
            const float e[4] = {fmaf(-2.f, __uint_as_float(v[i]), nn.x), fmaf(-2.f, __uint_as_float(v[i + 1]), nn.y),
                                fmaf(-2.f, __uint_as_float(v[i + 2]), nn.z),
                                fmaf(-2.f, __uint_as_float(v[i + 3]), nn.w)};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (e[j] < best) {
                best = e[j];
                besti = c0 + i + j;
              }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + buf);
      }
      if (!ok) break;
      const int first = p.n_sink + (p.slot0 ? p.slot0[u / p.Hkv] : 0);
      const int j = (first & ~(kAsRows - 1)) + t * kAsM + r - first;
      if (j >= 0 && j < p.n_train) {
        const int a = besti < p.C ? besti : 0;   // NaN keys only
        p.assign[static_cast<size_t>(u) * p.n_train + j] = a;
        if (p.assign_out) p.assign_out[static_cast<size_t>(u) * p.n_train + j] = a;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

size_t assign_mma_smem_bytes() { return kAsSmemBytes; }

cudaError_t launch_centroid_terms(const TrainParams& p, cudaStream_t stream) {
  centroid_terms_kernel<<<dim3(p.B * p.Hkv, (p.Cpad + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_assign_mma(const CUtensorMap& tmk, const CUtensorMap& tmb, const TrainParams& p, int grid,
                              cudaStream_t stream) {
  cudaError_t e = ensure_dyn_smem<assign_mma_kernel>(kAsSmemBytes);
  if (e != cudaSuccess) return e;
  assign_mma_kernel<<<grid, kAsThreads, kAsSmemBytes, stream>>>(tmk, tmb, p);
  return cudaGetLastError();
}

}  // namespace pqhsa
