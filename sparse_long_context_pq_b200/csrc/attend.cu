// Split-K decode attention over a paged bf16 KV cache (dense decode and the
// exact part of PQ-HSA), the cluster-background partial and the log-sum-exp
// merge of all partials.
//
// PQ-HSA source: rit.work "pq-hsa-long-context-attention", section
// "Как приблизительные оценки возвращают отброшенный контекст": selected,
// sink and recent tokens are attended exactly; unselected tokens enter the
// shared normalisation through their approximate logits and contribute
// (their cluster's summed weight) x (the cluster's mean value). The merge of
// partial numerators/denominators is O = sum_i e^{m_i-M} acc_i / sum_i e^{m_i-M} l_i.
//
// Design (sm_100a): one producer warp streams K/V rows into a ring of
// shared-memory tiles with mbarrier completion: dense reads use tensor TMA with
// one box per head-page (128-byte swizzle, 1024-byte aligned boxes); gathered
// rows (sink + selected + tail) use one 1-D bulk copy per 256-byte row into a
// 272-byte-stride layout. Both layouts are bank-conflict free for the two read
// patterns below. Four consumer warps each own every fourth 32-token tile:
// lane t computes token t's G logits, the warp keeps an online softmax, and
// each lane accumulates 4 output dims for all G heads. Partials are (m, l, acc)
// in log2 units.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace pqhsa {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 6;
constexpr int kHalfBytes = kTile * 128;        // swizzled: 32 rows x 128 B (64 bf16)
constexpr int kRowPitch = 272;                 // padded: 256-byte row + 16
constexpr int kStageBytes = 2 * kTile * kRowPitch;  // 17408 = 17 KB: K then V (either layout)
static_assert(kStageBytes % 1024 == 0, "stage bases must stay 1024-byte aligned");
static_assert(4 * kHalfBytes <= kStageBytes, "swizzled tiles fit a stage");

// Byte offset of 16-byte chunk c (0..15) of row r inside the K (or V) area of a stage.
template <bool kRows>
__device__ __forceinline__ uint32_t chunk_off(int r, int c) {
  if (kRows) return r * kRowPitch + c * 16;
  return (c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}
template <bool kRows>
__device__ __forceinline__ uint32_t v_area() { return kRows ? kTile * kRowPitch : 2 * kHalfBytes; }

template <int G>
struct AttendSmem {
  static constexpr int GP = (G + 3) / 4;
  static constexpr size_t stages = static_cast<size_t>(kStages) * kStageBytes;
  static constexpr size_t qs = kD * GP * 16;
  static constexpr size_t pbuf = kConsumerWarps * kTile * GP * 16;
  static constexpr size_t bars = 2 * kStages * 8;
  static constexpr size_t total = 1024 /*alignment slack*/ + stages + qs + pbuf + bars + 64;
};

// Position of row v of a unit's exact list: sink [0,s0), then the k selected
// positions (ascending), then the tail [s0+N, T).
__device__ __forceinline__ int exact_row_pos(int v, int s0, int k, int N, const int32_t* sel_u) {
  if (v < s0) return v;
  if (v < s0 + k) return sel_u[v - s0];
  return s0 + N + (v - s0 - k);
}

template <int G, bool kExact, bool kRows>
__global__ void __launch_bounds__(kThreads, 2)
    attend_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                  AttendParams p) {
  static_assert(kRows || !kExact, "gathered rows use bulk row copies");
  constexpr int GP = (G + 3) / 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float4* qs = reinterpret_cast<float4*>(smem + AttendSmem<G>::stages);               // [kD][GP]
  float4* pbuf = qs + kD * GP;                                                          // [warps][32][GP]
  uint64_t* full = reinterpret_cast<uint64_t*>(pbuf + kConsumerWarps * kTile * GP);
  uint64_t* empty = full + kStages;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int total_attend = p.U * p.nsplit;

  if (kExact && static_cast<int>(blockIdx.x) >= total_attend) {
    background_block<G>(p, blockIdx.x - total_attend, smem);
    return;
  }

  const int u = blockIdx.x / p.nsplit;
  const int split = blockIdx.x % p.nsplit;
  const int b = u / p.Hkv;
  const int h = u % p.Hkv;

  pdl_wait();
  pdl_launch_dependents();

  // ---- row range of this split ------------------------------------------
  const int T = max(0, p.seq_lens[b]);
  int s0 = 0, N = 0, k = 0, E = T;
  if (kExact) {
    s0 = min(p.n_sink, T);
    N = max(0, min(p.n_indexed[b], T - s0));
    N = min(N, p.cap);
    k = decode_k(p.budget, p.k_override, N);
    E = s0 + k + (T - s0 - N);
  }
  const int r0 = split * p.chunk;
  const int r1 = min(E, r0 + p.chunk);
  const int ntiles = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  const int32_t* sel_u = kExact ? p.sel + static_cast<size_t>(u) * p.cap : nullptr;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;

  // ---- stage q (pre-scaled by scale*log2 e) -------------------------------
  for (int i = tid; i < kD * GP * 4; i += blockDim.x) {
    const int d = i / (GP * 4);
    const int g = i % (GP * 4);
    float v = 0.f;
    if (g < G) v = p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * kD + d] * p.qscale;
    reinterpret_cast<float*>(qs)[i] = v;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ===================== producer warp =====================
    if (!kRows && lane == 0) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
    }
    bool ok = true;
    const int box_rows = kRows ? 1 : min(p.page_size, kTile);
    for (int t = 0; t < ntiles && ok; ++t) {
      const int s = t % kStages;
      if (t >= kStages) {
        if (lane == 0) ok = mbar_wait(&empty[s], ((t / kStages) - 1) & 1, p.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      const int row0 = r0 + t * kTile;
      const int nvalid = min(kTile, r1 - row0);
      uint8_t* st = stage_base + static_cast<size_t>(s) * kStageBytes;
      const int nbox = kRows ? nvalid : (nvalid + box_rows - 1) / box_rows;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox) * 2u * box_rows * 256u);
      __syncwarp();
      for (int i = lane; i < nbox; i += 32) {
        const int pos = kExact ? exact_row_pos(row0 + i, s0, k, N, sel_u) : row0 + i * box_rows;
        int page = (pos >= 0 && pos < T && pos / p.page_size < p.max_pages) ? bt[pos / p.page_size] : -1;
        if (page < 0 || page >= p.num_pages) {
          record_error(p.err, HSA_DEVERR_PAGE);
          page = 0;
        }
        const int y = (page * p.Hkv + h) * p.page_size + (pos % p.page_size);
        if (kRows) {
          const size_t src = static_cast<size_t>(y) * (kD * 2);
          bulk_load(st + i * kRowPitch, p.k_cache + src, 256u, &full[s]);
          bulk_load(st + v_area<kRows>() + i * kRowPitch, p.v_cache + src, 256u, &full[s]);
        } else {
          const int off = i * box_rows * 128;
          tma_load_2d(st + 0 * kHalfBytes + off, &tmap_k, &full[s], 0, y);
          tma_load_2d(st + 1 * kHalfBytes + off, &tmap_k, &full[s], 64, y);
          tma_load_2d(st + 2 * kHalfBytes + off, &tmap_v, &full[s], 0, y);
          tma_load_2d(st + 3 * kHalfBytes + off, &tmap_v, &full[s], 64, y);
        }
      }
    }
    // Drain: make sure every issued copy has landed before the CTA can exit.
    if (lane == 0) {
      for (int t = max(0, ntiles - kStages); t < ntiles; ++t) mbar_wait(&full[t % kStages], (t / kStages) & 1, p.err);
    }
    return;
  }

  // ======================= consumer warps =======================
  float m_run[G], l_lane[G], acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_lane[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.f;
  }
  const int vchunk = lane >> 1;          // 16-byte chunk holding dims 4*lane .. 4*lane+3
  const int vsub = (lane & 1) * 8;
  float4* pw = pbuf + warp * kTile * GP;

  for (int t = warp; t < ntiles; t += kConsumerWarps) {
    const int s = t % kStages;
    if (!mbar_wait(&full[s], (t / kStages) & 1, p.err)) break;
    const int nvalid = min(kTile, r1 - (r0 + t * kTile));
    const uint8_t* st = stage_base + static_cast<size_t>(s) * kStageBytes;

    // ---- logits: lane = token row ----
    float sc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sc[g] = 0.f;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(st + chunk_off<kRows>(lane, hf * 8 + c));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float kv = e ? bf16hi(w[jj]) : bf16lo(w[jj]);
            const int d = hf * 64 + c * 8 + jj * 2 + e;
#pragma unroll
            for (int gp = 0; gp < GP; ++gp) {
              const float4 qv = qs[d * GP + gp];
              if (gp * 4 + 0 < G) sc[gp * 4 + 0] = fmaf(qv.x, kv, sc[gp * 4 + 0]);
              if (gp * 4 + 1 < G) sc[gp * 4 + 1] = fmaf(qv.y, kv, sc[gp * 4 + 1]);
              if (gp * 4 + 2 < G) sc[gp * 4 + 2] = fmaf(qv.z, kv, sc[gp * 4 + 2]);
              if (gp * 4 + 3 < G) sc[gp * 4 + 3] = fmaf(qv.w, kv, sc[gp * 4 + 3]);
            }
          }
        }
      }
    }
    const bool valid = lane < nvalid;
    float pr[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float sv = valid ? sc[g] : -INFINITY;
      const float m_new = fmaxf(m_run[g], warp_max(sv));   // finite: at least one valid row
      const float alpha = fast_exp2(m_run[g] - m_new);     // m_run = -inf -> 0
      pr[g] = valid ? fast_exp2(sv - m_new) : 0.f;
      l_lane[g] = l_lane[g] * alpha + pr[g];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[g][i] *= alpha;
      m_run[g] = m_new;
    }
#pragma unroll
    for (int gp = 0; gp < GP; ++gp) {
      float4 v;
      v.x = (gp * 4 + 0 < G) ? pr[gp * 4 + 0] : 0.f;
      v.y = (gp * 4 + 1 < G) ? pr[gp * 4 + 1] : 0.f;
      v.z = (gp * 4 + 2 < G) ? pr[gp * 4 + 2] : 0.f;
      v.w = (gp * 4 + 3 < G) ? pr[gp * 4 + 3] : 0.f;
      pw[lane * GP + gp] = v;
    }
    __syncwarp();

    // ---- PV: lane owns dims 4*lane .. 4*lane+3 ----
    const uint8_t* vbase = st + v_area<kRows>() + vsub;
    for (int r = 0; r < nvalid; ++r) {
      const uint2 raw = *reinterpret_cast<const uint2*>(vbase + chunk_off<kRows>(r, vchunk));
      const float v0 = bf16lo(raw.x), v1 = bf16hi(raw.x), v2 = bf16lo(raw.y), v3 = bf16hi(raw.y);
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) {
        const float4 pv = pw[r * GP + gp];
        const float pp[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int g = gp * 4 + e;
          if (g < G) {
            acc[g][0] = fmaf(pp[e], v0, acc[g][0]);
            acc[g][1] = fmaf(pp[e], v1, acc[g][1]);
            acc[g][2] = fmaf(pp[e], v2, acc[g][2]);
            acc[g][3] = fmaf(pp[e], v3, acc[g][3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---- combine the consumer warps (reuse stage 0 area after the pipeline) ----
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  float* cm = reinterpret_cast<float*>(stage_base);            // [warps][G]
  float* cl = cm + kConsumerWarps * G;                         // [warps][G]
  float* cacc = cl + kConsumerWarps * G;                       // [warps][G][kD]
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float lw = warp_sum(l_lane[g]);
    if (lane == 0) {
      cm[warp * G + g] = m_run[g];
      cl[warp * G + g] = lw;
    }
    *reinterpret_cast<float4*>(&cacc[(warp * G + g) * kD + lane * 4]) =
        make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  const size_t slot = static_cast<size_t>(u) * p.S_tot + split;
  const int d = tid;  // 128 consumer threads, one output dim each
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * G + g]);
    float L = 0.f, a = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float f = fast_exp2(cm[w * G + g] - M);
        L += f * cl[w * G + g];
        a += f * cacc[(w * G + g) * kD + d];
      }
    }
    p.pacc[(slot * G + g) * kD + d] = a;
    if (d == 0) {
      p.pm[slot * G + g] = M;
      p.pl[slot * G + g] = L;
    }
  }
}

}  // namespace

// Background partial of one chunk of clusters: l_g = sum_c W_gc, acc_g = sum_c W_gc mean_v_c,
// relative to the reference ub_g (W was accumulated as e^{shat - ub}).
template <int G>
__device__ void background_block(const AttendParams& p, int j, uint8_t* smem) {
  const int u = j / p.nbg;
  const int cb = j % p.nbg;
  const int b = u / p.Hkv;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int NW = kThreads / 32;
  pdl_wait();
  pdl_launch_dependents();
  const int T = max(0, p.seq_lens[b]);
  const int s0 = min(p.n_sink, T);
  int N = max(0, min(p.n_indexed[b], T - s0));
  N = min(N, p.cap);
  const int k = decode_k(p.budget, p.k_override, N);
  const bool active = p.bg_enabled && N > k;
  const size_t slot = static_cast<size_t>(u) * p.S_tot + p.nsplit + cb;
  if (!active) {
    for (int i = tid; i < G * kD; i += blockDim.x) p.pacc[slot * G * kD + i] = 0.f;
    if (tid < G) {
      p.pm[slot * G + tid] = -INFINITY;
      p.pl[slot * G + tid] = 0.f;
    }
    return;
  }
  const int c0 = cb * kBgClusters;
  const int c1 = min(p.C, c0 + kBgClusters);
  const float* W = p.W + static_cast<size_t>(u) * G * p.C;
  const float* mv = p.mean_v + static_cast<size_t>(u) * p.C * kD;
  float acc[G][4], lsum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    lsum[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.f;
  }
  for (int c = c0 + warp; c < c1; c += NW) {
    const float4 m4 = *reinterpret_cast<const float4*>(mv + static_cast<size_t>(c) * kD + lane * 4);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float w = fmaxf(W[g * p.C + c], 0.f);
      lsum[g] += w;
      acc[g][0] = fmaf(w, m4.x, acc[g][0]);
      acc[g][1] = fmaf(w, m4.y, acc[g][1]);
      acc[g][2] = fmaf(w, m4.z, acc[g][2]);
      acc[g][3] = fmaf(w, m4.w, acc[g][3]);
    }
  }
  float* red = reinterpret_cast<float*>(smem);  // [NW][G][kD] + [NW][G]
  float* redl = red + NW * G * kD;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    *reinterpret_cast<float4*>(&red[(warp * G + g) * kD + lane * 4]) =
        make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    if (lane == 0) redl[warp * G + g] = lsum[g];
  }
  __syncthreads();
  float ub[G];
  unit_upper_bounds<G>(p.bounds, u, p.nq, ub);
  for (int i = tid; i < G * kD; i += blockDim.x) {
    const int g = i / kD;
    float a = 0.f;
    for (int w = 0; w < NW; ++w) a += red[(w * G + g) * kD + (i % kD)];
    p.pacc[slot * G * kD + i] = a;
  }
  if (tid < G) {
    float l = 0.f;
    for (int w = 0; w < NW; ++w) l += redl[w * G + tid];
    p.pm[slot * G + tid] = ub[tid] * kLog2e;
    p.pl[slot * G + tid] = l;
  }
}

namespace {

// out[b, qh] = sum_s e^{m_s - M} acc_s / sum_s e^{m_s - M} l_s over the S_tot partials of its unit.
template <int G>
__global__ void __launch_bounds__(128) merge_kernel(MergeParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int bq = blockIdx.x;            // b * Hq + qh
  const int b = bq / p.Hq, qh = bq % p.Hq;
  const int h = qh / G, g = qh % G;
  const size_t u = static_cast<size_t>(b) * p.Hkv + h;
  const int d = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < p.S_tot; ++s) M = fmaxf(M, p.pm[(u * p.S_tot + s) * G + g]);
  float L = 0.f, a = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.S_tot; ++s) {
      const size_t sl = (u * p.S_tot + s) * G + g;
      const float m = p.pm[sl];
      if (m == -INFINITY) continue;
      const float f = fast_exp2(m - M);
      L += f * p.pl[sl];
      a += f * p.pacc[sl * kD + d];
    }
  }
  p.out[static_cast<size_t>(bq) * kD + d] = (L > 0.f) ? a / L : 0.f;
}

template <int G, bool kExact, bool kRows>
cudaError_t launch_attend_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttendParams& p, int grid,
                            cudaStream_t stream, bool pdl) {
  auto kern = attend_kernel<G, kExact, kRows>;
  const size_t smem = AttendSmem<G>::total;
  cudaError_t e = ensure_dyn_smem<attend_kernel<G, kExact, kRows>>(smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, p);
}

template <int G>
cudaError_t launch_merge_t(const MergeParams& p, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * p.Hq);
  cfg.blockDim = dim3(kD);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<G>, p);
}

}  // namespace

int attend_slots_per_sm() { return 2; }
size_t attend_smem_bytes(int G) {
  switch (G) {
    case 1: return AttendSmem<1>::total;
    case 2: return AttendSmem<2>::total;
    case 4: return AttendSmem<4>::total;
    default: return AttendSmem<8>::total;
  }
}

cudaError_t launch_attend(int G, bool exact, bool rows, const CUtensorMap& tk, const CUtensorMap& tv,
                          const AttendParams& p, int grid, cudaStream_t stream, bool pdl) {
#define PQHSA_ATT(GG)                                                                  \
  case GG:                                                                             \
    if (exact) return launch_attend_t<GG, true, true>(tk, tv, p, grid, stream, pdl);   \
    if (rows) return launch_attend_t<GG, false, true>(tk, tv, p, grid, stream, pdl);   \
    return launch_attend_t<GG, false, false>(tk, tv, p, grid, stream, pdl);
  switch (G) {
    PQHSA_ATT(1)
    PQHSA_ATT(2)
    PQHSA_ATT(4)
    PQHSA_ATT(8)
    default: return cudaErrorInvalidValue;
  }
#undef PQHSA_ATT
}

cudaError_t launch_merge(int G, const MergeParams& p, cudaStream_t stream, bool pdl) {
  switch (G) {
    case 1: return launch_merge_t<1>(p, stream, pdl);
    case 2: return launch_merge_t<2>(p, stream, pdl);
    case 4: return launch_merge_t<4>(p, stream, pdl);
    case 8: return launch_merge_t<8>(p, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pqhsa
