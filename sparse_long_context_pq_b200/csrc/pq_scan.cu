// PQ-HSA scoring and selection kernels:
//   tables   - per-query PQ look-up tables and centroid terms (q . codeword, q . centroid),
//              plus exact upper/lower bounds of every head's approximate logit;
//   scan     - one pass over the uint8 codes: approximate logits of every indexed
//              token, the selection score sigma = max over the group's heads,
//              per-cluster exp-weight sums and a histogram of sigma;
//   filter   - marks tokens above the threshold histogram bin, collects the
//              tokens in that bin as candidates;
//   finalize - resolves the candidates exactly (score desc, position asc),
//              compacts the selected positions in ascending order and removes
//              the selected tokens' weights from the cluster sums.
//
// Source: rit.work "pq-hsa-long-context-attention", section
// "Как приблизительные оценки возвращают отброшенный контекст" (an approximate
// logit for every indexed token from the IVF-PQ index; the best ones are read
// exactly under a 1 % budget; the rest stay in the normalisation), and section
// "Фоновый вклад сохранил точность, а длина дала ускорение" (the fixed costs:
// building tables, scanning compressed codes, selecting candidates).
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace pqhsa {

namespace {

__device__ __forceinline__ int unit_n(const int32_t* seq_lens, const int32_t* n_indexed, int b, int n_sink,
                                      int cap) {
  const int T = max(0, seq_lens[b]);
  const int s0 = min(n_sink, T);
  const int N = max(0, min(n_indexed[b], T - s0));
  return min(N, cap);
}

template <int G>
__device__ __forceinline__ void hist_range(const float* bounds, int u, int nq, float& lo, float& inv) {
  float ub[G], lb[G];
  unit_upper_bounds<G>(bounds, u, nq, ub);
  unit_lower_bounds<G>(bounds, u, nq, lb);
  float hi = ub[0];
  lo = lb[0];
#pragma unroll
  for (int g = 1; g < G; ++g) {
    hi = fmaxf(hi, ub[g]);
    lo = fmaxf(lo, lb[g]);   // sigma = max_g shat_g >= lb_g for every g
  }
  inv = (hi > lo) ? __fdiv_rn(static_cast<float>(kNB), __fsub_rn(hi, lo)) : 0.f;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One full warp: over counts cnt[0..nbins) (nbins a multiple of 32), find the bin
// b such that sum_{b' > b} cnt < need <= sum_{b' >= b} cnt. Writes *bin/*above
// only when such a bin exists.
__device__ void find_threshold_desc(const uint32_t* cnt, int nbins, uint32_t need, int* bin, uint32_t* above) {
  const int lane = threadIdx.x & 31;
  const int per = nbins / 32;
  const int hi = nbins - per * lane;   // lane 0 holds the highest bins
  const int lo = hi - per;
  uint32_t local = 0;
  for (int i = lo; i < hi; ++i) local += cnt[i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - local;
  if (need > 0 && excl < need && incl >= need) {
    uint32_t cum = excl;
    for (int i = hi - 1; i >= lo; --i) {
      if (cum + cnt[i] >= need) {
        *bin = i;
        *above = cum;
        break;
      }
      cum += cnt[i];
    }
  }
}

// ===========================================================================
// tables
// ===========================================================================
template <int G>
__global__ void __launch_bounds__(256) tables_kernel(TablesParams p) {
  constexpr int GP = (G + 3) / 4;
  constexpr int G4 = GP * 4;
  __shared__ float qsh[G4][kD];
  __shared__ float red[2][kM][G4];
  __shared__ float wred[2][8][G4];
  const int u = blockIdx.x;
  const int part = blockIdx.y;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  for (int i = tid; i < G4 * kD; i += blockDim.x) {
    const int g = i / kD, d = i % kD;
    qsh[g][d] = (g < G) ? p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * kD + d] * p.scale : 0.f;
  }
  __syncthreads();

  if (part == 0) {
    for (int i = tid; i < kNB; i += blockDim.x) p.hist[static_cast<size_t>(u) * kNB + i] = 0u;
    for (int i = tid; i < p.bitmap_words; i += blockDim.x) p.bitmap[static_cast<size_t>(u) * p.bitmap_words + i] = 0u;
    if (tid < static_cast<int>(sizeof(UnitState) / 4)) reinterpret_cast<int32_t*>(p.units + u)[tid] = 0;
    // LUT[m][s][g] = sum_d q'_g[8s+d] * codeword[s][m][d]; warp w owns subspaces w and w+8.
    for (int si = 0; si < 2; ++si) {
      const int s = warp + 8 * si;
      float mx[G4], mn[G4];
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        mx[g] = -INFINITY;
        mn[g] = INFINITY;
      }
      for (int jm = 0; jm < kNcode / 32; ++jm) {
        const int m = lane + 32 * jm;
        const float4* cwp =
            reinterpret_cast<const float4*>(p.codebooks + ((static_cast<size_t>(u) * kM + s) * kNcode + m) * kDsub);
        const float4 c0 = cwp[0], c1 = cwp[1];
        const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        float val[G4];
#pragma unroll
        for (int g = 0; g < G4; ++g) {
          float v = 0.f;
#pragma unroll
          for (int d = 0; d < kDsub; ++d) v = fmaf(qsh[g][s * kDsub + d], cw[d], v);
          val[g] = v;
          if (g < G) {
            mx[g] = fmaxf(mx[g], v);
            mn[g] = fminf(mn[g], v);
          }
        }
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) {
          float4* dst = reinterpret_cast<float4*>(p.lut) + ((static_cast<size_t>(u) * GP + gp) * kNcode + m) * kM + s;
          *dst = make_float4(val[gp * 4 + 0], val[gp * 4 + 1], val[gp * 4 + 2], val[gp * 4 + 3]);
        }
      }
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        const float a = warp_max(mx[g]);
        const float c = warp_min(mn[g]);
        if (lane == 0) {
          red[0][s][g] = (g < G) ? a : 0.f;
          red[1][s][g] = (g < G) ? c : 0.f;
        }
      }
    }
    __syncthreads();
    if (tid < 2 * G4) {
      const int mm = tid / G4, g = tid % G4;
      float acc = 0.f;
      for (int s = 0; s < kM; ++s) acc += red[mm][s][g];
      p.bounds[(static_cast<size_t>(u) * (1 + p.nq) * 2 + mm) * G4 + g] = acc;
    }
  } else {
    const int c0 = (part - 1) * 128;
    const int c1 = min(p.C, c0 + 128);
    const int nc = c1 - c0;
    for (int i = tid; i < G * nc; i += blockDim.x)
      p.W[(static_cast<size_t>(u) * G + i / nc) * p.C + c0 + (i % nc)] = 0.f;
    float mx[G4], mn[G4];
#pragma unroll
    for (int g = 0; g < G4; ++g) {
      mx[g] = -INFINITY;
      mn[g] = INFINITY;
    }
    for (int c = c0 + warp; c < c1; c += 8) {
      const float4 cv = *reinterpret_cast<const float4*>(p.centroids + (static_cast<size_t>(u) * p.C + c) * kD + lane * 4);
      float val[G4];
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        float v = qsh[g][lane * 4 + 0] * cv.x;
        v = fmaf(qsh[g][lane * 4 + 1], cv.y, v);
        v = fmaf(qsh[g][lane * 4 + 2], cv.z, v);
        v = fmaf(qsh[g][lane * 4 + 3], cv.w, v);
        val[g] = warp_sum(v);
        if (g < G) {
          mx[g] = fmaxf(mx[g], val[g]);
          mn[g] = fminf(mn[g], val[g]);
        }
      }
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) {
        if (lane == gp) {
          float4* dst = reinterpret_cast<float4*>(p.qc) + (static_cast<size_t>(u) * GP + gp) * p.C + c;
          *dst = make_float4(val[gp * 4 + 0], val[gp * 4 + 1], val[gp * 4 + 2], val[gp * 4 + 3]);
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        wred[0][warp][g] = mx[g];
        wred[1][warp][g] = mn[g];
      }
    }
    __syncthreads();
    if (tid < 2 * G4) {
      const int mm = tid / G4, g = tid % G4;
      float v = mm == 0 ? -INFINITY : INFINITY;
      for (int w = 0; w < 8; ++w) v = mm == 0 ? fmaxf(v, wred[0][w][g]) : fminf(v, wred[1][w][g]);
      if (g >= G) v = 0.f;
      p.bounds[((static_cast<size_t>(u) * (1 + p.nq) + part) * 2 + mm) * G4 + g] = v;
    }
  }
}

// ===========================================================================
// scan
// ===========================================================================
constexpr int kScanThreads = 256;
constexpr int kScanUnroll = 4;

template <int G>
struct ScanSmem {
  static constexpr int GP = (G + 3) / 4;
  static size_t bytes(int C) {
    return static_cast<size_t>(GP) * kNcode * kM * 16 + static_cast<size_t>(GP) * C * 16 +
           static_cast<size_t>(G) * C * 4 + kNB * 4;
  }
};

// Segment [j0, j1) of unit u: score every slot.
template <int G>
__device__ __forceinline__ void scan_segment(const ScanParams& p, int u, int j0, int j1, uint8_t* smem,
                                             const uint32_t ysoff[8], const uint32_t sel[4], bool swap_words) {
  constexpr int GP = (G + 3) / 4;
  const int tid = threadIdx.x;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int C = p.C;
  float4* lut_s = reinterpret_cast<float4*>(smem);                               // [GP][256][16]
  float4* qc_s = lut_s + GP * kNcode * kM;                                       // [GP][C]
  float* w_s = reinterpret_cast<float*>(qc_s + GP * C);                          // [G][C]
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(w_s + G * C);                   // [NB]

  __syncthreads();  // previous segment finished with shared memory
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.lut) + static_cast<size_t>(u) * GP * kNcode * kM;
    uint4* dst = reinterpret_cast<uint4*>(lut_s);
    for (int i = tid; i < GP * kNcode * kM; i += blockDim.x) dst[i] = src[i];
    const uint4* srcq = reinterpret_cast<const uint4*>(p.qc) + static_cast<size_t>(u) * GP * C;
    uint4* dstq = reinterpret_cast<uint4*>(qc_s);
    for (int i = tid; i < GP * C; i += blockDim.x) dstq[i] = srcq[i];
    for (int i = tid; i < G * C; i += blockDim.x) w_s[i] = 0.f;
    for (int i = tid; i < kNB; i += blockDim.x) hist_s[i] = 0u;
  }
  float ub2[G];
  {
    float ub[G];
    unit_upper_bounds<G>(p.bounds, u, p.nq, ub);
#pragma unroll
    for (int g = 0; g < G; ++g) ub2[g] = ub[g] * kLog2e;
  }
  float lo, inv;
  hist_range<G>(p.bounds, u, p.nq, lo, inv);
  __syncthreads();

  const uint8_t* codes_u = p.codes + static_cast<size_t>(u) * p.cap * kM;
  const uint16_t* ids_u = p.ids + static_cast<size_t>(u) * p.cap;
  float* sig_u = p.sigma + static_cast<size_t>(u) * p.cap;
  const uint8_t* lut_b = reinterpret_cast<const uint8_t*>(lut_s);
  bool bad_id = false;

  for (int base = j0; base < j1; base += kScanUnroll * kScanThreads) {
    uint4 cw[kScanUnroll];
    uint32_t idv[kScanUnroll];
#pragma unroll
    for (int r = 0; r < kScanUnroll; ++r) {
      const int j = base + r * kScanThreads + tid;
      if (j < j1) {
        cw[r] = __ldcs(reinterpret_cast<const uint4*>(codes_u) + j);
        idv[r] = __ldcs(ids_u + j);
      }
    }
#pragma unroll
    for (int r = 0; r < kScanUnroll; ++r) {
      const int j = base + r * kScanThreads + tid;
      if (j >= j1) continue;
      uint32_t w0 = cw[r].x, w1 = cw[r].y, w2 = cw[r].z, w3 = cw[r].w;
      if (swap_words) {
        uint32_t t = w0; w0 = w1; w1 = t;
        t = w2; w2 = w3; w3 = t;
      }
      uint32_t id = idv[r];
      if (id >= static_cast<uint32_t>(C)) {
        bad_id = true;
        id = 0;
      }
      float4 acc[GP];
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) acc[gp] = qc_s[gp * C + id];
#pragma unroll
      for (int i = 0; i < kM; ++i) {
        const uint32_t wd = (i < 4) ? w0 : (i < 8) ? w1 : (i < 12) ? w2 : w3;
        // offset of LUT entry [code][s] with s = i ^ (lane & 7): code*256 + s*16
        const uint32_t off = __byte_perm(wd, ysoff[i >> 1], sel[i & 3]);
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) {
          const float4 v = *reinterpret_cast<const float4*>(lut_b + gp * (kNcode * kM * 16) + off);
          acc[gp].x = __fadd_rn(acc[gp].x, v.x);
          acc[gp].y = __fadd_rn(acc[gp].y, v.y);
          acc[gp].z = __fadd_rn(acc[gp].z, v.z);
          acc[gp].w = __fadd_rn(acc[gp].w, v.w);
        }
      }
      float sh[G];
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) {
        if (gp * 4 + 0 < G) sh[gp * 4 + 0] = acc[gp].x;
        if (gp * 4 + 1 < G) sh[gp * 4 + 1] = acc[gp].y;
        if (gp * 4 + 2 < G) sh[gp * 4 + 2] = acc[gp].z;
        if (gp * 4 + 3 < G) sh[gp * 4 + 3] = acc[gp].w;
      }
      float sg = sh[0];
#pragma unroll
      for (int g = 1; g < G; ++g) sg = fmaxf(sg, sh[g]);
      __stcs(sig_u + j, sg);
      if (p.approx_logits) {
#pragma unroll
        for (int g = 0; g < G; ++g)
          p.approx_logits[(static_cast<size_t>(b) * p.Hq + h * G + g) * p.cap + j] = sh[g];
      }
#pragma unroll
      for (int g = 0; g < G; ++g) atomicAdd(&w_s[g * C + id], fast_exp2(fmaf(sh[g], kLog2e, -ub2[g])));
      atomicAdd(&hist_s[score_bin(sg, lo, inv)], 1u);
    }
  }
  if (bad_id) record_error(p.err, HSA_DEVERR_CLUSTER);
  __syncthreads();
  float* Wg = p.W + static_cast<size_t>(u) * G * C;
  for (int i = tid; i < G * C; i += blockDim.x) {
    const float v = w_s[i];
    if (v != 0.f) atomicAdd(Wg + i, v);
  }
  uint32_t* hg = p.hist + static_cast<size_t>(u) * kNB;
  for (int i = tid; i < kNB; i += blockDim.x) {
    const uint32_t v = hist_s[i];
    if (v) atomicAdd(hg + i, v);
  }
}

// Walk the balanced global slot range of this CTA over the units.
template <typename F>
__device__ __forceinline__ void for_each_segment(const int32_t* seq_lens, const int32_t* n_indexed, int B, int Hkv,
                                                 int n_sink, int cap, F&& f) {
  long long total = 0;
  for (int b = 0; b < B; ++b) total += static_cast<long long>(Hkv) * unit_n(seq_lens, n_indexed, b, n_sink, cap);
  const long long start = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  if (start >= end) return;
  long long acc = 0;
  for (int b = 0; b < B && acc < end; ++b) {
    const int n = unit_n(seq_lens, n_indexed, b, n_sink, cap);
    for (int h = 0; h < Hkv && acc < end; ++h) {
      if (start < acc + n && end > acc) {
        const int j0 = static_cast<int>(max(start - acc, 0LL));
        const int j1 = static_cast<int>(min(end - acc, static_cast<long long>(n)));
        f(b * Hkv + h, j0, j1);
      }
      acc += n;
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kScanThreads, 2) scan_kernel(ScanParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const uint32_t l7 = lane & 7;
  // Per-lane subspace skew: lookup i reads subspace s = i ^ (lane & 7), so the 8
  // lanes of a quarter-warp hit 8 different 16-byte bank groups.
  uint32_t ysoff[8], sel[4];
#pragma unroll
  for (int k2 = 0; k2 < 8; ++k2) {
    const uint32_t s_lo = ((2 * k2) ^ l7) & 15, s_hi = ((2 * k2 + 1) ^ l7) & 15;
    ysoff[k2] = (s_lo * 16u) | ((s_hi * 16u) << 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t bi = (i ^ l7) & 3;              // byte of the (swapped) word holding code s
    sel[i] = (4u + 2u * (i & 1)) | (bi << 4) | (5u << 8) | (5u << 12);
  }
  const bool swap_words = (l7 >> 2) & 1;
  pdl_wait();
  pdl_launch_dependents();
  for_each_segment(p.seq_lens, p.n_indexed, p.B, p.Hkv, p.n_sink, p.cap,
                   [&](int u, int j0, int j1) { scan_segment<G>(p, u, j0, j1, smem, ysoff, sel, swap_words); });
}

// ===========================================================================
// filter: tokens above the threshold bin are selected, the bin's tokens are candidates
// ===========================================================================
template <int G>
__global__ void __launch_bounds__(256) filter_kernel(SelectParams p) {
  __shared__ uint32_t hist_s[kNB];
  __shared__ int sh_bstar;
  __shared__ uint32_t sh_above;
  pdl_wait();
  pdl_launch_dependents();
  for_each_segment(p.seq_lens, p.n_indexed, p.B, p.Hkv, p.n_sink, p.cap, [&](int u, int j0, int j1) {
    const int b = u / p.Hkv;
    const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
    const int k = decode_k(p.budget, p.k_override, N);
    __syncthreads();
    for (int i = threadIdx.x; i < kNB; i += blockDim.x) hist_s[i] = p.hist[static_cast<size_t>(u) * kNB + i];
    if (threadIdx.x == 0) {
      sh_bstar = kNB;   // k == 0: nothing selected
      sh_above = 0;
    }
    __syncthreads();
    if (threadIdx.x < 32) find_threshold_desc(hist_s, kNB, static_cast<uint32_t>(k), &sh_bstar, &sh_above);
    __syncthreads();
    const int bstar = sh_bstar;
    if (threadIdx.x == 0) {
      p.units[u].bstar = bstar;
      p.units[u].above = static_cast<int32_t>(sh_above);
    }
    if (bstar >= kNB) return;
    float lo, inv;
    hist_range<G>(p.bounds, u, p.nq, lo, inv);
    const float* sig = p.sigma + static_cast<size_t>(u) * p.cap;
    uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;
    for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
      const float s = __ldcs(sig + j);
      const int bin = score_bin(s, lo, inv);
      if (bin > bstar) {
        atomicOr(bm + (j >> 5), 1u << (j & 31));
      } else if (bin == bstar) {
        const int slot = atomicAdd(&p.units[u].ncand, 1);
        if (slot < p.cap)
          p.cand[static_cast<size_t>(u) * p.cap + slot] =
              (static_cast<unsigned long long>(float_key(s)) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
      }
    }
  });
}

// ===========================================================================
// finalize (one CTA per unit)
// ===========================================================================
constexpr int kFinThreads = 1024;
constexpr int kFinSmemCand = 4096;

__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < nw ? warp_tot[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < nw) warp_tot[lane] = xi - x;   // exclusive prefix of warp totals
    if (lane == nw - 1) warp_tot[32] = xi;
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return r;
}

template <int G>
__global__ void __launch_bounds__(kFinThreads) finalize_kernel(SelectParams p) {
  constexpr int GP = (G + 3) / 4;
  __shared__ unsigned long long ck[kFinSmemCand];
  __shared__ uint32_t dig[256];
  __shared__ uint32_t warp_tot[33];
  __shared__ int sh_bin;
  __shared__ uint32_t sh_above;
  const int u = blockIdx.x;
  const int b = u / p.Hkv;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const int T = max(0, p.seq_lens[b]);
  const int s0 = min(p.n_sink, T);
  const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
  const int k = decode_k(p.budget, p.k_override, N);
  int32_t* sel_u = p.sel + static_cast<size_t>(u) * p.cap;
  uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;
  if (k == 0) {
    if (tid == 0 && p.dbg_nselected) p.dbg_nselected[u] = 0;
    return;
  }
  const UnitState st = p.units[u];
  const int m = min(st.ncand, p.cap);
  const int r = k - st.above;
  if (r < 1 || r > m) {
    if (tid == 0) record_error(p.err, HSA_DEVERR_SELECT);
  }
  const unsigned long long* cg = p.cand + static_cast<size_t>(u) * p.cap;
  const bool in_smem = m <= kFinSmemCand;
  if (in_smem)
    for (int i = tid; i < m; i += blockDim.x) ck[i] = cg[i];
  __syncthreads();
  const unsigned long long* keys = in_smem ? ck : cg;

  // ---- threshold key: the r-th largest candidate key (keys are distinct) ----
  unsigned long long tau = ~0ull;
  if (r >= 1 && r <= m) {
    if (m <= 256) {
      // rank selection; slot kFinSmemCand-1 is free because m <= 256
      if (tid == 0) ck[kFinSmemCand - 1] = ~0ull;
      __syncthreads();
      for (int i = tid; i < m; i += blockDim.x) {
        const unsigned long long key = keys[i];
        int rank = 0;
        for (int j = 0; j < m; ++j) rank += keys[j] > key;
        if (rank == r - 1) ck[kFinSmemCand - 1] = key;   // unique writer: keys are distinct
      }
      __syncthreads();
      tau = ck[kFinSmemCand - 1];
      __syncthreads();
    } else {
      unsigned long long prefix = 0, mask = 0;
      uint32_t need = static_cast<uint32_t>(r);
      for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += blockDim.x) dig[i] = 0u;
        if (tid == 0) {
          sh_bin = -1;
          sh_above = 0;
        }
        __syncthreads();
        for (int i = tid; i < m; i += blockDim.x) {
          const unsigned long long key = keys[i];
          if ((key & mask) == prefix) atomicAdd(&dig[(key >> shift) & 255ull], 1u);
        }
        __syncthreads();
        if (tid < 32) find_threshold_desc(dig, 256, need, &sh_bin, &sh_above);
        __syncthreads();
        const int d = sh_bin < 0 ? 0 : sh_bin;
        need -= sh_above;
        prefix |= static_cast<unsigned long long>(d) << shift;
        mask |= 255ull << shift;
        __syncthreads();
      }
      tau = prefix;
    }
    for (int i = tid; i < m; i += blockDim.x) {
      const unsigned long long key = keys[i];
      if (key >= tau) {
        const uint32_t j = 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
        atomicOr(bm + (j >> 5), 1u << (j & 31));
      }
    }
  }
  __threadfence_block();
  __syncthreads();

  // ---- compaction of the selection bitmap into ascending positions ----
  const int nw = (N + 31) / 32;
  uint32_t running = 0;
  for (int w0 = 0; w0 < nw; w0 += 4 * kFinThreads) {
    uint32_t words[4];
    uint32_t pc = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int wi = w0 + 4 * tid + e;
      words[e] = wi < nw ? bm[wi] : 0u;
      pc += __popc(words[e]);
    }
    uint32_t tot;
    uint32_t off = running + block_excl_scan(pc, warp_tot, tot);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t wv = words[e];
      const int wi = w0 + 4 * tid + e;
      while (wv) {
        const int bit = __ffs(wv) - 1;
        wv &= wv - 1;
        if (off < static_cast<uint32_t>(p.cap)) sel_u[off] = s0 + wi * 32 + bit;
        ++off;
      }
    }
    running += tot;
  }
  if (tid == 0) {
    p.units[u].nsel = static_cast<int32_t>(running);
    if (running != static_cast<uint32_t>(k)) record_error(p.err, HSA_DEVERR_SELECT);
    if (p.dbg_nselected) p.dbg_nselected[u] = static_cast<int32_t>(running);
  }
  __syncthreads();
  const int nsel = min(static_cast<int>(running), k);
  if (p.dbg_selected)
    for (int i = tid; i < nsel; i += blockDim.x) p.dbg_selected[static_cast<size_t>(u) * p.cap + i] = sel_u[i];

  // ---- remove the selected tokens' weights from the cluster sums ----
  if (p.background && N > k) {
    float ub[G];
    unit_upper_bounds<G>(p.bounds, u, p.nq, ub);
    const float4* lut4 = reinterpret_cast<const float4*>(p.lut) + static_cast<size_t>(u) * GP * kNcode * kM;
    const float4* qc4 = reinterpret_cast<const float4*>(p.qc) + static_cast<size_t>(u) * GP * p.C;
    float* Wu = p.W + static_cast<size_t>(u) * G * p.C;
    for (int i = tid; i < nsel; i += blockDim.x) {
      const int j = sel_u[i] - s0;
      uint32_t id = p.ids[static_cast<size_t>(u) * p.cap + j];
      if (id >= static_cast<uint32_t>(p.C)) id = 0;
      const uint8_t* cj = p.codes + (static_cast<size_t>(u) * p.cap + j) * kM;
      float4 acc[GP];
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) acc[gp] = qc4[gp * p.C + id];
#pragma unroll
      for (int s = 0; s < kM; ++s) {
        const int code = cj[s];
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) {
          const float4 v = lut4[(gp * kNcode + code) * kM + s];
          acc[gp].x = __fadd_rn(acc[gp].x, v.x);
          acc[gp].y = __fadd_rn(acc[gp].y, v.y);
          acc[gp].z = __fadd_rn(acc[gp].z, v.z);
          acc[gp].w = __fadd_rn(acc[gp].w, v.w);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 a = acc[g / 4];
        const float sh = (g % 4 == 0) ? a.x : (g % 4 == 1) ? a.y : (g % 4 == 2) ? a.z : a.w;
        atomicAdd(&Wu[g * p.C + id], -fast_exp2(fmaf(sh, kLog2e, -ub[g] * kLog2e)));
      }
    }
  }
}

template <typename Kern, typename P>
cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl, const P& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int scan_threads() { return kScanThreads; }

size_t scan_smem_bytes(int G, int C) {
  switch (G) {
    case 1: return ScanSmem<1>::bytes(C);
    case 2: return ScanSmem<2>::bytes(C);
    case 4: return ScanSmem<4>::bytes(C);
    default: return ScanSmem<8>::bytes(C);
  }
}

#define PQHSA_G_SWITCH(G, CALL) \
  switch (G) {                  \
    case 1: CALL(1);            \
    case 2: CALL(2);            \
    case 4: CALL(4);            \
    case 8: CALL(8);            \
    default: return cudaErrorInvalidValue; \
  }

cudaError_t launch_tables(int G, const TablesParams& p, cudaStream_t stream, bool pdl) {
  const dim3 grid(p.B * p.Hkv, 1 + p.nq);
#define CALL(GG) return launch_ex(tables_kernel<GG>, grid, dim3(256), 0, stream, pdl, p)
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

cudaError_t launch_scan(int G, const ScanParams& p, int grid, cudaStream_t stream, bool pdl) {
  const size_t smem = scan_smem_bytes(G, p.C);
#define CALL(GG)                                                                                         \
  {                                                                                                      \
    cudaError_t e = ensure_dyn_smem<scan_kernel<GG>>(smem);                                             \
    if (e != cudaSuccess) return e;                                                                      \
    return launch_ex(scan_kernel<GG>, dim3(grid), dim3(kScanThreads), smem, stream, pdl, p);            \
  }
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

cudaError_t launch_filter(int G, const SelectParams& p, int grid, cudaStream_t stream, bool pdl) {
#define CALL(GG) return launch_ex(filter_kernel<GG>, dim3(grid), dim3(256), 0, stream, pdl, p)
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

cudaError_t launch_finalize(int G, const SelectParams& p, cudaStream_t stream, bool pdl) {
#define CALL(GG) return launch_ex(finalize_kernel<GG>, dim3(p.B * p.Hkv), dim3(kFinThreads), 0, stream, pdl, p)
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

}  // namespace pqhsa
