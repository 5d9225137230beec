// PQ-HSA scoring and selection kernels:
//   tables   - per-query PQ look-up tables and centroid terms (q . codeword, q . centroid),
//              plus exact upper/lower bounds of every head's approximate logit;
//   scan     - one pass over the uint8 codes: approximate logits of every indexed
//              token, the selection score sigma = max over the group's heads,
//              per-cluster exp-weight sums, a histogram of sigma, each chunk's
//              largest sigma and the final logit bounds;
//   filter   - marks tokens above the threshold histogram bin, collects the
//              tokens in that bin as candidates (reading only chunks that reach
//              the bin) and removes the definite selections' weights;
//   finalize - resolves the candidates exactly (score desc, position asc),
//              writes the selected tokens as KV-pool rows in ascending position
//              order, removes the winners' weights and publishes the unit.
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

// ===========================================================================
// tables
// ===========================================================================
// q'_g = scale * q_g of the unit's heads into shared memory: every load of the thread in
// flight before the first store (256 threads).
template <int G4, int G>
__device__ __forceinline__ void stage_q(const TablesParams& p, int b, int h, int tid, float (*qsh)[kD]) {
  constexpr int kPer = G4 * kD / 256;
  float v[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int i = tid + r * 256, g = i / kD, d = i % kD;
    v[r] = (g < G) ? p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * kD + d] * p.scale : 0.f;
  }
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int i = tid + r * 256;
    qsh[i / kD][i % kD] = v[r];
  }
}
template <int G>
__global__ void __launch_bounds__(256) tables_kernel(TablesParams p) {
  constexpr int GP = (G + 3) / 4;
  constexpr int G4 = GP * 4;
  constexpr int kSubPerPart = kM / kLutParts;   // 4 subspaces per LUT CTA
  constexpr int kQcPerWarp = kQcSlice / 8;      // clusters per warp (8 warps per slice)
  __shared__ float qsh[G4][kD];
  __shared__ float wred[2][8][kSubPerPart][G4];
  const int u = blockIdx.x;
  const int part = blockIdx.y;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  float* bnd = p.bounds + static_cast<size_t>(u) * (kLutParts + p.nq) * 2 * G4;

  if (part < kLutParts) {
    // ---- LUT[m][s][g] = sum_d q'_g[8s+d] * codeword[s][m][d] for 4 subspaces; thread = codeword m ----
    const int m = tid;
    float4 cw[kSubPerPart][2];
#pragma unroll
    for (int i = 0; i < kSubPerPart; ++i) {
      const float4* src = reinterpret_cast<const float4*>(
          p.codebooks + ((static_cast<size_t>(u) * kM + part * kSubPerPart + i) * kNcode + m) * kDsub);
      cw[i][0] = src[0];
      cw[i][1] = src[1];
    }
    stage_q<G4, G>(p, b, h, tid, qsh);
    // zero this unit's selection state (spread over the LUT CTAs)
    for (int i = part * blockDim.x + tid; i < kNB; i += kLutParts * blockDim.x)
      p.hist[static_cast<size_t>(u) * kNB + i] = 0u;
    for (int i = part * blockDim.x + tid; i < p.bitmap_words; i += kLutParts * blockDim.x)
      p.bitmap[static_cast<size_t>(u) * p.bitmap_words + i] = 0u;
    if (part == 0 && tid < static_cast<int>(sizeof(UnitState) / 4)) reinterpret_cast<int32_t*>(p.units + u)[tid] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kSubPerPart; ++i) {
      const int s = part * kSubPerPart + i;
      const float c8[8] = {cw[i][0].x, cw[i][0].y, cw[i][0].z, cw[i][0].w,
                           cw[i][1].x, cw[i][1].y, cw[i][1].z, cw[i][1].w};
      float val[G4];
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        float v = 0.f;
#pragma unroll
        for (int d = 0; d < kDsub; ++d) v = fmaf(qsh[g][s * kDsub + d], c8[d], v);
        val[g] = v;
      }
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) {
        float4* dst = reinterpret_cast<float4*>(p.lut) + ((static_cast<size_t>(u) * GP + gp) * kNcode + m) * kM + s;
        *dst = make_float4(val[gp * 4 + 0], val[gp * 4 + 1], val[gp * 4 + 2], val[gp * 4 + 3]);
      }
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        const float a = warp_max(val[g]);
        const float c = warp_min(val[g]);
        if (lane == 0) {
          wred[0][warp][i][g] = a;
          wred[1][warp][i][g] = c;
        }
      }
    }
    __syncthreads();
    if (tid < 2 * G4) {
      const int mm = tid / G4, g = tid % G4;
      float acc = 0.f;
      for (int i = 0; i < kSubPerPart; ++i) {
        float v = wred[mm][0][i][g];
        for (int w = 1; w < 8; ++w) v = mm == 0 ? fmaxf(v, wred[0][w][i][g]) : fminf(v, wred[1][w][i][g]);
        acc += v;
      }
      bnd[(part * 2 + mm) * G4 + g] = (g < G) ? acc : 0.f;
    }
  } else {
    // ---- qc[c][g] = q'_g . centroid_c for one kQcSlice-cluster slice; lane = 4 dims ----
    const int slice = part - kLutParts;
    const int c0 = slice * kQcSlice + warp * kQcPerWarp;
    float4 cv[kQcPerWarp];
#pragma unroll
    for (int i = 0; i < kQcPerWarp; ++i) {
      const int c = c0 + i;
      cv[i] = c < p.C ? *reinterpret_cast<const float4*>(p.centroids + (static_cast<size_t>(u) * p.C + c) * kD + lane * 4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    stage_q<G4, G>(p, b, h, tid, qsh);
    {   // zero this slice's cluster weights
      const int cs = slice * kQcSlice, ce = min(p.C, cs + kQcSlice), nc = ce - cs;
      for (int i = tid; i < G * nc; i += blockDim.x)
        p.W[(static_cast<size_t>(u) * G + i / nc) * p.C + cs + (i % nc)] = 0.f;
    }
    __syncthreads();
    float mx[G4], mn[G4];
#pragma unroll
    for (int g = 0; g < G4; ++g) {
      mx[g] = -INFINITY;
      mn[g] = INFINITY;
    }
#pragma unroll
    for (int i = 0; i < kQcPerWarp; ++i) {
      const int c = c0 + i;
      float val[G4];
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        float v = qsh[g][lane * 4 + 0] * cv[i].x;
        v = fmaf(qsh[g][lane * 4 + 1], cv[i].y, v);
        v = fmaf(qsh[g][lane * 4 + 2], cv[i].z, v);
        v = fmaf(qsh[g][lane * 4 + 3], cv[i].w, v);
        val[g] = warp_sum(v);
      }
      if (c < p.C) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          mx[g] = fmaxf(mx[g], val[g]);
          mn[g] = fminf(mn[g], val[g]);
        }
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) {
          if (lane == gp) {
            float4* dst = reinterpret_cast<float4*>(p.qc) + (static_cast<size_t>(u) * GP + gp) * p.C + c;
            *dst = make_float4(val[gp * 4 + 0], val[gp * 4 + 1], val[gp * 4 + 2], val[gp * 4 + 3]);
          }
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        wred[0][warp][0][g] = mx[g];
        wred[1][warp][0][g] = mn[g];
      }
    }
    __syncthreads();
    if (tid < 2 * G4) {
      const int mm = tid / G4, g = tid % G4;
      float v = wred[mm][0][0][g];
      for (int w = 1; w < 8; ++w) v = mm == 0 ? fmaxf(v, wred[0][w][0][g]) : fminf(v, wred[1][w][0][g]);
      bnd[(part * 2 + mm) * G4 + g] = (g < G) ? v : 0.f;
    }
  }
}

// ===========================================================================
// scan
// ===========================================================================
// One CTA per SM: 16 warps share one copy of the tables. Each lane streams the codes
// (16 B) and index slot (4 B) of its own list slot, for the warp's next D chunks, into a
// private ring with LSU async copies (one commit group per chunk), so D chunks per warp
// are in flight while it scores the current one.
// threads per scan CTA (one CTA per SM; registers bound the warp count)
template <int G>
__host__ __device__ constexpr int scan_threads_of() { return 512; }
constexpr int kRingCodeBytes = 32 * kM;                     // 512 per chunk
constexpr int kRingJsBytes = 32 * 4;                        // index slots
constexpr int kRingSlotBytes = kRingCodeBytes + kRingJsBytes + 16;   // + cluster word (16-B cell) = 656
constexpr size_t kScanSmemLimit = 226 * 1024;   // dynamic; the rest of 227 KB is static

template <int G>
struct ScanSmem {
  static constexpr int GP = (G + 3) / 4;
  // tables (LUT, centroid terms) and the score histogram; then the warps' rings
  // ([D][32][16 B] codes, [D][32] index slots, [D] 16-B cells holding the 4-byte word
  // with the chunk's cluster id, per warp); then the tables mbarrier
  __host__ __device__ static size_t tables(int C) {
    return align_up(static_cast<size_t>(GP) * kNcode * kM * 16 + static_cast<size_t>(GP) * C * 16 + kNB * 4, 128);
  }
  __host__ __device__ static size_t bytes(int C, int depth) {
    return tables(C) + static_cast<size_t>(scan_threads_of<G>() / 32) * depth * kRingSlotBytes + 8;
  }
  // deepest ring (8, 4 or 2 chunks per warp) that fits; 0 if none does
  static int depth(int C) {
    for (int d = 8; d >= 2; d >>= 1)
      if (bytes(C, d) <= kScanSmemLimit) return d;
    return 0;
  }
};

template <int G>
__device__ __forceinline__ void score_token(const uint4& code, uint32_t id, const uint8_t* lut_b, const float4* qc_s,
                                            int C, const uint32_t ysoff[8], const uint32_t sel[4], bool swap_words,
                                            float* sh) {
  constexpr int GP = (G + 3) / 4;
  uint32_t w0 = code.x, w1 = code.y, w2 = code.z, w3 = code.w;
  if (swap_words) {
    uint32_t t = w0; w0 = w1; w1 = t;
    t = w2; w2 = w3; w3 = t;
  }
  // Two independent partial sums per head (even / odd lookups) halve the dependent add
  // chain; each float4 of 4 heads is two packed f32x2 additions.
  ulonglong2 acc[2][GP];
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) {
    acc[0][gp] = reinterpret_cast<const ulonglong2*>(qc_s)[gp * C + id];
    acc[1][gp] = make_ulonglong2(0ull, 0ull);
  }
#pragma unroll
  for (int i = 0; i < kM; ++i) {
    const uint32_t wd = (i < 4) ? w0 : (i < 8) ? w1 : (i < 12) ? w2 : w3;
    // offset of LUT entry [code][s] with s = i ^ (lane & 7): code*256 + s*16
    const uint32_t off = __byte_perm(wd, ysoff[i >> 1], sel[i & 3]);
#pragma unroll
    for (int gp = 0; gp < GP; ++gp) {
      const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(lut_b + gp * (kNcode * kM * 16) + off);
      ulonglong2& a = acc[i & 1][gp];
      a.x = fadd2_rn(a.x, v.x);
      a.y = fadd2_rn(a.y, v.y);
    }
  }
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) {
    const unsigned long long xy = fadd2_rn(acc[0][gp].x, acc[1][gp].x);
    const unsigned long long zw = fadd2_rn(acc[0][gp].y, acc[1][gp].y);
    if (gp * 4 + 0 < G) sh[gp * 4 + 0] = lo_f(xy);
    if (gp * 4 + 1 < G) sh[gp * 4 + 1] = hi_f(xy);
    if (gp * 4 + 2 < G) sh[gp * 4 + 2] = lo_f(zw);
    if (gp * 4 + 3 < G) sh[gp * 4 + 3] = hi_f(zw);
  }
}

// Warp sum of G per-lane values, scattered: after log2(G) halving exchanges each lane
// holds a partial of one value, then plain butterflies finish it. Returns the total of
// value (lane >> (5 - log2 G)) in every lane of that group (lane (32/G)*g holds head g).
template <int G>
__device__ __forceinline__ float warp_sum_scatter(float* v) {
  const int lane = threadIdx.x & 31;
  int n = G;
  int o = 16;
#pragma unroll
  for (int step = 0; (1 << step) < G; ++step) {
    const bool up = (lane & o) != 0;
    const int half = n >> 1;
#pragma unroll
    for (int i = 0; i < G / 2; ++i) {
      if (i < half) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    n = half;
    o >>= 1;
  }
  float t = v[0];
  for (; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// Chunks [ch0, ch1) of unit u's cluster-ordered list: one warp scores one 32-slot
// chunk (all members of one cluster), so the centroid term is warp-uniform and the
// chunk's cluster weights are one warp reduction. Warp w takes chunks ch0 + w + 16 i
// through its D-slot ring; `phase` counts segments (tables mbarrier parity).
template <int G, int D>
__device__ __forceinline__ void scan_segment(const ScanParams& p, int u, int ch0, int ch1, uint8_t* smem,
                                             uint64_t* bar, uint32_t phase, float* sh_bounds,
                                             const uint32_t ysoff[8], const uint32_t sel[4], bool swap_words) {
  constexpr int GP = (G + 3) / 4;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int C = p.C;
  const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
  const uint32_t lut_bytes = GP * kNcode * kM * 16;
  const uint32_t qc_bytes = GP * C * 16;
  float4* lut_s = reinterpret_cast<float4*>(smem);                               // [GP][256][16]
  float4* qc_s = lut_s + GP * kNcode * kM;                                       // [GP][C]
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(qc_s + GP * C);                 // [NB]
  uint8_t* wring = smem + ScanSmem<G>::tables(C) + static_cast<size_t>(warp) * D * kRingSlotBytes;
  uint4* ring_code = reinterpret_cast<uint4*>(wring) + lane;                              // [D][32]
  int32_t* ring_js = reinterpret_cast<int32_t*>(wring + D * kRingCodeBytes) + lane;       // [D][32]
  uint32_t* ring_cl = reinterpret_cast<uint32_t*>(wring + D * (kRingCodeBytes + kRingJsBytes));   // [D][4]

  __syncthreads();  // previous segment finished with shared memory
  if (tid == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, lut_bytes + qc_bytes);
    const uint8_t* lg = reinterpret_cast<const uint8_t*>(p.lut) + static_cast<size_t>(u) * lut_bytes;
    for (uint32_t o = 0; o < lut_bytes; o += 32768u)
      bulk_load(reinterpret_cast<uint8_t*>(lut_s) + o, lg + o, min(32768u, lut_bytes - o), bar);
    const uint8_t* qg = reinterpret_cast<const uint8_t*>(p.qc) + static_cast<size_t>(u) * qc_bytes;
    for (uint32_t o = 0; o < qc_bytes; o += 32768u)
      bulk_load(reinterpret_cast<uint8_t*>(qc_s) + o, qg + o, min(32768u, qc_bytes - o), bar);
  }
  const uint4* lcodes = reinterpret_cast<const uint4*>(p.list_codes) + static_cast<size_t>(u) * p.list_slots;
  const int32_t* lslot = p.list_slot + static_cast<size_t>(u) * p.list_slots;
  const uint16_t* ccl = p.chunk_cluster + static_cast<size_t>(u) * (p.list_slots / 32);
  float* sig_u = p.sigma + static_cast<size_t>(u) * p.list_slots;
  float* Wu = p.W + static_cast<size_t>(u) * G * C;
  const uint8_t* lut_b = reinterpret_cast<const uint8_t*>(lut_s);

  // this warp's chunks; the first D go out while the tables land (one commit group per
  // chunk, empty groups past the end keep the count regular). The chunk's cluster id
  // (u16) comes with lane 0's group as the aligned 4-byte word that holds it.
  const int first = ch0 + warp;
  constexpr int kScanWarps = scan_threads_of<G>() / 32;
  const int cnt = first < ch1 ? (ch1 - first + kScanWarps - 1) / kScanWarps : 0;
  auto issue = [&](int i) {
    if (i < cnt) {
      const int ch = first + kScanWarps * i;
      const int slot = i % D;
      cp_async_16(ring_code + slot * 32, lcodes + static_cast<size_t>(ch) * 32 + lane);
      cp_async_4(ring_js + slot * 32, lslot + static_cast<size_t>(ch) * 32 + lane);
      if (lane == 0)
        cp_async_4(ring_cl + slot * 4,
                   reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(ccl + ch) & ~uintptr_t(3)));
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < D; ++i) issue(i);

  for (int i = tid; i < kNB; i += blockDim.x) hist_s[i] = 0u;
  if (warp == 0) {   // final bounds of the unit, once: this CTA's copy and the later kernels'
    reduce_bounds_warp<G>(p.bounds, u, p.nq, sh_bounds, sh_bounds + G);
    __syncwarp();
    if (lane < 2 * G) p.fbounds[static_cast<size_t>(u) * 2 * G + lane] = sh_bounds[lane];
  }
  __syncthreads();                       // zeroed histogram and bounds visible
  float ub2[G], lo, inv;
  {
    float ub[G], lb[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      ub[g] = sh_bounds[g];
      lb[g] = sh_bounds[G + g];
    }
    float hi = ub[0];
    lo = lb[0];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      ub2[g] = ub[g] * kLog2e;
      hi = fmaxf(hi, ub[g]);
      lo = fmaxf(lo, lb[g]);
    }
    inv = (hi > lo) ? __fdiv_rn(static_cast<float>(kNB), __fsub_rn(hi, lo)) : 0.f;
  }
  mbar_wait(bar, phase & 1, p.err);      // tables landed
  bool bad_id = false;

  for (int i = 0; i < cnt; ++i) {
    const int slot = i % D;
    cp_async_wait<D - 1>();              // this lane's copies of chunk i have landed
    __syncwarp();                        // ... and lane 0's cluster word
    const uint4 code = ring_code[slot * 32];
    const int32_t js = ring_js[slot * 32];
    const int ch = first + kScanWarps * i;
    const uint32_t cw = ring_cl[slot * 4];
    uint32_t id = ((reinterpret_cast<uintptr_t>(ccl + ch) >> 1) & 1) ? (cw >> 16) : (cw & 0xffffu);
    if (id >= static_cast<uint32_t>(C)) {
      bad_id = true;
      id = 0;
    }
    const bool valid = js >= 0 && js < N;
    float sh[G];
    score_token<G>(code, id, lut_b, qc_s, C, ysoff, sel, swap_words, sh);
    float sg = sh[0];
#pragma unroll
    for (int g = 1; g < G; ++g) sg = fmaxf(sg, sh[g]);
    __stcs(sig_u + static_cast<size_t>(ch) * 32 + lane, valid ? sg : -INFINITY);
    {   // the chunk's largest score lets the filter skip chunks below the threshold
      const float cmx = warp_max(valid ? sg : -INFINITY);
      if (lane == 0) p.chunk_max[static_cast<size_t>(u) * (p.list_slots / 32) + ch] = cmx;
    }
    if (p.approx_logits && valid) {
#pragma unroll
      for (int g = 0; g < G; ++g) p.approx_logits[(static_cast<size_t>(b) * p.Hq + h * G + g) * p.cap + js] = sh[g];
    }
    {
      float ev[G];
#pragma unroll
      for (int g = 0; g < G; ++g) ev[g] = valid ? fast_exp2(fmaf(sh[g], kLog2e, -ub2[g])) : 0.f;
      const float e = warp_sum_scatter<G>(ev);
      constexpr int kGroup = 32 / G;
      if ((lane & (kGroup - 1)) == 0) atomicAdd(Wu + (lane / kGroup) * C + id, e);
    }
    if (valid) atomicAdd(&hist_s[score_bin(sg, lo, inv)], 1u);
    __syncwarp();                        // every lane has read the slot
    issue(i + D);                        // refill it with the chunk D ahead
  }
  cp_async_wait<0>();
  if (bad_id) record_error(p.err, HSA_DEVERR_CLUSTER);
  __syncthreads();
  uint32_t* hg = p.hist + static_cast<size_t>(u) * kNB;
  for (int i = tid; i < kNB; i += blockDim.x) {
    const uint32_t v = hist_s[i];
    if (v) atomicAdd(hg + i, v);
  }
}

// Walk the balanced global item range of this CTA over the units; count(b, h) gives
// the items of unit (b, h). f(u, i0, i1) is called for every overlapped unit range.
template <typename Count, typename F>
__device__ __forceinline__ void for_each_range(int B, int Hkv, Count&& count, F&& f) {
  long long total = 0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) total += count(b, h);
  const long long start = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  if (start >= end) return;
  long long acc = 0;
  for (int b = 0; b < B && acc < end; ++b) {
    for (int h = 0; h < Hkv && acc < end; ++h) {
      const int n = count(b, h);
      if (start < acc + n && end > acc) {
        const int j0 = static_cast<int>(max(start - acc, 0LL));
        const int j1 = static_cast<int>(min(end - acc, static_cast<long long>(n)));
        f(b * Hkv + h, j0, j1);
      }
      acc += n;
    }
  }
}

// Work split for kernels whose items are grouped by unit. With at least as many CTAs as
// units that have work, every CTA takes one part of exactly one unit (1 + a share of the
// spare CTAs in proportion to the unit's items), so no CTA pays a second unit's set-up;
// a few CTAs may be left idle. Otherwise the balanced range walk. Calls f(u, i0, i1).
template <typename Count, typename F>
__device__ __forceinline__ void for_each_unit_part(int B, int Hkv, Count&& count, F&& f) {
  long long total = 0;
  int active = 0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const int n = count(b, h);
      total += n;
      active += n > 0;
    }
  const int grid = static_cast<int>(gridDim.x);
  if (active == 0) return;
  if (active > grid) {
    for_each_range(B, Hkv, count, f);
    return;
  }
  const long long spare = grid - active;
  int base = 0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const int n = count(b, h);
      if (n <= 0) continue;
      const int parts = 1 + static_cast<int>(spare * n / total);
      const int k = static_cast<int>(blockIdx.x) - base;
      if (k >= 0 && k < parts) {
        const int i0 = static_cast<int>(static_cast<long long>(n) * k / parts);
        const int i1 = static_cast<int>(static_cast<long long>(n) * (k + 1) / parts);
        if (i1 > i0) f(b * Hkv + h, i0, i1);
        return;
      }
      base += parts;
    }
}

__device__ __forceinline__ int unit_chunks(const int32_t* list_meta, int u, int C, int max_chunks) {
  const int n = list_meta[static_cast<size_t>(u) * (2 + 2 * static_cast<size_t>(C))];
  return max(0, min(n, max_chunks));
}

template <int G, int D>
__global__ void __launch_bounds__(scan_threads_of<G>(), 1) scan_kernel(ScanParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float sh_bounds[2 * G];
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
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + ScanSmem<G>::tables(p.C) +
                                              static_cast<size_t>(scan_threads_of<G>() / 32) * D * kRingSlotBytes);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  pdl_wait();
  pdl_launch_dependents();
  uint32_t phase = 0;
  const int max_chunks = p.list_slots / 32;
  for_each_unit_part(
      p.B, p.Hkv, [&](int b, int h) { return unit_chunks(p.list_meta, b * p.Hkv + h, p.C, max_chunks); },
      [&](int u, int c0, int c1) {
        scan_segment<G, D>(p, u, c0, c1, smem, bar, phase, sh_bounds, ysoff, sel, swap_words);
        ++phase;
      });
}

// ===========================================================================
// filter: tokens above the threshold bin are selected, the bin's tokens are candidates
// ===========================================================================
// Head weights e^{shat_g - ub_g} of one indexed token (cluster id, code words cw), from
// the decode tables: the same quantities the scan added into its cluster's sums.
template <int G>
__device__ __forceinline__ void token_weights(const SelectParams& p, int u, uint32_t id, const uint4 cw,
                                              const float* ub2, float* e) {
  constexpr int GP = (G + 3) / 4;
  const uint32_t cwords[4] = {cw.x, cw.y, cw.z, cw.w};
  const float4* lut4 = reinterpret_cast<const float4*>(p.lut) + static_cast<size_t>(u) * GP * kNcode * kM;
  const float4* qc4 = reinterpret_cast<const float4*>(p.qc) + static_cast<size_t>(u) * GP * p.C;
  float4 acc[GP];
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) acc[gp] = qc4[gp * p.C + id];
#pragma unroll
  for (int s = 0; s < kM; ++s) {
    const int code = (cwords[s >> 2] >> (8 * (s & 3))) & 255;
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
    e[g] = fast_exp2(fmaf(sh, kLog2e, -ub2[g]));
  }
}

// Take a selected token's head weights out of its cluster's sums.
template <int G>
__device__ __forceinline__ void remove_weights(const SelectParams& p, int u, uint32_t id, const float* e) {
  float* Wu = p.W + static_cast<size_t>(u) * G * p.C;
#pragma unroll
  for (int g = 0; g < G; ++g) atomicAdd(&Wu[g * p.C + id], -e[g]);
}

// Filter over chunks: the scan left each 32-slot chunk's largest score, so a chunk whose
// maximum falls below the threshold bin holds no selected or candidate token (the bin is
// monotone in the score) and is skipped; only the few chunks that reach it are read.
constexpr int kFilterThreads = 256;
constexpr int kCmPerThread = 4;                                    // chunk maxima per thread per pass
constexpr int kCmPass = kCmPerThread * kFilterThreads;             // chunks examined per pass
constexpr int kActPerWarp = 4;                                     // active chunks per warp per round
constexpr int kFixCap = kActPerWarp * kFilterThreads;              // queued tokens per round (<= one per slot)

template <int G>
__global__ void __launch_bounds__(kFilterThreads, 2) filter_kernel(SelectParams p) {
  __shared__ __align__(16) uint32_t hist_s[kNB];
  __shared__ uint32_t scan_tot[33];
  __shared__ int sh_bstar;
  __shared__ uint32_t sh_above;
  __shared__ int32_t act[kCmPass];          // active chunks of the current pass
  __shared__ int n_act;
  __shared__ uint32_t fix_list[kFixCap];   // list slots
  __shared__ int32_t fix_cand[kFixCap];     // candidate slot, or -1 for a definite selection
  __shared__ uint32_t fix_n;
  static_assert(kNB == 8 * kFilterThreads, "filter threshold search: 256 threads x 8 bins");
  constexpr int NW = kFilterThreads / 32;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  const int max_chunks = p.list_slots / 32;
  for_each_unit_part(
      p.B, p.Hkv, [&](int b, int h) { return unit_chunks(p.list_meta, b * p.Hkv + h, p.C, max_chunks); },
      [&](int u, int c0, int c1) {
    const int b = u / p.Hkv;
    const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
    const int k = decode_k(p.budget, p.k_override, N);
    const float* sig = p.sigma + static_cast<size_t>(u) * p.list_slots;
    const int32_t* lslot = p.list_slot + static_cast<size_t>(u) * p.list_slots;
    const float* cmax = p.chunk_max + static_cast<size_t>(u) * max_chunks;
    // bounds and the first pass of chunk maxima load with the histogram
    float ub[G], lb[G];
    final_bounds<G>(p.fbounds, u, ub, lb);
    float cm[kCmPerThread];
#pragma unroll
    for (int e = 0; e < kCmPerThread; ++e) {
      const int c = c0 + tid + e * kFilterThreads;
      cm[e] = c < c1 ? cmax[c] : -INFINITY;
    }
    __syncthreads();   // shared state of a previous unit range is no longer read
    {
      const uint4* hg = reinterpret_cast<const uint4*>(p.hist + static_cast<size_t>(u) * kNB);
      uint4 hv[kNB / 4 / kFilterThreads];
#pragma unroll
      for (int r = 0; r < kNB / 4 / kFilterThreads; ++r) hv[r] = hg[r * kFilterThreads + tid];
#pragma unroll
      for (int r = 0; r < kNB / 4 / kFilterThreads; ++r) reinterpret_cast<uint4*>(hist_s)[r * kFilterThreads + tid] = hv[r];
    }
    if (tid == 0) {
      sh_bstar = kNB;   // k == 0: nothing selected
      sh_above = 0;
      fix_n = 0;
    }
    __syncthreads();
    {
      // thread t owns the 8 bins [kNB-8(t+1), kNB-8t): block scan of counts from the top
      const int hi = kNB - 8 * tid;
      uint32_t c8[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c8[i] = hist_s[hi - 1 - i];
        local += c8[i];
      }
      uint32_t tot;
      const uint32_t excl = block_excl_scan(local, scan_tot, tot);
      const uint32_t need = static_cast<uint32_t>(k);
      if (need > 0 && excl < need && excl + local >= need) {
        uint32_t cum = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum < need && cum + c8[i] >= need) {
            sh_bstar = hi - 1 - i;
            sh_above = cum;
          }
          cum += c8[i];
        }
      }
    }
    __syncthreads();
    const int bstar = sh_bstar;
    if (tid == 0) {
      p.units[u].bstar = bstar;
      p.units[u].above = static_cast<int32_t>(sh_above);
    }
    if (bstar >= kNB) return;
    float hi = ub[0], lo = lb[0];
#pragma unroll
    for (int g = 1; g < G; ++g) {
      hi = fmaxf(hi, ub[g]);
      lo = fmaxf(lo, lb[g]);
    }
    const float inv = (hi > lo) ? __fdiv_rn(static_cast<float>(kNB), __fsub_rn(hi, lo)) : 0.f;
    float ub2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) ub2[g] = ub[g] * kLog2e;
    const bool fix = p.background && N > k;
    const uint4* lcodes = reinterpret_cast<const uint4*>(p.list_codes) + static_cast<size_t>(u) * p.list_slots;
    const uint16_t* ccl = p.chunk_cluster + static_cast<size_t>(u) * max_chunks;
    uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;

    for (int cb = c0; cb < c1; cb += kCmPass) {
      if (cb != c0) {
#pragma unroll
        for (int e = 0; e < kCmPerThread; ++e) {
          const int c = cb + tid + e * kFilterThreads;
          cm[e] = c < c1 ? cmax[c] : -INFINITY;
        }
        __syncthreads();   // the previous pass is done with act[]
      }
      if (tid == 0) n_act = 0;
      __syncthreads();
      // chunks whose maximum reaches the threshold bin, compacted warp by warp
#pragma unroll
      for (int e = 0; e < kCmPerThread; ++e) {
        const int c = cb + tid + e * kFilterThreads;
        const bool active = c < c1 && score_bin(cm[e], lo, inv) >= bstar;
        const uint32_t m = __ballot_sync(0xffffffffu, active);
        if (m) {
          const uint32_t leader = __ffs(m) - 1;
          int at = 0;
          if (lane == leader) at = atomicAdd(&n_act, __popc(m));
          at = __shfl_sync(0xffffffffu, at, leader);
          if (active) act[at + __popc(m & ((1u << lane) - 1u))] = c;
        }
      }
      __syncthreads();
      const int na = n_act;
      for (int a0 = 0; a0 < na; a0 += NW * kActPerWarp) {
        // each warp reads up to kActPerWarp active chunks at once; lane = slot of the chunk
        float sv[kActPerWarp];
        int32_t jv[kActPerWarp];
        int chv[kActPerWarp];
#pragma unroll
        for (int r = 0; r < kActPerWarp; ++r) {
          const int a = a0 + warp + NW * r;
          chv[r] = a < na ? act[a] : -1;
          sv[r] = chv[r] >= 0 ? sig[static_cast<size_t>(chv[r]) * 32 + lane] : -INFINITY;
          jv[r] = chv[r] >= 0 ? lslot[static_cast<size_t>(chv[r]) * 32 + lane] : -1;
        }
#pragma unroll
        for (int r = 0; r < kActPerWarp; ++r) {
          const int j = jv[r];            // index slot of this list slot
          const bool valid = j >= 0 && j < N;
          const int bin = valid ? score_bin(sv[r], lo, inv) : -1;
          const bool definite = bin > bstar;
          if (definite) atomicOr(bm + (j >> 5), 1u << (j & 31));
          int slot = -1;
          if (bin == bstar) {
            slot = atomicAdd(&p.units[u].ncand, 1);
            if (slot < p.cap)
              p.cand[static_cast<size_t>(u) * p.cap + slot] =
                  (static_cast<unsigned long long>(float_key(sv[r])) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
          }
          if (fix) {
            // queue the list slot: a definite selection's weight leaves its cluster's sums
            // below; a candidate's weights are stored for the finalize's winners
            const bool queued = definite || (slot >= 0 && slot < kCandWeights);
            const uint32_t m = __ballot_sync(0xffffffffu, queued);
            if (m) {
              const uint32_t leader = __ffs(m) - 1;
              uint32_t at = 0;
              if (lane == leader) at = atomicAdd(&fix_n, static_cast<uint32_t>(__popc(m)));
              at = __shfl_sync(0xffffffffu, at, leader);
              if (queued) {
                at += __popc(m & ((1u << lane) - 1u));
                fix_list[at] = static_cast<uint32_t>(chv[r]) * 32 + lane;
                fix_cand[at] = definite ? -1 : slot;
              }
            }
          }
        }
        if (fix) {
          // queued tokens of this round: one per thread, every look-up of a token in flight together
          __syncthreads();
          const uint32_t n = fix_n;
          for (uint32_t i = tid; i < n; i += kFilterThreads) {
            const uint32_t ls = fix_list[i];
            const int cs = fix_cand[i];
            uint32_t id = ccl[ls >> 5];
            if (id >= static_cast<uint32_t>(p.C)) id = 0;
            float e[G];
            token_weights<G>(p, u, id, lcodes[ls], ub2, e);
            if (cs < 0) {
              remove_weights<G>(p, u, id, e);
            } else {
              float* cw = p.cand_w + (static_cast<size_t>(u) * kCandWeights + cs) * G;
#pragma unroll
              for (int g = 0; g < G; ++g) cw[g] = e[g];
              p.cand_c[static_cast<size_t>(u) * kCandWeights + cs] = static_cast<int32_t>(id);
            }
          }
          __syncthreads();
          if (tid == 0) fix_n = 0;
          __syncthreads();
        }
      }
    }
  });
}

// ===========================================================================
// finalize (one CTA per unit)
// ===========================================================================
constexpr int kFinThreads = 1024;
constexpr int kFinWordsPerThread = 4;
constexpr int kFinChunkWords = kFinWordsPerThread * kFinThreads;   // 131072 slots per pass
constexpr int kFinSmemCand = kFinThreads;                          // candidates resolved in shared memory
constexpr int kFinBtCache = 8192;   // block-table entries cached in shared memory (longer tables: global)

__host__ __device__ inline int fin_bt_cached(int max_pages) { return max_pages <= kFinBtCache ? max_pages : 0; }

// One CTA per unit: resolve the threshold bin's candidates exactly (score desc, position
// asc), compact the selection bitmap into ascending positions, and take the selected
// tokens' weights out of the cluster sums. Unit state, candidates and the first bitmap
// pass are loaded in one round trip.
template <int G>
__global__ void __launch_bounds__(kFinThreads) finalize_kernel(SelectParams p) {
  __shared__ unsigned long long ck[kFinSmemCand];
  __shared__ uint32_t bmc[kFinChunkWords];
  __shared__ uint32_t woff[kFinChunkWords];   // exclusive count of selected bits before each word
  __shared__ uint32_t wins[kFinSmemCand];
  __shared__ uint32_t dig[256];
  __shared__ uint32_t warp_tot[33];
  __shared__ int sh_bin;
  __shared__ uint32_t sh_above, sh_nwin;
  extern __shared__ int32_t bt_s[];   // the sequence's block table when it fits
  const int u = blockIdx.x;
  const int b = u / p.Hkv;
  const int h = u % p.Hkv;
  const int tid = threadIdx.x;
  const int nbt = fin_bt_cached(p.max_pages);
  const int32_t* bt_row = p.block_table + static_cast<size_t>(b) * p.max_pages;
  {   // the block table predates the step: all of this thread's entries in flight at once
    constexpr int kPer = kFinBtCache / kFinThreads;
    int32_t v[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) v[e] = tid + e * kFinThreads < nbt ? bt_row[tid + e * kFinThreads] : 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (tid + e * kFinThreads < nbt) bt_s[tid + e * kFinThreads] = v[e];
  }
  pdl_wait();
  pdl_launch_dependents();
  // ---- one round trip: lengths, unit state, candidates and the first bitmap pass (speculative) ----
  const int T_raw = p.seq_lens[b];
  const int n_raw = p.n_indexed[b];
  const UnitState st = p.units[u];
  const unsigned long long* cg = p.cand + static_cast<size_t>(u) * p.cap;
  const unsigned long long ck_mine = tid < p.cap ? cg[tid] : 0ull;
  const uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;
  uint32_t words[kFinWordsPerThread];
#pragma unroll
  for (int e = 0; e < kFinWordsPerThread; ++e) {
    const int wi = kFinWordsPerThread * tid + e;
    words[e] = wi < p.bitmap_words ? bm[wi] : 0u;
  }
  // bounds, and this thread's candidate weights (slot tid) as stored by the filter
  float ub2[G];
  {
    float ub[G], lb[G];
    final_bounds<G>(p.fbounds, u, ub, lb);
#pragma unroll
    for (int g = 0; g < G; ++g) ub2[g] = ub[g] * kLog2e;
  }
  static_assert(kCandWeights <= kFinThreads, "one stored candidate per thread");
  float cwr[G];
  int32_t ccr = 0;
  if (p.background) {
    const float* cw = p.cand_w + (static_cast<size_t>(u) * kCandWeights + tid) * G;
#pragma unroll
    for (int g = 0; g < G; ++g) cwr[g] = tid < kCandWeights ? cw[g] : 0.f;
    ccr = tid < kCandWeights ? p.cand_c[static_cast<size_t>(u) * kCandWeights + tid] : 0;
  }
  const int T = max(0, T_raw);
  const int s0 = min(p.n_sink, T);
  const int N = min(max(0, min(n_raw, T - s0)), p.cap);
  const int k = decode_k(p.budget, p.k_override, N);
  const bool fix = p.background && N > k;
  // A winner's weights leave its cluster's sums: from registers (slot tid), from the
  // filter's store (slot < kCandWeights), else recomputed from the tables.
  auto fix_winner = [&](int i, uint32_t j) {
    if (!fix) return;
    float e[G];
    uint32_t id;
    if (i == tid && i < kCandWeights) {
#pragma unroll
      for (int g = 0; g < G; ++g) e[g] = cwr[g];
      id = static_cast<uint32_t>(ccr);
    } else if (i < kCandWeights) {
      const float* cw = p.cand_w + (static_cast<size_t>(u) * kCandWeights + i) * G;
#pragma unroll
      for (int g = 0; g < G; ++g) e[g] = cw[g];
      id = static_cast<uint32_t>(p.cand_c[static_cast<size_t>(u) * kCandWeights + i]);
    } else {
      id = p.ids[static_cast<size_t>(u) * p.cap + j];
      const uint4 cwd = *reinterpret_cast<const uint4*>(p.codes + (static_cast<size_t>(u) * p.cap + j) * kM);
      if (id >= static_cast<uint32_t>(p.C)) id = 0;
      token_weights<G>(p, u, id, cwd, ub2, e);
    }
    if (id >= static_cast<uint32_t>(p.C)) id = 0;
    remove_weights<G>(p, u, id, e);
  };
  int32_t* sel_u = p.sel + static_cast<size_t>(u) * p.cap;
  if (k == 0) {
    if (tid == 0 && p.dbg_nselected) p.dbg_nselected[u] = 0;
    publish_flag(&p.units[u].ready);
    return;
  }
  const int m = min(st.ncand, p.cap);
  const int r = k - st.above;
  const bool ok = r >= 1 && r <= m;
  if (!ok && tid == 0) record_error(p.err, HSA_DEVERR_SELECT);
  const bool in_smem = m <= kFinSmemCand;
  if (in_smem && tid < m) ck[tid] = ck_mine;
  if (tid == 0) sh_nwin = 0;
  __syncthreads();
  const unsigned long long* keys = in_smem ? ck : cg;

  // ---- threshold key: the r-th largest candidate key (keys are distinct) ----
  if (ok) {
    unsigned long long tau;
    if (m <= 256) {
      if (tid < m) {
        const unsigned long long key = keys[tid];
        int rank = 0;
        for (int j = 0; j < m; ++j) rank += keys[j] > key;
        if (rank < r) {
          const uint32_t j = 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
          wins[atomicAdd(&sh_nwin, 1u)] = j;
          fix_winner(tid, j);
        }
      }
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
      for (int i = tid; i < m; i += blockDim.x) {
        const unsigned long long key = keys[i];
        if (key >= tau) {
          const uint32_t j = 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
          const uint32_t w = atomicAdd(&sh_nwin, 1u);
          if (w < kFinSmemCand) wins[w] = j;
          else atomicOr(p.bitmap + static_cast<size_t>(u) * p.bitmap_words + (j >> 5), 1u << (j & 31));
          fix_winner(i, j);
        }
      }
    }
  }
  __syncthreads();
  const uint32_t nwin = min(sh_nwin, static_cast<uint32_t>(kFinSmemCand));
  if (nwin < sh_nwin) __threadfence_block();   // overflowed winners went to the global bitmap


  // ---- compaction of the selection bitmap into ascending positions ----
  const int nw = (N + 31) / 32;
  uint32_t running = 0;
  for (int w0 = 0; w0 < nw; w0 += kFinChunkWords) {
    if (w0 > 0 || sh_nwin > kFinSmemCand) {
#pragma unroll
      for (int e = 0; e < kFinWordsPerThread; ++e) {
        const int wi = w0 + kFinWordsPerThread * tid + e;
        words[e] = wi < nw ? bm[wi] : 0u;
      }
    }
#pragma unroll
    for (int e = 0; e < kFinWordsPerThread; ++e) {
      const int wi = w0 + kFinWordsPerThread * tid + e;
      bmc[kFinWordsPerThread * tid + e] = wi < nw ? words[e] : 0u;
    }
    __syncthreads();
    for (uint32_t i = tid; i < nwin; i += blockDim.x) {
      const uint32_t j = wins[i];
      const int w = static_cast<int>(j >> 5) - w0;
      if (w >= 0 && w < kFinChunkWords) atomicOr(&bmc[w], 1u << (j & 31));
    }
    __syncthreads();
    uint32_t pc = 0;
#pragma unroll
    for (int e = 0; e < kFinWordsPerThread; ++e) {
      words[e] = bmc[kFinWordsPerThread * tid + e];
      pc += __popc(words[e]);
    }
    uint32_t tot;
    {
      uint32_t o = block_excl_scan(pc, warp_tot, tot);
#pragma unroll
      for (int e = 0; e < kFinWordsPerThread; ++e) {
        woff[kFinWordsPerThread * tid + e] = o;
        o += __popc(words[e]);
      }
    }
    __syncthreads();
    // Output entry i of this pass: the word holding it by binary search over the word
    // offsets, then its bit; every thread writes about tot / 1024 entries whatever the
    // positions of the selected tokens.
    for (uint32_t i = tid; i < tot; i += kFinThreads) {
      int lo_w = 0, hi_w = kFinChunkWords - 1;   // largest word with woff <= i
      while (lo_w < hi_w) {
        const int mid = (lo_w + hi_w + 1) >> 1;
        if (woff[mid] <= i) lo_w = mid;
        else hi_w = mid - 1;
      }
      uint32_t wv = bmc[lo_w];
      for (uint32_t c = i - woff[lo_w]; c > 0; --c) wv &= wv - 1;
      const int j = (w0 + lo_w) * 32 + (__ffs(wv) - 1);
      const uint32_t off = running + i;
      if (off < static_cast<uint32_t>(p.cap)) {
        // the token's KV-pool row, so the exact attend reads it in one step
        const int pos = s0 + j;
        const int pi = pos / p.page_size;
        int page = pi < p.max_pages ? (pi < nbt ? bt_s[pi] : bt_row[pi]) : -1;
        if (page < 0 || page >= p.num_pages) {
          record_error(p.err, HSA_DEVERR_PAGE);
          page = 0;
        }
        sel_u[off] = (page * p.Hkv + h) * p.page_size + (pos % p.page_size);
        if (p.dbg_selected) p.dbg_selected[static_cast<size_t>(u) * p.cap + off] = pos;
      }
    }
    running += tot;
    __syncthreads();   // woff / bmc are rewritten by the next pass
  }
  if (tid == 0) {
    p.units[u].nsel = static_cast<int32_t>(running);
    if (running != static_cast<uint32_t>(k)) record_error(p.err, HSA_DEVERR_SELECT);
    if (p.dbg_nselected) p.dbg_nselected[u] = static_cast<int32_t>(running);
  }
  // the exact attend and the background of this unit may start (selection rows and
  // the winners' weight fix-up are written)
  publish_flag(&p.units[u].ready);
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


int scan_ring_depth(int G, int C) {
  switch (G) {
    case 1: return ScanSmem<1>::depth(C);
    case 2: return ScanSmem<2>::depth(C);
    case 4: return ScanSmem<4>::depth(C);
    default: return ScanSmem<8>::depth(C);
  }
}

size_t scan_smem_bytes(int G, int C) {
  const int d = scan_ring_depth(G, C);
  switch (G) {
    case 1: return ScanSmem<1>::bytes(C, d);
    case 2: return ScanSmem<2>::bytes(C, d);
    case 4: return ScanSmem<4>::bytes(C, d);
    default: return ScanSmem<8>::bytes(C, d);
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
  const dim3 grid(p.B * p.Hkv, kLutParts + p.nq);
#define CALL(GG) return launch_ex(tables_kernel<GG>, grid, dim3(256), 0, stream, pdl, p)
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

template <int G, int D>
cudaError_t launch_scan_t(const ScanParams& p, int grid, cudaStream_t stream, bool pdl) {
  const size_t smem = ScanSmem<G>::bytes(p.C, D);
  cudaError_t e = ensure_dyn_smem<scan_kernel<G, D>>(smem);
  if (e != cudaSuccess) return e;
  return launch_ex(scan_kernel<G, D>, dim3(grid), dim3(scan_threads_of<G>()), smem, stream, pdl, p);
}

template <int G>
cudaError_t launch_scan_g(const ScanParams& p, int grid, cudaStream_t stream, bool pdl) {
  switch (p.ring_depth) {
    case 8: return launch_scan_t<G, 8>(p, grid, stream, pdl);
    case 4: return launch_scan_t<G, 4>(p, grid, stream, pdl);
    case 2: return launch_scan_t<G, 2>(p, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_scan(int G, const ScanParams& p, int grid, cudaStream_t stream, bool pdl) {
  switch (G) {
    case 1: return launch_scan_g<1>(p, grid, stream, pdl);
    case 2: return launch_scan_g<2>(p, grid, stream, pdl);
    case 4: return launch_scan_g<4>(p, grid, stream, pdl);
    case 8: return launch_scan_g<8>(p, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_filter(int G, const SelectParams& p, int grid, cudaStream_t stream, bool pdl) {
#define CALL(GG) return launch_ex(filter_kernel<GG>, dim3(grid), dim3(kFilterThreads), 0, stream, pdl, p)
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

cudaError_t launch_finalize(int G, const SelectParams& p, cudaStream_t stream, bool pdl) {
  const size_t smem = static_cast<size_t>(fin_bt_cached(p.max_pages)) * sizeof(int32_t);
#define CALL(GG)                                                                                     \
  {                                                                                                  \
    cudaError_t e = ensure_dyn_smem<finalize_kernel<GG>>(smem);                                      \
    if (e != cudaSuccess) return e;                                                                  \
    return launch_ex(finalize_kernel<GG>, dim3(p.B * p.Hkv), dim3(kFinThreads), smem, stream, pdl, p); \
  }
  PQHSA_G_SWITCH(G, CALL)
#undef CALL
}

}  // namespace pqhsa
