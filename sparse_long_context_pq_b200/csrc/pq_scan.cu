// PQ-HSA scoring and selection kernels:
//   tables      - per-query PQ look-up tables and centroid terms (q . codeword, q . centroid),
//                 plus exact upper/lower bounds of every head's approximate logit;
//   scan+select - one launch: a pass over the uint8 codes (approximate logits of every
//                 indexed token, the selection score sigma = max over the group's heads,
//                 per-cluster exp-weight sums, a histogram of sigma, each chunk's largest
//                 sigma); then, per unit, the tokens above the threshold histogram bin
//                 (selected, their KV-pool rows written at once) and in it (candidates),
//                 the selected tokens' weights taken out of the cluster sums; then the
//                 part that completes the unit's count resolves the candidates exactly
//                 (score desc, position asc), writes the winners' rows after the others
//                 (in no particular position order) and publishes the unit.
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
  // the dependency wait: first thing, or (index_early) once this CTA's codebook or
  // centroid loads are on their way
  if (!p.index_early) {
    pdl_wait();
    pdl_launch_dependents();
  }
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
    if (p.index_early) {
      pdl_wait();
      pdl_launch_dependents();
    }
    stage_q<G4, G>(p, b, h, tid, qsh);
    // zero this unit's selection state (spread over the LUT CTAs)
    for (int i = part * blockDim.x + tid; i < kNB; i += kLutParts * blockDim.x)
      p.hist[static_cast<size_t>(u) * kNB + i] = 0u;
    for (int i = part * blockDim.x + tid; i < p.bitmap_words; i += kLutParts * blockDim.x)
      p.bitmap[static_cast<size_t>(u) * p.bitmap_words + i] = 0u;
    if (part == 0)
      for (int i = tid; i < static_cast<int>(sizeof(UnitState) / 4); i += blockDim.x)
        reinterpret_cast<int32_t*>(p.units + u)[i] = 0;
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
        const float a = warp_max_f32(val[g]);
        const float c = warp_min_f32(val[g]);
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
    if (p.index_early) {
      pdl_wait();
      pdl_launch_dependents();
    }
    stage_q<G4, G>(p, b, h, tid, qsh);
    {   // zero this slice's cluster weights
      const int cs = slice * kQcSlice, ce = min(p.C, cs + kQcSlice), nc = ce - cs;
      for (int i = tid; i < G * nc; i += blockDim.x)
        p.W[(static_cast<size_t>(u) * G + i / nc) * p.C + cs + (i % nc)] = 0.f;
    }
    __syncthreads();
    // The G4 dot products of a cluster are reduced together (scattered halving): head g's
    // total ends in the lanes of group g = lane / (32 / G4), which keep its extremes.
    constexpr int kGroup = 32 / G4;
    const int hg = lane / kGroup;
    float mx = -INFINITY, mn = INFINITY;
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
        val[g] = v;
      }
      const float tot = warp_sum_scatter<G4>(val);
      if (c < p.C) {
        if (hg < G) {
          mx = fmaxf(mx, tot);
          mn = fminf(mn, tot);
        }
        if ((lane & (kGroup - 1)) == 0)   // component hg % 4 of float4 [hg / 4][c]
          reinterpret_cast<float*>(p.qc)[((static_cast<size_t>(u) * GP + hg / 4) * p.C + c) * 4 + (hg % 4)] = tot;
      }
    }
    if ((lane & (kGroup - 1)) == 0) {
      wred[0][warp][0][hg] = mx;
      wred[1][warp][0][hg] = mn;
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
// scan + select: one launch, one 512-thread CTA per SM
// ===========================================================================
// Phase 1 (scan): every CTA streams its chunks of the cluster-ordered code lists and
// scores them against the unit's tables in shared memory: approximate logits, the
// selection score sigma, per-cluster exp-weight sums, a histogram of sigma and each
// chunk's largest sigma. Phase 2 (filter), per unit, once every CTA of the unit has
// scanned its chunks: the threshold bin from the unit's histogram, then, over this CTA's
// share of the unit's chunks (spread over the whole list), the definite selections' rows,
// the threshold-bin candidates and the weight fix-ups. Phase 3 (resolution), by the part
// that completes the unit's filter count: the exact order of the candidates (score desc,
// position asc), the winners' KV-pool rows after the others and their weight fix-ups, the
// ready flag. The attention needs the rows in no particular order; only the debug output
// of the selected positions is written in ascending order.
//
// The per-unit wait of phase 2 only waits on CTAs of the same grid, which are all
// resident: the grid has one CTA per SM and each CTA needs a whole SM's registers,
// and a dependent launch starts only after every CTA of this grid has started.
constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kRingCodeBytes = 32 * kM;                    // 512 per chunk
constexpr int kRingSlotBytes = kRingCodeBytes + 16;        // + a 16-B cell with the cluster word
constexpr size_t kScanSmemLimit = 226 * 1024;   // dynamic; the rest of 227 KB is static

template <int G>
struct ScanSmem {
  static constexpr int GP = (G + 3) / 4;
  // LUT [GP][256][16] float4, centroid terms [GP][C] float4, the open chunk and fill of
  // every cluster [C] u32, the score histogram [NB] u32; then the warps' rings ([D][32]
  // 16-B code rows and [D] 16-B cells holding the 4-byte word with the chunk's cluster id,
  // per warp); then the tables mbarrier.
  __host__ __device__ static size_t meta_off(int C) {
    return static_cast<size_t>(GP) * kNcode * kM * 16 + static_cast<size_t>(GP) * C * 16;
  }
  __host__ __device__ static size_t hist_off(int C) { return meta_off(C) + align_up(static_cast<size_t>(C) * 4, 16); }
  __host__ __device__ static size_t tables(int C) { return align_up(hist_off(C) + kNB * 4, 128); }
  __host__ __device__ static size_t bytes(int C, int depth) {
    return tables(C) + static_cast<size_t>(kScanWarps) * depth * kRingSlotBytes + 8;
  }
  // deepest ring (8, 4 or 2 chunks per warp) that fits; 0 if none does
  static int depth(int C) {
    for (int d = 8; d >= 2; d >>= 1)
      if (bytes(C, d) <= kScanSmemLimit) return d;
    return 0;
  }
};

// Phase-2 scratch (after the tables; over the histogram and the rings) and phase-3
// scratch (from the start of dynamic shared memory, over the tables).
constexpr int kCmPerThread = 4;                                  // chunk maxima per thread per pass
constexpr int kCmPass = kCmPerThread * kScanThreads;             // chunks examined per pass
constexpr int kActPerWarp = 1;                                   // active chunks per warp per round
constexpr size_t kFilterScratch = kCmPass * 4;
constexpr int kFinWordsPerThread = 8;
constexpr int kFinChunkWords = kFinWordsPerThread * kScanThreads;   // 131072 slots per pass
constexpr int kFinSmemCand = 1024;                                  // candidates resolved in shared memory
constexpr int kFinBt = 8192;                                        // block-table entries staged in shared memory
constexpr size_t kFinScratch =
    kFinSmemCand * 8 + 2 * kFinChunkWords * 4 + kFinSmemCand * 4 + 256 * 4 + kFinBt * 4;
static_assert(kFilterScratch <= kNB * 4 + kScanWarps * 2 * kRingSlotBytes, "filter scratch fits");
// the smallest scan layout (G = 1, C = 1, 8-deep rings) is 141 KB of dynamic shared memory
static_assert(kFinScratch <= 128 * 1024, "resolution scratch fits in the scan's shared memory");
static_assert(kCandWeights <= kFinSmemCand, "stored candidate weights are resolved in shared memory");

constexpr int kMaxParts = 24;   // (unit, chunk range) parts one CTA plans in shared memory

struct SelShared {
  uint32_t scan_tot[33];
  long long red[kScanWarps];
  int bstar;
  uint32_t above;
  int n_act;
  int flag;
  uint32_t nwin;
  int bin;
  uint32_t fin_above;
  unsigned long long tau;        // the unit's threshold key: candidates with keys >= tau are selected
  int res[kMaxParts];            // units this CTA resolves after its filter parts
  // this CTA's parts
  int nparts;                    // -1: more than kMaxParts, walk the units instead
  int pu[kMaxParts], pc0[kMaxParts], pc1[kMaxParts];
  uint32_t pst[kMaxParts];       // phase-2 chunk permutation stride of the part's unit
  long long total;
  int active;
};

// Chunks of unit u's lists to scan (0 if nothing is indexed); its three loads go out together.
__device__ __forceinline__ int unit_chunks(const StepParams& p, int u) {
  const int b = u / p.Hkv;
  const int n = p.list_meta[static_cast<size_t>(u) * (2 + 2 * static_cast<size_t>(p.C))];
  const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
  return N == 0 ? 0 : max(0, min(n, p.list_slots / 32));
}

// KV-pool row of position pos of KV head h through one block-table row; an entry outside
// the pool is recorded and replaced by page 0.
// Split in two so that the block-table read can go out before other round trips: the
// raw entry of position pos, then the row (an entry outside the pool recorded, page 0).
__device__ __forceinline__ int32_t kv_page_entry(const StepParams& p, const int32_t* bt_row, int pos) {
  const int pi = pos / p.page_size;
  return pi < p.max_pages ? bt_row[pi] : -1;
}
__device__ __forceinline__ int32_t kv_row_of(const StepParams& p, int32_t page, int h, int pos) {
  if (page < 0 || page >= p.num_pages) {
    record_error(p.err, HSA_DEVERR_PAGE);
    page = 0;
  }
  return (page * p.Hkv + h) * p.page_size + (pos % p.page_size);
}
__device__ __forceinline__ int32_t kv_row(const StepParams& p, const int32_t* bt_row, int h, int pos) {
  return kv_row_of(p, kv_page_entry(p, bt_row, pos), h, pos);
}

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

// Add the warp's per-lane weight sums of one cluster run to the cluster's sums.
template <int G>
__device__ __forceinline__ void flush_weights(const float* acc, float* Wu, int C, uint32_t c) {
  float v[G];
#pragma unroll
  for (int g = 0; g < G; ++g) v[g] = acc[g];
  const float e = warp_sum_scatter<G>(v);
  constexpr int kGroup = 32 / G;
  const int lane = threadIdx.x & 31;
  if ((lane & (kGroup - 1)) == 0) atomicAdd(Wu + (lane / kGroup) * C + c, e);
}

// Phase 1 for chunks [ch0, ch1) of unit u: one warp scores one 32-slot chunk (members of
// one cluster) at a time, so the centroid term is warp-uniform. Warp w takes a contiguous
// run of the range through its D-slot ring of async copies (one commit group per chunk);
// consecutive chunks of one cluster add their weights in registers, and the warp reduces
// them once per cluster run. A chunk's valid slots are a prefix: all 32, or the cluster's
// fill count for its open chunk. `phase` counts segments (tables mbarrier parity).
template <int G, int D>
__device__ __forceinline__ void scan_segment(const StepParams& p, int u, int ch0, int ch1, uint8_t* smem,
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
  uint32_t* meta_s = reinterpret_cast<uint32_t*>(smem + ScanSmem<G>::meta_off(C));   // [C]
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + ScanSmem<G>::hist_off(C));   // [NB]
  uint8_t* wring = smem + ScanSmem<G>::tables(C) + static_cast<size_t>(warp) * D * kRingSlotBytes;
  uint4* ring_code = reinterpret_cast<uint4*>(wring) + lane;                              // [D][32]
  uint32_t* ring_cl = reinterpret_cast<uint32_t*>(wring + D * kRingCodeBytes);            // [D][4]

  __syncthreads();  // previous segment (or planning) finished with shared memory
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
  const int max_chunks = p.list_slots / 32;
  const uint4* lcodes = reinterpret_cast<const uint4*>(p.list_codes) + static_cast<size_t>(u) * p.list_slots;
  const uint16_t* ccl = p.chunk_cluster + static_cast<size_t>(u) * max_chunks;
  float* sig_u = p.sigma + static_cast<size_t>(u) * p.list_slots;
  float* cmax_u = p.chunk_max + static_cast<size_t>(u) * max_chunks;
  float* Wu = p.W + static_cast<size_t>(u) * G * C;
  const uint8_t* lut_b = reinterpret_cast<const uint8_t*>(lut_s);

  // this warp's contiguous run [wb, we); the first D chunks go out while the tables land
  const int nch = ch1 - ch0;
  const int wb = ch0 + static_cast<int>(static_cast<long long>(nch) * warp / kScanWarps);
  const int we = ch0 + static_cast<int>(static_cast<long long>(nch) * (warp + 1) / kScanWarps);
  const int cnt = we - wb;
  // The chunk's cluster id (u16) comes with lane 0's group as the aligned 4-byte word
  // that holds it; empty commit groups past the end keep the group count regular.
  auto issue = [&](int i) {
    if (i < cnt) {
      const int ch = wb + i;
      const int slot = i % D;
      cp_async_16(ring_code + slot * 32, lcodes + static_cast<size_t>(ch) * 32 + lane);
      if (lane == 0)
        cp_async_4(ring_cl + slot * 4,
                   reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(ccl + ch) & ~uintptr_t(3)));
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < D; ++i) issue(i);

  {   // open chunk (26 bits) and its fill (6 bits) of every cluster; all-ones: no open chunk
    const int32_t* mg = p.list_meta + static_cast<size_t>(u) * (2 + 2 * static_cast<size_t>(C));
    for (int c = tid; c < C; c += kScanThreads) {
      const int op = mg[2 + 2 * c], fl = mg[3 + 2 * c];
      meta_s[c] = (op >= 0 && op < (1 << 26)) ? ((static_cast<uint32_t>(op) << 6) |
                                                  static_cast<uint32_t>(min(max(fl, 0), 32)))
                                              : 0xffffffffu;
    }
  }
  for (int i = tid; i < kNB; i += kScanThreads) hist_s[i] = 0u;
  if (warp == 0) {   // final bounds of the unit: this CTA's copy and the later phases'
    reduce_bounds_warp<G>(p.bounds, u, p.nq, sh_bounds, sh_bounds + G);
    __syncwarp();
    if (lane < 2 * G) p.fbounds[static_cast<size_t>(u) * 2 * G + lane] = sh_bounds[lane];
  }
  __syncthreads();                       // histogram, cluster fills and bounds visible
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
  uint32_t cur = 0xffffffffu;            // cluster of the current run
  float wacc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) wacc[g] = 0.f;

  // Chunk (slot) -> its code row, cluster and fill; then the scores of the chunk's valid
  // slots are stored, reduced and binned (the weight run is per chunk, in list order).
  auto chunk_in = [&](int i, uint4& code, uint32_t& id, int& fill) {
    const int slot = i % D;
    const int ch = wb + i;
    code = ring_code[slot * 32];
    const uint32_t cw = ring_cl[slot * 4];
    id = ((reinterpret_cast<uintptr_t>(ccl + ch) >> 1) & 1) ? (cw >> 16) : (cw & 0xffffu);
    fill = 32;
    if (id >= static_cast<uint32_t>(C)) {
      bad_id = true;
      id = 0;
      fill = 0;
    } else {
      const uint32_t m = meta_s[id];
      if (m != 0xffffffffu && static_cast<int>(m >> 6) == ch) fill = static_cast<int>(m & 63u);
    }
  };
  auto chunk_out = [&](int i, uint32_t id, int fill, const float* sh) {
    const int ch = wb + i;
    const bool valid = lane < fill;
    float sg = sh[0];
#pragma unroll
    for (int g = 1; g < G; ++g) sg = fmaxf(sg, sh[g]);
    const float sv = valid ? sg : -INFINITY;
    sig_u[static_cast<size_t>(ch) * 32 + lane] = sv;
    const float cmx = warp_max_f32(sv);  // lets the filter skip chunks below the threshold
    if (lane == 0) cmax_u[ch] = cmx;
    if (p.approx_logits && valid) {
      const int js = p.list_slot[static_cast<size_t>(u) * p.list_slots + static_cast<size_t>(ch) * 32 + lane];
      if (js >= 0 && js < N) {
#pragma unroll
        for (int g = 0; g < G; ++g) p.approx_logits[(static_cast<size_t>(b) * p.Hq + h * G + g) * p.cap + js] = sh[g];
      }
    }
    if (id != cur) {                     // warp-uniform: a new cluster run starts
      if (cur != 0xffffffffu) flush_weights<G>(wacc, Wu, C, cur);
      cur = id;
#pragma unroll
      for (int g = 0; g < G; ++g) wacc[g] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) wacc[g] += valid ? fast_exp2(fmaf(sh[g], kLog2e, -ub2[g])) : 0.f;
    if (valid) atomicAdd(&hist_s[score_bin(sg, lo, inv)], 1u);
  };
  for (int i = 0; i < cnt; ++i) {
    cp_async_wait<D - 1>();            // this lane's copies of chunk i have landed
    __syncwarp();                      // ... and lane 0's cluster word
    uint4 code;
    uint32_t id;
    int fill;
    chunk_in(i, code, id, fill);
    float sh[G];
    score_token<G>(code, id, lut_b, qc_s, C, ysoff, sel, swap_words, sh);
    chunk_out(i, id, fill, sh);
    __syncwarp();                      // every lane has read the slot
    issue(i + D);                      // refill it with the chunk D ahead
  }
  if (cur != 0xffffffffu) flush_weights<G>(wacc, Wu, C, cur);
  cp_async_wait<0>();
  if (bad_id) record_error(p.err, HSA_DEVERR_CLUSTER);
  __syncthreads();
  uint32_t* hg = p.hist + static_cast<size_t>(u) * kNB;
  for (int i = tid; i < kNB; i += kScanThreads) {
    const uint32_t v = hist_s[i];
    if (v) atomicAdd(hg + i, v);
  }
  // publish this range: scores, chunk maxima, weights and histogram before the count (the
  // barrier orders the CTA's writes before thread 0's release, which is cumulative; the
  // waiters read the count with acquire loads)
  __syncthreads();
  if (tid == 0)
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(&p.units[u].scan_done), "r"(nch) : "memory");
}

// Head weights e^{shat_g - ub_g} of one indexed token (cluster id, code words cw) from the
// decode tables (global or shared copies, layout [GP][256][16] and [GP][C] float4): the
// same quantities the scan added into its cluster's sums.
template <int G>
__device__ __forceinline__ void token_weights(const float4* lut4, const float4* qc4, int C, uint32_t id,
                                              const uint4 cw, const float* ub2, float* e) {
  constexpr int GP = (G + 3) / 4;
  const uint32_t cwords[4] = {cw.x, cw.y, cw.z, cw.w};
  float4 acc[GP];
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) acc[gp] = qc4[gp * C + id];
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

// token_weights for many lanes at once (the filter's selections): lane l visits subspace
// s = i ^ (l & 7) at step i, so the 8 lanes of a quarter-warp read 8 different 16-byte bank
// groups of the shared-memory tables instead of one (same sums up to rounding order).
template <int G>
__device__ __forceinline__ void token_weights_skewed(const float4* lut4, const float4* qc4, int C, uint32_t id,
                                                     const uint4 cw, const float* ub2, float* e) {
  constexpr int GP = (G + 3) / 4;
  const uint32_t l7 = threadIdx.x & 7;
  const uint32_t wlo[2] = {(l7 & 4) ? cw.y : cw.x, (l7 & 4) ? cw.x : cw.y};   // words i>>2 = 0, 1 after the skew
  const uint32_t whi[2] = {(l7 & 4) ? cw.w : cw.z, (l7 & 4) ? cw.z : cw.w};   // words i>>2 = 2, 3
  float4 acc[GP];
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) acc[gp] = qc4[gp * C + id];
#pragma unroll
  for (int i = 0; i < kM; ++i) {
    const uint32_t s = static_cast<uint32_t>(i) ^ l7;
    const uint32_t wd = (i < 4) ? wlo[0] : (i < 8) ? wlo[1] : (i < 12) ? whi[0] : whi[1];
    const uint32_t code = (wd >> (8u * (s & 3u))) & 255u;
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
__device__ __forceinline__ void remove_weights(const StepParams& p, int u, uint32_t id, const float* e) {
  float* Wu = p.W + static_cast<size_t>(u) * G * p.C;
#pragma unroll
  for (int g = 0; g < G; ++g) atomicAdd(&Wu[g * p.C + id], -e[g]);
}

// Stride of the chunk permutation c -> (c * stride) mod n of phase 2: about n / golden
// ratio and coprime with n, so the map is a bijection of [0, n) and any run of consecutive
// chunks (a high-scoring cluster's) is spread evenly over every range of c. Every CTA of a
// unit derives the same stride from n alone. Terminates: n - 1 is coprime with n.
__device__ __forceinline__ uint32_t gcd_u32(uint32_t a, uint32_t b) {   // binary gcd, a, b > 0
  const int sh = __ffs(a | b) - 1;
  a >>= __ffs(a) - 1;
  do {
    b >>= __ffs(b) - 1;
    if (a > b) {
      const uint32_t t = a;
      a = b;
      b = t;
    }
    b -= a;
  } while (b);
  return a << sh;
}
__device__ __forceinline__ uint32_t scatter_stride(uint32_t n) {
  if (n <= 2) return 1u;
  uint32_t s = static_cast<uint32_t>((static_cast<unsigned long long>(n) * 2654435769ull) >> 32);
  if (s == 0) s = 1;
  while (gcd_u32(n, s) != 1u) ++s;
  return s;
}

// Phase 2 for part [c0, c1) of unit u (after every CTA of the unit has scanned): the
// threshold bin, then the part's chunks, c -> (c * stride) mod total with
// stride = scatter_stride(total), whose maximum reaches
// it (the bin is monotone in the score). The permutation only decides which part handles
// a chunk (parts still partition the unit's chunks); it keeps the chunks of high-scoring
// clusters, which are consecutive in list order, from piling up in one part. Tokens above
// the bin are selected: their KV-pool rows join the unit's rows and their weights leave
// their clusters' sums here (from the tables in shared memory when this CTA holds the
// unit's, `tables`, else from the global copy). The bin's tokens are candidates; the
// first ones' weights are stored for the resolution. Every lane handles its own slot, so
// a warp's chunks need no block-wide step. Returns true in the part that completes the
// unit's filter count (it then resolves the unit).
template <int G>
__device__ bool filter_part(const StepParams& p, int u, int c0, int c1, uint32_t stride, const uint8_t* tables,
                            uint8_t* smem, SelShared& ss) {
  constexpr int GP = (G + 3) / 4;
  constexpr int NW = kScanWarps;
  constexpr int T = kScanThreads;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane = tid & 31;
  const int b = u / p.Hkv;
  const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
  // read with N, before this part's first global store (which the compiler cannot rule
  // out as aliasing it, so a later read would be another round trip)
  const int s0 = min(p.n_sink, max(0, p.seq_lens[b]));
  const int k = decode_k(p.budget, p.k_override, N);
  const int max_chunks = p.list_slots / 32;
  const int total = unit_chunks(p, u);
  int32_t* act = reinterpret_cast<int32_t*>(smem + ScanSmem<G>::hist_off(p.C));   // active chunks of the pass
  const float4* lut4 = tables ? reinterpret_cast<const float4*>(tables)
                              : reinterpret_cast<const float4*>(p.lut) + static_cast<size_t>(u) * GP * kNcode * kM;
  const float4* qc4 = tables ? reinterpret_cast<const float4*>(tables) + GP * kNcode * kM
                             : reinterpret_cast<const float4*>(p.qc) + static_cast<size_t>(u) * GP * p.C;
  // chunk of local index c0 + tid, and the step to local index + T (both mod total)
  const uint32_t nt = static_cast<uint32_t>(max(total, 1));   // parts exist only for units with chunks
  const uint32_t step = static_cast<uint32_t>((static_cast<unsigned long long>(T) * stride) % nt);
  uint32_t pc = static_cast<uint32_t>((static_cast<unsigned long long>(c0 + tid) * stride) % nt);

  __syncthreads();   // shared state of the previous part is no longer read
  if (tid == 0) {
    wait_count(&p.units[u].scan_done, total, p.err);   // every CTA of the unit has scanned
    ss.bstar = kNB;   // k == 0: nothing selected
    ss.above = 0;
  }
  __syncthreads();
  // one round trip: this thread's histogram bins, the first pass of chunk maxima, the bounds
  static_assert(kNB == 4 * kScanThreads, "threshold search: 512 threads x 4 bins");
  const uint4 hv = __ldcg(reinterpret_cast<const uint4*>(p.hist + static_cast<size_t>(u) * kNB) +
                          (kNB / 4 - 1 - tid));
  const float* cmax = p.chunk_max + static_cast<size_t>(u) * max_chunks;
  float cm[kCmPerThread];
  auto next_chunk = [&]() {   // chunk of this thread's next local index, then advance
    const int32_t c = static_cast<int32_t>(pc);
    pc += step;
    if (pc >= nt) pc -= nt;
    return c;
  };
  uint32_t pc_pass = pc;      // the pass's first chunk; the compaction replays the sequence
#pragma unroll
  for (int e = 0; e < kCmPerThread; ++e) {
    const int c = c0 + tid + e * T;
    const int32_t ch = next_chunk();
    cm[e] = c < c1 ? __ldcg(cmax + ch) : -INFINITY;
  }
  float ub[G], lb[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    ub[g] = __ldcg(p.fbounds + (static_cast<size_t>(u) * 2 + 0) * G + g);
    lb[g] = __ldcg(p.fbounds + (static_cast<size_t>(u) * 2 + 1) * G + g);
  }
  {
    // thread t owns the 4 bins [kNB-4(t+1), kNB-4t): block scan of counts from the top
    const int hi = kNB - 4 * tid;
    const uint32_t c4[4] = {hv.w, hv.z, hv.y, hv.x};
    const uint32_t local = c4[0] + c4[1] + c4[2] + c4[3];
    uint32_t tot;
    const uint32_t excl = block_excl_scan(local, ss.scan_tot, tot);
    const uint32_t need = static_cast<uint32_t>(k);
    if (need > 0 && excl < need && excl + local >= need) {
      uint32_t cum = excl;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (cum < need && cum + c4[i] >= need) {
          ss.bstar = hi - 1 - i;
          ss.above = cum;
        }
        cum += c4[i];
      }
    }
  }
  __syncthreads();
  const int bstar = ss.bstar;
  if (tid == 0) {   // every CTA of the unit stores the same values
    p.units[u].bstar = bstar;
    p.units[u].above = static_cast<int32_t>(ss.above);
  }
  if (bstar < kNB) {
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
    const float* sig = p.sigma + static_cast<size_t>(u) * p.list_slots;
    const int32_t* lslot = p.list_slot + static_cast<size_t>(u) * p.list_slots;
    const uint4* lcodes = reinterpret_cast<const uint4*>(p.list_codes) + static_cast<size_t>(u) * p.list_slots;
    const uint16_t* ccl = p.chunk_cluster + static_cast<size_t>(u) * max_chunks;
    uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;
    int32_t* sel_u = p.sel + static_cast<size_t>(u) * p.cap;
    unsigned long long* cand_u = p.cand + static_cast<size_t>(u) * p.cap;
    int32_t* cand_row_u = p.cand_row + static_cast<size_t>(u) * p.cap;
    // low word: candidates, high word: definite selections (neither count exceeds N < 2^31)
    unsigned long long* counts = reinterpret_cast<unsigned long long*>(&p.units[u].ncand);
    const int32_t* bt_row = p.block_table + static_cast<size_t>(b) * p.max_pages;
    const int h = u % p.Hkv;

    for (int cb = c0; cb < c1; cb += kCmPass) {
      if (cb != c0) {
        pc_pass = pc;
#pragma unroll
        for (int e = 0; e < kCmPerThread; ++e) {
          const int c = cb + tid + e * T;
          const int32_t ch = next_chunk();
          cm[e] = c < c1 ? __ldcg(cmax + ch) : -INFINITY;
        }
      }
      if (tid == 0) ss.n_act = 0;
      __syncthreads();
      // chunks whose maximum reaches the threshold bin, compacted warp by warp
      uint32_t pr = pc_pass;
#pragma unroll
      for (int e = 0; e < kCmPerThread; ++e) {
        const int c = cb + tid + e * T;
        const int32_t ch = static_cast<int32_t>(pr);
        pr += step;
        if (pr >= nt) pr -= nt;
        const bool active = c < c1 && score_bin(cm[e], lo, inv) >= bstar;
        const uint32_t m = __ballot_sync(0xffffffffu, active);
        if (m) {
          const uint32_t leader = __ffs(m) - 1;
          int at = 0;
          if (lane == leader) at = atomicAdd(&ss.n_act, __popc(m));
          at = __shfl_sync(0xffffffffu, at, leader);
          if (active) act[at + __popc(m & ((1u << lane) - 1u))] = ch;
        }
      }
      __syncthreads();
      const int na = ss.n_act;
      for (int a0 = warp * kActPerWarp; a0 < na; a0 += NW * kActPerWarp) {
        // up to kActPerWarp active chunks of this warp, every load in one round trip;
        // lane = slot of the chunk
        float sv[kActPerWarp];
        int32_t jv[kActPerWarp];
        uint4 cwv[kActPerWarp];
        uint32_t idv[kActPerWarp];
#pragma unroll
        for (int r = 0; r < kActPerWarp; ++r) {
          const int ch = a0 + r < na ? act[a0 + r] : -1;
          const size_t ls = static_cast<size_t>(max(ch, 0)) * 32 + lane;
          sv[r] = ch >= 0 ? __ldcg(sig + ls) : -INFINITY;
          jv[r] = ch >= 0 ? __ldg(lslot + ls) : -1;
          cwv[r] = (ch >= 0 && fix) ? __ldg(lcodes + ls) : make_uint4(0u, 0u, 0u, 0u);
          idv[r] = (ch >= 0 && fix) ? static_cast<uint32_t>(__ldg(ccl + ch)) : 0u;
        }
        // classify both chunks, then one atomic per warp for all their selections and
        // candidates; the block-table reads go out before the counts come back
        bool defv[kActPerWarp], candv[kActPerWarp];
        uint32_t dmv[kActPerWarp], cmv[kActPerWarp];
        int32_t pagev[kActPerWarp];
        uint32_t ndm = 0, ncm = 0;
#pragma unroll
        for (int r = 0; r < kActPerWarp; ++r) {
          const int j = jv[r];            // index slot of this list slot
          const bool valid = j >= 0 && j < N;
          const int bin = valid ? score_bin(sv[r], lo, inv) : -1;
          defv[r] = bin > bstar;
          candv[r] = bin == bstar;
          dmv[r] = __ballot_sync(0xffffffffu, defv[r]);
          cmv[r] = __ballot_sync(0xffffffffu, candv[r]);
          pagev[r] = (defv[r] || candv[r]) ? kv_page_entry(p, bt_row, s0 + j) : 0;
          ndm += __popc(dmv[r]);
          ncm += __popc(cmv[r]);
        }
        if ((ndm | ncm) == 0u) continue;   // warp-uniform
        unsigned long long old = 0ull;
        if (lane == 0) old = atomicAdd(counts, (static_cast<unsigned long long>(ndm) << 32) | ncm);
        old = __shfl_sync(0xffffffffu, old, 0);
        uint32_t dbase = static_cast<uint32_t>(old >> 32), cbase = static_cast<uint32_t>(old & 0xffffffffull);
        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int r = 0; r < kActPerWarp; ++r) {
          const int j = jv[r];
          int slot = -1;
          const int32_t row = (defv[r] || candv[r]) ? kv_row_of(p, pagev[r], h, s0 + j) : 0;
          if (defv[r]) {
            const uint32_t o = dbase + __popc(dmv[r] & below);
            if (o < static_cast<uint32_t>(p.cap)) sel_u[o] = row;
            if (p.dbg_selected) atomicOr(bm + (j >> 5), 1u << (j & 31));   // for the ascending positions
          } else if (candv[r]) {
            slot = static_cast<int>(cbase + __popc(cmv[r] & below));
            if (slot < p.cap) {
              cand_u[slot] = (static_cast<unsigned long long>(float_key(sv[r])) << 32) |
                             (0xffffffffu - static_cast<uint32_t>(j));
              cand_row_u[slot] = row;
            }
          }
          dbase += __popc(dmv[r]);
          cbase += __popc(cmv[r]);
          // the definite selections' weights leave their cluster's sums (a chunk holds one
          // cluster: the warp adds them up and sends one atomic per head); a candidate's
          // weights are stored for the resolution's winners
          const bool keep = candv[r] && slot >= 0 && slot < kCandWeights;
          if (fix && (dmv[r] != 0u || __any_sync(0xffffffffu, keep))) {   // warp-uniform
            uint32_t id = idv[r];
            if (id >= static_cast<uint32_t>(p.C)) id = 0;
            float e[G];
#pragma unroll
            for (int g = 0; g < G; ++g) e[g] = 0.f;
            // only the lanes that need them look their weights up
            if (defv[r] || keep) token_weights_skewed<G>(lut4, qc4, p.C, id, cwv[r], ub2, e);
            if (keep) {
              float* cw = p.cand_w + (static_cast<size_t>(u) * kCandWeights + slot) * G;
#pragma unroll
              for (int g = 0; g < G; ++g) cw[g] = e[g];
              p.cand_c[static_cast<size_t>(u) * kCandWeights + slot] = static_cast<int32_t>(id);
            }
            if (dmv[r] != 0u) {
              float neg[G];
#pragma unroll
              for (int g = 0; g < G; ++g) neg[g] = defv[r] ? -e[g] : 0.f;   // candidates add nothing
              flush_weights<G>(neg, p.W + static_cast<size_t>(u) * G * p.C, p.C, id);
            }
          }
        }
      }
      __syncthreads();   // this pass is done with act[] and n_act
    }
  }
  // publish this range's selections, candidates and fix-ups, then count it in; the part
  // that completes the count resolves the unit
  // (the barrier orders the CTA's writes before thread 0's release, which is cumulative;
  // the acquire half lets the part that completes the count read every other part's writes)
  __syncthreads();
  if (tid == 0) {
    const int n = c1 - c0;
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(&p.units[u].filt_done), "r"(n)
                 : "memory");
    ss.flag = (old < total && old + n >= total) ? 1 : 0;
  }
  __syncthreads();
  return ss.flag != 0;
}

// One full warp: over counts cnt[0..nbins) (nbins a multiple of 32), find the bin b such
// that sum_{b' > b} cnt < need <= sum_{b' >= b} cnt. Writes *bin/*above only when such a
// bin exists.
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

// Phase 3 for unit u, in the part that completed its filter count: the threshold bin's
// candidates are resolved exactly (the r largest keys, score desc then position asc, with
// r = k - tokens above the bin); the winners' KV-pool rows follow the definite selections'
// rows in key order, their weights leave their clusters' sums, and the unit is published.
// The rows are in no particular position order (the attention does not need one); only
// the debug positions are written in ascending order, after the unit is published.
// `fsm` holds kFinScratch bytes (over the tables: this CTA's filter parts are done).
template <int G>
__device__ void resolve_unit(const StepParams& p, int u, uint8_t* fsm, SelShared& ss) {
  constexpr int GP = (G + 3) / 4;
  constexpr int T = kScanThreads;
  constexpr int kKeysPer = kFinSmemCand / T;   // candidate keys fetched per thread
  unsigned long long* ck = reinterpret_cast<unsigned long long*>(fsm);   // [kFinSmemCand]
  uint32_t* bmc = reinterpret_cast<uint32_t*>(ck + kFinSmemCand);         // [kFinChunkWords]
  uint32_t* woff = bmc + kFinChunkWords;                                  // [kFinChunkWords]
  uint32_t* dig = woff + kFinChunkWords;                                  // [256]
  const int b = u / p.Hkv;
  const int tid = threadIdx.x;
  const unsigned long long* cg = p.cand + static_cast<size_t>(u) * p.cap;
  int32_t* sel_u = p.sel + static_cast<size_t>(u) * p.cap;
  const int T_len = max(0, p.seq_lens[b]);
  const int s0 = min(p.n_sink, T_len);
  const int N = unit_n(p.seq_lens, p.n_indexed, b, p.n_sink, p.cap);
  const int k = decode_k(p.budget, p.k_override, N);
  const bool fix = p.background && N > k;
  __syncthreads();   // the scratch overlays the tables and the filter queues

  // ---- one round trip ----
  const int ncand = __ldcg(&p.units[u].ncand);
  const int above = __ldcg(&p.units[u].above);
  const int ndef = __ldcg(&p.units[u].ndef);
  unsigned long long kr[kKeysPer];   // candidate keys of slots tid + r T (speculative: any count)
#pragma unroll
  for (int r = 0; r < kKeysPer; ++r) {
    const int i = tid + r * T;
    kr[r] = i < p.cap ? __ldcg(cg + i) : 0ull;
  }
  const int32_t* crow = p.cand_row + static_cast<size_t>(u) * p.cap;
  const int32_t rowr = tid < p.cap ? __ldcg(crow + tid) : 0;   // KV-pool row of candidate slot tid
  float cwr[G];                      // stored weights of candidate slot tid
  int32_t ccr = 0;
  if (fix) {
    const float* cw = p.cand_w + (static_cast<size_t>(u) * kCandWeights + tid) * G;
#pragma unroll
    for (int g = 0; g < G; ++g) cwr[g] = tid < kCandWeights ? __ldcg(cw + g) : 0.f;
    ccr = tid < kCandWeights ? __ldcg(p.cand_c + static_cast<size_t>(u) * kCandWeights + tid) : 0;
  }
  float ub2[G];
#pragma unroll
  for (int g = 0; g < G; ++g) ub2[g] = __ldcg(p.fbounds + (static_cast<size_t>(u) * 2 + 0) * G + g) * kLog2e;

  const int m = k > 0 ? min(ncand, p.cap) : 0;
  const int r = k - above;
  const bool ok = k == 0 || (r >= 1 && r <= m);
  const bool in_smem = m <= kFinSmemCand;
#pragma unroll
  for (int rr = 0; rr < kKeysPer; ++rr)
    if (tid + rr * T < min(m, kFinSmemCand)) ck[tid + rr * T] = kr[rr];
  if (tid == 0) {
    ss.tau = ~0ull;
    ss.nwin = 0;
  }
  __syncthreads();
  auto key_at = [&](int i) -> unsigned long long { return in_smem ? ck[i] : __ldcg(cg + i); };
  // A winner: its row after the definite rows (at `o`), its weights out of its cluster's sums.
  auto take_winner = [&](int i, unsigned long long key, int o) {
    const uint32_t j = 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
    if (ndef + o < p.cap) sel_u[ndef + o] = i == tid ? rowr : __ldcg(crow + i);
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
      for (int g = 0; g < G; ++g) e[g] = __ldcg(cw + g);
      id = static_cast<uint32_t>(__ldcg(p.cand_c + static_cast<size_t>(u) * kCandWeights + i));
    } else {
      id = p.ids[static_cast<size_t>(u) * p.cap + j];
      const uint4 cwd = *reinterpret_cast<const uint4*>(p.codes + (static_cast<size_t>(u) * p.cap + j) * kM);
      if (id >= static_cast<uint32_t>(p.C)) id = 0;
      token_weights<G>(reinterpret_cast<const float4*>(p.lut) + static_cast<size_t>(u) * GP * kNcode * kM,
                       reinterpret_cast<const float4*>(p.qc) + static_cast<size_t>(u) * GP * p.C, p.C, id, cwd,
                       ub2, e);
    }
    if (id >= static_cast<uint32_t>(p.C)) id = 0;
    remove_weights<G>(p, u, id, e);
  };

  // ---- winners: the r largest candidate keys (keys are distinct) ----
  if (k > 0 && ok) {
    if (m <= T) {
      if (tid < m) {   // rank = place in descending key order; the r first win, in rank order
        const unsigned long long key = key_at(tid);
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < m; ++j) rank += key_at(j) > key;
        if (rank < r) take_winner(tid, key, rank);
        if (rank == r - 1) ss.tau = key;
      }
    } else {
      unsigned long long prefix = 0, mask = 0;
      uint32_t need = static_cast<uint32_t>(r);
      for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += T) dig[i] = 0u;
        if (tid == 0) {
          ss.bin = -1;
          ss.fin_above = 0;
        }
        __syncthreads();
        for (int i = tid; i < m; i += T) {
          const unsigned long long key = key_at(i);
          if ((key & mask) == prefix) atomicAdd(&dig[(key >> shift) & 255ull], 1u);
        }
        __syncthreads();
        if (tid < 32) find_threshold_desc(dig, 256, need, &ss.bin, &ss.fin_above);
        __syncthreads();
        const int d = ss.bin < 0 ? 0 : ss.bin;
        need -= ss.fin_above;
        prefix |= static_cast<unsigned long long>(d) << shift;
        mask |= 255ull << shift;
        __syncthreads();
      }
      if (tid == 0) ss.tau = prefix;
      for (int i = tid; i < m; i += T) {
        const unsigned long long key = key_at(i);
        if (key >= prefix) take_winner(i, key, static_cast<int>(atomicAdd(&ss.nwin, 1u)));
      }
    }
  }
  // publish: the rows and the winners' fix-ups are written
  __syncthreads();
  const int nsel = ndef + ((k > 0 && ok) ? r : 0);
  if (tid == 0) {   // release after the barrier: cumulative over the CTA's writes
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(&p.units[u].ready), "r"(1) : "memory");
    if (!ok || nsel != k) record_error(p.err, HSA_DEVERR_SELECT);
    if (p.dbg_nselected) p.dbg_nselected[u] = nsel;
  }
  if (!p.dbg_selected || k == 0) return;

  // ---- debug: the selected positions in ascending order (definite bits and winners) ----
  const uint32_t* bm = p.bitmap + static_cast<size_t>(u) * p.bitmap_words;
  const unsigned long long tau = ss.tau;
  const int nw = (N + 31) / 32;
  uint32_t running = 0;
  for (int w0 = 0; w0 < nw; w0 += kFinChunkWords) {
    const int we = min(nw, w0 + kFinChunkWords);
#pragma unroll
    for (int e = 0; e < kFinWordsPerThread; ++e) {
      const int wi = w0 + kFinWordsPerThread * tid + e;
      bmc[kFinWordsPerThread * tid + e] = wi < we ? __ldcg(bm + wi) : 0u;
    }
    __syncthreads();
    for (int i = tid; i < m; i += T) {
      const unsigned long long key = key_at(i);
      if (key < tau) continue;
      const uint32_t j = 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
      const int w = static_cast<int>(j >> 5) - w0;
      if (w >= 0 && w < we - w0) atomicOr(&bmc[w], 1u << (j & 31));
    }
    __syncthreads();
    uint32_t words[kFinWordsPerThread], pc = 0;
#pragma unroll
    for (int e = 0; e < kFinWordsPerThread; ++e) {
      words[e] = bmc[kFinWordsPerThread * tid + e];
      pc += __popc(words[e]);
    }
    uint32_t tot;
    {
      uint32_t o = block_excl_scan(pc, ss.scan_tot, tot);
#pragma unroll
      for (int e = 0; e < kFinWordsPerThread; ++e) {
        woff[kFinWordsPerThread * tid + e] = o;
        o += __popc(words[e]);
      }
    }
    __syncthreads();
    for (uint32_t i = tid; i < tot; i += T) {
      int lo_w = 0, hi_w = kFinChunkWords - 1;   // largest word with woff <= i
      while (lo_w < hi_w) {
        const int mid = (lo_w + hi_w + 1) >> 1;
        if (woff[mid] <= i) lo_w = mid;
        else hi_w = mid - 1;
      }
      uint32_t wv = bmc[lo_w];
      for (uint32_t c = i - woff[lo_w]; c > 0; --c) wv &= wv - 1;
      const uint32_t off = running + i;
      if (off < static_cast<uint32_t>(p.cap))
        p.dbg_selected[static_cast<size_t>(u) * p.cap + off] = s0 + (w0 + lo_w) * 32 + (__ffs(wv) - 1);
    }
    running += tot;
    __syncthreads();   // woff / bmc are rewritten by the next pass
  }
}

// A unit with no chunks to scan (nothing indexed): nothing is selected; publish it.
__device__ void publish_empty_unit(const StepParams& p, int u) {
  if (threadIdx.x == 0) {
    const int N = unit_n(p.seq_lens, p.n_indexed, u / p.Hkv, p.n_sink, p.cap);
    if (decode_k(p.budget, p.k_override, N) != 0) record_error(p.err, HSA_DEVERR_SELECT);
    if (p.dbg_nselected) p.dbg_nselected[u] = 0;
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(&p.units[u].ready), "r"(1) : "memory");
  }
}

// Work split over the units' chunks, planned cooperatively by the CTA (one pass over the
// units per mode, thread t taking units t, t + T, ...). With at least as many CTAs as
// units that have chunks, every CTA takes one part of exactly one unit (1 + a share of
// the spare CTAs in proportion to the unit's chunks), so no CTA pays a second unit's
// set-up; a few CTAs may be left idle. Otherwise every CTA takes a balanced range of the
// concatenated chunks, which may span several units. The parts land in ss.pu/pc0/pc1;
// ss.nparts = -1 when a range spans more than kMaxParts units (then walk_parts is used).
__device__ void plan_parts(const StepParams& p, SelShared& ss) {
  const int U = p.B * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long grid = gridDim.x, me = blockIdx.x;
  long long tot = 0;
  int act = 0;
  int n_first = 0;   // chunks of unit tid (reused by the first pass below)
  for (int u = tid; u < U; u += kScanThreads) {
    const int n = unit_chunks(p, u);
    if (u == tid) n_first = n;
    tot += n;
    act += n > 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    act += __shfl_xor_sync(0xffffffffu, act, o);
  }
  if (lane == 0) {
    ss.red[warp] = tot;
    ss.scan_tot[warp] = static_cast<uint32_t>(act);
  }
  if (tid == 0) ss.nparts = 0;
  __syncthreads();
  if (tid == 0) {
    long long t = 0;
    int a = 0;
    for (int w = 0; w < kScanWarps; ++w) {
      t += ss.red[w];
      a += static_cast<int>(ss.scan_tot[w]);
    }
    ss.total = t;
    ss.active = a;
  }
  __syncthreads();
  const long long total = ss.total;
  const int active = ss.active;
  if (active == 0) return;
  const bool per_unit = active <= grid;
  const long long spare = grid - active;
  const long long start = total * me / grid, end = total * (me + 1) / grid;
  long long run = 0;   // items (or CTAs) of the units before this pass
  for (int u0 = 0; u0 < U; u0 += kScanThreads) {
    const int u = u0 + tid;
    const int n = u0 == 0 ? n_first : (u < U ? unit_chunks(p, u) : 0);
    const int w = per_unit ? (n > 0 ? 1 + static_cast<int>(spare * n / total) : 0) : n;
    uint32_t pass_tot;
    const long long base = run + block_excl_scan(static_cast<uint32_t>(w), ss.scan_tot, pass_tot);
    int i0 = 0, i1 = 0;
    if (per_unit) {
      if (n > 0 && me >= base && me < base + w) {
        const int kk = static_cast<int>(me - base);
        i0 = static_cast<int>(static_cast<long long>(n) * kk / w);
        i1 = static_cast<int>(static_cast<long long>(n) * (kk + 1) / w);
      }
    } else if (n > 0 && start < base + n && end > base) {
      i0 = static_cast<int>(max(start - base, 0LL));
      i1 = static_cast<int>(min(end - base, static_cast<long long>(n)));
    }
    if (i1 > i0) {
      const int at = atomicAdd(&ss.nparts, 1);
      if (at < kMaxParts) {
        ss.pu[at] = u;
        ss.pc0[at] = i0;
        ss.pc1[at] = i1;
        ss.pst[at] = scatter_stride(static_cast<uint32_t>(n));
      }
    }
    run += pass_tot;
    __syncthreads();
  }
  if (tid == 0) {
    if (ss.nparts > kMaxParts) {
      ss.nparts = -1;
    } else {   // unit order (the atomic appends may interleave within a pass)
      for (int i = 1; i < ss.nparts; ++i)
        for (int j = i; j > 0 && ss.pu[j - 1] > ss.pu[j]; --j) {
          int t = ss.pu[j]; ss.pu[j] = ss.pu[j - 1]; ss.pu[j - 1] = t;
          t = ss.pc0[j]; ss.pc0[j] = ss.pc0[j - 1]; ss.pc0[j - 1] = t;
          t = ss.pc1[j]; ss.pc1[j] = ss.pc1[j - 1]; ss.pc1[j - 1] = t;
          const uint32_t st = ss.pst[j]; ss.pst[j] = ss.pst[j - 1]; ss.pst[j - 1] = st;
        }
    }
  }
  __syncthreads();
}

// The balanced-range split of plan_parts walked unit by unit (for a CTA whose range spans
// more than kMaxParts units). Calls f(u, i0, i1) in unit order.
template <typename F>
__device__ void walk_parts(const StepParams& p, long long total, F&& f) {
  const long long grid = gridDim.x;
  const long long start = total * blockIdx.x / grid;
  const long long end = total * (blockIdx.x + 1) / grid;
  long long acc = 0;
  for (int u = 0; u < p.B * p.Hkv && acc < end; ++u) {
    const int n = unit_chunks(p, u);
    if (n > 0 && start < acc + n && end > acc) {
      const int j0 = static_cast<int>(max(start - acc, 0LL));
      const int j1 = static_cast<int>(min(end - acc, static_cast<long long>(n)));
      f(u, j0, j1);
    }
    acc += n;
  }
}

template <int G, int D>
__global__ void __launch_bounds__(kScanThreads, 1) scan_select_kernel(StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float sh_bounds[2 * G];
  __shared__ SelShared ss;
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
                                              static_cast<size_t>(kScanWarps) * D * kRingSlotBytes);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  // The work split reads only the index lists and lengths, which predate the tables kernel
  // (it started only once every earlier kernel had completed): plan while the tables finish.
  plan_parts(p, ss);
  pdl_wait();
  pdl_launch_dependents();
  const int nparts = ss.nparts;
  const long long total = ss.total;
  uint32_t phase = 0;
  int tables_unit = -1;
  // ---- phase 1: scan ----
  auto scan = [&](int u, int c0, int c1) {
    scan_segment<G, D>(p, u, c0, c1, smem, bar, phase, sh_bounds, ysoff, sel, swap_words);
    tables_unit = u;
    ++phase;
  };
  if (nparts >= 0) {
    for (int i = 0; i < nparts; ++i) scan(ss.pu[i], ss.pc0[i], ss.pc1[i]);
  } else {
    walk_parts(p, total, scan);
  }
  // ---- phase 2: selection per unit; phase 3: the part that completes a unit's filter
  // resolves it, after all of this CTA's filter parts (no unit's filter waits behind it) ----
  int nres = 0;
  auto filt = [&](int u, int c0, int c1, uint32_t stride) {
    if (filter_part<G>(p, u, c0, c1, stride, tables_unit == u ? smem : nullptr, smem, ss)) {
      if (nres < kMaxParts) {
        if (threadIdx.x == 0) ss.res[nres] = u;
        ++nres;
      } else {   // more units to resolve than the list holds: resolve this one now
        __threadfence();
        resolve_unit<G>(p, u, smem, ss);
        tables_unit = -1;
      }
    }
  };
  if (nparts >= 0) {
    for (int i = 0; i < nparts; ++i) filt(ss.pu[i], ss.pc0[i], ss.pc1[i], ss.pst[i]);
  } else {
    walk_parts(p, total, [&](int u, int c0, int c1) {
      filt(u, c0, c1, scatter_stride(static_cast<uint32_t>(unit_chunks(p, u))));
    });
  }
  if (nres > 0) {
    __syncthreads();   // thread 0's acquiring count orders the other parts' writes before the reads
    for (int i = 0; i < min(nres, kMaxParts); ++i) resolve_unit<G>(p, ss.res[i], smem, ss);
  }
  // units without chunks (nothing indexed) are published by CTA u mod grid
  for (int u = blockIdx.x; u < p.B * p.Hkv; u += gridDim.x)
    if (unit_chunks(p, u) == 0) publish_empty_unit(p, u);
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
cudaError_t launch_scan_t(const StepParams& p, int grid, cudaStream_t stream, bool pdl) {
  const size_t smem = ScanSmem<G>::bytes(p.C, D);
  cudaError_t e = ensure_dyn_smem<scan_select_kernel<G, D>>(smem);
  if (e != cudaSuccess) return e;
  return launch_ex(scan_select_kernel<G, D>, dim3(grid), dim3(kScanThreads), smem, stream, pdl, p);
}

template <int G>
cudaError_t launch_scan_g(const StepParams& p, int grid, cudaStream_t stream, bool pdl) {
  switch (p.ring_depth) {
    case 8: return launch_scan_t<G, 8>(p, grid, stream, pdl);
    case 4: return launch_scan_t<G, 4>(p, grid, stream, pdl);
    case 2: return launch_scan_t<G, 2>(p, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_scan_select(int G, const StepParams& p, int grid, cudaStream_t stream, bool pdl) {
  switch (G) {
    case 1: return launch_scan_g<1>(p, grid, stream, pdl);
    case 2: return launch_scan_g<2>(p, grid, stream, pdl);
    case 4: return launch_scan_g<4>(p, grid, stream, pdl);
    case 8: return launch_scan_g<8>(p, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pqhsa
