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
// rows (sink + tail + selected) are copied in 16-byte pieces by the producer lanes
// (LSU async copies, 16 lanes per 256-byte row) into a 272-byte-stride layout. Both layouts are bank-conflict free for the two read
// patterns below (and for ldmatrix). Four consumer warps each own every fourth
// 32-token tile and run it on the tensor cores (mma.sync m16n8k16 bf16, with q
// and P split into bf16 hi + lo so the result keeps fp32-level accuracy), with an
// online softmax per query head. Partials are (m, l, acc) in log2 units.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace pqhsa {

namespace {

constexpr int kHalfBytes = kTile * 128;        // swizzled: 32 rows x 128 B (64 bf16)
constexpr int kRowPitch = 272;                 // padded: 256-byte row + 16

// Pipeline shape per loading mode. Tile t goes to consumer warp t % CW and stage
// t % S. S is a multiple of CW, so every stage is always consumed by the same warp
// and its mbarrier phases are awaited strictly in order: a parity wait can then
// never alias a phase two steps ahead (which returns immediately on a parity barrier).
// Dense page tiles use tensor TMA into 16 KB stages, gathered rows 16-byte async copies
// into 272-byte-pitch rows (17 KB stages); both run 4 consumer warps over 4 stages (a
// deeper 2-warp x 6-stage ring for dense reads measured no faster).
template <bool kRows>
struct Pipe {
  static constexpr int CW = 4;
  static constexpr int S = 4;
  static constexpr int threads = (CW + 1) * 32;
  static constexpr int stage_bytes = kRows ? 2 * kTile * kRowPitch : 4 * kHalfBytes;
  static_assert(S % CW == 0, "each stage must belong to one consumer warp");
  static_assert(stage_bytes % 1024 == 0, "stage bases must stay 1024-byte aligned");
};
constexpr int kThreads = Pipe<true>::threads;   // the exact+background launch (background CTAs use it)

template <int G, bool kRows>
struct AttendSmem {
  static constexpr int GP = (G + 3) / 4;
  static constexpr size_t stages = static_cast<size_t>(Pipe<kRows>::S) * Pipe<kRows>::stage_bytes;
  static constexpr size_t qs = kD * GP * 16;
  static constexpr size_t pbuf = Pipe<kRows>::CW * 2 * 8 * kTile * 2;   // P hi/lo bf16 [8 heads][32 tokens]
  static constexpr size_t bars = 2 * Pipe<kRows>::S * 8;
  // swizzled TMA boxes need 1024-byte aligned stages; gathered rows only 16-byte ones
  static constexpr size_t align = kRows ? 128 : 1024;
  static constexpr size_t total = align /*alignment slack*/ + stages + qs + pbuf + bars + 64;
};

// Byte offset of 16-byte chunk c (0..15) of row r inside the K (or V) area of a stage.
template <bool kRows>
__device__ __forceinline__ uint32_t chunk_off(int r, int c) {
  if (kRows) return r * kRowPitch + c * 16;
  return (c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}
template <bool kRows>
__device__ __forceinline__ uint32_t v_area() { return kRows ? kTile * kRowPitch : 2 * kHalfBytes; }


// Position of row v of a unit's sink + tail list: the sink [0, s0), then the R tail rows
// [s0+N, T). Each split takes these rows first, because they do not depend on the
// selection: their copies and math run while the selection is still finishing. The
// selection hands over its k tokens as KV-pool rows (in no particular order).
__device__ __forceinline__ int exact_tail_pos(int v, int s0, int N) { return v < s0 ? v : s0 + N + (v - s0); }

// kMinB resident CTAs per SM: 2, or 3 for the exact part of G <= 4 when its grid holds more
// CTAs than two per SM (128 registers and 76 KB of shared memory each: more gathered rows in
// flight; with at most two CTAs per SM the wider register budget is faster).
template <int G, bool kExact, bool kRows, int kMinB>
__global__ void __launch_bounds__(Pipe<kRows>::threads, kMinB)
    attend_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                  AttendParams p) {
  static_assert(kRows || !kExact, "gathered rows use bulk row copies");
  constexpr int kConsumerWarps = Pipe<kRows>::CW;
  constexpr int kStages = Pipe<kRows>::S;
  constexpr int kStageBytes = Pipe<kRows>::stage_bytes;
  constexpr int GP = (G + 3) / 4;
  extern __shared__ uint8_t smem_raw[];
  constexpr uintptr_t kAlign = AttendSmem<G, kRows>::align;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + kAlign - 1) & ~(kAlign - 1));
  uint8_t* stage_base = smem;
  float4* qs = reinterpret_cast<float4*>(smem + AttendSmem<G, kRows>::stages);               // [kD][GP]
  uint8_t* pbuf = reinterpret_cast<uint8_t*>(qs + kD * GP);                            // [warps] P buffers
  uint64_t* full = reinterpret_cast<uint64_t*>(pbuf + AttendSmem<G, kRows>::pbuf);
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

  // Dense decode waits for the previous kernel at once (its partials may still be read by
  // the previous merge). The exact part starts while the selection's last kernel runs
  // (every kernel before it has completed, the previous step's merge included: each waited
  // for its predecessor before letting the next one start). Sink and tail rows need
  // nothing from the selection; the producer waits for its unit's ready flag before the
  // first selected row.
  if (!kExact) pdl_wait();
  pdl_launch_dependents();

  // ---- row range of this split ------------------------------------------
  const int T = max(0, p.seq_lens[b]);
  int s0 = 0, N = 0, R = 0, E = T;
  if (kExact) {
    s0 = min(p.n_sink, T);
    N = max(0, min(p.n_indexed[b], T - s0));
    N = min(N, p.cap);
    R = T - s0 - N;
    E = s0 + R + decode_k(p.budget, p.k_override, N);
  }
  // Dense: rows [r0, r1) of the T tokens. Exact: the split's share of the sink and tail rows
  // (the first ta tiles, rows [a0, a1) of the sink + tail list) and then its share of the
  // selected rows (tb tiles, entries [e0, e1) of the selection), so every split has some of
  // each: the tiles before the selection is published are spread over all splits, and so
  // are the ones after.
  int r0 = 0, r1 = 0, ta = 0, e0 = 0, e1 = 0;
  if (kExact) {
    const int A = s0 + R, K = E - A;
    const int ca = (A + p.nsplit - 1) / p.nsplit, ce = (K + p.nsplit - 1) / p.nsplit;
    r0 = min(A, split * ca);
    r1 = min(A, r0 + ca);
    e0 = min(K, split * ce);
    e1 = min(K, e0 + ce);
    ta = (r1 - r0 + kTile - 1) / kTile;
  } else {
    r0 = split * p.chunk;
    r1 = min(E, r0 + p.chunk);
    ta = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  }
  const int ntiles = ta + (e1 - e0 + kTile - 1) / kTile;
  const int first_sel_tile = ta;   // first tile of selected rows (ntiles if none)
  // rows of tile t: first row (of the sink + tail list, or of the selection) and count
  auto tile_first = [&](int t) { return t < ta ? r0 + t * kTile : e0 + (t - ta) * kTile; };
  auto tile_rows = [&](int t) { return t < ta ? min(kTile, r1 - (r0 + t * kTile)) : min(kTile, e1 - (e0 + (t - ta) * kTile)); };
  const int32_t* sel_u = kExact ? p.sel + static_cast<size_t>(u) * p.cap : nullptr;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;

  // ---- stage q (pre-scaled by scale*log2 e): every load in flight before the stores ----
  {
    constexpr int kQ = kD * GP * 4;
    constexpr int kPer = (kQ + Pipe<kRows>::threads - 1) / Pipe<kRows>::threads;
    float v[kPer];
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int i = tid + r * Pipe<kRows>::threads;
      const int d = i / (GP * 4), g = i % (GP * 4);
      v[r] = (i < kQ && g < G) ? p.q[(static_cast<size_t>(b) * p.Hq + h * G + g) * kD + d] * p.qscale : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int i = tid + r * Pipe<kRows>::threads;
      if (i < kQ) reinterpret_cast<float*>(qs)[i] = v[r];
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], kRows ? 32 : 1);   // rows: one cp.async arrival per producer lane
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
    bool ok = true, waited = !kExact;
    const int box_rows = kRows ? 1 : min(p.page_size, kTile);
    // Tiles go in groups of up to kStages: each lane first resolves its box of every tile of
    // the group (selected-position and block-table loads of the group in flight together),
    // then the copies are issued tile by tile as stages are released. A group never mixes
    // tiles before and after first_sel_tile, so selection-free tiles never wait.
    for (int t0 = 0, t1; t0 < ntiles && ok; t0 = t1) {
      t1 = min(ntiles, t0 + kStages);
      if (t0 < first_sel_tile) t1 = min(t1, first_sel_tile);
      if (!waited && t0 >= first_sel_tile) {
        ok = __shfl_sync(0xffffffffu, lane == 0 ? (wait_flag(&p.units[u].ready, p.err) ? 1 : 0) : 0, 0) != 0;
        __syncwarp();   // the other lanes' reads of the selection follow lane 0's acquire
        waited = true;
        if (!ok) break;
      }
      int ys[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) {
        ys[i] = -1;
        const int t = t0 + i;
        if (t >= t1) continue;
        const int row0 = tile_first(t);
        const int nvalid = tile_rows(t);
        const int nbox = kRows ? nvalid : (nvalid + box_rows - 1) / box_rows;
        if (lane < nbox) {
          const int v = row0 + lane;
          if (kExact && t >= ta) {
            // already a KV-pool row (checked by the selection); an entry the selection did
            // not write cannot become an out-of-range read
            int y = sel_u[v];
            if (y < 0 || y >= p.num_pages * p.Hkv * p.page_size) {
              record_error(p.err, HSA_DEVERR_SELECT);
              y = 0;
            }
            ys[i] = y;
          } else {
            const int pos = kExact ? exact_tail_pos(v, s0, N) : row0 + lane * box_rows;
            int page = (pos >= 0 && pos < T && pos / p.page_size < p.max_pages) ? bt[pos / p.page_size] : -1;
            if (page < 0 || page >= p.num_pages) {
              record_error(p.err, HSA_DEVERR_PAGE);
              page = 0;
            }
            ys[i] = (page * p.Hkv + h) * p.page_size + (pos % p.page_size);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kStages; ++i) {
        const int t = t0 + i;
        if (t >= t1) break;
        const int s = t % kStages;
        if (t >= kStages) {
          ok = mbar_wait_warp(&empty[s], ((t / kStages) - 1) & 1, p.err);
          if (!ok) break;
        }
        const int nvalid = tile_rows(t);
        uint8_t* st = stage_base + static_cast<size_t>(s) * kStageBytes;
        const int nbox = kRows ? nvalid : (nvalid + box_rows - 1) / box_rows;
        if (kRows) {
          // Gathered rows: 16 lanes copy one 256-byte row in 16-byte pieces (LSU async
          // copies; a bulk copy per row would be bound by the copy engine's per-copy
          // cost), two rows per step; each lane then arrives once its copies have landed.
          const int c16 = lane & 15, half = lane >> 4;
#pragma unroll 4
          for (int rr = 0; rr < kTile / 2; ++rr) {
            const int r = 2 * rr + half;
            const int y = __shfl_sync(0xffffffffu, ys[i], r);
            if (r < nvalid) {
              const size_t src = static_cast<size_t>(y) * (kD * 2) + c16 * 16;
              cp_async_16(st + r * kRowPitch + c16 * 16, p.k_cache + src);
              cp_async_16(st + v_area<kRows>() + r * kRowPitch + c16 * 16, p.v_cache + src);
            }
          }
          cp_async_arrive(&full[s]);
        } else {
          if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox) * 2u * box_rows * 256u);
          __syncwarp();
          if (lane < nbox) {
            const int y = ys[i];
            const int off = lane * box_rows * 128;
            tma_load_2d(st + 0 * kHalfBytes + off, &tmap_k, &full[s], 0, y);
            tma_load_2d(st + 1 * kHalfBytes + off, &tmap_k, &full[s], 64, y);
            tma_load_2d(st + 2 * kHalfBytes + off, &tmap_v, &full[s], 0, y);
            tma_load_2d(st + 3 * kHalfBytes + off, &tmap_v, &full[s], 64, y);
          }
        }
      }
    }
    // Drain: make sure every issued copy has landed before the CTA can exit.
    if (kRows) cp_async_wait<0>();
    if (lane == 0) {
      for (int t = max(0, ntiles - kStages); t < ntiles; ++t) mbar_wait(&full[t % kStages], (t / kStages) & 1, p.err);
    }
    return;
  }

  // ======================= consumer warps (tensor cores) =======================
  // QK^T: S[tok][head] = K[tok][:] . q'[head][:] with m16n8k16 bf16 MMAs: A = K tile (ldmatrix),
  // B = q' split into bf16 hi + lo (the bf16 x bf16 products are exact in fp32, so S carries
  // ~16 mantissa bits of q'). PV: O^T[dim][head] += V^T[dim][tok] P[tok][head]: A = V^T
  // (ldmatrix.trans), B = P split into hi + lo and transposed through a per-warp buffer.
  const int grp = lane >> 2, tig = lane & 3;
  uint32_t qb[8][2][2];   // [k-step][hi, lo][b0, b1]
  {
    const float* qsf = reinterpret_cast<const float*>(qs);   // [kD][GP * 4]
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int d0 = 16 * kk + 8 * r + 2 * tig;
        const float x0 = grp < G ? qsf[d0 * (GP * 4) + grp] : 0.f;
        const float x1 = grp < G ? qsf[(d0 + 1) * (GP * 4) + grp] : 0.f;
        uint32_t hi, lo;
        split_bf16x2(x0, x1, hi, lo);
        qb[kk][0][r] = hi;
        qb[kk][1][r] = lo;
      }
    }
  }
  float oacc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[i][e] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint16_t* pbw = reinterpret_cast<uint16_t*>(pbuf) + warp * (2 * 8 * kTile);   // [hi, lo][8 heads][32 tokens]

  for (int t = warp; t < ntiles; t += kConsumerWarps) {
    const int s = t % kStages;
    if (!mbar_wait_warp(&full[s], (t / kStages) & 1, p.err)) break;   // converged before ldmatrix/mma
    const int nvalid = tile_rows(t);
    uint8_t* st = stage_base + static_cast<size_t>(s) * kStageBytes;
    const uint32_t sa = smem_addr(st);
    if (nvalid < kTile) {
      // stale V rows of a partial tile meet P = 0 in the MMA: make them finite zeros
      for (int r = nvalid + (lane >> 4); r < kTile; r += 2)
        *reinterpret_cast<uint4*>(st + v_area<kRows>() + chunk_off<kRows>(r, lane & 15)) = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }

    // ---- S = K q'^T: two 16-token row blocks x 8 k-steps x (hi, lo) ----
    float sc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
      const int trow = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, sa + chunk_off<kRows>(trow, 2 * kk + (lane >> 4)));
        mma_bf16_16816(sc[mt], a0, a1, a2, a3, qb[kk][0][0], qb[kk][0][1]);
        mma_bf16_16816(sc[mt], a0, a1, a2, a3, qb[kk][1][0], qb[kk][1][1]);
      }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (16 * mt + grp + 8 * (e >> 1) >= nvalid) sc[mt][e] = -INFINITY;

    // ---- online softmax, heads 2*tig + j ----
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float mx = fmaxf(fmaxf(sc[0][j], sc[0][2 + j]), fmaxf(sc[1][j], sc[1][2 + j]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[j], mx);            // finite: every tile has a valid row
      const float alpha = fast_exp2(m_run[j] - m_new);    // m_run = -inf -> 0
      m_run[j] = m_new;
      l_run[j] *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        oacc[i][j] *= alpha;
        oacc[i][2 + j] *= alpha;
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const float pv = fast_exp2(sc[mt][2 * h2 + j] - m_new);
          l_run[j] += pv;
          sc[mt][2 * h2 + j] = pv;
        }
      }
    }
    // ---- P (bf16 hi, lo) to the warp buffer as [head][token] ----
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 16 * mt + grp + 8 * (e >> 1);
        const int head = 2 * tig + (e & 1);
        uint16_t hb, lb;
        split_bf16(sc[mt][e], hb, lb);
        pbw[(0 * 8 + head) * kTile + tok] = hb;
        pbw[(1 * 8 + head) * kTile + tok] = lb;
      }
    }
    __syncwarp();

    // ---- O^T += V^T P: 8 blocks of 16 dims x 2 k-steps of 16 tokens x (hi, lo) ----
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const uint32_t* ph = reinterpret_cast<const uint32_t*>(pbw + (0 * 8 + grp) * kTile + 16 * kk);
      const uint32_t* pl = reinterpret_cast<const uint32_t*>(pbw + (1 * 8 + grp) * kTile + 16 * kk);
      const uint32_t bh0 = ph[tig], bh1 = ph[4 + tig], bl0 = pl[tig], bl1 = pl[4 + tig];
      const int vrow = 16 * kk + (lane & 7) + 8 * (lane >> 4);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(a0, a1, a2, a3, sa + v_area<kRows>() + chunk_off<kRows>(vrow, 2 * i + ((lane >> 3) & 1)));
        mma_bf16_16816(oacc[i], a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(oacc[i], a0, a1, a2, a3, bl0, bl1);
      }
    }
    if (nvalid < kTile) fence_proxy_async_smem();   // zero-fill before the stage's next async fill
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---- combine the consumer warps (reuse the stage area after the pipeline) ----
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  float* cm = reinterpret_cast<float*>(stage_base);            // [warps][8]
  float* cl = cm + kConsumerWarps * 8;                         // [warps][8]
  float* cacc = cl + kConsumerWarps * 8;                       // [warps][8][kD]
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float lw = l_run[j];
    lw += __shfl_xor_sync(0xffffffffu, lw, 4);
    lw += __shfl_xor_sync(0xffffffffu, lw, 8);
    lw += __shfl_xor_sync(0xffffffffu, lw, 16);
    if (grp == 0) {
      cm[warp * 8 + 2 * tig + j] = m_run[j];
      cl[warp * 8 + 2 * tig + j] = lw;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      cacc[(warp * 8 + 2 * tig + (e & 1)) * kD + 16 * i + grp + 8 * (e >> 1)] = oacc[i][e];
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  const size_t slot = static_cast<size_t>(u) * p.S_tot + split;
  for (int d = tid; d < kD; d += kConsumerWarps * 32) {   // the consumer threads cover the output dims
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * 8 + g]);
      float L = 0.f, a = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float f = fast_exp2(cm[w * 8 + g] - M);
          L += f * cl[w * 8 + g];
          a += f * cacc[(w * 8 + g) * kD + d];
        }
      }
      p.pacc[(slot * G + g) * kD + d] = a;
      if (d == 0) {
        p.pm[slot * G + g] = M;
        p.pl[slot * G + g] = L;
      }
    }
  }
}

}  // namespace

// Background partial of one chunk of clusters: l_g = sum_c W_gc, acc_g = sum_c W_gc mean_v_c,
// relative to the reference ub_g (W was accumulated as e^{shat - ub}).
template <int G>
__device__ void background_block(const AttendParams& p, int j, uint8_t* smem) {
  constexpr int NW = kThreads / 32;
  constexpr int kPerWarp = (kBgClusters + NW - 1) / NW;   // clusters per warp: c0 + warp + r * NW
  const int u = j / p.nbg;
  const int cb = j % p.nbg;
  const int b = u / p.Hkv;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  const int T = max(0, p.seq_lens[b]);
  const int s0 = min(p.n_sink, T);
  int N = max(0, min(p.n_indexed[b], T - s0));
  N = min(N, p.cap);
  const int k = decode_k(p.budget, p.k_override, N);
  const bool active = p.bg_enabled && N > k;
  const int c0 = cb * kBgClusters;
  const int c1 = active ? min(p.C, c0 + kBgClusters) : c0;
  // The cluster means predate the step: their loads go out before waiting for the selection.
  const float* mv = p.mean_v + static_cast<size_t>(u) * p.C * kD;
  float4 m4[kPerWarp];
#pragma unroll
  for (int r = 0; r < kPerWarp; ++r) {
    const int c = c0 + warp + r * NW;
    m4[r] = c < c1 ? *reinterpret_cast<const float4*>(mv + static_cast<size_t>(c) * kD + lane * 4)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const size_t slot = static_cast<size_t>(u) * p.S_tot + p.nsplit + cb;
  if (!active) {
    for (int i = tid; i < G * kD; i += blockDim.x) p.pacc[slot * G * kD + i] = 0.f;
    if (tid < G) {
      p.pm[slot * G + tid] = -INFINITY;
      p.pl[slot * G + tid] = 0.f;
    }
    return;
  }
  if (tid == 0) wait_flag(&p.units[u].ready, p.err);   // W is final once the unit's selection is published
  __syncthreads();
  float* ws = reinterpret_cast<float*>(smem);          // [G][kBgClusters] cluster weights
  float* red = ws + G * kBgClusters;                   // [NW][G][kD]
  float* redl = red + NW * G * kD;                     // [NW][G]
  {
    const float* W = p.W + static_cast<size_t>(u) * G * p.C;
    constexpr int kLoads = (G * kBgClusters + kThreads - 1) / kThreads;
    float wv[kLoads];
#pragma unroll
    for (int r = 0; r < kLoads; ++r) {
      const int i = tid + r * kThreads;
      const int g = i / kBgClusters, c = c0 + i % kBgClusters;
      wv[r] = (i < G * kBgClusters && c < c1) ? fmaxf(W[static_cast<size_t>(g) * p.C + c], 0.f) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kLoads; ++r) {
      const int i = tid + r * kThreads;
      if (i < G * kBgClusters) ws[i] = wv[r];
    }
  }
  __syncthreads();
  float acc[G][4], lsum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    lsum[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.f;
  }
#pragma unroll
  for (int r = 0; r < kPerWarp; ++r) {
    const int cl = warp + r * NW;   // cluster c0 + cl (weight 0 past c1)
    if (cl >= kBgClusters) break;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float w = ws[g * kBgClusters + cl];
      lsum[g] += w;
      acc[g][0] = fmaf(w, m4[r].x, acc[g][0]);
      acc[g][1] = fmaf(w, m4[r].y, acc[g][1]);
      acc[g][2] = fmaf(w, m4[r].z, acc[g][2]);
      acc[g][3] = fmaf(w, m4[r].w, acc[g][3]);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    *reinterpret_cast<float4*>(&red[(warp * G + g) * kD + lane * 4]) =
        make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    if (lane == 0) redl[warp * G + g] = lsum[g];
  }
  __syncthreads();
  float ub[G], lb[G];
  final_bounds<G>(p.fbounds, u, ub, lb);
  for (int i = tid; i < G * kD; i += blockDim.x) {
    const int g = i / kD;
    float a = 0.f;
    for (int w = 0; w < NW; ++w) a += red[(w * G + g) * kD + (i % kD)];
    p.pacc[slot * G * kD + i] = a;
  }
  if (tid < G) {
    float l = 0.f, ubt = 0.f;
    for (int w = 0; w < NW; ++w) l += redl[w * G + tid];
#pragma unroll
    for (int g = 0; g < G; ++g) ubt = g == tid ? ub[g] : ubt;   // no run-time index into registers
    p.pm[slot * G + tid] = ubt * kLog2e;
    p.pl[slot * G + tid] = l;
  }
}

namespace {

// out[b, qh] = sum_s e^{m_s - M} acc_s / sum_s e^{m_s - M} l_s over the S_tot partials of its unit.
// 8 warps; warp w owns splits w, w+8, ... (at most kMergePerWarp); lane = 4 dims. Every
// partial (m, l and the 128-wide acc row) is loaded in one round trip, before any math.
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergePerWarp = 16;
static_assert(kMaxSplits + kMaxBgChunks <= kMergeWarps * kMergePerWarp, "merge covers every partial");
template <int G>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(MergeParams p) {
  __shared__ float sh_m[kMergeWarps], sh_l[kMergeWarps];
  __shared__ float4 red[kMergeWarps][32];
  pdl_wait();
  pdl_launch_dependents();
  const int bq = blockIdx.x;               // b * Hq + qh
  const int b = bq / p.Hq, qh = bq % p.Hq;
  const int h = qh / G, g = qh % G;
  const size_t u = static_cast<size_t>(b) * p.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = min(p.S_tot, kMergeWarps * kMergePerWarp);
  float4 v[kMergePerWarp];
  float mv[kMergePerWarp], lv[kMergePerWarp];
#pragma unroll
  for (int r = 0; r < kMergePerWarp; ++r) {
    const int s = warp + r * kMergeWarps;
    const bool ok = s < S;
    const size_t row = (u * S + s) * G + g;
    mv[r] = ok ? p.pm[row] : -INFINITY;
    lv[r] = ok ? p.pl[row] : 0.f;
    v[r] = ok ? *reinterpret_cast<const float4*>(p.pacc + row * kD + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float mx = -INFINITY;
#pragma unroll
  for (int r = 0; r < kMergePerWarp; ++r) mx = fmaxf(mx, mv[r]);
  if (lane == 0) sh_m[warp] = mx;
  __syncthreads();
  float M = sh_m[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) M = fmaxf(M, sh_m[w]);
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
#pragma unroll
  for (int r = 0; r < kMergePerWarp; ++r) {
    const float f = (M == -INFINITY || mv[r] == -INFINITY) ? 0.f : fast_exp2(mv[r] - M);
    L = fmaf(f, lv[r], L);
    a.x = fmaf(f, v[r].x, a.x);
    a.y = fmaf(f, v[r].y, a.y);
    a.z = fmaf(f, v[r].z, a.z);
    a.w = fmaf(f, v[r].w, a.w);
  }
  red[warp][lane] = a;
  if (lane == 0) sh_l[warp] = L;
  __syncthreads();
  if (tid < 32) {
    float4 t = red[0][tid];
    float Lt = sh_l[0];
#pragma unroll
    for (int w = 1; w < kMergeWarps; ++w) {
      const float4 x = red[w][tid];
      t.x += x.x;
      t.y += x.y;
      t.z += x.z;
      t.w += x.w;
      Lt += sh_l[w];
    }
    float4 o;
    o.x = Lt > 0.f ? t.x / Lt : 0.f;
    o.y = Lt > 0.f ? t.y / Lt : 0.f;
    o.z = Lt > 0.f ? t.z / Lt : 0.f;
    o.w = Lt > 0.f ? t.w / Lt : 0.f;
    *reinterpret_cast<float4*>(p.out + static_cast<size_t>(bq) * kD + tid * 4) = o;
  }
}

template <int G, bool kExact, bool kRows, int kMinB = 2>
cudaError_t launch_attend_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttendParams& p, int grid,
                            cudaStream_t stream, bool pdl) {
  static_assert(kMinB == 2 || (kMinB == 3 && kExact && G <= 4), "three CTAs per SM only fit the exact G <= 4 part");
  auto kern = attend_kernel<G, kExact, kRows, kMinB>;
  const size_t smem = AttendSmem<G, kRows>::total;
  cudaError_t e = ensure_dyn_smem<attend_kernel<G, kExact, kRows, kMinB>>(smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Pipe<kRows>::threads);
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
  cfg.blockDim = dim3(kMergeThreads);
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

// CTAs per SM the split planner sizes its waves with (measured on B200, L2 flushed before
// every step): for G <= 4 two, as for dense decode (counting a third resident CTA gave more,
// shorter splits that were slower at 128K); for G = 8, which holds two, three (finer splits
// of each unit's rows were about 4 % faster per step at the Qwen shape).
int attend_slots_per_sm(int G, bool exact, bool rows) {
  (void)rows;
  return (exact && G >= 8) ? 3 : 2;
}

template <int G>
cudaError_t launch_exact_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttendParams& p, int grid,
                           bool wide, cudaStream_t stream, bool pdl) {
  if constexpr (G <= 4) {
    if (wide) return launch_attend_t<G, true, true, 3>(tk, tv, p, grid, stream, pdl);
  }
  return launch_attend_t<G, true, true, 2>(tk, tv, p, grid, stream, pdl);
}

cudaError_t launch_attend(int G, bool exact, bool rows, const CUtensorMap& tk, const CUtensorMap& tv,
                          const AttendParams& p, int grid, bool wide, cudaStream_t stream, bool pdl) {
#define PQHSA_ATT(GG)                                                                   \
  case GG:                                                                              \
    if (exact) return launch_exact_t<GG>(tk, tv, p, grid, wide, stream, pdl);           \
    if (rows) return launch_attend_t<GG, false, true>(tk, tv, p, grid, stream, pdl);    \
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
