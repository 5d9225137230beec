// IVF-PQ index maintenance for PQ-HSA: cluster statistics of the indexed
// tokens' values (count, sum, mean) and batched encoding of new tokens.
//
// Source: rit.work "pq-hsa-long-context-attention", section
// "Как приблизительные оценки возвращают отброшенный контекст": the index is
// built after prefill, new tokens are kept outside it and added in batches,
// and an unread token's value is represented by its index group's mean value.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace pqhsa {

namespace {

__device__ __forceinline__ int slot_base(const IndexParams& p, int b) {
  return p.slot_lo_from_indexed ? max(0, p.n_indexed[b]) : 0;
}
__device__ __forceinline__ int slot_count(const IndexParams& p, int b) {
  return p.n_slots >= 0 ? p.n_slots : max(0, p.n_indexed[b]);
}

// Row address of (position pos, KV head h) of sequence b, or null for an invalid page.
__device__ __forceinline__ const uint16_t* kv_row(const IndexParams& p, const uint16_t* cache, int b, int h, int pos) {
  const int lp = pos / p.page_size;
  const int page = (pos >= 0 && lp < p.max_pages) ? p.block_table[static_cast<size_t>(b) * p.max_pages + lp] : -1;
  if (page < 0 || page >= p.num_pages) {
    record_error(p.err, HSA_DEVERR_PAGE);
    return nullptr;
  }
  return cache + ((static_cast<size_t>(page) * p.Hkv + h) * p.page_size + (pos % p.page_size)) * kD;
}

__global__ void zero_stats_kernel(IndexParams p) {
  const size_t per_unit = static_cast<size_t>(p.C) * kD;
  const size_t U = static_cast<size_t>(p.B) * p.Hkv;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < U * per_unit;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(i / per_unit);
    if (p.zero_if_empty && p.n_indexed[u / p.Hkv] != 0) continue;
    p.sum_v[i] = 0.f;
    if (i % kD == 0) p.count[i / kD] = 0;
  }
}

// Warp per token: add the token's value row to its cluster's sum and count.
__global__ void __launch_bounds__(256) accumulate_kernel(IndexParams p) {
  const int u = blockIdx.x;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.seq_lens[b];
  const int lo = slot_base(p, b);
  const int n = slot_count(p, b);
  for (int t = blockIdx.y * 64 + warp; t < min(n, (static_cast<int>(blockIdx.y) + 1) * 64); t += 8) {
    const int slot = lo + t;
    const int pos = p.n_sink + slot;
    if (slot >= p.cap || pos >= T) continue;
    uint32_t id = p.ids[static_cast<size_t>(u) * p.cap + slot];
    if (id >= static_cast<uint32_t>(p.C)) {
      if (lane == 0) record_error(p.err, HSA_DEVERR_CLUSTER);
      continue;
    }
    const uint16_t* row = kv_row(p, p.v_cache, b, h, pos);
    if (!row) continue;
    const uint2 raw = *reinterpret_cast<const uint2*>(row + lane * 4);
    const float4 v = make_float4(bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y));
    float* dst = p.sum_v + (static_cast<size_t>(u) * p.C + id) * kD + lane * 4;
    atomicAdd(reinterpret_cast<float4*>(dst), v);
    if (lane == 0) atomicAdd(p.count + static_cast<size_t>(u) * p.C + id, 1);
  }
}

// mean_v = sum_v / count (0 for an empty cluster); optionally advance n_indexed.
__global__ void means_kernel(IndexParams p) {
  const size_t total = static_cast<size_t>(p.B) * p.Hkv * p.C * kD;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int c = p.count[i / kD];
    p.mean_v[i] = c > 0 ? __fdiv_rn(p.sum_v[i], static_cast<float>(c)) : 0.f;
  }
  if (p.bump_indexed && blockIdx.x == 0 && threadIdx.x == 0) {
    for (int b = 0; b < p.B; ++b) p.n_indexed[b] = min(p.cap, p.n_indexed[b] + p.n_slots);
  }
}

// Encode 32 new tokens of one unit: lane t of every warp holds token t's key in
// registers; warp w scans centroids w, w+8, ...; then warp w finds the nearest
// codeword of subspaces 2w and 2w+1 for all 32 residuals.
constexpr int kEncTok = 32;

__global__ void __launch_bounds__(256, 1) encode_kernel(IndexParams p) {
  __shared__ float bd[8][kEncTok];
  __shared__ int bc[8][kEncTok];
  __shared__ int assign[kEncTok];
  __shared__ float rs[kEncTok][kD + 1];
  __shared__ uint8_t cs[kEncTok][kM];
  const int u = blockIdx.x;
  const int b = u / p.Hkv, h = u % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.seq_lens[b];
  const int base = slot_base(p, b);
  const int n = slot_count(p, b);
  const int t_idx = blockIdx.y * kEncTok + lane;
  const int slot = base + t_idx;
  const int pos = p.n_sink + slot;
  const bool valid = t_idx < n && slot < p.cap && pos < T;

  float kf[kD];
  const uint16_t* row = valid ? kv_row(p, p.k_cache, b, h, pos) : nullptr;
#pragma unroll
  for (int c = 0; c < kD / 8; ++c) {
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (row) raw = *reinterpret_cast<const uint4*>(row + c * 8);
    kf[c * 8 + 0] = bf16lo(raw.x);
    kf[c * 8 + 1] = bf16hi(raw.x);
    kf[c * 8 + 2] = bf16lo(raw.y);
    kf[c * 8 + 3] = bf16hi(raw.y);
    kf[c * 8 + 4] = bf16lo(raw.z);
    kf[c * 8 + 5] = bf16hi(raw.z);
    kf[c * 8 + 6] = bf16lo(raw.w);
    kf[c * 8 + 7] = bf16hi(raw.w);
  }

  // nearest centroid: direct sum of squared differences, ties to the lower index
  const float* cent = p.centroids + static_cast<size_t>(u) * p.C * kD;
  float best = INFINITY;
  int besti = 0x7fffffff;
  for (int c = warp; c < p.C; c += 8) {
    const float4* cr = reinterpret_cast<const float4*>(cent + static_cast<size_t>(c) * kD);
    float dist = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < kD / 4; ++q4) {
      const float4 cv = __ldg(cr + q4);
      float t0 = __fsub_rn(kf[q4 * 4 + 0], cv.x);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 1], cv.y);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 2], cv.z);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 3], cv.w);
      dist = fmaf(t0, t0, dist);
    }
    if (dist < best) {
      best = dist;
      besti = c;
    }
  }
  bd[warp][lane] = best;
  bc[warp][lane] = besti;
  __syncthreads();
  if (warp == 0) {
    float bb = bd[0][lane];
    int bi = bc[0][lane];
    for (int w = 1; w < 8; ++w) {
      const float d = bd[w][lane];
      const int ci = bc[w][lane];
      if (d < bb || (d == bb && ci < bi)) {
        bb = d;
        bi = ci;
      }
    }
    if (bi >= p.C || bi < 0) bi = 0;   // only for an empty centroid set / NaN keys
    assign[lane] = bi;
    const float* ca = cent + static_cast<size_t>(bi) * kD;
#pragma unroll
    for (int d = 0; d < kD; ++d) rs[lane][d] = __fsub_rn(kf[d], __ldg(ca + d));
  }
  __syncthreads();

  // nearest codeword per subspace of the residual
  const float* cb = p.codebooks + static_cast<size_t>(u) * kM * kNcode * kDsub;
  for (int si = 0; si < 2; ++si) {
    const int s = warp * 2 + si;
    float r[kDsub];
#pragma unroll
    for (int d = 0; d < kDsub; ++d) r[d] = rs[lane][s * kDsub + d];
    float bb = INFINITY;
    int bm = 0;
    const float4* cw = reinterpret_cast<const float4*>(cb + static_cast<size_t>(s) * kNcode * kDsub);
    for (int m = 0; m < kNcode; ++m) {
      const float4 a = __ldg(cw + 2 * m), c2 = __ldg(cw + 2 * m + 1);
      const float w8[8] = {a.x, a.y, a.z, a.w, c2.x, c2.y, c2.z, c2.w};
      float dist = 0.f;
#pragma unroll
      for (int d = 0; d < kDsub; ++d) {
        const float t0 = __fsub_rn(r[d], w8[d]);
        dist = fmaf(t0, t0, dist);
      }
      if (dist < bb) {
        bb = dist;
        bm = m;
      }
    }
    cs[lane][s] = static_cast<uint8_t>(bm);
  }
  __syncthreads();
  if (warp == 0 && valid) {
    p.ids[static_cast<size_t>(u) * p.cap + slot] = static_cast<uint16_t>(assign[lane]);
    uint4 packed;
    const uint8_t* c8 = cs[lane];
    packed.x = c8[0] | (c8[1] << 8) | (c8[2] << 16) | (static_cast<uint32_t>(c8[3]) << 24);
    packed.y = c8[4] | (c8[5] << 8) | (c8[6] << 16) | (static_cast<uint32_t>(c8[7]) << 24);
    packed.z = c8[8] | (c8[9] << 8) | (c8[10] << 16) | (static_cast<uint32_t>(c8[11]) << 24);
    packed.w = c8[12] | (c8[13] << 8) | (c8[14] << 16) | (static_cast<uint32_t>(c8[15]) << 24);
    *reinterpret_cast<uint4*>(p.codes + (static_cast<size_t>(u) * p.cap + slot) * kM) = packed;
  }
}

// ---------------------------------------------------------------------------
// Cluster-ordered lists. A unit's list slots form 32-slot chunks; every chunk holds
// members of one cluster, so the scan sees one cluster per warp-sized chunk. Meta per
// unit: [0] chunks in use, [1] unused, then per cluster c: [2+2c] its open (last)
// chunk or -1, [3+2c] members in that chunk.
// ---------------------------------------------------------------------------
__global__ void list_reset_kernel(IndexParams p) {
  const size_t per_unit = 2 + 2 * static_cast<size_t>(p.C);
  const size_t total = static_cast<size_t>(p.B) * p.Hkv * per_unit;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(i / per_unit);
    if (p.zero_if_empty && p.n_indexed[u / p.Hkv] != 0) continue;
    const size_t r = i % per_unit;
    p.list_meta[i] = r < 2 ? 0 : ((r & 1) == 0 ? -1 : 32);   // no open chunk: treat as full
  }
}

// One CTA per unit: add index slots [lo, lo + n) to their clusters' lists. Count the
// new members per cluster, give each cluster the room left in its open chunk plus
// fresh chunks, then place every member (any order inside a cluster).
constexpr int kListThreads = 1024;
__global__ void __launch_bounds__(kListThreads) list_append_kernel(IndexParams p) {
  extern __shared__ int32_t lsm[];
  const int C = p.C;
  int32_t* cnt = lsm;
  int32_t* put = cnt + C;
  int32_t* base = put + C;
  int32_t* room = base + C;
  int32_t* open0 = room + C;
  int32_t* fill0 = open0 + C;
  __shared__ int32_t nch_s;
  const int u = blockIdx.x;
  const int b = u / p.Hkv;
  const int tid = threadIdx.x;
  const int lo = slot_base(p, b);
  const int n = slot_count(p, b);
  const int max_chunks = p.list_slots / 32;
  int32_t* meta = p.list_meta + static_cast<size_t>(u) * (2 + 2 * static_cast<size_t>(C));
  const uint16_t* ids_u = p.ids + static_cast<size_t>(u) * p.cap;
  int32_t* lslot = p.list_slot + static_cast<size_t>(u) * p.list_slots;
  uint4* lcodes = reinterpret_cast<uint4*>(p.list_codes) + static_cast<size_t>(u) * p.list_slots;
  const uint4* codes_u = reinterpret_cast<const uint4*>(p.codes) + static_cast<size_t>(u) * p.cap;
  uint16_t* ccl = p.chunk_cluster + static_cast<size_t>(u) * max_chunks;
  for (int c = tid; c < C; c += blockDim.x) {
    cnt[c] = 0;
    put[c] = 0;
  }
  if (tid == 0) nch_s = min(max(meta[0], 0), max_chunks);   // garbage metadata cannot index out of range
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int slot = lo + i;
    if (slot >= p.cap) continue;
    const uint32_t id = ids_u[slot];
    if (id < static_cast<uint32_t>(C)) atomicAdd(&cnt[id], 1);
  }
  __syncthreads();
  for (int c = tid; c < C; c += blockDim.x) {
    const int k = cnt[c];
    if (k == 0) continue;
    int op = meta[2 + 2 * c], fl = meta[3 + 2 * c];
    if (op < 0 || op >= max_chunks || fl < 0 || fl > 32) {   // no (valid) open chunk
      op = -1;
      fl = 32;
    }
    const int free = op >= 0 ? 32 - fl : 0;
    const int extra = max(0, k - free);
    const int nn = (extra + 31) / 32;
    int bs = nn ? atomicAdd(&nch_s, nn) : 0;
    if (bs + nn > max_chunks) {   // cannot happen with list_slots >= 32*(ceil(cap/32)+C)
      record_error(p.err, HSA_DEVERR_SELECT);
      bs = -1;
    }
    base[c] = bs;
    room[c] = free;
    open0[c] = op;
    fill0[c] = fl;
    if (bs >= 0) {
      for (int q = 0; q < nn; ++q) ccl[bs + q] = static_cast<uint16_t>(c);
      if (nn > 0) {
        const int used = extra - 32 * (nn - 1);
        for (int r = used; r < 32; ++r) lslot[(bs + nn - 1) * 32 + r] = -1;
        meta[2 + 2 * c] = bs + nn - 1;
        meta[3 + 2 * c] = used;
      } else {
        meta[3 + 2 * c] = fl + k;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int slot = lo + i;
    if (slot >= p.cap) continue;
    const uint32_t id = ids_u[slot];
    if (id >= static_cast<uint32_t>(C)) continue;
    const int r = atomicAdd(&put[id], 1);
    int ls;
    if (r < room[id]) {
      ls = open0[id] * 32 + fill0[id] + r;
    } else {
      if (base[id] < 0) continue;
      const int e = r - room[id];
      ls = (base[id] + e / 32) * 32 + (e % 32);
    }
    lcodes[ls] = codes_u[slot];
    lslot[ls] = slot;
  }
  __syncthreads();
  if (tid == 0) meta[0] = min(nch_s, max_chunks);
}

int grid_for(size_t work, int threads) {
  size_t g = (work + threads - 1) / threads;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// ---------------------------------------------------------------------------
// Index training. The article builds the index after prefill and leaves the training
// open; the reading here is the plain Lloyd k-means: coarse centroids on the unit's keys
// at positions [n_sink, n_sink + n_train), then per subspace a codebook on the residuals
// (key minus its centroid). Initial centres are the given training rows. Distances are
// direct sums of squared differences in fp32, ties to the lower index; a centre that
// gets no rows keeps its value.
// ---------------------------------------------------------------------------
// Key row of training key j of unit (b, h): position n_sink + slot0[b] + j (slot0 null: 0).
__device__ __forceinline__ const uint16_t* train_key(const TrainParams& p, int b, int h, int slot) {
  if (slot < 0 || slot >= p.n_train) {
    record_error(p.err, HSA_DEVERR_SLOT);
    slot = 0;
  }
  const int pos = p.n_sink + (p.slot0 ? p.slot0[b] : 0) + slot;
  const int lp = pos / p.page_size;
  const int page = lp < p.max_pages ? p.block_table[static_cast<size_t>(b) * p.max_pages + lp] : -1;
  if (page < 0 || page >= p.num_pages) {
    record_error(p.err, HSA_DEVERR_PAGE);
    return nullptr;
  }
  return p.k_cache + ((static_cast<size_t>(page) * p.Hkv + h) * p.page_size + (pos % p.page_size)) * kD;
}

__device__ __forceinline__ size_t init_stride(const TrainParams& p) {
  return static_cast<size_t>(p.C) + static_cast<size_t>(kM) * kNcode;
}

// Warp per centroid: centroid c = the key of training slot init_slots[c].
__global__ void __launch_bounds__(256) train_init_kernel(TrainParams p) {
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.y * 8 + warp;
  if (c >= p.C) return;
  const uint16_t* row = train_key(p, b, h, p.init_slots[u * init_stride(p) + c]);
  uint2 raw = make_uint2(0, 0);
  if (row) raw = *reinterpret_cast<const uint2*>(row + lane * 4);
  *reinterpret_cast<float4*>(p.centroids + (static_cast<size_t>(u) * p.C + c) * kD + lane * 4) =
      make_float4(bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y));
}

// Nearest centroid of 32 training keys per CTA: lane t of every warp holds key t in
// registers; warp w scans centroids w, w + 8, ...; the 8 warps' best are merged.
__global__ void __launch_bounds__(256, 1) train_assign_kernel(TrainParams p) {
  __shared__ float bd[8][32];
  __shared__ int bc[8][32];
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.y * 32 + lane;
  const bool valid = j < p.n_train;
  float kf[kD];
  const uint16_t* row = valid ? train_key(p, b, h, j) : nullptr;
#pragma unroll
  for (int c = 0; c < kD / 8; ++c) {
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (row) raw = *reinterpret_cast<const uint4*>(row + c * 8);
    kf[c * 8 + 0] = bf16lo(raw.x);
    kf[c * 8 + 1] = bf16hi(raw.x);
    kf[c * 8 + 2] = bf16lo(raw.y);
    kf[c * 8 + 3] = bf16hi(raw.y);
    kf[c * 8 + 4] = bf16lo(raw.z);
    kf[c * 8 + 5] = bf16hi(raw.z);
    kf[c * 8 + 6] = bf16lo(raw.w);
    kf[c * 8 + 7] = bf16hi(raw.w);
  }
  const float* cent = p.centroids + static_cast<size_t>(u) * p.C * kD;
  float best = INFINITY;
  int besti = 0x7fffffff;
  for (int c = warp; c < p.C; c += 8) {
    const float4* cr = reinterpret_cast<const float4*>(cent + static_cast<size_t>(c) * kD);
    float dist = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < kD / 4; ++q4) {
      const float4 cv = __ldg(cr + q4);
      float t0 = __fsub_rn(kf[q4 * 4 + 0], cv.x);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 1], cv.y);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 2], cv.z);
      dist = fmaf(t0, t0, dist);
      t0 = __fsub_rn(kf[q4 * 4 + 3], cv.w);
      dist = fmaf(t0, t0, dist);
    }
    if (dist < best) {
      best = dist;
      besti = c;
    }
  }
  bd[warp][lane] = best;
  bc[warp][lane] = besti;
  __syncthreads();
  if (warp == 0 && valid) {
    float bb = bd[0][lane];
    int bi = bc[0][lane];
    for (int w = 1; w < 8; ++w) {
      const float d = bd[w][lane];
      const int ci = bc[w][lane];
      if (d < bb || (d == bb && ci < bi)) {
        bb = d;
        bi = ci;
      }
    }
    if (bi >= p.C || bi < 0) bi = 0;   // NaN keys only
    p.assign[static_cast<size_t>(u) * p.n_train + j] = bi;
    if (p.assign_out) p.assign_out[static_cast<size_t>(u) * p.n_train + j] = bi;
  }
}

// Warp per training key: add it to its centre's sum and count.
__global__ void __launch_bounds__(256) train_accumulate_kernel(TrainParams p) {
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = blockIdx.y * 64 + warp; j < min(p.n_train, (static_cast<int>(blockIdx.y) + 1) * 64); j += 8) {
    const int a = p.assign[static_cast<size_t>(u) * p.n_train + j];
    const uint16_t* row = train_key(p, b, h, j);
    if (!row) continue;
    const uint2 raw = *reinterpret_cast<const uint2*>(row + lane * 4);
    atomicAdd(reinterpret_cast<float4*>(p.sums + (static_cast<size_t>(u) * p.C + a) * kD + lane * 4),
              make_float4(bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y)));
    if (lane == 0) atomicAdd(p.counts + static_cast<size_t>(u) * p.C + a, 1);
  }
}

// centre = sum / count where the centre got rows (else unchanged); then clear the sums.
__global__ void train_update_kernel(float* centres, float* sums, int32_t* counts, size_t n, int dim) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int c = counts[i / dim];
    if (c > 0) centres[i] = __fdiv_rn(sums[i], static_cast<float>(c));
    sums[i] = 0.f;
  }
}
__global__ void train_clear_counts_kernel(int32_t* counts, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    counts[i] = 0;
}

// Thread per codeword m of subspace s: its initial value is the subspace-s residual of
// training slot init_slots[C + s * ncode + m] under the final coarse assignment.
__global__ void __launch_bounds__(256) train_pq_init_kernel(TrainParams p) {
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int s = blockIdx.y, m = threadIdx.x;
  int slot = p.init_slots[u * init_stride(p) + p.C + s * kNcode + m];
  const uint16_t* row = train_key(p, b, h, slot);
  if (slot < 0 || slot >= p.n_train) slot = 0;
  const int a = p.assign[static_cast<size_t>(u) * p.n_train + slot];
  uint4 raw = make_uint4(0, 0, 0, 0);
  if (row) raw = *reinterpret_cast<const uint4*>(row + s * kDsub);
  const float kv8[8] = {bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y),
                        bf16lo(raw.z), bf16hi(raw.z), bf16lo(raw.w), bf16hi(raw.w)};
  const float* ca = p.centroids + (static_cast<size_t>(u) * p.C + a) * kD + s * kDsub;
  float* dst = p.codebooks + ((static_cast<size_t>(u) * kM + s) * kNcode + m) * kDsub;
#pragma unroll
  for (int d = 0; d < kDsub; ++d) dst[d] = __fsub_rn(kv8[d], ca[d]);
}

// ---- nearest codeword of residual sub-vectors (training step and encoding) ----------
// A CTA takes kPqGroup subspaces of one unit: the group's codebooks and, per codeword, the
// pair (|w|^2 / 2, |w|^2 / 2) sit in shared memory; each warp works on one subspace (every
// codeword read is a broadcast) and each lane on kPqLane keys, which share the reads. The
// distance is evaluated as |w|^2 - 2 r.w (|r - w|^2 minus the key's constant |r|^2) with
// packed fp32x2 fused multiply-adds; ties go to the lower codeword index.
constexpr int kPqGroup = 2;
constexpr int kPqLane = 4;                                       // keys per lane
constexpr int kPqKeys = 2048;                                    // keys per CTA
constexpr int kPqThreads = 256;
constexpr int kPqWarpKeys = 32 * kPqLane;
constexpr int kPqKeyStride = (kPqThreads / 32 / kPqGroup) * kPqWarpKeys;   // keys per loop round of a CTA
constexpr size_t kPqBookFloats = static_cast<size_t>(kPqGroup) * kNcode * kDsub;
constexpr size_t kPqSmemCodes = (kPqBookFloats + kPqGroup * kNcode * 2) * sizeof(float);
constexpr size_t kPqSmemStep = kPqSmemCodes + (kPqBookFloats + kPqGroup * kNcode) * sizeof(float);

// Stage the codebooks of subspaces [s0, s0 + kPqGroup) of unit u and their half norms.
__device__ __forceinline__ void stage_books(const float* codebooks, int u, int s0, float* book, float2* hn) {
  const float* g = codebooks + (static_cast<size_t>(u) * kM + s0) * kNcode * kDsub;
  for (int i = threadIdx.x; i < static_cast<int>(kPqBookFloats / 4); i += blockDim.x)
    reinterpret_cast<float4*>(book)[i] = reinterpret_cast<const float4*>(g)[i];
  __syncthreads();
  for (int i = threadIdx.x; i < kPqGroup * kNcode; i += blockDim.x) {
    const float* w = book + i * kDsub;
    float n = 0.f;
#pragma unroll
    for (int d = 0; d < kDsub; ++d) n = fmaf(w[d], w[d], n);
    hn[i] = make_float2(0.5f * n, 0.5f * n);
  }
  __syncthreads();
}

// Residual sub-vector s of key j: key - its centroid (fp32); zeros and false for a key
// outside [0, j_end) or on an invalid page.
__device__ __forceinline__ bool residual_sub(const TrainParams& p, int u, int b, int h, int j, int j_end, int s,
                                             float* r) {
  const uint16_t* row = j < j_end ? train_key(p, b, h, j) : nullptr;
  if (!row) {
#pragma unroll
    for (int d = 0; d < kDsub; ++d) r[d] = 0.f;
    return false;
  }
  const int a = p.assign[static_cast<size_t>(u) * p.n_train + j];
  const uint4 raw = *reinterpret_cast<const uint4*>(row + s * kDsub);
  const float kv8[8] = {bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y),
                        bf16lo(raw.z), bf16hi(raw.z), bf16lo(raw.w), bf16hi(raw.w)};
  const float4* ca = reinterpret_cast<const float4*>(p.centroids + (static_cast<size_t>(u) * p.C + a) * kD +
                                                     s * kDsub);
  const float4 c0 = __ldg(ca), c1 = __ldg(ca + 1);
  const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int d = 0; d < kDsub; ++d) r[d] = __fsub_rn(kv8[d], cv[d]);
  return true;
}

// Nearest codewords of kPqLane residual sub-vectors in one subspace's staged codebook.
__device__ __forceinline__ void nearest_codewords(const float (&r)[kPqLane][kDsub], const float* book,
                                                  const float2* hn, int (&best_m)[kPqLane]) {
  unsigned long long pr[kPqLane][4];
  float best[kPqLane];
#pragma unroll
  for (int k = 0; k < kPqLane; ++k) {
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[k][i] = pack_f2(-2.f * r[k][2 * i], -2.f * r[k][2 * i + 1]);
    best[k] = INFINITY;
    best_m[k] = 0;
  }
  const ulonglong2* w = reinterpret_cast<const ulonglong2*>(book);
  const unsigned long long* h = reinterpret_cast<const unsigned long long*>(hn);
#pragma unroll 2
  for (int m = 0; m < kNcode; ++m) {
    const ulonglong2 w0 = w[2 * m], w1 = w[2 * m + 1];
    const unsigned long long hm = h[m];
#pragma unroll
    for (int k = 0; k < kPqLane; ++k) {
      unsigned long long x = ffma2_rn(pr[k][0], w0.x, hm);
      x = ffma2_rn(pr[k][1], w0.y, x);
      x = ffma2_rn(pr[k][2], w1.x, x);
      x = ffma2_rn(pr[k][3], w1.y, x);
      const float d = lo_f(x) + hi_f(x);
      if (d < best[k]) {
        best[k] = d;
        best_m[k] = m;
      }
    }
  }
}

// One Lloyd step of the codebooks: nearest codeword of every residual sub-vector, added to
// the CTA's shared sums, which are then added to the global ones.
__global__ void __launch_bounds__(kPqThreads, 3) train_pq_step_kernel(TrainParams p) {
  extern __shared__ __align__(16) float pq_sh[];
  float* book = pq_sh;
  float2* hn = reinterpret_cast<float2*>(book + kPqBookFloats);
  float* sums = reinterpret_cast<float*>(hn + kPqGroup * kNcode);
  int* cnt = reinterpret_cast<int*>(sums + kPqBookFloats);
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int s0 = blockIdx.y * kPqGroup;
  for (int i = threadIdx.x; i < static_cast<int>(kPqBookFloats); i += kPqThreads) sums[i] = 0.f;
  for (int i = threadIdx.x; i < kPqGroup * kNcode; i += kPqThreads) cnt[i] = 0;
  stage_books(p.codebooks, u, s0, book, hn);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sl = warp % kPqGroup, s = s0 + sl;
  const int j_end = min(p.n_train, static_cast<int>(blockIdx.z + 1) * kPqKeys);
  for (int j = blockIdx.z * kPqKeys + (warp / kPqGroup) * kPqWarpKeys + lane; j < j_end; j += kPqKeyStride) {
    float r[kPqLane][kDsub];
    bool v[kPqLane];
#pragma unroll
    for (int k = 0; k < kPqLane; ++k) v[k] = residual_sub(p, u, b, h, j + 32 * k, j_end, s, r[k]);
    int m[kPqLane];
    nearest_codewords(r, book + sl * kNcode * kDsub, hn + sl * kNcode, m);
#pragma unroll
    for (int k = 0; k < kPqLane; ++k) {
      if (!v[k]) continue;
      float* dst = sums + (sl * kNcode + m[k]) * kDsub;
#pragma unroll
      for (int d = 0; d < kDsub; ++d) atomicAdd(dst + d, r[k][d]);
      atomicAdd(cnt + sl * kNcode + m[k], 1);
    }
  }
  __syncthreads();
  float* gsum = p.pq_sums + (static_cast<size_t>(u) * kM + s0) * kNcode * kDsub;
  int* gcnt = p.pq_counts + (static_cast<size_t>(u) * kM + s0) * kNcode;
  for (int i = threadIdx.x; i < kPqGroup * kNcode; i += kPqThreads) {
    const int c = cnt[i];
    if (c == 0) continue;
    const float4* src = reinterpret_cast<const float4*>(sums + i * kDsub);
    atomicAdd(reinterpret_cast<float4*>(gsum + i * kDsub), src[0]);
    atomicAdd(reinterpret_cast<float4*>(gsum + i * kDsub + 4), src[1]);
    atomicAdd(gcnt + i, c);
  }
}

// Encoding: ids and codes of keys [0, n_train) of every unit, i.e. index slots
// slot0[b] + j, from the nearest-centroid assignment in p.assign.
__global__ void __launch_bounds__(kPqThreads, 3) encode_codes_kernel(TrainParams p, uint8_t* codes, uint16_t* ids,
                                                                  int cap) {
  extern __shared__ __align__(16) float pq_sh[];
  float* book = pq_sh;
  float2* hn = reinterpret_cast<float2*>(book + kPqBookFloats);
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  const int s0 = blockIdx.y * kPqGroup;
  stage_books(p.codebooks, u, s0, book, hn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sl = warp % kPqGroup, s = s0 + sl;
  const int first = p.slot0 ? p.slot0[b] : 0;
  const int j_end = min(p.n_train, static_cast<int>(blockIdx.z + 1) * kPqKeys);
  for (int j = blockIdx.z * kPqKeys + (warp / kPqGroup) * kPqWarpKeys + lane; j < j_end; j += kPqKeyStride) {
    float r[kPqLane][kDsub];
    bool v[kPqLane];
#pragma unroll
    for (int k = 0; k < kPqLane; ++k) v[k] = residual_sub(p, u, b, h, j + 32 * k, j_end, s, r[k]);
    int m[kPqLane];
    nearest_codewords(r, book + sl * kNcode * kDsub, hn + sl * kNcode, m);
#pragma unroll
    for (int k = 0; k < kPqLane; ++k) {
      if (!v[k]) continue;
      const int jk = j + 32 * k;
      const size_t slot = static_cast<size_t>(u) * cap + first + jk;
      codes[slot * kM + s] = static_cast<uint8_t>(m[k]);
      if (s == 0) ids[slot] = static_cast<uint16_t>(p.assign[static_cast<size_t>(u) * p.n_train + jk]);
    }
  }
}

}  // namespace

cudaError_t launch_zero_stats(const IndexParams& p, cudaStream_t stream) {
  const size_t work = static_cast<size_t>(p.B) * p.Hkv * p.C * kD;
  zero_stats_kernel<<<grid_for(work, 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_encode(const IndexParams& p, int max_new, cudaStream_t stream) {
  if (max_new <= 0) return cudaSuccess;
  const dim3 grid(p.B * p.Hkv, (max_new + kEncTok - 1) / kEncTok);
  encode_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_accumulate(const IndexParams& p, int max_slots, cudaStream_t stream) {
  if (max_slots <= 0) return cudaSuccess;
  const dim3 grid(p.B * p.Hkv, (max_slots + 63) / 64);
  accumulate_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_list_reset(const IndexParams& p, cudaStream_t stream) {
  const size_t work = static_cast<size_t>(p.B) * p.Hkv * (2 + 2 * static_cast<size_t>(p.C));
  list_reset_kernel<<<grid_for(work, 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_list_append(const IndexParams& p, cudaStream_t stream) {
  const size_t smem = 6 * static_cast<size_t>(p.C) * sizeof(int32_t);
  cudaError_t e = ensure_dyn_smem<list_append_kernel>(smem);
  if (e != cudaSuccess) return e;
  list_append_kernel<<<p.B * p.Hkv, kListThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_means(const IndexParams& p, cudaStream_t stream) {
  const size_t work = static_cast<size_t>(p.B) * p.Hkv * p.C * kD;
  means_kernel<<<grid_for(work, 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_train_init(const TrainParams& p, cudaStream_t stream) {
  train_init_kernel<<<dim3(p.B * p.Hkv, (p.C + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_train_assign(const TrainParams& p, cudaStream_t stream) {
  train_assign_kernel<<<dim3(p.B * p.Hkv, (p.n_train + 31) / 32), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_train_accumulate(const TrainParams& p, cudaStream_t stream) {
  train_accumulate_kernel<<<dim3(p.B * p.Hkv, (p.n_train + 63) / 64), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// New centroids from the sums (clears sums and counts for the next iteration).
cudaError_t launch_train_update(const TrainParams& p, cudaStream_t stream) {
  const size_t n = static_cast<size_t>(p.B) * p.Hkv * p.C * kD;
  train_update_kernel<<<grid_for(n, 256), 256, 0, stream>>>(p.centroids, p.sums, p.counts, n, kD);
  const size_t nc = static_cast<size_t>(p.B) * p.Hkv * p.C;
  train_clear_counts_kernel<<<grid_for(nc, 256), 256, 0, stream>>>(p.counts, nc);
  return cudaGetLastError();
}

cudaError_t launch_train_pq_init(const TrainParams& p, cudaStream_t stream) {
  train_pq_init_kernel<<<dim3(p.B * p.Hkv, kM), kNcode, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_train_pq_step(const TrainParams& p, cudaStream_t stream) {
  static_assert(kM % kPqGroup == 0, "subspace groups must tile the subspaces");
  static_assert(kPqKeys % kPqKeyStride == 0, "a key block is whole loop rounds");
  cudaError_t e = ensure_dyn_smem<train_pq_step_kernel>(kPqSmemStep);
  if (e != cudaSuccess) return e;
  train_pq_step_kernel<<<dim3(p.B * p.Hkv, kM / kPqGroup, (p.n_train + kPqKeys - 1) / kPqKeys), kPqThreads,
                         kPqSmemStep, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_encode_codes(const TrainParams& p, uint8_t* codes, uint16_t* ids, int cap, cudaStream_t stream) {
  cudaError_t e = ensure_dyn_smem<encode_codes_kernel>(kPqSmemCodes);
  if (e != cudaSuccess) return e;
  encode_codes_kernel<<<dim3(p.B * p.Hkv, kM / kPqGroup, (p.n_train + kPqKeys - 1) / kPqKeys), kPqThreads,
                        kPqSmemCodes, stream>>>(p, codes, ids, cap);
  return cudaGetLastError();
}

// New codewords from the sums (clears sums and counts for the next iteration).
cudaError_t launch_train_pq_update(const TrainParams& p, cudaStream_t stream) {
  const size_t n = static_cast<size_t>(p.B) * p.Hkv * kM * kNcode * kDsub;
  train_update_kernel<<<grid_for(n, 256), 256, 0, stream>>>(p.codebooks, p.pq_sums, p.pq_counts, n, kDsub);
  const size_t nc = static_cast<size_t>(p.B) * p.Hkv * kM * kNcode;
  train_clear_counts_kernel<<<grid_for(nc, 256), 256, 0, stream>>>(p.pq_counts, nc);
  return cudaGetLastError();
}

}  // namespace pqhsa
