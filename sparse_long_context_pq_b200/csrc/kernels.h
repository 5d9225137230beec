// Internal launch interfaces between the C-ABI host code and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace pqhsa {

// Upper/lower bound of the (scaled) approximate logit of every head of unit u:
//   ub_g = sum_s max_m LUT_s[m][g] + max_c qc[c][g],  lb_g likewise with min.
// The table builder leaves partial extremes in `bounds`, layout
// [U][kLutParts + nq][2 (max, min)][4 * GP]: parts 0..kLutParts-1 hold partial sums over
// their subspaces of the per-subspace extremes, parts kLutParts.. the extremes of one
// kQcSlice-cluster slice of the centroid term. The scan reduces them once per unit (one
// warp) into the final bounds `fbounds` [U][2][G] that every later kernel reads.
template <int G>
__device__ __forceinline__ void reduce_bounds_warp(const float* bounds, int u, int nq, float* ub, float* lb) {
  constexpr int G4 = ((G + 3) / 4) * 4;
  const int lane = threadIdx.x & 31;
  const float* bu = bounds + static_cast<size_t>(u) * (kLutParts + nq) * 2 * G4;
  // one head at a time (few live registers); lane l takes centroid slices l, l + 32, ...
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    float qmax = -INFINITY, qmin = INFINITY;
    for (int sl = lane; sl < nq; sl += 32) {
      qmax = fmaxf(qmax, bu[((kLutParts + sl) * 2 + 0) * G4 + g]);
      qmin = fminf(qmin, bu[((kLutParts + sl) * 2 + 1) * G4 + g]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
      qmin = fminf(qmin, __shfl_xor_sync(0xffffffffu, qmin, o));
    }
    float smax = 0.f, smin = 0.f;
#pragma unroll
    for (int part = 0; part < kLutParts; ++part) {   // fixed order: the same sums in every CTA
      smax += bu[(part * 2 + 0) * G4 + g];
      smin += bu[(part * 2 + 1) * G4 + g];
    }
    if (lane == 0) {
      ub[g] = smax + qmax;
      lb[g] = smin + qmin;
    }
  }
}
// Final bounds of unit u as the scan stored them.
template <int G>
__device__ __forceinline__ void final_bounds(const float* fbounds, int u, float* ub, float* lb) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    ub[g] = fbounds[(static_cast<size_t>(u) * 2 + 0) * G + g];
    lb[g] = fbounds[(static_cast<size_t>(u) * 2 + 1) * G + g];
  }
}

struct AttendParams {
  const uint8_t* k_cache;    // bf16 rows (row-gather modes)
  const uint8_t* v_cache;
  const float* q;            // [B][Hq][D]
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* n_indexed;  // exact mode
  const int32_t* sel;        // exact mode: [U][cap] KV-pool rows of the selected tokens
  const UnitState* units;    // exact mode: per-unit ready flags set by the selection
  int32_t* err;
  float* pm;                 // [U][S_tot][G]
  float* pl;
  float* pacc;               // [U][S_tot][G][D]
  // background (exact mode)
  const float* W;            // [U][G][C]
  const float* mean_v;       // [U][C][D]
  const float* bounds;
  const float* fbounds;      // [U][2][G] final (ub, lb) from the scan
  int U, B, Hq, Hkv, page_size, max_pages, num_pages, cap, n_sink;
  int nsplit, chunk, S_tot, C, nbg, nq, bg_enabled, k_override;
  double budget;
  float qscale;              // scale * log2(e)
};

struct MergeParams {
  const float* pm;
  const float* pl;
  const float* pacc;
  float* out;
  int B, Hq, Hkv, S_tot;
};

template <int G>
__device__ void background_block(const AttendParams& p, int j, uint8_t* smem);

// Host-side helpers shared by the entry points (api.cu).
hsa_status check_kv(const hsa_kv_cache* kv);   // shapes, alignment and lengths of a KV-cache view
// Tensor map over a paged cache viewed as rows of D bf16, box = 64 columns x box_rows rows.
bool make_kv_tmap(CUtensorMap* map, const void* base, const hsa_kv_cache* kv, int box_rows);

int attend_slots_per_sm(int G, bool exact, bool rows);   // resident attend CTAs per SM
// Row sources: kExact = sink + selected + tail list of hsa_decode, else every token.
// Loading: page tiles by tensor TMA (dense, page_size >= 8) or 16-byte async copies per row.
// wide: the grid holds more CTAs than two per SM (the exact part of G <= 4 then runs three).
cudaError_t launch_attend(int G, bool exact, bool rows, const CUtensorMap& tk, const CUtensorMap& tv,
                          const AttendParams& p, int grid, bool wide, cudaStream_t stream, bool pdl);
cudaError_t launch_merge(int G, const MergeParams& p, cudaStream_t stream, bool pdl);

// ---- PQ tables, scan, top-k ------------------------------------------------
struct TablesParams {
  const float* q;            // [B][Hq][D]
  const float* centroids;    // [U][C][D]
  const float* codebooks;    // [U][M][256][8]
  float* lut;                // [U][GP][256][16][4]
  float* qc;                 // [U][GP][C][4]
  float* bounds;
  float* W;                  // [U][G][C] zeroed here
  uint32_t* hist;            // [U][NB] zeroed here
  uint32_t* bitmap;          // [U][bitmap_words] zeroed here
  UnitState* units;          // zeroed here
  int B, Hq, Hkv, C, nq, bitmap_words;
  float scale;
  // 1: the codebooks and centroids may be read before the dependency wait (the previous
  // kernel is the q staging of a host-buffer step, which itself follows every earlier one)
  int index_early;
};
cudaError_t launch_tables(int G, const TablesParams& p, cudaStream_t stream, bool pdl);

// One launch after the tables: the scan of the codes (phase 1), then, per unit, the
// selection (phase 2: threshold bin from the unit's histogram; over this CTA's share of
// the unit's chunks, the definite selections' rows, the threshold-bin candidates and the
// weight fix-ups) and its resolution by the part that completes the unit's count (phase
// 3: exact order of the candidates, the winners' rows and fix-ups, ready flag).
struct StepParams {
  const uint8_t* list_codes;     // [U][list_slots][16] cluster-ordered codes
  const int32_t* list_slot;      // [U][list_slots] index slot of each list slot (-1 empty)
  const uint16_t* chunk_cluster; // [U][list_slots / 32]
  const int32_t* list_meta;      // [U][2 + 2C]; [0] = chunks in use
  int list_slots;
  const int32_t* seq_lens;
  const int32_t* n_indexed;
  const uint8_t* codes;          // [U][cap][16] (weights of winners past the stored candidates)
  const uint16_t* ids;           // [U][cap]
  const float* lut;
  const float* qc;
  const float* bounds;
  float* fbounds;                // [U][2][G] final (ub, lb), written by the scan
  float* W;
  uint32_t* hist;
  float* sigma;                  // [U][list_slots]
  float* chunk_max;              // [U][list_slots / 32] largest sigma of each chunk
  uint32_t* bitmap;              // [U][bitmap_words] selected index slots
  unsigned long long* cand;      // [U][cap] threshold-bin candidates (score key, slot)
  float* cand_w;                 // [U][kCandWeights][G] e^{shat_g - ub_g} of the first candidates
  int32_t* cand_c;               // [U][kCandWeights] their clusters
  int32_t* cand_row;             // [U][cap] KV-pool row of each candidate
  UnitState* units;
  int32_t* sel;                  // [U][cap] KV-pool row of each selected token, ascending position
  const int32_t* block_table;    // [B][max_pages]
  int page_size, max_pages, num_pages;
  float* approx_logits;          // debug [B][Hq][cap] or null
  int32_t* dbg_selected;         // [U][cap] or null (positions)
  int32_t* dbg_nselected;        // [U] or null
  int32_t* err;
  int B, Hq, Hkv, cap, C, nq, n_sink, bitmap_words, k_override, background;
  int ring_depth;                // chunk slots per warp (scan_ring_depth)
  double budget;
};
cudaError_t launch_scan_select(int G, const StepParams& p, int grid, cudaStream_t stream, bool pdl);
int scan_ring_depth(int G, int C);   // 0: the tables do not fit in shared memory
size_t scan_smem_bytes(int G, int C);

// ---- index maintenance -----------------------------------------------------
struct IndexParams {
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const float* centroids;
  const float* codebooks;
  uint8_t* codes;
  uint16_t* ids;
  float* sum_v;
  float* mean_v;
  int32_t* count;
  int32_t* n_indexed;
  int32_t* err;
  // cluster-ordered lists
  uint8_t* list_codes;       // [U][list_slots][16]
  int32_t* list_slot;        // [U][list_slots]
  uint16_t* chunk_cluster;   // [U][list_slots / 32]
  int32_t* list_meta;        // [U][2 + 2C]
  int B, Hkv, page_size, max_pages, num_pages, C, cap, n_sink, list_slots;
  int slot_lo_from_indexed;  // 1: slots start at n_indexed[b]; 0: slots start at 0
  int n_slots;               // slots per unit to process (n_new), or -1 = n_indexed[b]
  int bump_indexed;          // add n_slots to n_indexed[b] in the mean pass
  int zero_if_empty;         // zero stats of units whose sequence has n_indexed == 0
};
cudaError_t launch_zero_stats(const IndexParams& p, cudaStream_t stream);
cudaError_t launch_encode(const IndexParams& p, int max_new, cudaStream_t stream);
cudaError_t launch_accumulate(const IndexParams& p, int max_slots, cudaStream_t stream);
cudaError_t launch_means(const IndexParams& p, cudaStream_t stream);
cudaError_t launch_list_reset(const IndexParams& p, cudaStream_t stream);
cudaError_t launch_list_append(const IndexParams& p, cudaStream_t stream);

// ---- index training (k-means centroids, residual PQ codebooks) --------------
struct TrainParams {
  const uint16_t* k_cache;
  const int32_t* block_table;
  float* centroids;            // [U][C][D] written
  float* codebooks;            // [U][M][ncode][dsub] written
  const int32_t* init_slots;   // [U][C + M * ncode] training slots seeding the centres
  int32_t* assign;             // [U][n_train] coarse assignment (workspace)
  int32_t* assign_out;         // [U][n_train] final coarse assignment, or null
  float* sums;                 // [U][C][D]
  int32_t* counts;             // [U][C]
  float* pq_sums;              // [U][M][ncode][dsub]
  int32_t* pq_counts;          // [U][M][ncode]
  int32_t* err;
  uint16_t* terms;             // [U][3][Cpad][D] bf16 terms of the centroids (tensor-core assignment)
  float* cnorm;                // [U][Cpad] |c|^2, +inf for the padding rows
  int B, Hkv, C, n_sink, n_train, page_size, max_pages, num_pages;
  const int32_t* slot0;        // [B] first slot of each sequence's keys (null: 0), as for encoding
  int Cpad;                    // C rounded up to the 256-centroid tile
  int tiles_per_unit, items;   // 128-key tiles per unit, units x tiles
};
cudaError_t launch_train_init(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_assign(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_accumulate(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_update(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_pq_init(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_pq_step(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_train_pq_update(const TrainParams& p, cudaStream_t stream);
size_t assign_mma_smem_bytes();
cudaError_t launch_centroid_terms(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_encode_codes(const TrainParams& p, uint8_t* codes, uint16_t* ids, int cap, cudaStream_t stream);
cudaError_t launch_assign_mma(const CUtensorMap& tmk, const CUtensorMap& tmb, const TrainParams& p, int grid,
                              cudaStream_t stream);

}  // namespace pqhsa
