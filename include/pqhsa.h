/*
 * pqhsa.h - C ABI of a B200 (sm_100a) library for one decode step of PQ-HSA
 * sparse attention over a paged bf16 KV cache.
 *
 * Method: the rit.work article "pq-hsa-long-context-attention" (PQ-HSA),
 * section "Как приблизительные оценки возвращают отброшенный контекст":
 * an IVF-PQ index over the keys yields an approximate logit for every indexed
 * token; the top tokens under a read budget, plus the first tokens and a
 * recent window, are attended exactly from the KV cache; every other indexed
 * token stays in the softmax normalisation through its approximate logit, and
 * its value contribution is its cluster's summed weight times the cluster's
 * mean value. The index is built after prefill and new tokens are added to it
 * in batches. At full budget the same machinery is plain dense split-K GQA
 * decode (dense_decode), the in-library baseline.
 *
 * Conventions shared by every entry point
 * - Pointers are DEVICE pointers unless their name ends in _host (host memory).
 *   The caller owns all memory; the library allocates no device memory, keeps
 *   no state between calls, and touches only the buffers it is given - except
 *   where an entry point says otherwise: dense_decode_static's static scratch
 *   array, and a prepared decode step (hsa_decode_step_*), which holds a small
 *   host object, a private stream and a CUDA graph until it is destroyed.
 * - Every call validates its arguments on the host (from the *_host arrays)
 *   before any launch and returns a status; on an error nothing is launched.
 *   HSA_ERR_CUDA means a launch failed (the CUDA error is left pending).
 * - Work is enqueued on `stream` only; calls are asynchronous with respect to
 *   the host. The *_host arrays are read during the call (and, for
 *   hsa_append_encode, n_indexed_host is advanced by the call).
 * - Device-side faults never trap: an out-of-range block-table entry, cluster
 *   id or a timed-out wait is recorded in the workspace error word (see
 *   hsa_read_error) and the offending access is skipped.
 * - Workspaces must be 256-byte aligned and at least as large as the
 *   matching *_workspace_bytes() says. Their first 4 bytes are the device error
 *   word: it must be zero before the workspace's first use (allocate it zeroed,
 *   or clear those bytes once); calls only OR bits into it, and hsa_read_error
 *   reads and clears it. The rest of a workspace needs no initialisation and is
 *   clobbered by every call.
 *
 * KV cache layout (bf16): [num_pages][Hkv][page_size][D], so one head-page is
 * page_size contiguous 256-byte rows. Token t of sequence b lives in page
 * block_table[b * max_pages + t / page_size], slot t % page_size.
 *
 * Token sets of sequence b (T = seq_lens[b], s0 = n_sink, N = n_indexed[b]):
 *   sink S = [0, s0), indexed I = [s0, s0 + N), exact tail R = [s0 + N, T).
 * Index slot i of a (sequence, KV head) holds the code of position s0 + i.
 */
#ifndef PQHSA_H
#define PQHSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSA_OK = 0,
  HSA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent shapes */
  HSA_ERR_UNSUPPORTED = 2,   /* D != 128, M * dsub != D, dsub != 8, ncode != 256, G not in {1,2,4,8},
                                page_size not a power of two in [1, 128], C too large for shared memory */
  HSA_ERR_CAPACITY = 3,      /* index capacity or sequence length exceeded */
  HSA_ERR_ALIGNMENT = 4,     /* a pointer is not aligned as documented */
  HSA_ERR_WORKSPACE = 5,     /* workspace missing or smaller than required */
  HSA_ERR_CUDA = 6           /* a CUDA launch or query failed */
} hsa_status;

/* Paged KV cache view (read only). */
typedef struct {
  const void* k_cache;             /* bf16 [num_pages][Hkv][page_size][D], 256-B aligned */
  const void* v_cache;             /* same layout as k_cache */
  const int32_t* block_table;      /* [B][max_pages] page ids, each in [0, num_pages) */
  const int32_t* seq_lens;         /* [B] tokens in each sequence */
  const int32_t* seq_lens_host;    /* [B] host copy of seq_lens (used for planning/validation) */
  int32_t B, Hq, Hkv, D, page_size, max_pages, num_pages;
} hsa_kv_cache;

/* IVF-PQ index storage, one index per (sequence, KV head) "unit" u = b * Hkv + h. */
typedef struct {
  float* centroids;                /* fp32 [B][Hkv][C][D]            (caller fills; 16-B aligned) */
  float* codebooks;                /* fp32 [B][Hkv][M][ncode][dsub]  (caller fills; 16-B aligned) */
  uint8_t* codes;                  /* u8  [B][Hkv][cap][M]  residual PQ code of slot i */
  uint16_t* ids;                   /* u16 [B][Hkv][cap]     cluster of slot i, < C */
  float* sum_v;                    /* fp32 [B][Hkv][C][D]   sum of member values */
  float* mean_v;                   /* fp32 [B][Hkv][C][D]   mean member value (0 if empty); 16-B aligned */
  int32_t* count;                  /* [B][Hkv][C]           members per cluster */
  int32_t* n_indexed;              /* [B] indexed tokens per sequence (device) */
  int32_t* n_indexed_host;         /* [B] host copy of n_indexed */
  /* Cluster-ordered copy of the codes, kept by hsa_build_from_codes / hsa_append_encode
     and read by hsa_decode: the list slots of a unit form 32-slot chunks, each chunk
     holding members of one cluster (its last chunk may be partly empty). */
  uint8_t* list_codes;             /* u8  [B][Hkv][list_slots][M], 16-B aligned */
  int32_t* list_slot;              /* [B][Hkv][list_slots]  index slot of the member, -1 = empty;
                                      16-B aligned (both are streamed by bulk copies) */
  uint16_t* chunk_cluster;         /* [B][Hkv][list_slots / 32] cluster of each chunk; 4-B aligned */
  int32_t* list_meta;              /* [B][Hkv][2 + 2*C]: chunks in use, unused, then per cluster
                                      (its open chunk or -1, members in that chunk) */
  int32_t C, M, dsub, ncode, cap, n_sink;
  int32_t list_slots;              /* >= hsa_index_list_slots(cap, C) */
} hsa_index;

/* List capacity (slots per unit) an index of `cap` tokens and C clusters needs:
   32 * (ceil(cap / 32) + C). */
int64_t hsa_index_list_slots(int32_t cap, int32_t C);

typedef struct {
  float scale;                     /* logit scale, e.g. 1/sqrt(D) */
  double budget;                   /* k = floor(budget * N) selected tokens per unit */
  int32_t k_override;              /* >= 0: use min(k_override, N) instead of the budget */
  int32_t background;              /* 1: PQ-HSA (unselected tokens enter through the
                                      cluster background); 0: plain top-k sparse attention */
} hsa_decode_params;

/* Optional debug outputs of hsa_decode (any member may be NULL). */
typedef struct {
  float* approx_logits;            /* fp32 [B][Hq][cap]: approximate logit of slot i (scaled) */
  int32_t* selected;               /* [B][Hkv][cap]: selected token positions, ascending */
  int32_t* n_selected;             /* [B][Hkv]: number of selected tokens */
  cudaEvent_t* stage_events;       /* NULL, or HSA_STAGE_EVENTS events recorded on `stream`
                                      before each stage and after the last one */
} hsa_debug;

/* Stages of hsa_decode, in launch order: tables, scan+selection, exact+background
   attention, merge. stage_events[i] precedes stage i. */
#define HSA_NUM_STAGES 4
#define HSA_STAGE_EVENTS (HSA_NUM_STAGES + 1)

/* ---- decode -------------------------------------------------------------- */

/* Workspace bytes hsa_decode needs for these shapes (0 on invalid arguments). */
size_t hsa_decode_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* index);

/*
 * One PQ-HSA decode step (rit.work "pq-hsa-long-context-attention", section
 * "Как приблизительные оценки возвращают отброшенный контекст").
 * q: fp32 [B][Hq][D]; out: fp32 [B][Hq][D]; both 16-B aligned. For every unit:
 *   shat_gj = scale * (q_g . centroid_{a_j} + sum_s q_g,s . codeword_s[code_js]) for j in I;
 *   K = the k slots of largest max_g shat_gj (ties to the smaller position),
 *       k = floor(budget * N) computed in double;
 *   out_g = (sum_{j in S+K+R} e^{s_gj} v_j + sum_c W_gc mean_v_c)
 *           / (sum_{j in S+K+R} e^{s_gj} + sum_{j in I\K} e^{shat_gj}),
 *   s_gj = scale * q_g . k_j,  W_gc = sum_{j in I\K, a_j = c} e^{shat_gj}.
 * Needs mean_v consistent with the index (hsa_build_from_codes / hsa_append_encode).
 * A unit with N = 0 is dense attention over [0, T).
 */
hsa_status hsa_decode(const hsa_kv_cache* kv, const hsa_index* index, const float* q, float* out,
                      const hsa_decode_params* params, const hsa_debug* debug,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes hsa_decode_host needs: hsa_decode's (first, 256-byte aligned), then
   device room for q and for out (fp32 [B][Hq][D] each, 256-byte aligned). 0 on invalid
   arguments. */
size_t hsa_decode_host_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* index);

/*
 * hsa_decode with q and out in host memory, for callers whose query and result live
 * on the host. On `stream`: q_host is brought into the workspace, the decode step runs
 * (as hsa_decode, without debug outputs), and the result goes to out_host. Page-locked
 * (device-addressable) buffers are read by a copy kernel and written by the last kernel
 * of the step directly; pageable ones take one cudaMemcpyAsync each way.
 * q_host, out_host: fp32 [B][Hq][D] host memory, caller-owned. Returns once all of it
 * is queued; out_host holds the result when `stream` reaches the end of this call
 * (synchronise the stream or an event recorded after it before reading). Arguments
 * are checked before anything is queued; status, workspace and error word otherwise
 * as for hsa_decode.
 */
hsa_status hsa_decode_host(const hsa_kv_cache* kv, const hsa_index* index, const float* q_host, float* out_host,
                           const hsa_decode_params* params, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* ---- prepared decode step (graph replay) --------------------------------- */

/* A decode step prepared for one cache, index, parameter set and workspace (opaque), for
   decode loops: each run replays a recorded CUDA graph of the step while its launch shape
   and buffers stay the same. */
typedef struct hsa_decode_step hsa_decode_step;

/*
 * Prepare hsa_decode_host for a decode loop. Copies the cache and index views and the
 * parameters, not the arrays they point to: those stay caller-owned, must outlive the
 * step, and may change in place between runs (lengths, appends, lists). The workspace
 * must hold hsa_decode_host_workspace_bytes. Validates as hsa_decode_host does and makes
 * no CUDA call. *step receives the handle, or NULL on error (HSA_ERR_CUDA also when the
 * step's host memory cannot be allocated).
 */
hsa_status hsa_decode_step_create(const hsa_kv_cache* kv, const hsa_index* index, const hsa_decode_params* params,
                                  void* workspace, size_t workspace_bytes, hsa_decode_step** step);

/*
 * One decode step, queued on `stream` as one CUDA graph launch. q, out: fp32 [B][Hq][D],
 * both page-locked host memory (the step is hsa_decode_host's) or both device memory
 * (hsa_decode's, 16-B aligned); anything else, pageable host memory included, is
 * HSA_ERR_INVALID_ARG. Every run validates the views and the current lengths again and
 * recomputes the split-K plan of the exact part (the only launch shape that depends on
 * host-side values). While that plan, q and out are those of the previous run, the run
 * replays the previous run's graph; otherwise (the first run, lengths that moved the plan,
 * other buffers) it records the step on a private stream of the step and updates the
 * graph. Result and error word as for hsa_decode_host / hsa_decode. One thread at a time
 * per step; runs of steps that share a workspace must not overlap.
 */
hsa_status hsa_decode_step_run(hsa_decode_step* step, const float* q, float* out, cudaStream_t stream);

/* Release a step (its graph and private stream). NULL is ignored. It does not wait:
   let the step's queued work finish before the arrays it reads are freed. */
void hsa_decode_step_destroy(hsa_decode_step* step);

/* Workspace bytes dense_decode needs. */
size_t dense_decode_workspace_bytes(const hsa_kv_cache* kv);

/*
 * Dense split-K GQA decode: out_g = softmax(scale * q_g K^T) V over all T tokens of
 * each sequence. q, out: fp32 [B][Hq][D] (16-B aligned); the workspace as
 * dense_decode_workspace_bytes says (its error word as for hsa_decode).
 * The in-library baseline that PQ-HSA is measured against. The rit.work article
 * "activation-kv-cache-sparsity-crossover", section "Почему один и тот же способ
 * даёт разное ускорение", asks that dense and sparse decode read the cache through
 * the same split-K kernel, so that a measured speed-up reflects the data saved and
 * not a change of attention kernel: this call runs the same split-K engine (same
 * tiles, same tensor-core consumers, same merge) as the exact part of hsa_decode.
 */
hsa_status dense_decode(const hsa_kv_cache* kv, const float* q, float* out, float scale,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * dense_decode_static: dense_decode that allocates nothing and takes no workspace.
 * The PQ-HSA article has no counterpart to this call. It serves callers that cannot
 * obtain device memory when they decode: a plain host program with no device
 * allocator of its own, a serving runtime whose memory pool is fixed before traffic
 * starts, or a decode loop that must never call cudaMalloc (an allocation there can
 * stall or fail at the worst moment). Arguments and result are those of dense_decode.
 * - Scratch: a static 8 MiB device array inside this library, reserved on every GPU
 *   that loads the library until the process exits.
 * - The first call on a device looks up that array's device address (once per
 *   device, with that device current). Make that first call before any stream capture.
 * - Limit: the split-K partials need B*Hkv*G*520 bytes per chunk; shapes for which
 *   even one chunk does not fit in 8 MiB (B*Hkv*G above about 16000) return
 *   HSA_ERR_WORKSPACE; otherwise the number of chunks is capped to fit.
 * - Every call uses the same array and rewrites what it reads (nothing has to start
 *   at zero; the array keeps the last call's partials). Calls that overlap on the
 *   GPU (other streams or threads) race on it: serialise them.
 * - There is no error word: out-of-range block-table entries are skipped and a wait
 *   that gives up (after 2 s) ends the call's copies early; neither is reported, and
 *   in the second case the output is wrong. Callers that need these reported use
 *   dense_decode with a workspace.
 */
hsa_status dense_decode_static(const hsa_kv_cache* kv, const float* q, float* out, float scale,
                               cudaStream_t stream);

/* ---- index maintenance --------------------------------------------------- */

/* Workspace bytes of hsa_append_encode of n_new tokens (n_new = 0: of
 * hsa_build_from_codes, the error word only). With pages of at least 8 rows the
 * encoding's nearest-centroid search runs on the tensor cores and the workspace also
 * holds the centroids as bf16 terms [B*Hkv][3][C rounded up to 256][128], their squared
 * norms and the new tokens' assignment [B*Hkv][n_new]. Never 0. */
size_t hsa_index_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* index, int32_t n_new);

/*
 * Index build after prefill from caller-provided codes (same article, section
 * above: "after the prompt is filled the index is built"). The caller fills
 * centroids, codebooks, codes and ids for slots [0, n_indexed[b]); this call
 * computes count, sum_v and mean_v of every cluster from the value rows of the
 * indexed tokens, and builds the cluster-ordered lists read by hsa_decode.
 */
hsa_status hsa_build_from_codes(const hsa_kv_cache* kv, hsa_index* index,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Batched encoding of new tokens into the index (same article: new tokens are
 * kept outside the index and added in batches). For every sequence b and KV
 * head, positions [s0 + N_b, s0 + N_b + n_new) are encoded:
 *   a = argmin_c sum_d (k_d - centroid_c,d)^2 (ties to the lower c),
 *   code_s = argmin_m sum_{d<dsub} (k - centroid_a)_{s*dsub+d} - codeword_s,m,d)^2
 *   (ties to the lower m). The decisions are taken in fp32: with pages of at least 8
 *   rows as |c|^2 - 2 k.c on the tensor cores (centroids as three bf16 terms, fp32
 *   accumulation) and |w|^2 - 2 r.w for the codewords; results can differ from an
 *   exact evaluation only where two candidates' distances nearly tie.
 * written to slots [N_b, N_b + n_new); the members' values are added to sum_v
 * and count, mean_v is recomputed, the new members join their clusters' lists
 * (list_codes / list_slot), and n_indexed (device and host) grows by n_new.
 * Requires s0 + N_b + n_new <= seq_lens_host[b] and N_b + n_new <= cap, and
 * lists built by earlier calls (a unit with n_indexed = 0 starts them afresh).
 * With n_indexed = 0 this is the whole index build from raw keys. The workspace is
 * hsa_index_workspace_bytes(kv, index, n_new) bytes.
 */
hsa_status hsa_append_encode(const hsa_kv_cache* kv, hsa_index* index, int32_t n_new,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * hsa_train_index: trains the index's centroids and codebooks on raw keys, the step
 * before hsa_append_encode when no trained index exists (rit.work PQ-HSA article,
 * section "Как приблизительные оценки возвращают отброшенный контекст": the index
 * is built after prefill; how its groups and codes are found is left open, and this
 * is the plain Lloyd k-means).
 *
 * For every sequence b and KV head the training set is the keys at positions
 * [s0, s0 + n_train) (training slot j = position s0 + j):
 *   centroids: start at the keys of slots init_slots[0 .. C); coarse_iters times
 *     assign every key to its nearest centroid (squared Euclidean distance, ties to
 *     the lower index) and move each centroid to the mean of its keys (a centroid
 *     with no keys keeps its value); then assign once more;
 *   codebook s: start at the subspace-s residuals (key - centroid of its final
 *     assignment) of slots init_slots[C + s*ncode .. C + (s+1)*ncode); pq_iters times
 *     the same assign/move on the residuals' subspace s.
 * Decisions are taken in fp32: with pages of at least 8 rows the nearest centroid
 *   minimises |c|^2 - 2 k.c with k.c on the tensor cores (each centroid as three bf16
 *   terms, fp32 accumulation; 4-row pages: direct fp32 sums of squared differences),
 *   the nearest codeword minimises |w|^2 - 2 r.w; the means are fp32 sums (atomics,
 *   so the last bits depend on the order of addition).
 * init_slots: device int32 [B][Hkv][C + M*ncode], each in [0, n_train) (the caller
 *   draws them; an out-of-range slot is replaced by 0 and flagged HSA_DEVERR_SLOT).
 * assign_out: NULL, or device int32 [B][Hkv][n_train] receiving the final coarse
 *   assignment. Writes index->centroids and index->codebooks only.
 * Requires 1 <= n_train <= 2097120, s0 + n_train <= seq_lens_host[b], M = 16, dsub = 8,
 * ncode = 256, C <= 4096, 0 <= iterations <= 1000; the workspace as
 * hsa_train_workspace_bytes says (its error word is read by hsa_read_error).
 */
size_t hsa_train_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* index, int32_t n_train);
hsa_status hsa_train_index(const hsa_kv_cache* kv, hsa_index* index, int32_t n_train,
                           const int32_t* init_slots, int32_t coarse_iters, int32_t pq_iters,
                           int32_t* assign_out, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* ---- diagnostics --------------------------------------------------------- */

/* Human-readable name of a status. */
const char* hsa_strerror(hsa_status status);

/*
 * Copies the workspace error word (0 = none; otherwise a HSA_DEVERR_* bit set)
 * to *error_host and clears it. Synchronises `stream`.
 */
hsa_status hsa_read_error(void* workspace, int32_t* error_host, cudaStream_t stream);

#define HSA_DEVERR_PAGE 1          /* block-table entry outside [0, num_pages) */
#define HSA_DEVERR_CLUSTER 2       /* cluster id >= C */
#define HSA_DEVERR_TIMEOUT 4       /* a bounded wait gave up */
#define HSA_DEVERR_SELECT 8        /* top-k bookkeeping inconsistent */
#define HSA_DEVERR_SLOT 16         /* a training slot outside [0, n_train) */

/* ABI self-description: sizeof of the public structs, for bindings to check. */
void hsa_abi_sizes(int64_t* kv_cache, int64_t* index, int64_t* decode_params, int64_t* debug);

#ifdef __cplusplus
}
#endif

#endif /* PQHSA_H */
