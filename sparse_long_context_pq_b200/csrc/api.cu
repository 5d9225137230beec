// Host side of the C ABI declared in include/pqhsa.h: argument validation,
// workspace layout, split planning and kernel launches. No allocation, no
// state across calls beyond a per-device cache of immutable properties.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <dlfcn.h>
#include <stdint.h>

#include <algorithm>
#include <cstdlib>
#include <cmath>
#include <mutex>
#include <new>

#include "../../include/pqhsa.h"
#include "common.cuh"
#include "kernels.h"

using namespace pqhsa;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 148;
  int scan_ctas_per_sm[9] = {0};
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
bool g_encode_tried = false;

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    d.sms = sms;
    d.ready = true;
  }
  return &d;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode_tried) {
    g_encode_tried = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn) {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    } else if (void* h = dlopen("libcuda.so.1", RTLD_NOW | RTLD_LOCAL)) {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(dlsym(h, "cuTensorMapEncodeTiled"));
    }
  }
  return g_encode;
}

// Programmatic dependent launch between the kernels of a call (and with the
// previous call): every kernel waits on griddepcontrol before touching memory a
// predecessor writes. PQHSA_NO_PDL=1 turns it off.
bool use_pdl() {
  static const bool on = [] {
    const char* e = getenv("PQHSA_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

}  // namespace

namespace pqhsa {

// Tensor map over a paged cache viewed as rows of D bf16: [num_pages*Hkv*page_size][128],
// box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_kv_tmap(CUtensorMap* map, const void* base, const hsa_kv_cache* kv, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD),
                        static_cast<cuuint64_t>(kv->num_pages) * kv->Hkv * kv->page_size};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Validation of a KV-cache view shared by every entry point that reads the cache.
hsa_status check_kv(const hsa_kv_cache* kv) {
  if (!kv || !kv->k_cache || !kv->v_cache || !kv->block_table || !kv->seq_lens || !kv->seq_lens_host)
    return HSA_ERR_INVALID_ARG;
  if (kv->B < 1 || kv->Hkv < 1 || kv->Hq < 1 || kv->max_pages < 1 || kv->num_pages < 1) return HSA_ERR_INVALID_ARG;
  if (kv->Hq % kv->Hkv) return HSA_ERR_INVALID_ARG;
  const int G = kv->Hq / kv->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return HSA_ERR_UNSUPPORTED;
  if (kv->D != kD) return HSA_ERR_UNSUPPORTED;
  if (!pow2(kv->page_size) || kv->page_size > 128) return HSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(kv->num_pages) * kv->Hkv * kv->page_size >= (1LL << 31)) return HSA_ERR_UNSUPPORTED;
  if (!aligned(kv->k_cache, 256) || !aligned(kv->v_cache, 256) || !aligned(kv->block_table, 4) ||
      !aligned(kv->seq_lens, 4))
    return HSA_ERR_ALIGNMENT;
  const long long tmax = static_cast<long long>(kv->max_pages) * kv->page_size;
  for (int b = 0; b < kv->B; ++b)
    if (kv->seq_lens_host[b] < 0 || kv->seq_lens_host[b] > tmax) return HSA_ERR_CAPACITY;
  return HSA_OK;
}

}  // namespace pqhsa

namespace {

hsa_status check_index(const hsa_kv_cache* kv, const hsa_index* ix, bool need_codes) {
  if (!ix || !ix->centroids || !ix->codebooks || !ix->ids || !ix->mean_v || !ix->n_indexed || !ix->n_indexed_host)
    return HSA_ERR_INVALID_ARG;
  if (need_codes && !ix->codes) return HSA_ERR_INVALID_ARG;
  if (ix->M != kM || ix->dsub != kDsub || ix->ncode != kNcode || ix->M * ix->dsub != kv->D) return HSA_ERR_UNSUPPORTED;
  if (ix->C < 1 || ix->C > 65535 || ix->cap < 1 || ix->n_sink < 0) return HSA_ERR_INVALID_ARG;
  if (!aligned(ix->centroids, 16) || !aligned(ix->codebooks, 16) || !aligned(ix->mean_v, 16) ||
      (ix->codes && !aligned(ix->codes, 16)) || !aligned(ix->ids, 2))
    return HSA_ERR_ALIGNMENT;
  // cluster-ordered lists
  if (!ix->list_codes || !ix->list_slot || !ix->chunk_cluster || !ix->list_meta) return HSA_ERR_INVALID_ARG;
  if (ix->C > kMaxClusters) return HSA_ERR_UNSUPPORTED;
  if (ix->list_slots < list_slots_needed(ix->cap, ix->C) || ix->list_slots % 32) return HSA_ERR_CAPACITY;
  if (!aligned(ix->list_codes, 16) || !aligned(ix->list_slot, 16) || !aligned(ix->list_meta, 4) ||
      !aligned(ix->chunk_cluster, 4))
    return HSA_ERR_ALIGNMENT;
  for (int b = 0; b < kv->B; ++b) {
    const int T = kv->seq_lens_host[b];
    const int n = ix->n_indexed_host[b];
    if (n < 0) return HSA_ERR_INVALID_ARG;
    if (n > ix->cap) return HSA_ERR_CAPACITY;
    if (n > 0 && ix->n_sink + n > T) return HSA_ERR_CAPACITY;
  }
  return HSA_OK;
}

int host_unit_n(const hsa_kv_cache* kv, const hsa_index* ix, int b) {
  const int T = std::max(0, kv->seq_lens_host[b]);
  const int s0 = std::min(ix->n_sink, T);
  const int N = std::max(0, std::min(ix->n_indexed_host[b], T - s0));
  return std::min(N, ix->cap);
}

struct Split {
  int nsplit;
  int chunk;
};

// Choose the split-K chunking of E_max rows per unit: minimise (waves of CTAs) x (rows per CTA).
Split plan_splits(long long E_max, int U, int nbg, int slots) {
  Split best{1, static_cast<int>(std::max<long long>(kTile, (E_max + kTile - 1) / kTile * kTile))};
  if (E_max <= 0) return Split{1, kTile};
  double best_cost = 1e300;
  for (int ns = 1; ns <= kMaxSplits; ++ns) {
    long long chunk = (E_max + ns - 1) / ns;
    chunk = (chunk + kTile - 1) / kTile * kTile;
    const int ns_eff = static_cast<int>((E_max + chunk - 1) / chunk);
    const long long ctas = static_cast<long long>(U) * (ns_eff + nbg);
    const long long waves = (ctas + slots - 1) / slots;
    const double per_cta = std::max<double>(static_cast<double>(chunk), nbg ? kBgClusters : 0.0) + 96.0;
    const double cost = static_cast<double>(waves) * per_cta + 2.0 * ns_eff;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = Split{ns_eff, static_cast<int>(chunk)};
    }
  }
  return best;
}

// Split-K plan of hsa_decode's exact part for the current lengths: the longest unit's
// sink + selected + tail rows over the units' splits (the only launch shape that depends
// on host-side values).
Split decode_split_plan(const hsa_kv_cache* kv, const hsa_index* ix, const hsa_decode_params* prm, int nbg,
                        int sms) {
  long long Emax = 0;
  for (int b = 0; b < kv->B; ++b) {
    const int T = std::max(0, kv->seq_lens_host[b]);
    const int s0 = std::min(ix->n_sink, T);
    const int N = host_unit_n(kv, ix, b);
    const int k = decode_k(prm->budget, prm->k_override, N);
    Emax = std::max<long long>(Emax, static_cast<long long>(s0) + k + (T - s0 - N));
  }
  const int G = kv->Hq / kv->Hkv;
  return plan_splits(Emax, kv->B * kv->Hkv, nbg, sms * attend_slots_per_sm(G, true, true));
}

// q of hsa_decode_host from page-locked host memory (device-addressable) into the
// workspace: one 16-byte load and store per thread, so the step's many CTAs read q from
// device memory rather than each across the host link.
__global__ void __launch_bounds__(256) stage_q_kernel(const float4* __restrict__ src, float4* __restrict__ dst,
                                                      int n4) {
  pdl_launch_dependents();   // the tables kernel may start its index loads meanwhile
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x) dst[i] = src[i];
}

// Where a buffer of the prepared step lives: 1 page-locked host memory, 2 device (or
// managed) memory, 0 anything else (pageable host memory, an unknown pointer).
int buffer_kind(const void* p) {
  cudaPointerAttributes a = {};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  if (a.type == cudaMemoryTypeHost) return a.devicePointer ? 1 : 0;
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) ? 2 : 0;
}

// Device address of page-locked host memory (nullptr for pageable memory).
void* mapped_host_pointer(const void* p) {
  cudaPointerAttributes a = {};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

// Device room for q (or out) of hsa_decode_host at the end of its workspace.
size_t host_io_bytes(const hsa_kv_cache* kv) {
  return align_up(static_cast<size_t>(kv->B) * kv->Hq * kD * sizeof(float), 256);
}

size_t dense_layout_bytes(int U, int G) {
  const size_t parts = static_cast<size_t>(U) * kMaxSplits * G;
  size_t o = align_up(sizeof(WsHeader), 256);
  o += align_up(parts * sizeof(float), 256) * 2;
  o += align_up(parts * kD * sizeof(float), 256);
  return o;
}

#define RET_CUDA(x)                         \
  do {                                      \
    if ((x) != cudaSuccess) return HSA_ERR_CUDA; \
  } while (0)

}  // namespace

extern "C" {

const char* hsa_strerror(hsa_status s) {
  switch (s) {
    case HSA_OK: return "ok";
    case HSA_ERR_INVALID_ARG: return "invalid argument";
    case HSA_ERR_UNSUPPORTED: return "unsupported shape";
    case HSA_ERR_CAPACITY: return "capacity exceeded";
    case HSA_ERR_ALIGNMENT: return "misaligned pointer";
    case HSA_ERR_WORKSPACE: return "workspace too small";
    case HSA_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

void hsa_abi_sizes(int64_t* a, int64_t* b, int64_t* c, int64_t* d) {
  if (a) *a = sizeof(hsa_kv_cache);
  if (b) *b = sizeof(hsa_index);
  if (c) *c = sizeof(hsa_decode_params);
  if (d) *d = sizeof(hsa_debug);
}

size_t hsa_decode_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* ix) {
  if (check_kv(kv) != HSA_OK || !ix || ix->C < 1 || ix->cap < 1) return 0;
  if (ix->list_slots < 32) return 0;
  const DecodeLayout L =
      make_decode_layout(kv->B * kv->Hkv, kv->Hq / kv->Hkv, ix->C, ix->cap, ix->list_slots, kMaxSplits);
  return L.total;
}

size_t hsa_decode_host_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* ix) {
  const size_t base = hsa_decode_workspace_bytes(kv, ix);
  if (base == 0) return 0;
  return align_up(base, 256) + 2 * host_io_bytes(kv);
}

size_t dense_decode_workspace_bytes(const hsa_kv_cache* kv) {
  if (check_kv(kv) != HSA_OK) return 0;
  return dense_layout_bytes(kv->B * kv->Hkv, kv->Hq / kv->Hkv);
}



int64_t hsa_index_list_slots(int32_t cap, int32_t C) {
  if (cap < 1 || C < 1) return 0;
  return list_slots_needed(cap, C);
}

hsa_status hsa_read_error(void* ws, int32_t* error_host, cudaStream_t stream) {
  if (!ws || !error_host) return HSA_ERR_INVALID_ARG;
  RET_CUDA(cudaMemcpyAsync(error_host, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
  RET_CUDA(cudaMemsetAsync(ws, 0, sizeof(int32_t), stream));
  RET_CUDA(cudaStreamSynchronize(stream));
  return HSA_OK;
}

hsa_status dense_decode(const hsa_kv_cache* kv, const float* q, float* out, float scale, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  if (!q || !out) return HSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return HSA_ERR_ALIGNMENT;
  const int U = kv->B * kv->Hkv, G = kv->Hq / kv->Hkv;
  if (!ws || !aligned(ws, 256) || ws_bytes < dense_layout_bytes(U, G)) return HSA_ERR_WORKSPACE;
  const DeviceInfo* dev = device_info();
  if (!dev) return HSA_ERR_CUDA;
  long long Tmax = 0;
  for (int b = 0; b < kv->B; ++b) Tmax = std::max<long long>(Tmax, kv->seq_lens_host[b]);
  // Page tiles by tensor TMA need boxes of >= 8 rows (1024-byte aligned in shared memory).
  const bool rows = kv->page_size < 8;
  const Split sp = plan_splits(Tmax, U, 0, dev->sms * attend_slots_per_sm(G, false, rows));
  CUtensorMap tk = {}, tv = {};
  const int box_rows = std::min(kv->page_size, kTile);
  if (!rows && (!make_kv_tmap(&tk, kv->k_cache, kv, box_rows) || !make_kv_tmap(&tv, kv->v_cache, kv, box_rows)))
    return HSA_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t parts = static_cast<size_t>(U) * kMaxSplits * G;
  size_t o = align_up(sizeof(WsHeader), 256);
  float* pm = reinterpret_cast<float*>(base + o);
  o += align_up(parts * sizeof(float), 256);
  float* pl = reinterpret_cast<float*>(base + o);
  o += align_up(parts * sizeof(float), 256);
  float* pacc = reinterpret_cast<float*>(base + o);

  AttendParams p = {};
  p.k_cache = static_cast<const uint8_t*>(kv->k_cache);
  p.v_cache = static_cast<const uint8_t*>(kv->v_cache);
  p.q = q;
  p.block_table = kv->block_table;
  p.seq_lens = kv->seq_lens;
  p.err = reinterpret_cast<int32_t*>(base);
  p.pm = pm;
  p.pl = pl;
  p.pacc = pacc;
  p.U = U;
  p.B = kv->B;
  p.Hq = kv->Hq;
  p.Hkv = kv->Hkv;
  p.page_size = kv->page_size;
  p.max_pages = kv->max_pages;
  p.num_pages = kv->num_pages;
  p.nsplit = sp.nsplit;
  p.chunk = sp.chunk;
  p.S_tot = sp.nsplit;
  p.qscale = scale * kLog2e;
  p.k_override = -1;
  RET_CUDA(launch_attend(G, false, rows, tk, tv, p, U * sp.nsplit, false, stream, use_pdl()));
  MergeParams mp = {pm, pl, pacc, out, kv->B, kv->Hq, kv->Hkv, sp.nsplit};
  RET_CUDA(launch_merge(G, mp, stream, use_pdl()));
  return HSA_OK;
}

}  // extern "C"

namespace {
// hsa_decode; q_staged: the previous kernel on the stream is hsa_decode_host's q staging
// (the tables kernel may then read the index before its dependency wait).
hsa_status decode_impl(const hsa_kv_cache* kv, const hsa_index* ix, const float* q, float* out,
                       const hsa_decode_params* prm, const hsa_debug* dbg, void* ws, size_t ws_bytes,
                       cudaStream_t stream, bool q_staged) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  st = check_index(kv, ix, true);
  if (st != HSA_OK) return st;
  if (!q || !out || !prm) return HSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return HSA_ERR_ALIGNMENT;
  if (!(prm->budget >= 0.0) || !std::isfinite(prm->scale)) return HSA_ERR_INVALID_ARG;
  const int U = kv->B * kv->Hkv, G = kv->Hq / kv->Hkv;
  const int ring_depth = scan_ring_depth(G, ix->C);
  if (ring_depth < 2) return HSA_ERR_UNSUPPORTED;   // LUT + centroid terms too large for shared memory
  const DecodeLayout L = make_decode_layout(U, G, ix->C, ix->cap, ix->list_slots, kMaxSplits);
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HSA_ERR_WORKSPACE;
  const DeviceInfo* dev = device_info();
  if (!dev) return HSA_ERR_CUDA;

  // ---- plan the exact split-K over sink + selected + tail rows ----
  const Split sp = decode_split_plan(kv, ix, prm, L.nbg, dev->sms);
  CUtensorMap tk = {}, tv = {};   // unused: gathered rows are copied by the producer lanes
  cudaEvent_t* ev = dbg ? dbg->stage_events : nullptr;
  auto mark = [&](int i) -> cudaError_t { return ev ? cudaEventRecord(ev[i], stream) : cudaSuccess; };

  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* err = reinterpret_cast<int32_t*>(base);
  UnitState* units = reinterpret_cast<UnitState*>(base + L.off_units);
  float* bounds = reinterpret_cast<float*>(base + L.off_bounds);
  float* fbounds = reinterpret_cast<float*>(base + L.off_fbounds);
  float* lut = reinterpret_cast<float*>(base + L.off_lut);
  float* qc = reinterpret_cast<float*>(base + L.off_qc);
  float* W = reinterpret_cast<float*>(base + L.off_w);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.off_hist);
  float* sigma = reinterpret_cast<float*>(base + L.off_sigma);
  float* cmax = reinterpret_cast<float*>(base + L.off_cmax);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(base + L.off_bitmap);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(base + L.off_cand);
  float* cand_w = reinterpret_cast<float*>(base + L.off_candw);
  int32_t* cand_c = reinterpret_cast<int32_t*>(base + L.off_candc);
  int32_t* cand_row = reinterpret_cast<int32_t*>(base + L.off_candr);
  int32_t* sel = reinterpret_cast<int32_t*>(base + L.off_sel);
  float* pm = reinterpret_cast<float*>(base + L.off_pm);
  float* pl = reinterpret_cast<float*>(base + L.off_pl);
  float* pacc = reinterpret_cast<float*>(base + L.off_pacc);
  const int S_tot = sp.nsplit + L.nbg;
  if (S_tot > kMaxSplits + L.nbg) return HSA_ERR_WORKSPACE;

  TablesParams tp = {};
  tp.q = q;
  tp.centroids = ix->centroids;
  tp.codebooks = ix->codebooks;
  tp.lut = lut;
  tp.qc = qc;
  tp.bounds = bounds;
  tp.W = W;
  tp.hist = hist;
  tp.bitmap = bitmap;
  tp.units = units;
  tp.B = kv->B;
  tp.Hq = kv->Hq;
  tp.Hkv = kv->Hkv;
  tp.C = ix->C;
  tp.nq = L.nq;
  tp.bitmap_words = L.bitmap_words;
  tp.scale = prm->scale;
  tp.index_early = (q_staged && use_pdl()) ? 1 : 0;
  RET_CUDA(mark(0));
  RET_CUDA(launch_tables(G, tp, stream, use_pdl()));

  StepParams sc = {};
  sc.list_codes = ix->list_codes;
  sc.list_slot = ix->list_slot;
  sc.chunk_cluster = ix->chunk_cluster;
  sc.list_meta = ix->list_meta;
  sc.list_slots = ix->list_slots;
  sc.seq_lens = kv->seq_lens;
  sc.n_indexed = ix->n_indexed;
  sc.codes = ix->codes;
  sc.ids = ix->ids;
  sc.lut = lut;
  sc.qc = qc;
  sc.bounds = bounds;
  sc.fbounds = fbounds;
  sc.W = W;
  sc.hist = hist;
  sc.sigma = sigma;
  sc.chunk_max = cmax;
  sc.bitmap = bitmap;
  sc.cand = cand;
  sc.cand_w = cand_w;
  sc.cand_c = cand_c;
  sc.cand_row = cand_row;
  sc.units = units;
  sc.sel = sel;
  sc.block_table = kv->block_table;
  sc.page_size = kv->page_size;
  sc.max_pages = kv->max_pages;
  sc.num_pages = kv->num_pages;
  sc.approx_logits = dbg ? dbg->approx_logits : nullptr;
  sc.dbg_selected = dbg ? dbg->selected : nullptr;
  sc.dbg_nselected = dbg ? dbg->n_selected : nullptr;
  sc.err = err;
  sc.B = kv->B;
  sc.Hq = kv->Hq;
  sc.Hkv = kv->Hkv;
  sc.cap = ix->cap;
  sc.C = ix->C;
  sc.nq = L.nq;
  sc.n_sink = ix->n_sink;
  sc.bitmap_words = L.bitmap_words;
  sc.k_override = prm->k_override;
  sc.background = prm->background ? 1 : 0;
  sc.ring_depth = ring_depth;
  sc.budget = prm->budget;
  RET_CUDA(mark(1));
  RET_CUDA(launch_scan_select(G, sc, dev->sms, stream, use_pdl()));

  AttendParams p = {};
  p.k_cache = static_cast<const uint8_t*>(kv->k_cache);
  p.v_cache = static_cast<const uint8_t*>(kv->v_cache);
  p.q = q;
  p.block_table = kv->block_table;
  p.seq_lens = kv->seq_lens;
  p.n_indexed = ix->n_indexed;
  p.sel = sel;
  p.err = err;
  p.pm = pm;
  p.pl = pl;
  p.pacc = pacc;
  p.W = W;
  p.mean_v = ix->mean_v;
  p.bounds = bounds;
  p.U = U;
  p.B = kv->B;
  p.Hq = kv->Hq;
  p.Hkv = kv->Hkv;
  p.page_size = kv->page_size;
  p.max_pages = kv->max_pages;
  p.num_pages = kv->num_pages;
  p.cap = ix->cap;
  p.n_sink = ix->n_sink;
  p.nsplit = sp.nsplit;
  p.chunk = sp.chunk;
  p.S_tot = S_tot;
  p.C = ix->C;
  p.nbg = L.nbg;
  p.nq = L.nq;
  p.fbounds = fbounds;
  p.units = units;
  p.bg_enabled = prm->background ? 1 : 0;
  p.k_override = prm->k_override;
  p.budget = prm->budget;
  p.qscale = prm->scale * kLog2e;
  RET_CUDA(mark(2));
  const int attend_grid = U * (sp.nsplit + L.nbg);
  RET_CUDA(launch_attend(G, true, true, tk, tv, p, attend_grid, attend_grid > 2 * dev->sms, stream, use_pdl()));
  MergeParams mp = {pm, pl, pacc, out, kv->B, kv->Hq, kv->Hkv, S_tot};
  RET_CUDA(mark(3));
  RET_CUDA(launch_merge(G, mp, stream, use_pdl()));
  RET_CUDA(mark(4));
  return HSA_OK;
}
}  // namespace

extern "C" {

hsa_status hsa_decode(const hsa_kv_cache* kv, const hsa_index* ix, const float* q, float* out,
                      const hsa_decode_params* prm, const hsa_debug* dbg, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
  return decode_impl(kv, ix, q, out, prm, dbg, ws, ws_bytes, stream, false);
}

// Longest training set: the fallback assignment launches one grid row per 32 keys (at most 65535).
constexpr int32_t kMaxTrain = 65535 * 32;
constexpr size_t kAssignTileN = 256;   // centroids per tensor-core tile

// Tensor map over row-major [rows][128] bf16 (the centroid terms), box 64 x 256, 128-byte swizzle.
bool make_rows_tmap(CUtensorMap* map, const void* base, size_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(kAssignTileN)};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core nearest-centroid search of keys [0, n) of every unit (key j of sequence b at
// position n_sink + slot0[b] + j), p.assign receiving the centroid index: tensor maps,
// tile counts and grid. lead = the largest (n_sink + slot0[b]) mod 8 over the sequences.
static hsa_status plan_mma_assign(const hsa_kv_cache* kv, TrainParams& p, int lead, CUtensorMap* tmk,
                                  CUtensorMap* tmb, int* grid) {
  const DeviceInfo* di = device_info();
  if (!di) return HSA_ERR_CUDA;
  const int U = kv->B * kv->Hkv;
  p.Cpad = static_cast<int>(align_up(static_cast<size_t>(p.C), kAssignTileN));
  p.tiles_per_unit = (lead + p.n_train + 127) / 128;
  p.items = U * p.tiles_per_unit;
  if (!make_kv_tmap(tmk, kv->k_cache, kv, 8) || !make_rows_tmap(tmb, p.terms, static_cast<size_t>(U) * 3 * p.Cpad))
    return HSA_ERR_CUDA;
  *grid = std::min(p.items, di->sms);
  return HSA_OK;
}

static cudaError_t run_mma_assign(const CUtensorMap& tmk, const CUtensorMap& tmb, const TrainParams& p, int grid,
                                  cudaStream_t stream) {
  cudaError_t e = launch_centroid_terms(p, stream);
  if (e != cudaSuccess) return e;
  return launch_assign_mma(tmk, tmb, p, grid, stream);
}

// Encoding workspace (tensor-core path): error header, centroid terms [U][3][Cpad][D]
// bf16, |c|^2 [U][Cpad], assignment [U][n_new].
struct EncodeLayout {
  size_t terms, cnorm, assign, total;
};
static EncodeLayout encode_layout(int U, int C, int n_new) {
  EncodeLayout L;
  size_t o = align_up(sizeof(WsHeader), 256);
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + bytes, 256);
    return r;
  };
  const size_t cpad = align_up(static_cast<size_t>(C), kAssignTileN);
  L.terms = take(static_cast<size_t>(U) * 3 * cpad * kD * sizeof(uint16_t));
  L.cnorm = take(static_cast<size_t>(U) * cpad * sizeof(float));
  L.assign = take(static_cast<size_t>(U) * n_new * sizeof(int32_t));
  L.total = o;
  return L;
}

// Encoding runs on the tensor cores when the cache has pages of at least 8 rows.
static bool mma_encode(const hsa_kv_cache* kv, int n_new) { return kv->page_size >= 8 && n_new > 0; }

hsa_status hsa_decode_host(const hsa_kv_cache* kv, const hsa_index* ix, const float* q_host, float* out_host,
                           const hsa_decode_params* prm, void* ws, size_t ws_bytes, cudaStream_t stream) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  st = check_index(kv, ix, true);
  if (st != HSA_OK) return st;
  if (!q_host || !out_host || !prm) return HSA_ERR_INVALID_ARG;
  const size_t base = align_up(hsa_decode_workspace_bytes(kv, ix), 256);
  const size_t io = host_io_bytes(kv);
  if (!ws || !aligned(ws, 256) || ws_bytes < base + 2 * io) return HSA_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* q_dev = reinterpret_cast<float*>(w + base);
  float* out_dev = reinterpret_cast<float*>(w + base + io);
  const size_t bytes = static_cast<size_t>(kv->B) * kv->Hq * kD * sizeof(float);
  // Page-locked buffers are device-addressable: q is staged by a kernel and the merge writes
  // out across the host link itself (no copy-engine round trips). Pageable ones are copied.
  const void* q_map = mapped_host_pointer(q_host);
  void* out_map = mapped_host_pointer(out_host);
  if (q_map && out_map && aligned(q_map, 16) && aligned(out_map, 16)) {
    const int n4 = static_cast<int>(bytes / 16);
    stage_q_kernel<<<std::min(64, (n4 + 255) / 256), 256, 0, stream>>>(static_cast<const float4*>(q_map),
                                                                       reinterpret_cast<float4*>(q_dev), n4);
    RET_CUDA(cudaGetLastError());
    return decode_impl(kv, ix, q_dev, static_cast<float*>(out_map), prm, nullptr, ws, base, stream, true);
  }
  RET_CUDA(cudaMemcpyAsync(q_dev, q_host, bytes, cudaMemcpyHostToDevice, stream));
  st = hsa_decode(kv, ix, q_dev, out_dev, prm, nullptr, ws, base, stream);
  if (st != HSA_OK) return st;
  RET_CUDA(cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, stream));
  return HSA_OK;
}

}  // extern "C"

struct hsa_decode_step {
  hsa_kv_cache kv;
  hsa_index ix;
  hsa_decode_params prm;
  void* ws;
  size_t ws_bytes;
  int device;                   // device current at the first capture
  cudaStream_t cap;             // private capture stream (created at the first capture)
  cudaGraphExec_t exec;         // the last recorded step
  int key_nsplit, key_chunk;    // its split-K plan
  const float* key_q;
  float* key_out;
};

namespace {
hsa_status check_step_args(const hsa_kv_cache* kv, const hsa_index* ix, const hsa_decode_params* prm, void* ws,
                           size_t ws_bytes) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  st = check_index(kv, ix, true);
  if (st != HSA_OK) return st;
  if (!prm || !(prm->budget >= 0.0) || !std::isfinite(prm->scale)) return HSA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < hsa_decode_host_workspace_bytes(kv, ix)) return HSA_ERR_WORKSPACE;
  return HSA_OK;
}
}  // namespace

extern "C" {

hsa_status hsa_decode_step_create(const hsa_kv_cache* kv, const hsa_index* ix, const hsa_decode_params* prm,
                                  void* ws, size_t ws_bytes, hsa_decode_step** step) {
  if (!step) return HSA_ERR_INVALID_ARG;
  *step = nullptr;
  const hsa_status st = check_step_args(kv, ix, prm, ws, ws_bytes);
  if (st != HSA_OK) return st;
  hsa_decode_step* s = new (std::nothrow) hsa_decode_step();
  if (!s) return HSA_ERR_CUDA;
  s->kv = *kv;
  s->ix = *ix;
  s->prm = *prm;
  s->ws = ws;
  s->ws_bytes = ws_bytes;
  s->device = -1;
  s->cap = nullptr;
  s->exec = nullptr;
  *step = s;
  return HSA_OK;
}

hsa_status hsa_decode_step_run(hsa_decode_step* s, const float* q, float* out, cudaStream_t stream) {
  if (!s) return HSA_ERR_INVALID_ARG;
  hsa_status st = check_step_args(&s->kv, &s->ix, &s->prm, s->ws, s->ws_bytes);
  if (st != HSA_OK) return st;
  if (!q || !out) return HSA_ERR_INVALID_ARG;
  const DeviceInfo* dev = device_info();
  if (!dev) return HSA_ERR_CUDA;
  const int G = s->kv.Hq / s->kv.Hkv;
  const DecodeLayout L = make_decode_layout(s->kv.B * s->kv.Hkv, G, s->ix.C, s->ix.cap, s->ix.list_slots, kMaxSplits);
  const Split sp = decode_split_plan(&s->kv, &s->ix, &s->prm, L.nbg, dev->sms);
  const bool same = s->exec && sp.nsplit == s->key_nsplit && sp.chunk == s->key_chunk && q == s->key_q &&
                    out == s->key_out;
  if (!same) {
    // both page-locked host memory (the host-buffer step) or both device memory (hsa_decode);
    // a graph cannot copy pageable host memory
    const int kind = buffer_kind(q);
    if (kind == 0 || buffer_kind(out) != kind) return HSA_ERR_INVALID_ARG;
    int cur = 0;
    RET_CUDA(cudaGetDevice(&cur));
    if (s->cap && cur != s->device) return HSA_ERR_INVALID_ARG;   // a step stays on its first device
    if (!s->cap) {
      RET_CUDA(cudaStreamCreateWithFlags(&s->cap, cudaStreamNonBlocking));
      s->device = cur;
    }
    // record the step (nothing runs while the stream captures)
    RET_CUDA(cudaStreamBeginCapture(s->cap, cudaStreamCaptureModeThreadLocal));
    st = kind == 1 ? hsa_decode_host(&s->kv, &s->ix, q, out, &s->prm, s->ws, s->ws_bytes, s->cap)
                   : hsa_decode(&s->kv, &s->ix, q, out, &s->prm, nullptr, s->ws, s->ws_bytes, s->cap);
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(s->cap, &g);
    if (st != HSA_OK || ce != cudaSuccess || !g) {
      if (g) cudaGraphDestroy(g);
      (void)cudaGetLastError();   // an invalidated capture (e.g. pageable host memory) is not sticky
      return st != HSA_OK ? st : HSA_ERR_CUDA;
    }
    if (s->exec) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(s->exec, g, &info) != cudaSuccess) {
        (void)cudaGetLastError();   // the failed update is not sticky; instantiate afresh
        cudaGraphExecDestroy(s->exec);
        s->exec = nullptr;
      }
    }
    if (!s->exec && cudaGraphInstantiate(&s->exec, g, 0) != cudaSuccess) {
      s->exec = nullptr;
      cudaGraphDestroy(g);
      return HSA_ERR_CUDA;
    }
    cudaGraphDestroy(g);
    s->key_nsplit = sp.nsplit;
    s->key_chunk = sp.chunk;
    s->key_q = q;
    s->key_out = out;
  }
  RET_CUDA(cudaGraphLaunch(s->exec, stream));
  return HSA_OK;
}

void hsa_decode_step_destroy(hsa_decode_step* s) {
  if (!s) return;
  if (s->exec) cudaGraphExecDestroy(s->exec);
  if (s->cap) cudaStreamDestroy(s->cap);
  delete s;
}

size_t hsa_index_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* ix, int32_t n_new) {
  if (!kv || !ix || kv->B < 1 || kv->Hkv < 1 || ix->C < 1 || n_new < 0) return sizeof(WsHeader);
  if (!mma_encode(kv, n_new)) return sizeof(WsHeader);
  return encode_layout(kv->B * kv->Hkv, ix->C, n_new).total;
}

static IndexParams index_params(const hsa_kv_cache* kv, hsa_index* ix, void* ws) {
  IndexParams p = {};
  p.k_cache = static_cast<const uint16_t*>(kv->k_cache);
  p.v_cache = static_cast<const uint16_t*>(kv->v_cache);
  p.block_table = kv->block_table;
  p.seq_lens = kv->seq_lens;
  p.centroids = ix->centroids;
  p.codebooks = ix->codebooks;
  p.codes = ix->codes;
  p.ids = ix->ids;
  p.sum_v = ix->sum_v;
  p.mean_v = ix->mean_v;
  p.count = ix->count;
  p.n_indexed = ix->n_indexed;
  p.err = static_cast<int32_t*>(ws);
  p.list_codes = ix->list_codes;
  p.list_slot = ix->list_slot;
  p.chunk_cluster = ix->chunk_cluster;
  p.list_meta = ix->list_meta;
  p.B = kv->B;
  p.Hkv = kv->Hkv;
  p.page_size = kv->page_size;
  p.max_pages = kv->max_pages;
  p.num_pages = kv->num_pages;
  p.C = ix->C;
  p.cap = ix->cap;
  p.n_sink = ix->n_sink;
  p.list_slots = ix->list_slots;
  return p;
}

hsa_status hsa_build_from_codes(const hsa_kv_cache* kv, hsa_index* ix, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  st = check_index(kv, ix, true);
  if (st != HSA_OK) return st;
  if (!ix->sum_v || !ix->count) return HSA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(WsHeader)) return HSA_ERR_WORKSPACE;
  int nmax = 0;
  for (int b = 0; b < kv->B; ++b) nmax = std::max(nmax, ix->n_indexed_host[b]);
  IndexParams p = index_params(kv, ix, ws);
  p.slot_lo_from_indexed = 0;
  p.n_slots = -1;
  p.bump_indexed = 0;
  p.zero_if_empty = 0;
  RET_CUDA(launch_zero_stats(p, stream));
  RET_CUDA(launch_accumulate(p, nmax, stream));
  RET_CUDA(launch_list_reset(p, stream));
  RET_CUDA(launch_list_append(p, stream));
  RET_CUDA(launch_means(p, stream));
  return HSA_OK;
}

hsa_status hsa_append_encode(const hsa_kv_cache* kv, hsa_index* ix, int32_t n_new, void* ws, size_t ws_bytes,
                             cudaStream_t stream) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  st = check_index(kv, ix, true);
  if (st != HSA_OK) return st;
  if (!ix->sum_v || !ix->count) return HSA_ERR_INVALID_ARG;
  if (n_new < 0) return HSA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < hsa_index_workspace_bytes(kv, ix, n_new)) return HSA_ERR_WORKSPACE;
  for (int b = 0; b < kv->B; ++b) {
    const long long N = ix->n_indexed_host[b];
    if (N + n_new > ix->cap) return HSA_ERR_CAPACITY;
    if (ix->n_sink + N + n_new > kv->seq_lens_host[b]) return HSA_ERR_CAPACITY;
  }
  if (n_new == 0) return HSA_OK;
  IndexParams p = index_params(kv, ix, ws);
  p.slot_lo_from_indexed = 1;
  p.n_slots = n_new;
  p.bump_indexed = 1;
  p.zero_if_empty = 1;
  RET_CUDA(launch_zero_stats(p, stream));
  if (mma_encode(kv, n_new)) {
    const int U = kv->B * kv->Hkv;
    const EncodeLayout L = encode_layout(U, ix->C, n_new);
    uint8_t* base = static_cast<uint8_t*>(ws);
    TrainParams t = {};
    t.k_cache = static_cast<const uint16_t*>(kv->k_cache);
    t.block_table = kv->block_table;
    t.centroids = ix->centroids;
    t.codebooks = ix->codebooks;
    t.assign = reinterpret_cast<int32_t*>(base + L.assign);
    t.err = static_cast<int32_t*>(ws);
    t.terms = reinterpret_cast<uint16_t*>(base + L.terms);
    t.cnorm = reinterpret_cast<float*>(base + L.cnorm);
    t.slot0 = ix->n_indexed;   // read before the mean pass advances it
    t.B = kv->B;
    t.Hkv = kv->Hkv;
    t.C = ix->C;
    t.n_sink = ix->n_sink;
    t.n_train = n_new;
    t.page_size = kv->page_size;
    t.max_pages = kv->max_pages;
    t.num_pages = kv->num_pages;
    int lead = 0;
    for (int b = 0; b < kv->B; ++b) lead = std::max(lead, (ix->n_sink + ix->n_indexed_host[b]) & 7);
    CUtensorMap tmk = {}, tmb = {};
    int grid = 0;
    st = plan_mma_assign(kv, t, lead, &tmk, &tmb, &grid);
    if (st != HSA_OK) return st;
    RET_CUDA(run_mma_assign(tmk, tmb, t, grid, stream));
    RET_CUDA(launch_encode_codes(t, ix->codes, ix->ids, ix->cap, stream));
  } else {
    RET_CUDA(launch_encode(p, n_new, stream));
  }
  RET_CUDA(launch_accumulate(p, n_new, stream));
  RET_CUDA(launch_list_reset(p, stream));
  RET_CUDA(launch_list_append(p, stream));
  RET_CUDA(launch_means(p, stream));
  for (int b = 0; b < kv->B; ++b) ix->n_indexed_host[b] += n_new;
  return HSA_OK;
}

// Training workspace: error header, assignment [U][n_train], centroid sums [U][C][D] and
// counts [U][C], codeword sums [U][M][ncode][dsub] and counts [U][M][ncode].
struct TrainLayout {
  size_t assign, sums, counts, pq_sums, pq_counts, terms, cnorm, total;
};
static TrainLayout train_layout(int U, int C, int n_train) {
  TrainLayout L;
  size_t o = align_up(sizeof(WsHeader), 256);
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + bytes, 256);
    return r;
  };
  L.assign = take(static_cast<size_t>(U) * n_train * sizeof(int32_t));
  L.sums = take(static_cast<size_t>(U) * C * kD * sizeof(float));
  L.counts = take(static_cast<size_t>(U) * C * sizeof(int32_t));
  L.pq_sums = take(static_cast<size_t>(U) * kM * kNcode * kDsub * sizeof(float));
  L.pq_counts = take(static_cast<size_t>(U) * kM * kNcode * sizeof(int32_t));
  const size_t cpad = align_up(static_cast<size_t>(C), kAssignTileN);
  L.terms = take(static_cast<size_t>(U) * 3 * cpad * kD * sizeof(uint16_t));
  L.cnorm = take(static_cast<size_t>(U) * cpad * sizeof(float));
  L.total = o;
  return L;
}

size_t hsa_train_workspace_bytes(const hsa_kv_cache* kv, const hsa_index* ix, int32_t n_train) {
  if (!kv || !ix || n_train < 1 || ix->C < 1 || kv->B < 1 || kv->Hkv < 1) return 0;
  return train_layout(kv->B * kv->Hkv, ix->C, n_train).total;
}

hsa_status hsa_train_index(const hsa_kv_cache* kv, hsa_index* ix, int32_t n_train, const int32_t* init_slots,
                           int32_t coarse_iters, int32_t pq_iters, int32_t* assign_out, void* ws,
                           size_t ws_bytes, cudaStream_t stream) {
  hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  if (!ix || !ix->centroids || !ix->codebooks || !init_slots) return HSA_ERR_INVALID_ARG;
  if (ix->M != kM || ix->dsub != kDsub || ix->ncode != kNcode) return HSA_ERR_UNSUPPORTED;
  if (ix->C < 1 || ix->n_sink < 0) return HSA_ERR_INVALID_ARG;
  if (ix->C > kMaxClusters) return HSA_ERR_UNSUPPORTED;
  if (n_train < 1 || coarse_iters < 0 || pq_iters < 0 || coarse_iters > 1000 || pq_iters > 1000)
    return HSA_ERR_INVALID_ARG;
  if (n_train > kMaxTrain) return HSA_ERR_UNSUPPORTED;   // grid rows of the CUDA-core assignment
  if (!aligned(ix->centroids, 16) || !aligned(ix->codebooks, 16) || !aligned(init_slots, 4) ||
      (assign_out && !aligned(assign_out, 4)))
    return HSA_ERR_ALIGNMENT;
  for (int b = 0; b < kv->B; ++b)
    if (static_cast<long long>(ix->n_sink) + n_train > kv->seq_lens_host[b]) return HSA_ERR_CAPACITY;
  const int U = kv->B * kv->Hkv;
  const TrainLayout L = train_layout(U, ix->C, n_train);
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HSA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  TrainParams p = {};
  p.k_cache = static_cast<const uint16_t*>(kv->k_cache);
  p.block_table = kv->block_table;
  p.centroids = ix->centroids;
  p.codebooks = ix->codebooks;
  p.init_slots = init_slots;
  p.assign = reinterpret_cast<int32_t*>(base + L.assign);
  p.sums = reinterpret_cast<float*>(base + L.sums);
  p.counts = reinterpret_cast<int32_t*>(base + L.counts);
  p.pq_sums = reinterpret_cast<float*>(base + L.pq_sums);
  p.pq_counts = reinterpret_cast<int32_t*>(base + L.pq_counts);
  p.err = reinterpret_cast<int32_t*>(base);
  p.B = kv->B;
  p.Hkv = kv->Hkv;
  p.C = ix->C;
  p.n_sink = ix->n_sink;
  p.n_train = n_train;
  p.page_size = kv->page_size;
  p.max_pages = kv->max_pages;
  p.num_pages = kv->num_pages;
  p.terms = reinterpret_cast<uint16_t*>(base + L.terms);
  p.cnorm = reinterpret_cast<float*>(base + L.cnorm);

  // Nearest-centroid assignment: on the tensor cores (keys streamed by TMA in 8-row
  // boxes, so pages of at least 8 rows); 4-row pages use the CUDA-core kernel.
  const bool mma = kv->page_size >= 8;
  CUtensorMap tmk = {}, tmb = {};
  int grid = 0;
  if (mma) {
    st = plan_mma_assign(kv, p, ix->n_sink & 7, &tmk, &tmb, &grid);
    if (st != HSA_OK) return st;
  }
  auto assign = [&]() -> cudaError_t {
    if (!mma) return launch_train_assign(p, stream);
    return run_mma_assign(tmk, tmb, p, grid, stream);
  };

  // the sums start at zero; every update clears what it used
  RET_CUDA(cudaMemsetAsync(base + L.sums, 0, L.terms - L.sums, stream));
  RET_CUDA(launch_train_init(p, stream));
  for (int it = 0; it < coarse_iters; ++it) {
    RET_CUDA(assign());
    RET_CUDA(launch_train_accumulate(p, stream));
    RET_CUDA(launch_train_update(p, stream));
  }
  p.assign_out = assign_out;   // the final assignment is the one returned
  RET_CUDA(assign());
  RET_CUDA(launch_train_pq_init(p, stream));
  for (int it = 0; it < pq_iters; ++it) {
    RET_CUDA(launch_train_pq_step(p, stream));
    RET_CUDA(launch_train_pq_update(p, stream));
  }
  return HSA_OK;
}

}  // extern "C"
