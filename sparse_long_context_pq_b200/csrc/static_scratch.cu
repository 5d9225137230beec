// dense_decode_static: dense split-K decode whose scratch (the split-K partials)
// lives in a fixed, file-scope device array instead of a caller-provided
// workspace, for callers that cannot allocate device memory. The PQ-HSA
// article has no counterpart to this entry point; it is a deployment aid.
//
// Scratch: kStaticScratchBytes (8 MiB) of device memory, held by every GPU that
// loads this library until the process exits. Layout per call (all rewritten by
// the call, nothing needs to start at zero): pm[U][S][G], pl[U][S][G],
// pacc[U][S][G][128] floats, S = number of split-K chunks.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "../../include/pqhsa.h"
#include "common.cuh"
#include "kernels.h"

using namespace pqhsa;

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;

// The scratch array. In host code this name is only a stand-in for the symbol:
// its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_dense_scratch[kStaticScratchBytes];

constexpr int kDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kDevices] = {nullptr};
int g_sms[kDevices] = {0};

// Device address of the scratch array on the current device (looked up on the
// first call with that device current, then cached).
cudaError_t scratch_for_current_device(void** ptr, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dense_scratch);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_sms[dev] = n;
  }
  *ptr = g_scratch_ptr[dev];
  *sms = g_sms[dev];
  return cudaSuccess;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The KV-cache view is validated exactly as dense_decode validates it.
hsa_status validate(const hsa_kv_cache* kv, const float* q, const float* out) {
  const hsa_status st = check_kv(kv);
  if (st != HSA_OK) return st;
  if (!q || !out) return HSA_ERR_INVALID_ARG;
  if (!is_aligned(q, 16) || !is_aligned(out, 16)) return HSA_ERR_ALIGNMENT;
  return HSA_OK;
}

}  // namespace

extern "C" hsa_status dense_decode_static(const hsa_kv_cache* kv, const float* q, float* out, float scale,
                                          cudaStream_t stream) {
  hsa_status st = validate(kv, q, out);
  if (st != HSA_OK) return st;
  const int U = kv->B * kv->Hkv, G = kv->Hq / kv->Hkv;

  // Bytes of one split-K chunk for every (unit, head): m, l and 128 accumulators.
  const size_t header = align_up(sizeof(WsHeader), 256);
  const size_t per_split = static_cast<size_t>(U) * G * (2 + kD) * sizeof(float) + 3 * 256;
  if (header + per_split > kStaticScratchBytes) return HSA_ERR_WORKSPACE;   // shape too large for the array
  const int fit = static_cast<int>(std::min<size_t>(kMaxSplits, (kStaticScratchBytes - header) / per_split));

  void* scratch = nullptr;
  int sms = 0;
  if (scratch_for_current_device(&scratch, &sms) != cudaSuccess) return HSA_ERR_CUDA;

  // Split-K chunking: about two CTAs per SM over all units, at most `fit` chunks per unit.
  long long Tmax = 0;
  for (int b = 0; b < kv->B; ++b) Tmax = std::max<long long>(Tmax, kv->seq_lens_host[b]);
  int ns = static_cast<int>(std::max<long long>(1, (2LL * sms + U - 1) / U));
  ns = std::min(ns, fit);
  long long chunk = std::max<long long>(1, (Tmax + ns - 1) / ns);
  chunk = (chunk + kTile - 1) / kTile * kTile;
  ns = static_cast<int>(std::max<long long>(1, (Tmax + chunk - 1) / chunk));

  uint8_t* base = static_cast<uint8_t*>(scratch);
  const size_t parts = static_cast<size_t>(U) * ns * G;
  float* pm = reinterpret_cast<float*>(base + header);
  float* pl = reinterpret_cast<float*>(base + header + align_up(parts * sizeof(float), 256));
  float* pacc = reinterpret_cast<float*>(base + header + 2 * align_up(parts * sizeof(float), 256));

  const bool rows = kv->page_size < 8;
  CUtensorMap tk = {}, tv = {};
  const int box_rows = std::min(kv->page_size, kTile);
  if (!rows && (!make_kv_tmap(&tk, kv->k_cache, kv, box_rows) || !make_kv_tmap(&tv, kv->v_cache, kv, box_rows)))
    return HSA_ERR_CUDA;

  AttendParams p = {};
  p.k_cache = static_cast<const uint8_t*>(kv->k_cache);
  p.v_cache = static_cast<const uint8_t*>(kv->v_cache);
  p.q = q;
  p.block_table = kv->block_table;
  p.seq_lens = kv->seq_lens;
  p.err = nullptr;   // no error word here: bad block-table entries are still skipped on the device
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
  p.nsplit = ns;
  p.chunk = static_cast<int>(chunk);
  p.S_tot = ns;
  p.qscale = scale * kLog2e;
  p.k_override = -1;
  if (launch_attend(G, false, rows, tk, tv, p, U * ns, false, stream, false) != cudaSuccess) return HSA_ERR_CUDA;
  MergeParams mp = {pm, pl, pacc, out, kv->B, kv->Hq, kv->Hkv, ns};
  if (launch_merge(G, mp, stream, false) != cudaSuccess) return HSA_ERR_CUDA;
  return HSA_OK;
}
