// noalloc.cu -- csa_index_topk_noalloc: the indexer + top-k call for callers
// that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin loaded into a
// host process that owns every device allocation and exposes no allocator to
// the plugin, or a serving loop that forbids cudaMalloc once it has started
// (cudaMalloc can synchronise the device and its latency is unbounded).  For
// them this entry point takes its scratch from a fixed array compiled into the
// library instead of a caller-provided workspace.  It still takes the caller's
// inputs and outputs, runs exactly the kernels of csa_index_topk and never
// calls cudaMalloc, cudaFree or any allocating routine.
//
// The array lives in device memory on every GPU that loads the library and
// stays there until the process exits.  Host code cannot use the array's name
// as a device address (in host code it names a host-side stand-in), so the
// first call on each device looks the address up with cudaGetSymbolAddress,
// with that device current, and caches it; that first call should therefore
// happen before any stream capture.  Every call on a device shares the same
// array, which keeps whatever the previous call left in it: calls that can
// overlap on the GPU (different streams, or different host threads) race on
// it and must be serialised by the caller.  The indexer writes every scratch
// byte it later reads, except the cooperative selection's counters and
// histograms, which must start at zero: the array is zero at load time
// (static initialisation) and every call leaves them at zero.
#include <stdio.h>

#include <mutex>

#include "csa_internal.cuh"

namespace {

// Largest scratch a call may need (csa_index_topk_workspace_size); larger
// shapes are rejected with CSA_ERR_INVALID_ARG.
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_index_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_index_scratch on the current device (looked up once per
// device, with that device current).
csa_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return csa::set_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return csa::set_error(CSA_ERR_UNSUPPORTED, "csa_index_topk_noalloc: device ordinal beyond 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_index_scratch);
    if (e != cudaSuccess || p == nullptr)
      return csa::set_error(CSA_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                           : "cudaGetSymbolAddress returned NULL");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" csa_status_t csa_index_topk_noalloc(const void* qI, const void* qI_sf, const float* wI,
                                               const void* KI, const void* KI_sf, const int64_t* q_pos,
                                               int batch, int n_q, int64_t n_entries, int m, int n_heads,
                                               int dim, int k, csa_dtype_t dt, int32_t* idx_out,
                                               void* scores_out, void* stream) {
  const size_t need = csa_index_topk_workspace_size(batch, n_q, n_entries, k, n_heads, dim, dt);
  if (need > kStaticScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "csa_index_topk_noalloc: this shape needs %zu bytes of scratch but the built-in scratch "
             "holds %zu bytes; use csa_index_topk with a workspace",
             need, kStaticScratchBytes);
    return csa::set_error(CSA_ERR_INVALID_ARG, msg);
  }
  void* scratch = nullptr;
  const csa_status_t st = scratch_address(&scratch);
  if (st != CSA_OK) return st;
  return csa_index_topk(qI, qI_sf, wI, KI, KI_sf, q_pos, batch, n_q, n_entries, m, n_heads, dim, k, dt,
                        idx_out, scores_out, scratch, kStaticScratchBytes, stream);
}
