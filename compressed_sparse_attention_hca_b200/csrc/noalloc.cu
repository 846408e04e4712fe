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
// with that device current, and caches it together with the CUDA context it
// belongs to (a new context on the device, e.g. after cudaDeviceReset, is
// looked up again); that first call should therefore happen before any stream
// capture.  Every call on a device shares the same array, which keeps
// whatever the previous call left in it: calls that can overlap on the GPU
// (different streams, or different host threads) race on it and must be
// serialised by the caller.  The cooperative selection's counters and
// histograms must start at zero; the array is zero at load time (static
// initialisation), every call that ends normally leaves all of it at zero
// (the cooperative selection clears what it used, the merge kernel clears the
// candidate lists it consumed), and when csa_check_device_status reports a
// timed-out wait it zeroes the array of the current device again.
#include <stdio.h>

#include <cudaTypedefs.h>

#include <mutex>

#include "csa_internal.cuh"

namespace {

// Largest scratch a call may need (csa_index_topk_workspace_size); larger
// shapes are rejected with CSA_ERR_INVALID_ARG.
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_index_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  void* ctx;   // CUDA context the address belongs to
  void* addr;  // device address of g_index_scratch in that context
};
ScratchSlot g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The calling thread's current CUDA context (nullptr when it cannot be read).
void* current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_index_scratch on the current device, looked up with the
// device current and cached per (device, context).
csa_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return csa::set_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return csa::set_error(CSA_ERR_UNSUPPORTED, "csa_index_topk_noalloc: device ordinal beyond 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  const void* ctx = current_context();
  if (slot.addr == nullptr || ctx == nullptr || slot.ctx != ctx) {
    // the lookup also brings up the device's context when there is none yet,
    // so the context is read again afterwards
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_index_scratch);
    if (e != cudaSuccess || p == nullptr)
      return csa::set_error(CSA_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                           : "cudaGetSymbolAddress returned NULL");
    slot.ctx = current_context();
    slot.addr = p;
  }
  *out = slot.addr;
  return CSA_OK;
}

}  // namespace

// Zeroes the built-in scratch of the current device after a timed-out wait
// left counters set (called by csa_check_device_status, which has already
// synchronised the device).  A plain memset: nothing is allocated.
void csa::reset_static_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return;
  }
  void* addr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const ScratchSlot& slot = g_scratch[dev];
    if (slot.addr != nullptr && slot.ctx == current_context()) addr = slot.addr;
  }
  if (addr != nullptr && cudaMemset(addr, 0, kStaticScratchBytes) != cudaSuccess) cudaGetLastError();
}

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
