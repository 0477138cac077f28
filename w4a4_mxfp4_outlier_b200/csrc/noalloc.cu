// w4a4_linear_noalloc: the online layer (activation prep + dual-branch GEMM)
// with its scratch in a fixed, library-owned device array instead of a
// caller-provided workspace.  The paper has no counterpart; this is a service
// for callers that cannot allocate device memory where the layer runs -- a
// host framework or plugin interface that owns every device allocation and
// hands the library only inputs and outputs, or a serving loop whose device
// memory budget is fixed at start-up, where allocating per call (and the
// synchronisation cudaMalloc / cudaFree can imply) is not allowed.
//
// The layer still needs scratch for the quantised activations (E2M1 codes,
// E8M0 scales, the bf16 outlier columns); here it is a static __device__
// array, so the call allocates nothing.  Rules of the array:
//  * every device the library is used on holds W4A4_NOALLOC_SCRATCH_BYTES
//    for it until the process exits;
//  * a problem whose workspace (w4a4_workspace_size) exceeds the array is
//    rejected with W4A4_ERR_SCRATCH_LIMIT before anything is enqueued;
//  * all calls on a device share the array, which keeps the previous call's
//    contents.  Nothing needs clearing: the only bytes a call reads without
//    writing them first are scale rows past T in the last 128-row group, and
//    those reach only output rows past T, which are never stored.  Calls whose
//    GPU work overlaps (other streams, other host threads) race on the array
//    and must be serialised by the caller;
//  * the array's device address is looked up once per device, with that
//    device current, on the first call made there (a host-side query, no
//    allocation); make that first call before any stream capture.
#include <mutex>

#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands in for the symbol, so the address a kernel may use
// comes from the runtime, once per device.
static constexpr int kNoallocMaxDevices = 64;

static uint8_t* noalloc_scratch_ptr(cudaError_t* err) {
  static std::mutex mu;
  static void* ptrs[kNoallocMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    ptrs[dev] = p;
  }
  *err = cudaSuccess;
  return static_cast<uint8_t*>(ptrs[dev]);
}

}  // namespace w4a4

extern "C" w4a4_status w4a4_linear_noalloc(const void* X, int64_t T, int64_t ldx,
                                           const w4a4_packed_weight* pw, void* Y, int64_t ldy,
                                           void* stream) {
  using namespace w4a4;
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (T < 0 || ldx < g.d_in || ldy < g.d_out) return W4A4_ERR_INVALID_ARG;
  if (T == 0) return W4A4_OK;
  if (X == nullptr || Y == nullptr) return W4A4_ERR_INVALID_ARG;
  const WorkspaceLayout w = workspace_layout(T, g);
  if (w.total > static_cast<size_t>(W4A4_NOALLOC_SCRATCH_BYTES)) return W4A4_ERR_SCRATCH_LIMIT;
  cudaError_t e;
  uint8_t* base = noalloc_scratch_ptr(&e);
  if (base == nullptr) return W4A4_ERR_CUDA;
  uint8_t* aq = g.kj > 0 ? base + w.aq : nullptr;
  uint8_t* sfa = g.kj > 0 ? base + w.sfa : nullptr;
  void* xo = g.k > 0 ? base + w.xo : nullptr;
  st = w4a4_prep_act(X, T, ldx, pw, aq, sfa, xo, stream);
  if (st != W4A4_OK) return st;
  return w4a4_gemm_dual(aq, sfa, xo, T, pw, Y, ldy, stream);
}
