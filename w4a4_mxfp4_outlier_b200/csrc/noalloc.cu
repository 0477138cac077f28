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
//  * the array's device address is looked up, with the device current, on
//    the first call made in each CUDA context (a host-side query, no
//    allocation) -- normally once per device, in its primary context.  The
//    lookup is keyed on the context's unique id, so a caller that makes its
//    own driver-API context current, or a new primary context after
//    cudaDeviceReset, gets that context's address.  Make the first call in a
//    context before any stream capture.
#include <mutex>

#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  In host code
// the array's name only stands in for the symbol, so the address a kernel may
// use comes from the runtime.  A symbol's address belongs to a context, not to
// a device, so the cache is keyed on the context's unique id (ids are never
// reused within a process, unlike context handles).
typedef CUresult (*PFN_ctxGetCurrent)(CUcontext*);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long*);

template <class F>
static F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

static constexpr int kNoallocMaxContexts = 64;

// Unique id of the context current on this thread (0 if none or on error).
static unsigned long long current_context_id() {
  static const PFN_ctxGetCurrent get_current = driver_fn<PFN_ctxGetCurrent>("cuCtxGetCurrent");
  static const PFN_ctxGetId get_id = driver_fn<PFN_ctxGetId>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

static uint8_t* noalloc_scratch_ptr(cudaError_t* err) {
  static std::mutex mu;
  static unsigned long long ids[kNoallocMaxContexts] = {0};
  static void* ptrs[kNoallocMaxContexts] = {nullptr};
  static int used = 0;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = current_context_id();
  for (int i = 0; id != 0 && i < used; ++i) {
    if (ids[i] == id) {
      *err = cudaSuccess;
      return static_cast<uint8_t*>(ptrs[i]);
    }
  }
  // first call in this context (the lookup also makes the runtime's context
  // current when the thread had none)
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    return nullptr;
  }
  if (id == 0) id = current_context_id();
  // a full table keeps working, with one lookup per call for further contexts
  if (id != 0 && used < kNoallocMaxContexts) {
    ids[used] = id;
    ptrs[used] = p;
    ++used;
  }
  *err = cudaSuccess;
  return static_cast<uint8_t*>(p);
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
  // the caller's arguments are checked before the scratch lookup (the first
  // device query); plan_linear checks them again with the scratch pointers,
  // still before anything is enqueued
  if (T > (int64_t(1) << 31) - 256 || ldx % 8 != 0 || ldy % 8 != 0 || !aligned16(X) ||
      !aligned16(Y))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  cudaError_t e;
  uint8_t* base = noalloc_scratch_ptr(&e);
  if (base == nullptr) return W4A4_ERR_CUDA;
  LinearPlan lp;
  st = plan_linear(X, T, ldx, g, pw, base, Y, ldy, &lp);
  if (st != W4A4_OK) return st;
  return enqueue_linear(lp, X, T, ldx, g, pw, static_cast<cudaStream_t>(stream));
}
