// C-ABI entry points of libw4a4 (declared in include/w4a4.h): argument
// validation, workspace layout and kernel launches.  No entry point
// allocates device memory.
#include <cstdlib>
#include <cstring>

#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

int device_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("W4A4_NO_PDL");
    on = (e != nullptr && strcmp(e, "1") == 0) ? 0 : 1;
  }
  return on == 1;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static w4a4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA; }

static w4a4_status check_dims(int64_t d_in, int64_t d_out, int64_t k) {
  if (d_in <= 0 || d_out <= 0 || k < 0 || k > d_in) return W4A4_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || d_out % 16 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (d_in > 65535 || d_out > (int64_t(1) << 30)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

static w4a4_status check_pw(const w4a4_packed_weight* pw, Geometry* g) {
  if (pw == nullptr) return W4A4_ERR_INVALID_ARG;
  w4a4_status st = check_dims(pw->d_in, pw->d_out, pw->k);
  if (st != W4A4_OK) return st;
  if (pw->layout != W4A4_SF_32x1_KMAJOR && pw->layout != W4A4_SF_32x32_TILE &&
      pw->layout != W4A4_SF_128x1_KMAJOR)
    return W4A4_ERR_INVALID_ARG;
  *g = make_geometry(pw->d_in, pw->d_out, pw->k);
  if (g->kj > 0 && (pw->wq == nullptr || pw->sfb == nullptr || pw->jmap == nullptr))
    return W4A4_ERR_INVALID_ARG;
  if (g->k > 0 && (pw->w_hp == nullptr || pw->O == nullptr)) return W4A4_ERR_INVALID_ARG;
  if (pw->inv_s == nullptr) return W4A4_ERR_INVALID_ARG;
  if ((pw->wq && !aligned16(pw->wq)) || (pw->sfb && !aligned16(pw->sfb)) ||
      (pw->w_hp && !aligned16(pw->w_hp)))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (!prep_supported(*g)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

struct WorkspaceLayout {
  size_t aq, sfa, xo, total;
};

static WorkspaceLayout workspace_layout(int64_t T, const Geometry& g) {
  WorkspaceLayout w;
  const size_t aq_b = static_cast<size_t>(T) * static_cast<size_t>(g.kj_pad / 2);
  const size_t sfa_b = static_cast<size_t>(round_up(T, kSfaRowPad)) * static_cast<size_t>(g.nblk);
  const size_t xo_b = static_cast<size_t>(T) * static_cast<size_t>(g.k_pad) * 2;
  w.aq = 0;
  w.sfa = static_cast<size_t>(round_up(static_cast<int64_t>(aq_b), 1024));
  w.xo = w.sfa + static_cast<size_t>(round_up(static_cast<int64_t>(sfa_b), 1024));
  w.total = w.xo + static_cast<size_t>(round_up(static_cast<int64_t>(xo_b), 1024));
  return w;
}

// Arguments of the activation prep, checked without touching the device.
static w4a4_status validate_prep(const void* X, int64_t T, int64_t ldx, const Geometry& g,
                                 const void* aq, const void* sfa, const void* xo) {
  if (T < 0 || ldx < g.d_in) return W4A4_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 256) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return W4A4_OK;
  if (X == nullptr || (g.kj > 0 && (aq == nullptr || sfa == nullptr)) || (g.k > 0 && xo == nullptr))
    return W4A4_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned16(X) || (aq && !aligned16(aq)) || (sfa && !aligned16(sfa)) ||
      (xo && !aligned16(xo)))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

// Arguments of the dual-branch GEMM, checked without touching the device.
static w4a4_status validate_gemm(const void* aq, const void* sfa, const void* xo, int64_t T,
                                 const Geometry& g, const void* Y, int64_t ldy) {
  if (T < 0 || ldy < g.d_out) return W4A4_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 256) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return W4A4_OK;
  if (Y == nullptr || (g.kj > 0 && (aq == nullptr || sfa == nullptr)) || (g.k > 0 && xo == nullptr))
    return W4A4_ERR_INVALID_ARG;
  if (ldy % 8 != 0 || !aligned16(Y) || (aq && !aligned16(aq)) || (sfa && !aligned16(sfa)) ||
      (xo && !aligned16(xo)))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

// The online layer (prep into the workspace at `base`, then the GEMM) as two
// phases: plan_linear checks every argument of both kernels and builds the
// GEMM's tensor maps, enqueuing nothing; enqueue_linear launches.  Composite
// calls run the first before their first enqueue, so a non-OK status always
// means that nothing was enqueued.
struct LinearPlan {
  uint8_t* aq;
  uint8_t* sfa;
  void* xo;
  GemmPlan gemm;
};

static w4a4_status plan_linear(const void* X, int64_t T, int64_t ldx, const Geometry& g,
                               const w4a4_packed_weight* pw, uint8_t* base, void* Y, int64_t ldy,
                               LinearPlan* lp) {
  const WorkspaceLayout w = workspace_layout(T, g);
  lp->aq = g.kj > 0 ? base + w.aq : nullptr;
  lp->sfa = g.kj > 0 ? base + w.sfa : nullptr;
  lp->xo = g.k > 0 ? base + w.xo : nullptr;
  w4a4_status st = validate_prep(X, T, ldx, g, lp->aq, lp->sfa, lp->xo);
  if (st != W4A4_OK) return st;
  st = validate_gemm(lp->aq, lp->sfa, lp->xo, T, g, Y, ldy);
  if (st != W4A4_OK) return st;
  return from_cuda(plan_gemm(lp->aq, lp->sfa, lp->xo, T, g, pw->wq, pw->sfb, pw->w_hp, Y, ldy,
                             nullptr, &lp->gemm));
}

static w4a4_status enqueue_linear(const LinearPlan& lp, const void* X, int64_t T, int64_t ldx,
                                  const Geometry& g, const w4a4_packed_weight* pw,
                                  cudaStream_t stream) {
  cudaError_t e = launch_prep(X, T, ldx, pw->inv_s, pw->O, pw->jmap, g, lp.aq, lp.sfa, lp.xo,
                              stream);
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  return from_cuda(run_gemm(lp.gemm, stream));
}

}  // namespace w4a4

using namespace w4a4;

extern "C" {

int w4a4_abi_version(void) { return W4A4_ABI_VERSION; }

const char* w4a4_status_string(w4a4_status s) {
  switch (s) {
    case W4A4_OK: return "ok";
    case W4A4_ERR_INVALID_ARG: return "invalid argument";
    case W4A4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or alignment";
    case W4A4_ERR_CUDA: return "CUDA error";
    case W4A4_ERR_TIMEOUT: return "device pipeline wait timed out";
    case W4A4_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed no-alloc scratch";
    case W4A4_ERR_BAD_IMAGE: return "packed-weight image failed its header or checksum check";
    case W4A4_ERR_NONFINITE_CALIB: return "a calibration magnitude was inf or NaN";
  }
  return "unknown status";
}

int w4a4_num_sms(void) { return device_num_sms(); }

w4a4_status w4a4_get_dims(int64_t d_in, int64_t d_out, int64_t k, w4a4_dims* out) {
  if (out == nullptr || d_in < 0 || d_out < 0 || k < 0 || k > d_in) return W4A4_ERR_INVALID_ARG;
  const Geometry g = make_geometry(d_in, d_out, k);
  out->d_in = g.d_in;
  out->d_out = g.d_out;
  out->k = g.k;
  out->kj = g.kj;
  out->kj_pad = g.kj_pad;
  out->nblk = g.nblk;
  out->k_pad = g.k_pad;
  out->sfb_rows = g.sfb_rows;
  return W4A4_OK;
}

w4a4_status w4a4_calib_observe(const void* A, int64_t rows, int64_t cols, int64_t lda,
                               float* absmax, int reset, void* stream) {
  if (absmax == nullptr || rows < 0 || cols <= 0 || lda < cols) return W4A4_ERR_INVALID_ARG;
  if (rows > 0 && A == nullptr) return W4A4_ERR_INVALID_ARG;
  if (cols % 8 != 0 || lda % 8 != 0 || (A && !aligned16(A))) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_colabsmax(A, rows, cols, lda, absmax, reset,
                                    static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_calib_observe_layer(const void* X, int64_t T, int64_t ldx, const void* W,
                                     int64_t d_out, int64_t ldw, int64_t d_in, float* act_absmax,
                                     float* w_absmax, int reset, void* stream) {
  if (act_absmax == nullptr || w_absmax == nullptr || act_absmax == w_absmax || T < 0 ||
      d_out < 0 || d_in <= 0 || ldx < d_in || ldw < d_in)
    return W4A4_ERR_INVALID_ARG;
  if ((T > 0 && X == nullptr) || (d_out > 0 && W == nullptr)) return W4A4_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || ldx % 8 != 0 || ldw % 8 != 0 || (X && !aligned16(X)) || (W && !aligned16(W)))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_colabsmax2(X, T, ldx, act_absmax, W, d_out, ldw, w_absmax, d_in, reset,
                                     static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_calib_finalize(const float* act_scale, const float* w_scale, int64_t d_in,
                                double alpha, int64_t k, float* s, float* inv_s, float* score,
                                int32_t* O, int32_t* jmap, void* stream) {
  if (act_scale == nullptr || w_scale == nullptr || s == nullptr || inv_s == nullptr ||
      score == nullptr)
    return W4A4_ERR_INVALID_ARG;
  if (d_in <= 0 || k < 0 || k > d_in || !(alpha > 0.0 && alpha < 1.0)) return W4A4_ERR_INVALID_ARG;
  if ((k > 0 && O == nullptr) || (k < d_in && jmap == nullptr)) return W4A4_ERR_INVALID_ARG;
  if (d_in > finalize_max_d()) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_finalize(act_scale, w_scale, static_cast<int>(d_in), alpha,
                                   static_cast<int>(k), s, inv_s, score, O, jmap,
                                   static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_weight_sizes(int64_t d_in, int64_t d_out, int64_t k, w4a4_weight_bytes* out) {
  if (out == nullptr) return W4A4_ERR_INVALID_ARG;
  w4a4_status st = check_dims(d_in, d_out, k);
  if (st != W4A4_OK) return st;
  const Geometry g = make_geometry(d_in, d_out, k);
  out->wq = static_cast<size_t>(g.d_out) * static_cast<size_t>(g.kj_pad / 2);
  out->sfb = static_cast<size_t>(g.sfb_rows) * static_cast<size_t>(g.nblk);
  out->w_hp = static_cast<size_t>(g.d_out) * static_cast<size_t>(g.k_pad) * 2;
  return W4A4_OK;
}

w4a4_status w4a4_pack_weight(const void* W, int64_t ldw, const float* s,
                             const w4a4_packed_weight* pw, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (W == nullptr || s == nullptr || ldw < g.d_in) return W4A4_ERR_INVALID_ARG;
  if (ldw % 8 != 0 || !aligned16(W)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_pack(W, ldw, s, pw->O, pw->jmap, g, pw->layout, pw->wq, pw->sfb,
                               pw->w_hp, static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_workspace_size(int64_t T, int64_t d_in, int64_t d_out, int64_t k, size_t* bytes) {
  if (bytes == nullptr || T < 0) return W4A4_ERR_INVALID_ARG;
  w4a4_status st = check_dims(d_in, d_out, k);
  if (st != W4A4_OK) return st;
  *bytes = workspace_layout(T, make_geometry(d_in, d_out, k)).total;
  return W4A4_OK;
}

w4a4_status w4a4_prep_act(const void* X, int64_t T, int64_t ldx, const w4a4_packed_weight* pw,
                          uint8_t* aq, uint8_t* sfa, void* xo, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  st = validate_prep(X, T, ldx, g, aq, sfa, xo);
  if (st != W4A4_OK || T == 0) return st;
  return from_cuda(launch_prep(X, T, ldx, pw->inv_s, pw->O, pw->jmap, g, aq, sfa, xo,
                               static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_gemm_dual(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                           const w4a4_packed_weight* pw, void* Y, int64_t ldy, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  st = validate_gemm(aq, sfa, xo, T, g, Y, ldy);
  if (st != W4A4_OK || T == 0) return st;
  return from_cuda(launch_gemm(aq, sfa, xo, T, g, pw->wq, pw->sfb, pw->w_hp, Y, ldy,
                               static_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_linear(const void* X, int64_t T, int64_t ldx, const w4a4_packed_weight* pw,
                        void* workspace, size_t ws_bytes, void* Y, int64_t ldy, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (T < 0 || ldx < g.d_in || ldy < g.d_out) return W4A4_ERR_INVALID_ARG;
  if (T == 0) return W4A4_OK;
  if (workspace == nullptr || ws_bytes < workspace_layout(T, g).total || X == nullptr ||
      Y == nullptr)
    return W4A4_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  LinearPlan lp;
  st = plan_linear(X, T, ldx, g, pw, static_cast<uint8_t*>(workspace), Y, ldy, &lp);
  if (st != W4A4_OK) return st;
  return enqueue_linear(lp, X, T, ldx, g, pw, static_cast<cudaStream_t>(stream));
}

w4a4_status w4a4_linear_host(const void* X_host, int64_t T, const w4a4_packed_weight* pw,
                             void* X_dev, void* workspace, size_t ws_bytes, void* Y_dev,
                             void* Y_host, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (T < 0) return W4A4_ERR_INVALID_ARG;
  if (T == 0) return W4A4_OK;
  if (X_host == nullptr || Y_host == nullptr || X_dev == nullptr || Y_dev == nullptr)
    return W4A4_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < workspace_layout(T, g).total) return W4A4_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  // everything the two kernels need is checked (and the GEMM planned) before
  // the upload is enqueued
  LinearPlan lp;
  st = plan_linear(X_dev, T, g.d_in, g, pw, static_cast<uint8_t*>(workspace), Y_dev, g.d_out, &lp);
  if (st != W4A4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(T) * static_cast<size_t>(g.d_in) * 2;
  const size_t yb = static_cast<size_t>(T) * static_cast<size_t>(g.d_out) * 2;
  cudaError_t e = cudaMemcpyAsync(X_dev, X_host, xb, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  st = enqueue_linear(lp, X_dev, T, g.d_in, g, pw, s);
  if (st != W4A4_OK) return st;
  e = cudaMemcpyAsync(Y_host, Y_dev, yb, cudaMemcpyDeviceToHost, s);
  return from_cuda(e);
}

w4a4_status w4a4_test_fault(uint32_t mask, uint64_t wait_limit_ns) {
  if ((mask & ~static_cast<uint32_t>(FAULT_PREP_SKIP_LOADS)) != 0u) return W4A4_ERR_INVALID_ARG;
  const uint64_t limit = wait_limit_ns == 0 ? kWaitLimitNs : wait_limit_ns;
  if (limit > kWaitLimitNs) return W4A4_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  e = cudaMemcpyToSymbol(g_wait_limit_ns, &limit, sizeof(limit));
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  e = cudaMemcpyToSymbol(g_fault_mask, &mask, sizeof(mask));
  return from_cuda(e);
}

w4a4_status w4a4_last_error(void* stream, int clear, uint32_t* bits) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  if (clear) {
    const uint32_t z = 0;
    e = cudaMemcpyToSymbol(g_device_error, &z, sizeof(z));
    if (e != cudaSuccess) return W4A4_ERR_CUDA;
  }
  if (bits) *bits = v;
  if (v & (DEVERR_TIMEOUT_PRODUCER | DEVERR_TIMEOUT_MMA | DEVERR_TIMEOUT_EPILOGUE |
           DEVERR_TIMEOUT_PREP))
    return W4A4_ERR_TIMEOUT;
  return (v & DEVERR_NONFINITE_CALIB) ? W4A4_ERR_NONFINITE_CALIB : W4A4_OK;
}

}  // extern "C"
