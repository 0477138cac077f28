// Output-error sums for choosing alpha and k per layer: the review names
// layer-wise alpha and k as the way to narrow the gap further (sec. 4 table,
// "Layer-wise alpha and k"; sec. 6 "next step") without saying how to pick
// them; the search scores each candidate by the relative Frobenius error of
// its Y against a reference product, and this kernel supplies the two sums.
#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

constexpr int kErrThreads = 256;

// out[0] += sum (Y - R)^2, out[1] += sum R^2 over a T x d_out block (Y bf16,
// R float32), accumulated in float64.  Each block strides over whole rows.
__global__ void __launch_bounds__(kErrThreads)
    error_sums_kernel(const __nv_bfloat16* __restrict__ Y, int64_t ldy, const float* __restrict__ R,
                      int64_t ldr, int64_t T, int64_t d_out, double* __restrict__ out) {
  double num = 0.0, den = 0.0;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const __nv_bfloat16* y = Y + t * ldy;
    const float* rr = R + t * ldr;
    for (int64_t n = threadIdx.x; n < d_out; n += blockDim.x) {
      const double r = static_cast<double>(rr[n]);
      const double d = static_cast<double>(__bfloat162float(y[n])) - r;
      num += d * d;
      den += r * r;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xFFFFFFFFu, num, o);
    den += __shfl_xor_sync(0xFFFFFFFFu, den, o);
  }
  __shared__ double part[2][kErrThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    part[0][warp] = num;
    part[1][warp] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < kErrThreads / 32; ++w) {
      a += part[0][w];
      b += part[1][w];
    }
    atomicAdd(&out[0], a);
    atomicAdd(&out[1], b);
  }
}

}  // namespace w4a4

extern "C" w4a4_status w4a4_error_sums(const void* Y, int64_t ldy, const float* Yref, int64_t ldr,
                                       int64_t T, int64_t d_out, double* sums, void* stream) {
  using namespace w4a4;
  if (T < 0 || d_out < 0 || ldy < d_out || ldr < d_out || sums == nullptr) return W4A4_ERR_INVALID_ARG;
  if (T > 0 && d_out > 0 && (Y == nullptr || Yref == nullptr)) return W4A4_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sums, 0, 2 * sizeof(double), s) != cudaSuccess) return W4A4_ERR_CUDA;
  if (T == 0 || d_out == 0) return W4A4_OK;
  const int64_t sms = device_num_sms() > 0 ? device_num_sms() : 148;
  const int64_t grid = T < 4 * sms ? T : 4 * sms;
  error_sums_kernel<<<static_cast<unsigned>(grid), kErrThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(Y), ldy, Yref, ldr, T, d_out, sums);
  return cudaGetLastError() == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}
