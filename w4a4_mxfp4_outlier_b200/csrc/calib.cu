// Calibration kernels: per-column absolute maximum of a bf16 matrix, and the
// device-side finalisation (smoothing factor, score, top-k outlier set).
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.1-3.2 (per-channel magnitudes, s_j = a_j^alpha / w_j^(1-alpha)) and
// sec. 3.3 (score_j = max_t |x_tj|, static top-k set O).
#include "w4a4_internal.h"

namespace w4a4 {

// ---------------------------------------------------------------------------
// Column absmax.  Block = 32 x 8 threads; threadIdx.x owns 8 consecutive
// columns (one 16-byte load per row), threadIdx.y and blockIdx.y stride over
// rows.  Magnitudes are compared as bf16 bit patterns with the sign cleared
// (for non-NaN values the integer order is the magnitude order), packed two
// per 32-bit word.  The block result goes to global memory with an integer
// atomicMax on the float32 bits, which orders non-negative floats correctly.
// HBM-bound: 2 bytes read per element.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) colabsmax_kernel(const uint16_t* __restrict__ A,
                                                        int64_t rows, int64_t cols, int64_t lda,
                                                        uint32_t* __restrict__ out_bits) {
  __shared__ uint32_t red[8][32][4];
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x) * 8;
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  if (col0 < cols) {
    const int64_t rstep = static_cast<int64_t>(gridDim.y) * 8;
    int64_t r = static_cast<int64_t>(blockIdx.y) * 8 + threadIdx.y;
    const uint16_t* p = A + col0;
    // four rows in flight per iteration
    for (; r + 3 * rstep < rows; r += 4 * rstep) {
      uint4 v0 = __ldcs(reinterpret_cast<const uint4*>(p + r * lda));
      uint4 v1 = __ldcs(reinterpret_cast<const uint4*>(p + (r + rstep) * lda));
      uint4 v2 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 2 * rstep) * lda));
      uint4 v3 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 3 * rstep) * lda));
      m[0] = __vmaxu2(m[0], __vmaxu2(__vmaxu2(v0.x & 0x7FFF7FFFu, v1.x & 0x7FFF7FFFu),
                                     __vmaxu2(v2.x & 0x7FFF7FFFu, v3.x & 0x7FFF7FFFu)));
      m[1] = __vmaxu2(m[1], __vmaxu2(__vmaxu2(v0.y & 0x7FFF7FFFu, v1.y & 0x7FFF7FFFu),
                                     __vmaxu2(v2.y & 0x7FFF7FFFu, v3.y & 0x7FFF7FFFu)));
      m[2] = __vmaxu2(m[2], __vmaxu2(__vmaxu2(v0.z & 0x7FFF7FFFu, v1.z & 0x7FFF7FFFu),
                                     __vmaxu2(v2.z & 0x7FFF7FFFu, v3.z & 0x7FFF7FFFu)));
      m[3] = __vmaxu2(m[3], __vmaxu2(__vmaxu2(v0.w & 0x7FFF7FFFu, v1.w & 0x7FFF7FFFu),
                                     __vmaxu2(v2.w & 0x7FFF7FFFu, v3.w & 0x7FFF7FFFu)));
    }
    for (; r < rows; r += rstep) {
      uint4 v = __ldcs(reinterpret_cast<const uint4*>(p + r * lda));
      m[0] = __vmaxu2(m[0], v.x & 0x7FFF7FFFu);
      m[1] = __vmaxu2(m[1], v.y & 0x7FFF7FFFu);
      m[2] = __vmaxu2(m[2], v.z & 0x7FFF7FFFu);
      m[3] = __vmaxu2(m[3], v.w & 0x7FFF7FFFu);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) red[threadIdx.y][threadIdx.x][i] = m[i];
  __syncthreads();
  if (threadIdx.y == 0 && col0 < cols) {
#pragma unroll
    for (int y = 1; y < 8; ++y)
#pragma unroll
      for (int i = 0; i < 4; ++i) m[i] = __vmaxu2(m[i], red[y][threadIdx.x][i]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // low half = column col0 + 2i, high half = col0 + 2i + 1; bf16 -> f32 bits
      atomicMax(out_bits + col0 + 2 * i, (m[i] & 0xFFFFu) << 16);
      atomicMax(out_bits + col0 + 2 * i + 1, m[i] & 0xFFFF0000u);
    }
  }
}

cudaError_t launch_colabsmax(const void* A, int64_t rows, int64_t cols, int64_t lda, float* absmax,
                             int reset, cudaStream_t stream) {
  if (reset) {
    cudaError_t e = cudaMemsetAsync(absmax, 0, static_cast<size_t>(cols) * sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  if (rows == 0 || cols == 0) return cudaSuccess;
  const int sms = device_num_sms();
  const int64_t gx = (cols + 255) / 256;
  int64_t want = (static_cast<int64_t>(sms) * 8 + gx - 1) / gx;      // ~8 blocks per SM
  int64_t maxy = (rows + 31) / 32;                                    // >= 4 rows per thread
  int64_t gy = want < maxy ? want : maxy;
  if (gy < 1) gy = 1;
  if (gy > 65535) gy = 65535;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  colabsmax_kernel<<<grid, dim3(32, 8), 0, stream>>>(static_cast<const uint16_t*>(A), rows, cols,
                                                     lda, reinterpret_cast<uint32_t*>(absmax));
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Finalisation, step 1 (element-wise): s, inv_s, score.
// ---------------------------------------------------------------------------
__global__ void finalize_scales_kernel(const float* __restrict__ act, const float* __restrict__ wsc,
                                       int d_in, double alpha, float* __restrict__ s,
                                       float* __restrict__ inv_s, float* __restrict__ score) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d_in) return;
  const double a = fmax(static_cast<double>(act[j]), 1e-5);
  const double w = fmax(static_cast<double>(wsc[j]), 1e-5);
  const float sj = static_cast<float>(pow(a, alpha) / pow(w, 1.0 - alpha));
  const float ij = static_cast<float>(1.0 / static_cast<double>(sj));
  s[j] = sj;
  inv_s[j] = ij;
  score[j] = __fmul_rn(act[j], ij);
}

// Step 2 (one block): order the columns by (score descending, index
// ascending) with a bitonic sort of 64-bit keys in shared memory, flag the
// first k as outliers, then compact the flags into O and jmap (both
// ascending).  Keys: high word 0xFFFFFFFF - score bits (non-negative floats
// order like their bit patterns), low word the column index; padding keys
// are all-ones and sort last.
constexpr int kFinalizeMaxD = 16384;
constexpr int kFinalizeThreads = 1024;

__global__ void __launch_bounds__(kFinalizeThreads)
    finalize_select_kernel(const float* __restrict__ score, int d_in, int k,
                           int32_t* __restrict__ O, int32_t* __restrict__ jmap) {
  extern __shared__ __align__(16) uint8_t fsmem[];
  uint64_t* key = reinterpret_cast<uint64_t*>(fsmem);                  // [n]
  int* cnt = reinterpret_cast<int*>(fsmem + kFinalizeMaxD * 8);         // [1024]
  uint8_t* flag = fsmem + kFinalizeMaxD * 8 + kFinalizeThreads * 4;     // [d_in]
  int n = 1;
  while (n < d_in) n <<= 1;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    if (i < d_in) {
      const uint32_t b = __float_as_uint(score[i]);
      key[i] = (static_cast<uint64_t>(0xFFFFFFFFu - b) << 32) | static_cast<uint32_t>(i);
      flag[i] = 0;
    } else {
      key[i] = ~0ull;
    }
  }
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
        const int i = 2 * t - (t & (stride - 1));      // lower element of the pair
        const int j = i + stride;
        const bool up = (i & size) == 0;
        const uint64_t a = key[i], b = key[j];
        if ((a > b) == up) {
          key[i] = b;
          key[j] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int r = threadIdx.x; r < k; r += blockDim.x) flag[static_cast<uint32_t>(key[r])] = 1;
  __syncthreads();
  const int per = (d_in + kFinalizeThreads - 1) / kFinalizeThreads;
  const int lo = threadIdx.x * per < d_in ? threadIdx.x * per : d_in;
  const int hi = lo + per < d_in ? lo + per : d_in;
  int c = 0;
  for (int j = lo; j < hi; ++j) c += flag[j];
  cnt[threadIdx.x] = c;
  __syncthreads();
  for (int off = 1; off < kFinalizeThreads; off <<= 1) {     // inclusive scan
    const int v = threadIdx.x >= off ? cnt[threadIdx.x - off] : 0;
    __syncthreads();
    cnt[threadIdx.x] += v;
    __syncthreads();
  }
  int o = cnt[threadIdx.x] - c;          // outliers before this run
  int jj = lo - o;                       // kept columns before this run
  for (int j = lo; j < hi; ++j) {
    if (flag[j]) {
      O[o++] = j;
    } else {
      jmap[jj++] = j;
    }
  }
}

size_t finalize_smem_bytes() {
  return static_cast<size_t>(kFinalizeMaxD) * 8 + kFinalizeThreads * 4 + kFinalizeMaxD;
}

int finalize_max_d() { return kFinalizeMaxD; }

cudaError_t launch_finalize(const float* act, const float* wsc, int d_in, double alpha, int k,
                            float* s, float* inv_s, float* score, int32_t* O, int32_t* jmap,
                            cudaStream_t stream) {
  const int nb = (d_in + 255) / 256;
  finalize_scales_kernel<<<nb, 256, 0, stream>>>(act, wsc, d_in, alpha, s, inv_s, score);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = finalize_smem_bytes();
  e = cudaFuncSetAttribute(finalize_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  finalize_select_kernel<<<1, kFinalizeThreads, smem, stream>>>(score, d_in, k, O, jmap);
  return cudaGetLastError();
}

}  // namespace w4a4
