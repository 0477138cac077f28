// Calibration kernels: per-column absolute maximum of a bf16 matrix, and the
// device-side finalisation (smoothing factor, score, top-k outlier set).
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.1-3.2 (per-channel magnitudes, s_j = a_j^alpha / w_j^(1-alpha)) and
// sec. 3.3 (score_j = max_t |x_tj|, static top-k set O).
#include "w4a4_internal.h"

namespace w4a4 {

// ---------------------------------------------------------------------------
// Column absmax of one or two matrices with the same columns (a layer's X
// and W share d_in) in one launch.  Block = 32 x 8 threads; threadIdx.x owns
// 8 consecutive columns (one 16-byte load per row), threadIdx.y and the
// block row stride over rows; block rows 0 .. p0.gy-1 reduce p0, the others
// p1.  Magnitudes are compared as bf16 bit patterns with the sign cleared
// (for non-NaN values the integer order is the magnitude order; NaN patterns
// lie above +inf, so a NaN makes the column NaN), packed two per 32-bit
// word.  The block result goes to global memory with an integer atomicMax
// on the float32 bits, which orders non-negative floats correctly.
// HBM-bound: 2 bytes read per element.
// ---------------------------------------------------------------------------
struct AbsmaxPart {
  const uint16_t* A;
  int64_t rows, lda;
  uint32_t* out;     // float32 bits [cols]
  int gy;            // block rows given to this matrix
};

__global__ void __launch_bounds__(256) colabsmax_kernel(const AbsmaxPart p0, const AbsmaxPart p1,
                                                        int64_t cols) {
  __shared__ uint32_t red[8][32][4];
  pdl_wait();
  pdl_launch_dependents();
  const bool second = static_cast<int>(blockIdx.y) >= p0.gy;
  const uint16_t* A = second ? p1.A : p0.A;
  const int64_t rows = second ? p1.rows : p0.rows;
  const int64_t lda = second ? p1.lda : p0.lda;
  const int gy = second ? p1.gy : p0.gy;
  const int by = second ? static_cast<int>(blockIdx.y) - p0.gy : static_cast<int>(blockIdx.y);
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x) * 8;
  constexpr uint32_t kMag = 0x7FFF7FFFu;
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  if (col0 < cols) {
    const int64_t rstep = static_cast<int64_t>(gy) * 8;
    int64_t r = static_cast<int64_t>(by) * 8 + threadIdx.y;
    const uint16_t* p = A + col0;
    // eight rows in flight per iteration, folded pairwise (measured against
    // four: 5.98 -> 6.61 TB/s on a 57600 x 5120 X)
    for (; r + 7 * rstep < rows; r += 8 * rstep) {
      uint4 u0 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 4 * rstep) * lda));
      uint4 u1 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 5 * rstep) * lda));
      uint4 u2 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 6 * rstep) * lda));
      uint4 u3 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 7 * rstep) * lda));
      uint4 v0 = __ldcs(reinterpret_cast<const uint4*>(p + r * lda));
      uint4 v1 = __ldcs(reinterpret_cast<const uint4*>(p + (r + rstep) * lda));
      uint4 v2 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 2 * rstep) * lda));
      uint4 v3 = __ldcs(reinterpret_cast<const uint4*>(p + (r + 3 * rstep) * lda));
      v0.x = __vmaxu2(v0.x & kMag, u0.x & kMag); v0.y = __vmaxu2(v0.y & kMag, u0.y & kMag);
      v0.z = __vmaxu2(v0.z & kMag, u0.z & kMag); v0.w = __vmaxu2(v0.w & kMag, u0.w & kMag);
      v1.x = __vmaxu2(v1.x & kMag, u1.x & kMag); v1.y = __vmaxu2(v1.y & kMag, u1.y & kMag);
      v1.z = __vmaxu2(v1.z & kMag, u1.z & kMag); v1.w = __vmaxu2(v1.w & kMag, u1.w & kMag);
      v2.x = __vmaxu2(v2.x & kMag, u2.x & kMag); v2.y = __vmaxu2(v2.y & kMag, u2.y & kMag);
      v2.z = __vmaxu2(v2.z & kMag, u2.z & kMag); v2.w = __vmaxu2(v2.w & kMag, u2.w & kMag);
      v3.x = __vmaxu2(v3.x & kMag, u3.x & kMag); v3.y = __vmaxu2(v3.y & kMag, u3.y & kMag);
      v3.z = __vmaxu2(v3.z & kMag, u3.z & kMag); v3.w = __vmaxu2(v3.w & kMag, u3.w & kMag);
      m[0] = __vmaxu2(m[0], __vmaxu2(__vmaxu2(v0.x, v1.x), __vmaxu2(v2.x, v3.x)));
      m[1] = __vmaxu2(m[1], __vmaxu2(__vmaxu2(v0.y, v1.y), __vmaxu2(v2.y, v3.y)));
      m[2] = __vmaxu2(m[2], __vmaxu2(__vmaxu2(v0.z, v1.z), __vmaxu2(v2.z, v3.z)));
      m[3] = __vmaxu2(m[3], __vmaxu2(__vmaxu2(v0.w, v1.w), __vmaxu2(v2.w, v3.w)));
    }
    for (; r < rows; r += rstep) {
      uint4 v = __ldcs(reinterpret_cast<const uint4*>(p + r * lda));
      m[0] = __vmaxu2(m[0], v.x & kMag);
      m[1] = __vmaxu2(m[1], v.y & kMag);
      m[2] = __vmaxu2(m[2], v.z & kMag);
      m[3] = __vmaxu2(m[3], v.w & kMag);
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
    uint32_t* out = second ? p1.out : p0.out;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // low half = column col0 + 2i, high half = col0 + 2i + 1; bf16 -> f32 bits
      atomicMax(out + col0 + 2 * i, (m[i] & 0xFFFFu) << 16);
      atomicMax(out + col0 + 2 * i + 1, m[i] & 0xFFFF0000u);
    }
  }
}

// Resident blocks of colabsmax_kernel per SM (cached per device).
static int colabsmax_blocks_per_sm() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 4;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, colabsmax_kernel, 256, 0) != cudaSuccess ||
        n <= 0)
      n = 4;
    cached[dev] = n;
  }
  return cached[dev];
}

// One launch over A0 (rows0 rows) and, if rows1 > 0, A1, both `cols` wide.
// The grid is one wave of resident blocks (a second, partial wave left a
// tail: 0.1345 -> 0.1262 ms for X and W of the 5120-column layer at
// T = 57600 with both in one launch), its block rows split between the two
// matrices in proportion to their rows, at least 4 rows per thread.
cudaError_t launch_colabsmax2(const void* A0, int64_t rows0, int64_t lda0, float* out0,
                              const void* A1, int64_t rows1, int64_t lda1, float* out1,
                              int64_t cols, int reset, cudaStream_t stream) {
  if (reset) {
    cudaError_t e = cudaMemsetAsync(out0, 0, static_cast<size_t>(cols) * sizeof(float), stream);
    if (e == cudaSuccess && out1 != nullptr)
      e = cudaMemsetAsync(out1, 0, static_cast<size_t>(cols) * sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  if (cols == 0 || rows0 + rows1 == 0) return cudaSuccess;
  const int64_t sms = device_num_sms() > 0 ? device_num_sms() : 148;
  const int64_t gx = (cols + 255) / 256;
  int64_t total = sms * colabsmax_blocks_per_sm() / gx;
  if (total < 2) total = 2;
  auto cap = [](int64_t gy, int64_t rows) -> int64_t {
    if (rows == 0) return 0;
    const int64_t maxy = (rows + 31) / 32;               // >= 4 rows per thread
    if (gy > maxy) gy = maxy;
    return gy < 1 ? 1 : gy;
  };
  const int64_t gy0 = cap((total * rows0 + (rows0 + rows1) / 2) / (rows0 + rows1), rows0);
  const int64_t gy1 = cap(total - gy0, rows1);
  AbsmaxPart p0{static_cast<const uint16_t*>(A0), rows0, lda0, reinterpret_cast<uint32_t*>(out0),
                static_cast<int>(gy0)};
  AbsmaxPart p1{static_cast<const uint16_t*>(A1), rows1, lda1, reinterpret_cast<uint32_t*>(out1),
                static_cast<int>(gy1)};
  return launch_pdl(colabsmax_kernel, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy0 + gy1)),
                    dim3(32, 8), 0, stream, p0, p1, cols);
}

cudaError_t launch_colabsmax(const void* A, int64_t rows, int64_t cols, int64_t lda, float* absmax,
                             int reset, cudaStream_t stream) {
  return launch_colabsmax2(A, rows, lda, absmax, nullptr, 0, lda, nullptr, cols, reset, stream);
}

// ---------------------------------------------------------------------------
// Finalisation, step 1 (element-wise): s, inv_s, score.
// ---------------------------------------------------------------------------
__global__ void finalize_scales_kernel(const float* __restrict__ act, const float* __restrict__ wsc,
                                       int d_in, double alpha, float* __restrict__ s,
                                       float* __restrict__ inv_s, float* __restrict__ score) {
  pdl_wait();
  pdl_launch_dependents();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d_in) return;
  // s is defined for finite magnitudes only: an infinite or NaN one (from
  // non-finite calibration data) is reported, and that column's s, inv_s,
  // score and the selection are then unspecified
  if (!isfinite(act[j]) || !isfinite(wsc[j])) atomicOr(&g_device_error, DEVERR_NONFINITE_CALIB);
  const double a = fmax(static_cast<double>(act[j]), 1e-5);
  const double w = fmax(static_cast<double>(wsc[j]), 1e-5);
  const float sj = static_cast<float>(pow(a, alpha) / pow(w, 1.0 - alpha));
  const float ij = static_cast<float>(1.0 / static_cast<double>(sj));
  s[j] = sj;
  inv_s[j] = ij;
  score[j] = __fmul_rn(act[j], ij);
}

// Step 2 (one block): select the k columns of largest (score, -index) --
// score descending, lower index first among equal scores -- then compact the
// selection into O and the rest into jmap (both ascending).
//
// Selection is a radix select on a 48-bit key per column, 8 bits per pass
// from the top: key = score bits << 16 | (0xFFFF - index).  Non-negative
// floats order like their bit patterns and the low field breaks ties towards
// the lower index, so keys are distinct and the k largest keys are exactly the
// k columns wanted.  Each pass histograms the candidates that still match the
// prefix found so far, and one warp picks the digit holding the k-th largest
// key.  Thread t owns the contiguous columns [t*per, (t+1)*per), which keeps
// the final compaction in index order with one block-wide scan.
constexpr int kFinalizeMaxD = 16384;
constexpr int kFinalizeThreads = 1024;
constexpr int kFinalizePer = kFinalizeMaxD / kFinalizeThreads;   // columns per thread, at most

__global__ void __launch_bounds__(kFinalizeThreads)
    finalize_select_kernel(const float* __restrict__ score, int d_in, int k,
                           int32_t* __restrict__ O, int32_t* __restrict__ jmap) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_cnt[kFinalizeThreads / 32];
  __shared__ uint64_t sel_prefix;
  __shared__ uint32_t sel_remaining;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int per = (d_in + kFinalizeThreads - 1) / kFinalizeThreads;
  const int lo = tid * per < d_in ? tid * per : d_in;
  const int hi = lo + per < d_in ? lo + per : d_in;

  uint64_t key[kFinalizePer];
#pragma unroll
  for (int e = 0; e < kFinalizePer; ++e) {
    const int j = lo + e;
    key[e] = j < hi ? (static_cast<uint64_t>(__float_as_uint(score[j])) << 16) |
                          static_cast<uint64_t>(0xFFFFu - static_cast<uint32_t>(j))
                    : 0ull;
  }

  // threshold = the k-th largest key (keys are distinct); selected: key >= threshold
  uint64_t thr = ~0ull;                    // k == 0: nothing reaches it
  if (k > 0) {
    if (tid == 0) {
      sel_prefix = 0;
      sel_remaining = static_cast<uint32_t>(k);
    }
    for (int shift = 40; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += kFinalizeThreads) hist[b] = 0;
      __syncthreads();
      const uint64_t prefix = sel_prefix;
      const uint64_t above = shift + 8 < 64 ? ~0ull << (shift + 8) : 0ull;
#pragma unroll
      for (int e = 0; e < kFinalizePer; ++e)
        if (lo + e < hi && (key[e] & above) == prefix)
          atomicAdd(&hist[(key[e] >> shift) & 0xFFu], 1u);
      __syncthreads();
      if (warp == 0) {
        // lane l covers digits 8l .. 8l+7; count the candidates above each lane's range
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          c[q] = hist[8 * lane + q];
          sum += c[q];
        }
        uint32_t incl = sum;                 // inclusive suffix sum over lanes l..31
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, off);
          if (lane + off < 32) incl += v;
        }
        const uint32_t rem = sel_remaining;
        uint32_t acc = incl - sum;           // candidates with a digit above this lane's range
        if (acc < rem && rem <= incl) {      // exactly one lane
          int d = 7;
          while (d > 0 && acc + c[d] < rem) {
            acc += c[d];
            --d;
          }
          sel_prefix = prefix | (static_cast<uint64_t>(8 * lane + d) << shift);
          sel_remaining = rem - acc;
        }
      }
      __syncthreads();
    }
    thr = sel_prefix;
  }

  // compaction in index order
  uint32_t flags = 0, c = 0;
#pragma unroll
  for (int e = 0; e < kFinalizePer; ++e)
    if (lo + e < hi && key[e] >= thr) {
      flags |= 1u << e;
      ++c;
    }
  uint32_t incl = c;                         // inclusive scan over the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_cnt[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_cnt[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += v;
    }
    warp_cnt[lane] = w;                      // inclusive over warps
  }
  __syncthreads();
  int o = static_cast<int>(incl - c + (warp > 0 ? warp_cnt[warp - 1] : 0u));   // outliers before lo
  int jj = lo - o;                                                               // kept columns before lo
#pragma unroll
  for (int e = 0; e < kFinalizePer; ++e) {
    const int j = lo + e;
    if (j < hi) {
      if ((flags >> e) & 1u)
        O[o++] = j;
      else
        jmap[jj++] = j;
    }
  }
}

int finalize_max_d() { return kFinalizeMaxD; }

cudaError_t launch_finalize(const float* act, const float* wsc, int d_in, double alpha, int k,
                            float* s, float* inv_s, float* score, int32_t* O, int32_t* jmap,
                            cudaStream_t stream) {
  const int nb = (d_in + 255) / 256;
  cudaError_t e = launch_pdl(finalize_scales_kernel, dim3(nb), dim3(256), 0, stream, act, wsc, d_in,
                             alpha, s, inv_s, score);
  if (e != cudaSuccess) return e;
  return launch_pdl(finalize_select_kernel, dim3(1), dim3(kFinalizeThreads), 0, stream, score, d_in, k,
                    O, jmap);
}

}  // namespace w4a4
