// Offline weight packing: fold the smoothing factor into W, move the outlier
// channels into a bf16 matrix, MXFP4-encode the compacted remaining channels
// and write their E8M0 scales in the block-scaled MMA layout.
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.2 (s folded into the master weight offline), sec. 3.3 (O channels
// kept in high precision, J in 4 bits), sec. 3.4 (block-wise scales, 32x32
// tiles or K-major stripes; exponent stored beside the 4-bit payload).
#include "w4a4_internal.h"

namespace w4a4 {

// 32x32 tiles: one warp per (32-row group g, block b).  Lane l owns output row n = 32g + l
// and the 32 compacted positions p = 32b .. 32b+31 of that row.  For the 32x32
// tile layout the block maximum is reduced over the warp, so all 32 rows of
// the tile share one exponent.  Rows n >= d_out are zero (their scale code is
// 0) and only their scale bytes are stored (sfb is padded to sfb_rows).
__global__ void __launch_bounds__(256) pack_j_kernel(const uint16_t* __restrict__ W, int64_t ldw,
                                                     const float* __restrict__ s,
                                                     const int32_t* __restrict__ jmap, int kj,
                                                     int nblk, int d_out, int sfb_rows, int layout,
                                                     uint8_t* __restrict__ wq,
                                                     uint8_t* __restrict__ sfb,
                                                     const int32_t* __restrict__ rows) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int groups = sfb_rows / 32;
  if (warp >= groups * nblk) return;
  const int g = warp / nblk;
  const int b = warp % nblk;
  const int n = g * 32 + lane;
  const bool row_ok = n < d_out;
  const int64_t src_row = row_ok ? (rows ? rows[n] : n) : 0;
  float v[32];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int p = b * 32 + i;
    float x = 0.f;
    if (row_ok && p < kj) {
      const int j = jmap[p];
      x = __fmul_rn(__uint_as_float(static_cast<uint32_t>(W[src_row * ldw + j]) << 16), s[j]);
    }
    v[i] = x;
    amax = max_nan(amax, fabsf(x));       // NaN-propagating
  }
  if (layout == 1) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  }
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
  if (row_ok) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = cvt_e2m1x8(v[8 * q] * inv, v[8 * q + 1] * inv, v[8 * q + 2] * inv, v[8 * q + 3] * inv,
                        v[8 * q + 4] * inv, v[8 * q + 5] * inv, v[8 * q + 6] * inv,
                        v[8 * q + 7] * inv) &
             mx_nan_block_mask(code);
    const int64_t row_bytes = static_cast<int64_t>(nblk) * 16;
    *reinterpret_cast<uint4*>(wq + static_cast<int64_t>(n) * row_bytes + b * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  sfb[sf_offset(n, b, nblk)] = row_ok ? static_cast<uint8_t>(code) : static_cast<uint8_t>(0);
}

// W_hp[n, i] = bf16_rn(fl32(W[n, O[i]] * s[O[i]])) for i < k, 0 for k <= i < k_pad.
__global__ void pack_o_kernel(const uint16_t* __restrict__ W, int64_t ldw,
                              const float* __restrict__ s, const int32_t* __restrict__ O, int k,
                              int k_pad, int d_out, __nv_bfloat16* __restrict__ w_hp,
                              const int32_t* __restrict__ rows) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(d_out) * k_pad) return;
  const int n = static_cast<int>(idx / k_pad);
  const int i = static_cast<int>(idx % k_pad);
  float x = 0.f;
  if (i < k) {
    const int j = O[i];
    const int64_t src_row = rows ? rows[n] : n;
    x = __fmul_rn(__uint_as_float(static_cast<uint32_t>(W[src_row * ldw + j]) << 16), s[j]);
  }
  w_hp[idx] = __ushort_as_bfloat16(static_cast<unsigned short>(bf16_rn_bits(x)));
}

cudaError_t launch_pack(const void* W, int64_t ldw, const float* s, const int32_t* O,
                        const int32_t* jmap, const Geometry& g, int layout, uint8_t* wq,
                        uint8_t* sfb, void* w_hp, cudaStream_t stream, const int32_t* rows) {
  if (layout == W4A4_SF_32x1_KMAJOR || layout == W4A4_SF_128x1_KMAJOR) {
    // 32x1 / 128x1 stripes: the fold w * s_j, the compaction, the per-row
    // block encoding and the bf16 outlier columns are exactly what the
    // activation prep computes with s in place of inv_s (128x1: the amax
    // reduced over 4 blocks), so the rows of W stream through the prep
    // kernel (scale rows d_out .. sfb_rows are zeroed first).
    if (g.nblk > 0) {
      cudaError_t e = cudaMemsetAsync(sfb, 0, static_cast<size_t>(g.sfb_rows * g.nblk), stream);
      if (e != cudaSuccess) return e;
    }
    return launch_prep(W, g.d_out, ldw, s, O, jmap, g, wq, sfb, w_hp, stream,
                       layout == W4A4_SF_128x1_KMAJOR, rows);
  }
  if (g.nblk > 0) {
    const int64_t warps = (g.sfb_rows / 32) * g.nblk;
    const int64_t blocks = (warps * 32 + 255) / 256;
    pack_j_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(W), ldw, s, jmap, static_cast<int>(g.kj),
        static_cast<int>(g.nblk), static_cast<int>(g.d_out), static_cast<int>(g.sfb_rows), layout,
        wq, sfb, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (g.k_pad > 0) {
    const int64_t total = g.d_out * g.k_pad;
    pack_o_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint16_t*>(W), ldw, s, O, static_cast<int>(g.k), static_cast<int>(g.k_pad),
        static_cast<int>(g.d_out), static_cast<__nv_bfloat16*>(w_hp), rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace w4a4
