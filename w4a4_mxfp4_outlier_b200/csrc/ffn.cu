// The FFN of the Wan2.2 DiT block as two quantised projections with GELU
// between them.  The review quantises both projections (ffn.0 up, ffn.2 down;
// sec. 3.1, 3.5) with the same recipe; this file lets the up projection's
// GEMM hand its output to the down projection already quantised.
//
// The down layer's activation prep compacts its input channels (J first in
// ascending order, O removed) before forming 32-wide MX blocks.  If the up
// layer's output channels are stored in that same order -- its weight rows
// permuted to perm = [jmap_down..., O_down...] -- then compacted position p of
// the down layer is simply output column p of the up layer, an MX block is 32
// consecutive output columns, and the outliers are the last k columns.  The
// up GEMM's epilogue then applies GELU and the down layer's prep to each
// lane's 32 accumulator columns directly (see act_block in gemm.cu), and the
// bf16 Y of the up layer is never written.
#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

// X = bf16(gelu(Y)) elementwise (the unfused form of the FFN activation),
// with the same table and closed forms the fused GEMM epilogue uses.  Rows of
// 8-element multiples at 16-byte alignment (`vec`) move as 16-byte vectors,
// two per thread in flight; anything else goes element by element.
__device__ __forceinline__ uint32_t gelu_pair(uint32_t tab, uint32_t p) {
  return gelu_bf16(tab, p & 0xFFFFu) | (gelu_bf16(tab, p >> 16) << 16);
}

__device__ __forceinline__ uint4 gelu_vec8(uint32_t tab, uint4 v) {
  return make_uint4(gelu_pair(tab, v.x), gelu_pair(tab, v.y), gelu_pair(tab, v.z), gelu_pair(tab, v.w));
}

__global__ void __launch_bounds__(512) gelu_bf16_kernel(const uint16_t* __restrict__ Y, int64_t ldy,
                                                        uint16_t* __restrict__ X, int64_t ldx,
                                                        int64_t T, int64_t d, int vec) {
  __shared__ __align__(16) uint16_t tab[kGeluTabEntries];
  gelu_table_fill(tab, threadIdx.x, blockDim.x);
  __syncthreads();
  const uint32_t tab_s = smem_u32(tab);
  if (vec) {
    const int64_t nv = d >> 3;
    const int64_t bd = blockDim.x;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
      const uint4* y = reinterpret_cast<const uint4*>(Y + t * ldy);
      uint4* x = reinterpret_cast<uint4*>(X + t * ldx);
      for (int64_t j = threadIdx.x; j < nv; j += 2 * bd) {
        const bool two = j + bd < nv;
        const uint4 a = y[j];
        const uint4 b = two ? y[j + bd] : make_uint4(0u, 0u, 0u, 0u);
        x[j] = gelu_vec8(tab_s, a);
        if (two) x[j + bd] = gelu_vec8(tab_s, b);
      }
    }
    return;
  }
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* y = Y + t * ldy;
    uint16_t* x = X + t * ldx;
    for (int64_t j = threadIdx.x; j < d; j += blockDim.x)
      x[j] = static_cast<uint16_t>(gelu_bf16(tab_s, y[j]));
  }
}

// perm = [jmap..., O...]; inv_s_perm[c] = inv_s[perm[c]]
__global__ void ffn_link_kernel(const float* __restrict__ inv_s, const int32_t* __restrict__ O,
                                const int32_t* __restrict__ jmap, int kj, int k,
                                int32_t* __restrict__ perm, float* __restrict__ inv_s_perm) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= kj + k) return;
  const int j = c < kj ? jmap[c] : O[c - kj];
  perm[c] = j;
  inv_s_perm[c] = inv_s[j];
}

// dst row r = src row rows[r] for r < n (rows past n, the padding, copied in
// place); rows of row_vecs 16-byte vectors
__global__ void permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                    const int32_t* __restrict__ rows, int64_t n, int64_t nrows,
                                    int64_t row_vecs) {
  const int64_t total = nrows * row_vecs;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / row_vecs, c = i - r * row_vecs;
    const int64_t from = r < n ? rows[r] : r;
    dst[r * row_vecs + c] = src[from * row_vecs + c];
  }
}

// the same for the E8M0 scale bytes, which sit in the MMA's atom layout
__global__ void permute_sf_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                  const int32_t* __restrict__ rows, int64_t n, int64_t nrows,
                                  int64_t nblk) {
  const int64_t total = nrows * nblk;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / nblk, b = i - r * nblk;
    const int64_t from = r < n ? rows[r] : r;
    dst[sf_offset(r, b, nblk)] = src[sf_offset(from, b, nblk)];
  }
}

}  // namespace w4a4

using namespace w4a4;

extern "C" w4a4_status w4a4_gelu_bf16(const void* Y, int64_t T, int64_t d, int64_t ldy, void* X,
                                      int64_t ldx, void* stream) {
  if (T < 0 || d < 0 || ldy < d || ldx < d) return W4A4_ERR_INVALID_ARG;
  if (T == 0 || d == 0) return W4A4_OK;
  if (Y == nullptr || X == nullptr) return W4A4_ERR_INVALID_ARG;
  const int64_t sms = device_num_sms() > 0 ? device_num_sms() : 148;
  // every CTA first fills its own table, so keep the grid to about two per SM
  const int64_t grid = T < 2 * sms ? T : 2 * sms;
  const int vec = ((d | ldy | ldx) & 7) == 0 && aligned16(Y) && aligned16(X);
  gelu_bf16_kernel<<<static_cast<unsigned>(grid), 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(Y), ldy, static_cast<uint16_t*>(X), ldx, T, d, vec);
  return cudaGetLastError() == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

extern "C" w4a4_status w4a4_ffn_link(const w4a4_packed_weight* next, int32_t* perm,
                                     float* inv_s_perm, void* stream) {
  Geometry g;
  const w4a4_status st = check_pw(next, &g);
  if (st != W4A4_OK) return st;
  if (perm == nullptr || inv_s_perm == nullptr) return W4A4_ERR_INVALID_ARG;
  const int n = static_cast<int>(g.d_in);
  if (n == 0) return W4A4_OK;
  ffn_link_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      next->inv_s, next->O, next->jmap, static_cast<int>(g.kj), static_cast<int>(g.k), perm,
      inv_s_perm);
  return cudaGetLastError() == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

extern "C" w4a4_status w4a4_pack_weight_rows(const void* W, int64_t ldw, const float* s,
                                             const int32_t* rows, const w4a4_packed_weight* pw,
                                             void* stream) {
  Geometry g;
  const w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (W == nullptr || s == nullptr || rows == nullptr || ldw < g.d_in) return W4A4_ERR_INVALID_ARG;
  if (ldw % 8 != 0 || !aligned16(W)) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_pack(W, ldw, s, pw->O, pw->jmap, g, pw->layout, pw->wq, pw->sfb,
                               pw->w_hp, static_cast<cudaStream_t>(stream), rows));
}

extern "C" w4a4_status w4a4_gemm_dual_act(const uint8_t* aq, const uint8_t* sfa, const void* xo,
                                          int64_t T, const w4a4_packed_weight* pw,
                                          const w4a4_packed_weight* next, const float* inv_s_perm,
                                          uint8_t* aq_next, uint8_t* sfa_next, void* xo_next,
                                          void* stream) {
  Geometry g, gn;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  st = check_pw(next, &gn);
  if (st != W4A4_OK) return st;
  if (next->d_in != pw->d_out || T < 0 || inv_s_perm == nullptr) return W4A4_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 256) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return W4A4_OK;
  if ((g.kj > 0 && (aq == nullptr || sfa == nullptr)) || (g.k > 0 && xo == nullptr) ||
      (gn.kj > 0 && (aq_next == nullptr || sfa_next == nullptr)) || (gn.k > 0 && xo_next == nullptr))
    return W4A4_ERR_INVALID_ARG;
  if ((aq && !aligned16(aq)) || (sfa && !aligned16(sfa)) || (xo && !aligned16(xo)) ||
      (aq_next && !aligned16(aq_next)) || (xo_next && !aligned16(xo_next)))
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ActOut act;
  act.inv_s = inv_s_perm;
  act.aq = aq_next;
  act.sfa = sfa_next;
  act.xo = xo_next;
  act.kj = gn.kj;
  act.nblk = gn.nblk;
  act.k_pad = gn.k_pad;
  // the GEMM's tensor maps are built before anything is enqueued
  GemmPlan plan;
  if (plan_gemm(aq, sfa, xo, T, g, pw->wq, pw->sfb, pw->w_hp, nullptr, g.d_out, &act, &plan) !=
      cudaSuccess)
    return W4A4_ERR_CUDA;
  // X_O padding columns k .. k_pad that no output column reaches start at zero
  if (gn.k_pad > gn.k) {
    const cudaError_t e = cudaMemset2DAsync(static_cast<uint8_t*>(xo_next) + gn.k * 2,
                                            static_cast<size_t>(gn.k_pad) * 2, 0,
                                            static_cast<size_t>(gn.k_pad - gn.k) * 2,
                                            static_cast<size_t>(T), s);
    if (e != cudaSuccess) return W4A4_ERR_CUDA;
  }
  return from_cuda(run_gemm(plan, s));
}

extern "C" w4a4_status w4a4_permute_packed_rows(const w4a4_packed_weight* src, const int32_t* rows,
                                                const w4a4_packed_weight* dst, void* stream) {
  Geometry g, gd;
  w4a4_status st = check_pw(src, &g);
  if (st != W4A4_OK) return st;
  st = check_pw(dst, &gd);
  if (st != W4A4_OK) return st;
  if (rows == nullptr || src->d_in != dst->d_in || src->d_out != dst->d_out || src->k != dst->k ||
      src->layout != dst->layout)
    return W4A4_ERR_INVALID_ARG;
  if ((g.kj > 0 && (src->wq == dst->wq || src->sfb == dst->sfb)) ||
      (g.k > 0 && src->w_hp == dst->w_hp))
    return W4A4_ERR_INVALID_ARG;                       // not in place
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = device_num_sms() > 0 ? device_num_sms() : 148;
  const int grid = 4 * sms;
  if (g.kj > 0) {
    permute_rows_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(src->wq),
                                             reinterpret_cast<uint4*>(dst->wq), rows, g.d_out,
                                             g.d_out, g.kj_pad / 2 / 16);
    permute_sf_kernel<<<grid, 256, 0, s>>>(src->sfb, dst->sfb, rows, g.d_out, g.sfb_rows, g.nblk);
  }
  if (g.k > 0)
    permute_rows_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(src->w_hp),
                                             reinterpret_cast<uint4*>(dst->w_hp), rows, g.d_out,
                                             g.d_out, g.k_pad * 2 / 16);
  return cudaGetLastError() == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}
