// Internal declarations shared by the translation units of libw4a4.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "w4a4_device.cuh"

namespace w4a4 {

constexpr int kKTileElems = 256;   // compacted 4-bit K elements per GEMM K tile (128 bytes)
constexpr int kSfbRowPad = 256;    // scale rows of B are padded to the GEMM N tile
constexpr int kSfaRowPad = 128;    // scale rows of A are padded to the GEMM M tile

struct Geometry {
  int64_t d_in, d_out, k;
  int64_t kj, kj_pad, nblk, k_pad, sfb_rows;
};

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

inline Geometry make_geometry(int64_t d_in, int64_t d_out, int64_t k) {
  Geometry g;
  g.d_in = d_in;
  g.d_out = d_out;
  g.k = k;
  g.kj = d_in - k;
  g.kj_pad = round_up(g.kj, kKTileElems);
  g.nblk = g.kj_pad / 32;
  g.k_pad = round_up(k, 16);
  g.sfb_rows = round_up(d_out, kSfbRowPad);
  return g;
}

// Byte offset of the scale of (row r, block b) in the block-scaled MMA
// layout with nblk blocks per row (nblk a multiple of 4): 512-byte atoms of
// 128 rows x 4 blocks, K-major; inside an atom (r%32)*16 + ((r%128)/32)*4 + b%4.
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int64_t nblk) {
  return (((r >> 7) * (nblk >> 2) + (b >> 2)) << 9) + ((r & 31) << 4) + (((r & 127) >> 5) << 2) +
         (b & 3);
}

int device_num_sms();

// Launch attributes of a kernel that calls pdl_wait() before its first
// global-memory access: programmatic dependent launch, so its launch and
// setup overlap the end of the previous kernel in the stream.
// W4A4_NO_PDL=1 in the environment turns it off (read once per process).
bool pdl_enabled();
inline int pdl_attrs(cudaLaunchAttribute* attr) {
  if (!pdl_enabled()) return 0;
  attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr->val.programmaticStreamSerializationAllowed = 1;
  return 1;
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = static_cast<unsigned>(pdl_attrs(attr));
  cfg.attrs = attr;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_colabsmax(const void* A, int64_t rows, int64_t cols, int64_t lda, float* absmax,
                             int reset, cudaStream_t stream);
// both matrices in one launch (A1 may have 0 rows; out1 is then unused)
cudaError_t launch_colabsmax2(const void* A0, int64_t rows0, int64_t lda0, float* out0,
                              const void* A1, int64_t rows1, int64_t lda1, float* out1,
                              int64_t cols, int reset, cudaStream_t stream);
cudaError_t launch_finalize(const float* act, const float* wsc, int d_in, double alpha, int k,
                            float* s, float* inv_s, float* score, int32_t* O, int32_t* jmap,
                            cudaStream_t stream);
int finalize_max_d();
// rows (optional, device int32 [d_out]): packed row n is W row rows[n]
cudaError_t launch_pack(const void* W, int64_t ldw, const float* s, const int32_t* O,
                        const int32_t* jmap, const Geometry& g, int layout, uint8_t* wq,
                        uint8_t* sfb, void* w_hp, cudaStream_t stream,
                        const int32_t* rows = nullptr);
// stripe4 = true: one exponent per 4 consecutive blocks (128x1 weight stripes);
// rows (optional, device int32 [T]): output row r reads input row rows[r].
cudaError_t launch_prep(const void* X, int64_t T, int64_t ldx, const float* inv_s,
                        const int32_t* O, const int32_t* jmap, const Geometry& g, uint8_t* aq,
                        uint8_t* sfa, void* xo, cudaStream_t stream, bool stripe4 = false,
                        const int32_t* rows = nullptr);
bool prep_supported(const Geometry& g);
// The block-per-lane form of the same computation (prep_block.cu).
bool prep_block_supported(const Geometry& g);
cudaError_t launch_prep_block(const void* X, int64_t T, int64_t ldx, const float* inv_s,
                              const int32_t* O, const int32_t* jmap, const Geometry& g,
                              uint8_t* aq, uint8_t* sfa, void* xo, cudaStream_t stream,
                              bool stripe4, const int32_t* rows);
// Outputs of the fused FFN epilogue: the next layer's activation buffers
// (Aq, SFA, X_O) and its inv_s in this layer's output-column order.
struct ActOut {
  const float* inv_s;
  uint8_t* aq;
  uint8_t* sfa;
  void* xo;
  int64_t kj, nblk, k_pad;
};
// Kernel arguments of the dual-branch GEMM (both kernels of gemm.cu).
struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  __nv_bfloat16* Y;
  int64_t ldy;
  int T;
  int d_out;
  int nblk;          // scale blocks per row (kj_pad / 32)
  int kt_o;          // bf16 K tiles (64 columns each)
  int kt_j;          // MXFP4 K tiles (256 columns each)
  int k_pad;         // bf16 columns (multiple of 16)
  int tiles_m, tiles_n;
  // Fused FFN epilogue (kernels instantiated with kAct): Y is not stored;
  // column c of the tile row feeds the next layer, whose input channel c is
  // its compacted J position c for c < act_kj and outlier c - act_kj after:
  //   v = fl32(bf16(gelu(bf16(acc))) * act_inv_s[c])
  // J blocks are MXFP4-encoded into act_aq / act_sfa, outliers go to act_xo.
  const float* act_inv_s;   // [d_out] inv_s of the next layer in this column order
  uint8_t* act_aq;          // [T, act_nblk * 16]
  uint8_t* act_sfa;         // MMA layout, act_nblk blocks per row
  __nv_bfloat16* act_xo;    // [T, act_k_pad]
  int act_kj, act_nblk, act_k_pad;
};

// A GEMM launch split in two: plan_gemm does the host work (tile choice,
// tensor maps, arguments) and enqueues nothing; run_gemm enqueues the kernel.
struct GemmPlan {
  CUtensorMap tm_a, tm_b, tm_ao, tm_bo, tm_sfa, tm_sfb, tm_y;
  GemmArgs a;
  size_t smem;
  int grid, tile_n;
  bool pair, act, empty;
};
cudaError_t plan_gemm(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                      const Geometry& g, const uint8_t* wq, const uint8_t* sfb, const void* w_hp,
                      void* Y, int64_t ldy, const ActOut* act, GemmPlan* p);
cudaError_t run_gemm(const GemmPlan& p, cudaStream_t stream);
// act == nullptr: Y = bf16 product.  Otherwise Y is not written and the
// product feeds `act` (see GemmArgs).
cudaError_t launch_gemm(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                        const Geometry& g, const uint8_t* wq, const uint8_t* sfb, const void* w_hp,
                        void* Y, int64_t ldy, cudaStream_t stream, const ActOut* act = nullptr);

}  // namespace w4a4
