// Dual-branch GEMM  Y = X_J W^(q)_J + X_O W^(hp)_O  on the 5th-generation
// tensor cores (tcgen05) of sm_100a.
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.3 (eq. Y = X_J W^(q)_J + X_O W^(hp)_O; the J branch in W4A4 MXFP4,
// the O branch in 16-bit).
//
// One output tile is 128 tokens x 256 output channels; its float32
// accumulator lives in tensor memory (256 of the 512 columns).  The K loop
// first runs over the bf16 outlier columns (64 per K tile, kind::f16 MMAs
// with K = 16) and then over the compacted MXFP4 columns (256 per K tile,
// kind::mxf4 block-scaled MMAs with K = 64); both kinds accumulate into the
// same tensor-memory accumulator.  Every K tile is 128 bytes per row for
// both kinds, so one shared-memory ring (128-byte swizzle, filled by TMA)
// carries both.
//
// Roles (320 threads, persistent: CTA b handles tiles b, b+G, ...):
//   warp 0      TMA producer (one elected lane): A and B tiles by tensor-map
//               TMA, the matching E8M0 scale atoms by 1-D bulk copies.
//   warp 1      tensor-memory allocator; one lane issues tcgen05.cp (scales
//               into tensor memory) and tcgen05.mma, and commits to mbarriers.
//   warps 2-9   epilogue: each warp drains 32 lanes x 128 columns of the
//               accumulator (tcgen05.ld), releases it, converts to bf16 and
//               stores its rows of Y.
// Scale factors sit in tensor memory columns 256..279, rewritten for each
// K tile; tcgen05.cp and tcgen05.mma issued by one thread execute in order,
// so a rewrite never overtakes the MMAs that read the previous scales.
// Every wait is bounded (about 2 s); a role that gives up sets the device
// error word and an abort flag the others poll, and all roles then exit
// through the same teardown (drain in-flight copies / MMAs, free tensor
// memory).
#include <cuda.h>

#include "w4a4_internal.h"

namespace w4a4 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KT_BYTES = 128;                 // bytes per row per K tile (both kinds)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * KT_BYTES;        // 16 KB
constexpr int B_BYTES = BN * KT_BYTES;        // 32 KB
constexpr int SFA_BYTES = 1024;               // 2 K atoms x 512 B (128 rows)
constexpr int SFB_BYTES = 2048;               // 2 row blocks x 2 K atoms x 512 B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int GEMM_THREADS = 32 * (2 + NUM_EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SFA_COL = 256;             // 2 atoms x 4 columns
constexpr int TMEM_SFB_COL = 264;             // 2 atoms x 8 columns
constexpr int GROUP_M = 16;                   // tile raster: 16 M tiles per sweep of N

struct GemmSmem {
  uint8_t stage[STAGES][STAGE_BYTES];         // 1024-aligned (each part 1024-aligned)
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

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
};

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int per_group = GROUP_M * tiles_n;
  const int g = t / per_group;
  const int first_m = g * GROUP_M;
  const int gm = tiles_m - first_m < GROUP_M ? tiles_m - first_m : GROUP_M;
  const int w = t - g * per_group;
  tn = w / gm;
  tm = first_m + w % gm;
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_dual_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_ao, const __grid_constant__ CUtensorMap tm_bo,
                     const GemmArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile uint32_t* abort_flag = &sm.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = args.tiles_m * args.tiles_n;
  const int nkt = args.kt_o + args.kt_j;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, NUM_EPI_WARPS);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0u;
    fence_barrier_init();
    if (args.kt_j > 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
    }
    if (args.kt_o > 0) {
      prefetch_tmap(&tm_ao);
      prefetch_tmap(&tm_bo);
    }
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      uint32_t it = 0;                 // global K-tile counter (ring position)
      uint32_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, args.tiles_m, args.tiles_n, tm, tn);
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kt = 0; kt < nkt; ++kt, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const uint32_t ph = (it / STAGES) & 1u;
          if (it >= STAGES &&
              !mbar_wait_bounded(&sm.empty[s], ph ^ 1u, abort_flag, DEVERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* st = sm.stage[s];
          if (kt < args.kt_o) {
            mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
            tma_load_2d(st, &tm_ao, &sm.full[s], kt * 64, m0);
            tma_load_2d(st + A_BYTES, &tm_bo, &sm.full[s], kt * 64, n0);
          } else {
            const int kj = kt - args.kt_o;
            mbar_arrive_expect_tx(&sm.full[s], STAGE_BYTES);
            tma_load_2d(st, &tm_a, &sm.full[s], kj * KT_BYTES, m0);
            tma_load_2d(st + A_BYTES, &tm_b, &sm.full[s], kj * KT_BYTES, n0);
            const int atoms_k = args.nblk >> 2;
            const uint8_t* sa = args.sfa + (static_cast<int64_t>(tm) * atoms_k + 2 * kj) * 512;
            bulk_load(st + A_BYTES + B_BYTES, sa, SFA_BYTES, &sm.full[s]);
            for (int rb = 0; rb < 2; ++rb) {
              const uint8_t* sb =
                  args.sfb + (static_cast<int64_t>(2 * tn + rb) * atoms_k + 2 * kj) * 512;
              bulk_load(st + A_BYTES + B_BYTES + SFA_BYTES + rb * 1024, sb, 1024, &sm.full[s]);
            }
          }
          issued = it + 1;
        }
      }
      if (*abort_flag) {
        const uint32_t first = issued > STAGES ? issued - STAGES : 0;
        for (uint32_t i = first; i < issued; ++i)
          mbar_wait_bounded(&sm.full[i % STAGES], (i / STAGES) & 1u, nullptr,
                            DEVERR_TIMEOUT_PRODUCER);
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    if (lane == 0) {
      const uint32_t idesc_o = idesc_bf16(BM, BN);
      const uint32_t tsfa = tmem + TMEM_SFA_COL;
      const uint32_t tsfb = tmem + TMEM_SFB_COL;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
        // wait until the epilogue has drained the accumulator of the previous tile
        if (!mbar_wait_bounded(&sm.acc_empty, (tcount & 1u) ^ 1u, abort_flag, DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < nkt; ++kt, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(&sm.full[s], ph, abort_flag, DEVERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.stage[s]);
          const uint32_t b_addr = a_addr + A_BYTES;
          if (kt < args.kt_o) {
            const int rem = args.k_pad - kt * 64;
            const int nk = rem >= 64 ? 4 : rem / 16;
            for (int kk = 0; kk < nk; ++kk)
              mma_bf16(tmem, sdesc_kmajor_sw128(a_addr + kk * 32), sdesc_kmajor_sw128(b_addr + kk * 32),
                       idesc_o, (kt | kk) != 0 ? 1u : 0u);
          } else {
            const uint32_t sfa_s = b_addr + B_BYTES;
            const uint32_t sfb_s = sfa_s + SFA_BYTES;
            tc_cp_32x128b_warpx4(tsfa + 0, sdesc_sf_rows16(sfa_s));
            tc_cp_32x128b_warpx4(tsfa + 4, sdesc_sf_rows16(sfa_s + 512));
            tc_cp_32x128b_warpx4(tsfb + 0, sdesc_sf_rows16(sfb_s));
            tc_cp_32x128b_warpx4(tsfb + 8, sdesc_sf_rows16(sfb_s + 512));
            tc_cp_32x128b_warpx4(tsfb + 4, sdesc_sf_rows16(sfb_s + 1024));
            tc_cp_32x128b_warpx4(tsfb + 12, sdesc_sf_rows16(sfb_s + 1536));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t atom = static_cast<uint32_t>(kk >> 1);
              const uint32_t id = static_cast<uint32_t>((kk & 1) * 2);
              mma_mxf4(tmem, sdesc_kmajor_sw128(a_addr + kk * 32),
                       sdesc_kmajor_sw128(b_addr + kk * 32), idesc_mxf4(BM, BN, id, id),
                       (tsfa + 4 * atom) | (id << 30), (tsfb + 8 * atom) | (id << 30),
                       (kt | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty[s]);     // stage is free once these MMAs have read it
        }
        if (!ok) break;
        tc_commit(&sm.acc_full);       // accumulator complete
      }
      // wait for every MMA / copy this thread issued before tensor memory is freed
      tc_commit(&sm.drain);
      mbar_wait_bounded(&sm.drain, 0u, nullptr, DEVERR_TIMEOUT_MMA);
    }
  } else {
    // ============================ epilogue ================================
    const int ew = warp - 2;                 // 0..7
    const int sp = warp & 3;                 // tensor-memory lane quarter this warp may read
    const int half = ew >> 2;                // column half: 0 -> 0..127, 1 -> 128..255
    uint32_t tcount = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tcount) {
      int tm, tn;
      tile_coords(t, args.tiles_m, args.tiles_n, tm, tn);
      // one lane waits and the warp follows it, so the warp-collective
      // tcgen05.ld below runs converged
      int ready = 0;
      if (lane == 0)
        ready = mbar_wait_bounded(&sm.acc_full, tcount & 1u, abort_flag, DEVERR_TIMEOUT_EPILOGUE);
      ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      uint32_t r[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sp) << 16) + 128 * half;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);

      const int row = tm * BM + 32 * sp + lane;
      if (row < args.T) {
        __nv_bfloat16* yrow = args.Y + static_cast<int64_t>(row) * args.ldy;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col0 = tn * BN + 128 * half + 32 * c;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = col0 + 8 * q;
            if (col < args.d_out) {
              uint32_t p[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                    __uint_as_float(r[c][8 * q + 2 * h]), __uint_as_float(r[c][8 * q + 2 * h + 1]));
                p[h] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(yrow + col) = make_uint4(p[0], p[1], p[2], p[3]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// 2-D K-major tile map: inner dimension `inner` elements (row stride
// `row_bytes`), `rows` rows; box = 128 bytes x box_rows with 128-byte swizzle.
static bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                      uint64_t inner, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t gemm_smem_bytes() { return sizeof(GemmSmem) + 1024; }

cudaError_t launch_gemm(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                        const Geometry& g, const uint8_t* wq, const uint8_t* sfb, const void* w_hp,
                        void* Y, int64_t ldy, cudaStream_t stream) {
  if (T == 0 || g.d_out == 0) return cudaSuccess;
  CUtensorMap tm_a, tm_b, tm_ao, tm_bo;
  memset(&tm_a, 0, sizeof(tm_a));
  memset(&tm_b, 0, sizeof(tm_b));
  memset(&tm_ao, 0, sizeof(tm_ao));
  memset(&tm_bo, 0, sizeof(tm_bo));
  const uint64_t row_j = static_cast<uint64_t>(g.kj_pad / 2);
  if (g.kj_pad > 0) {
    if (!make_tmap(&tm_a, aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_j, T, row_j, BM) ||
        !make_tmap(&tm_b, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_j, g.d_out, row_j, BN))
      return cudaErrorInvalidValue;
  }
  if (g.k_pad > 0) {
    const uint64_t row_o = static_cast<uint64_t>(g.k_pad) * 2;
    if (!make_tmap(&tm_ao, xo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.k_pad, T, row_o, BM) ||
        !make_tmap(&tm_bo, w_hp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.k_pad, g.d_out, row_o, BN))
      return cudaErrorInvalidValue;
  }
  GemmArgs a;
  a.sfa = sfa;
  a.sfb = sfb;
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.ldy = ldy;
  a.T = static_cast<int>(T);
  a.d_out = static_cast<int>(g.d_out);
  a.nblk = static_cast<int>(g.nblk);
  a.kt_o = static_cast<int>((g.k_pad + 63) / 64);
  a.kt_j = static_cast<int>(g.kj_pad / 256);
  a.k_pad = static_cast<int>(g.k_pad);
  a.tiles_m = static_cast<int>((T + BM - 1) / BM);
  a.tiles_n = static_cast<int>((g.d_out + BN - 1) / BN);
  const int ntiles = a.tiles_m * a.tiles_n;
  const int sms = device_num_sms();
  const int grid = ntiles < sms ? ntiles : sms;
  const size_t smem = gemm_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(gemm_dual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  gemm_dual_kernel<<<grid, GEMM_THREADS, smem, stream>>>(tm_a, tm_b, tm_ao, tm_bo, a);
  return cudaGetLastError();
}

}  // namespace w4a4
