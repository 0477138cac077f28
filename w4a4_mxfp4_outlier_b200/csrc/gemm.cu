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
// Scale factors sit in tensor memory columns 256..279 and 288..311, the two
// buffers alternating by K tile, so the copy of one tile's scales does not
// have to wait for the MMAs still reading the previous tile's (tcgen05.cp
// and tcgen05.mma issued by one thread execute in order in any case).
// Every wait is bounded (about 2 s); a role that gives up sets the device
// error word and an abort flag the others poll, and all roles then exit
// through the same teardown (drain in-flight copies / MMAs, free tensor
// memory).
//
// Two kernels follow: gemm_dual_kernel (one CTA per 128 x 256 tile, for
// T <= 128) and gemm_dual_pair_kernel (a CTA pair per 256 x 256 or 256 x 384
// tile, see its own comment; its tensor-memory columns differ).  Both take a flag kAct: with it, the epilogue does not store
// Y but runs the fused FFN step (act_block: GELU, the next layer's smoothing
// and MXFP4 encoding) and writes the next layer's activation buffers.
#include <cuda.h>

#include <cstdlib>
#include <cstring>

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
constexpr int TMEM_SF_BUF = 32;               // scale buffers alternate by K tile: +0 / +32 columns
constexpr int GROUP_M = 16;                   // tile raster: 16 M tiles per sweep of N
constexpr int GROUP_M_384 = 24;               // the same for 384-wide pair tiles (measured best)

struct GemmSmem {
  uint8_t stage[STAGES][STAGE_BYTES];         // 1024-aligned (each part 1024-aligned)
  alignas(16) uint16_t gelu_tab[kGeluTabEntries];   // fused FFN epilogue only
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};


// Accumulator columns as bf16 pairs: the first step of the fused epilogue
// (bf16(acc), as the plain epilogue would store it), done right after the
// tensor-memory load so the pairs take half the registers.
struct BfPairs16 {
  uint32_t w[16];    // 32 consecutive columns of one row as bf16 pairs (low half: even column)
};

__device__ __forceinline__ void pack_bf16_pairs(const uint32_t (&acc)[32], BfPairs16& out) {
  uint32_t (&yb)[16] = out.w;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const __nv_bfloat162 b2 =
        __floats2bfloat162_rn(__uint_as_float(acc[2 * j]), __uint_as_float(acc[2 * j + 1]));
    yb[j] = *reinterpret_cast<const uint32_t*>(&b2);
  }
}

// One lane's 32 columns col0 .. col0+31 of row `row` (as bf16 pairs) through
// the fused FFN epilogue (see GemmArgs): writes the E2M1 codes of the MX
// block they form and the outlier columns among them, and returns the
// block's E8M0 scale code (0 where there is no block or no row), which the
// caller stores 4 blocks at a time.  No warp collectives: callable per lane.
// Not inlined: the epilogue calls it for 4 column chunks per tile, and with
// four inlined copies the epilogue warps' code was large enough to push the
// producer and MMA warps' instructions out of the instruction cache -- the
// fused up-projection GEMM then ran at 0.49x the speed of this form
// (T = 57600, 5120 -> 13824: 3.13 ms inlined, 1.87 ms called).
__device__ __noinline__ uint32_t act_block(const BfPairs16 y, int row, int col0, const GemmArgs* ap,
                                           uint32_t gelu_tab, uint32_t stg) {
  const uint32_t (&yb)[16] = y.w;
  const GemmArgs& a = *ap;
  if (row >= a.T) return 0u;
  // bf16(gelu(y)) of the 32 columns as bf16 pairs: table lookups, with the
  // inputs outside the table's range (rare) redone afterwards
  uint32_t hp[16];
  uint32_t bad = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t lo = yb[j] & 0xFFFFu, hi = yb[j] >> 16;
    const uint32_t rl = (lo & 0x7FFFu) - kGeluTabBase, rh = (hi & 0x7FFFu) - kGeluTabBase;
    bad |= rl | rh;
    hp[j] = gelu_bf16_table(gelu_tab, lo, rl) | (gelu_bf16_table(gelu_tab, hi, rh) << 16);
  }
  if (bad >= 2048u) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t lo = yb[j] & 0xFFFFu, hi = yb[j] >> 16;
      if ((lo & 0x7FFFu) - kGeluTabBase >= 2048u) hp[j] = (hp[j] & 0xFFFF0000u) | gelu_bf16_outside(lo);
      if ((hi & 0x7FFFu) - kGeluTabBase >= 2048u) hp[j] = (hp[j] & 0xFFFFu) | (gelu_bf16_outside(hi) << 16);
    }
  }
  // v = fl32(x * inv_s) column by column; columns past d_out are +0
  float2 v[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float4 is = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col0 + 4 * q < a.d_out) is = *reinterpret_cast<const float4*>(a.act_inv_s + col0 + 4 * q);
    const uint32_t p0 = hp[2 * q], p1 = hp[2 * q + 1];
    v[2 * q] = __fmul2_rn(make_float2(__uint_as_float(p0 << 16), __uint_as_float(p0 & 0xFFFF0000u)),
                          make_float2(is.x, is.y));
    v[2 * q + 1] = __fmul2_rn(make_float2(__uint_as_float(p1 << 16), __uint_as_float(p1 & 0xFFFF0000u)),
                              make_float2(is.z, is.w));
  }
  if (col0 + 32 > a.d_out) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (col0 + 2 * j >= a.d_out) v[j] = make_float2(0.f, 0.f);   // d_out is even
  }
  // outlier columns of the next layer (and its zero padding up to k_pad)
  if (col0 + 32 > a.act_kj && col0 < a.act_kj + a.act_k_pad) {
    __nv_bfloat16* xr = a.act_xo + static_cast<int64_t>(row) * a.act_k_pad;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int o = col0 + i - a.act_kj;
      const float vi = (i & 1) ? v[i >> 1].y : v[i >> 1].x;
      if (o >= 0 && o < a.act_k_pad)
        xr[o] = __ushort_as_bfloat16(static_cast<unsigned short>(bf16_rn_bits(vi)));
    }
  }
  // the MX block of compacted positions col0 .. col0+31 (zeros past act_kj)
  const int b = col0 >> 5;
  if (b < a.act_nblk) {
    if (col0 + 32 > a.act_kj) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (col0 + i >= a.act_kj) {
          if (i & 1) v[i >> 1].y = 0.0f;
          else v[i >> 1].x = 0.0f;
        }
      }
    }
    const float amax = block_absmax32(v);   // NaN if any element is NaN
    const uint32_t code = mx_scale_code(amax);
    const float inv = mx_inv_scale(code);
    const float2 inv2 = make_float2(inv, inv);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 a0 = __fmul2_rn(v[4 * q], inv2), a1 = __fmul2_rn(v[4 * q + 1], inv2);
      const float2 a2 = __fmul2_rn(v[4 * q + 2], inv2), a3 = __fmul2_rn(v[4 * q + 3], inv2);
      w[q] = cvt_e2m1x8(a0.x, a0.y, a1.x, a1.y, a2.x, a2.y, a3.x, a3.y) & mx_nan_block_mask(code);
    }
    if (stg != 0u) {
      // the staging row of this lane: 16-byte chunk (b & 3) at the 64-byte
      // swizzle position the tile store expects
      const uint32_t lane = threadIdx.x & 31u;
      st_shared_v4(stg + 64u * lane + 16u * ((static_cast<uint32_t>(b) & 3u) ^ ((lane >> 1) & 3u)),
                   w[0], w[1], w[2], w[3]);
    } else {
      *reinterpret_cast<uint4*>(a.act_aq + static_cast<int64_t>(row) * a.act_nblk * 16 + b * 16) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    return code;
  }
  return 0u;
}

// The scale codes of MX blocks b0 .. b0+3 of one row (b0 % 4 == 0): 4
// contiguous bytes of the MMA layout, one word store.  act_nblk % 4 == 0, so
// the 4 blocks are all J blocks or none is.
__device__ __forceinline__ void act_store_scales(const GemmArgs& a, int row, int b0, uint32_t codes) {
  if (b0 < a.act_nblk && row < a.T)
    *reinterpret_cast<uint32_t*>(a.act_sfa + sf_offset(row, b0, a.act_nblk)) = codes;
}

// Tile t of the raster: groups of kGroupM M tiles, each group swept N tile by
// N tile, M fastest within the group.
template <int kGroupM = GROUP_M>
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int per_group = kGroupM * tiles_n;
  const int g = t / per_group;
  const int first_m = g * kGroupM;
  const int gm = tiles_m - first_m < kGroupM ? tiles_m - first_m : kGroupM;
  const int w = t - g * per_group;
  tn = w / gm;
  tm = first_m + w % gm;
}

template <bool kAct>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_dual_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_ao, const __grid_constant__ CUtensorMap tm_bo,
                     const __grid_constant__ GemmArgs args) {
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
  pdl_wait();                  // barrier and tensor-memory setup overlap the previous kernel
  pdl_launch_dependents();

  if (warp == 0) {
    // ============================ TMA producer ============================
    // The whole warp runs the loop and waits; one elected lane issues.
    uint32_t it = 0;                   // global K-tile counter (ring position)
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
            !warp_wait_bounded(&sm.empty[s], ph ^ 1u, abort_flag, DEVERR_TIMEOUT_PRODUCER)) {
          ok = false;
          break;
        }
        if (elect_one()) {
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
        }
        __syncwarp();
        issued = it + 1;
      }
    }
    if (lane == 0 && *abort_flag) {
      // wait for the copies still in flight, so none lands after teardown
      const uint32_t first = issued > STAGES ? issued - STAGES : 0;
      for (uint32_t i = first; i < issued; ++i)
        mbar_wait_bounded(&sm.full[i % STAGES], (i / STAGES) & 1u, nullptr, DEVERR_TIMEOUT_PRODUCER);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    // The whole warp runs the loop and waits; one elected lane issues.
    const uint32_t idesc_o = idesc_bf16(BM, BN);
    const uint32_t tsfa = tmem + TMEM_SFA_COL;
    const uint32_t tsfb = tmem + TMEM_SFB_COL;
    uint32_t it = 0, tcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
      // wait until the epilogue has drained the accumulator of the previous tile
      if (!warp_wait_bounded(&sm.acc_empty, (tcount & 1u) ^ 1u, abort_flag, DEVERR_TIMEOUT_MMA)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kt = 0; kt < nkt; ++kt, ++it) {
        const int s = static_cast<int>(it % STAGES);
        const uint32_t ph = (it / STAGES) & 1u;
        if (!warp_wait_bounded(&sm.full[s], ph, abort_flag, DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a_addr = smem_u32(sm.stage[s]);
          const uint32_t b_addr = a_addr + A_BYTES;
          if (kt < args.kt_o) {
            const int rem = args.k_pad - kt * 64;
            const int nk = rem >= 64 ? 4 : rem / 16;
            for (int kk = 0; kk < nk; ++kk)
              mma_bf16(tmem, sdesc_kmajor_sw128(a_addr + kk * 32), sdesc_kmajor_sw128(b_addr + kk * 32),
                       idesc_o, (kt | kk) != 0 ? 1u : 0u);
          } else {
            // scales of this K tile go to the buffer the previous tile's MMAs
            // do not read, so the copy need not wait for them
            const uint32_t buf = static_cast<uint32_t>(it & 1u) * TMEM_SF_BUF;
            const uint32_t sa = tsfa + buf, sb = tsfb + buf;
            const uint32_t sfa_s = b_addr + B_BYTES;
            const uint32_t sfb_s = sfa_s + SFA_BYTES;
            tc_cp_32x128b_warpx4(sa + 0, sdesc_sf_rows16(sfa_s));
            tc_cp_32x128b_warpx4(sa + 4, sdesc_sf_rows16(sfa_s + 512));
            tc_cp_32x128b_warpx4(sb + 0, sdesc_sf_rows16(sfb_s));
            tc_cp_32x128b_warpx4(sb + 8, sdesc_sf_rows16(sfb_s + 512));
            tc_cp_32x128b_warpx4(sb + 4, sdesc_sf_rows16(sfb_s + 1024));
            tc_cp_32x128b_warpx4(sb + 12, sdesc_sf_rows16(sfb_s + 1536));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t atom = static_cast<uint32_t>(kk >> 1);
              const uint32_t id = static_cast<uint32_t>((kk & 1) * 2);
              mma_mxf4(tmem, sdesc_kmajor_sw128(a_addr + kk * 32),
                       sdesc_kmajor_sw128(b_addr + kk * 32), idesc_mxf4(BM, BN, id, id),
                       (sa + 4 * atom) | (id << 30), (sb + 8 * atom) | (id << 30),
                       (kt | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty[s]);     // stage is free once these MMAs have read it
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&sm.acc_full);   // accumulator complete
      __syncwarp();
    }
    // wait for every MMA / copy issued before tensor memory is freed (the
    // elected lane is the same one that issued them)
    if (elect_one()) tc_commit(&sm.drain);
    __syncwarp();
    mbar_wait_bounded(&sm.drain, 0u, nullptr, DEVERR_TIMEOUT_MMA);
    __syncwarp();
  } else {
    // ============================ epilogue ================================
    const int ew = warp - 2;                 // 0..7
    const int sp = warp & 3;                 // tensor-memory lane quarter this warp may read
    const int half = ew >> 2;                // column half: 0 -> 0..127, 1 -> 128..255
    uint32_t gelu_tab = 0;
    if constexpr (kAct) {
      gelu_table_fill(sm.gelu_tab, ew * 32 + lane, NUM_EPI_WARPS * 32);
      named_bar_sync(1, NUM_EPI_WARPS * 32);
      gelu_tab = smem_u32(sm.gelu_tab);
    }
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
      BfPairs16 yb[4];
      if constexpr (kAct) {
#pragma unroll
        for (int c = 0; c < 4; ++c) pack_bf16_pairs(r[c], yb[c]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);

      const int row = tm * BM + 32 * sp + lane;
      if constexpr (kAct) {
        {
          uint32_t codes = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            codes |= act_block(yb[c], row, tn * BN + 128 * half + 32 * c, &args, gelu_tab, 0u) << (8 * c);
          act_store_scales(args, row, (tn * BN + 128 * half) >> 5, codes);
        }
      } else if (row < args.T) {
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

// ===========================================================================
// CTA-pair kernel (tcgen05 cta_group::2): a cluster of two CTAs computes a
// 256 x kN output tile, kN = 256 or 384.  CTA r of the pair stages its own
// 128 token rows of A and its own half of the tile's B rows (so B's
// shared-memory traffic per SM halves against the single-CTA kernel), plus
// its A scales and the scales of all kN rows of B; the leader CTA (rank 0)
// issues the M=256 MMAs for both.  Each CTA's tensor memory holds the
// accumulator of its 128 rows (kN columns) and its scale factors.
//
// kN = 384 (plain epilogue only): each K step is one N=256 MMA into columns
// 0..255 and one N=128 MMA into columns 256..383 with the same A.  A is then
// fed once per 384 output columns instead of per 256 (a third fewer operand
// bytes per FLOP from A) and there are a third fewer tile hand-offs between
// the MMA issuer and the epilogue.  Per CTA and K tile, B is 128 rows for the
// first MMA (rows 128r .. 128r+127 of the tile) and 64 for the second (rows
// 256+64r .. 256+64r+63), stacked in shared memory; the tile's 384 scale rows
// are three 128-row atoms.
//
// Synchronisation: the TMA copies of both CTAs complete on the leader's
// "full" barrier (the leader posts the expected byte count of both); the
// leader's MMA completions are multicast to the "empty" and "acc_full"
// barriers of both CTAs; the epilogue warps of both CTAs arrive on the
// leader's "acc_empty".  No load uses cluster multicast.
// ===========================================================================
constexpr int P_A_BYTES = 128 * KT_BYTES;     // own 128 token rows
constexpr int P_SFA_BYTES = 1024;             // own 128 rows x 8 blocks
constexpr int P_EPI_ARRIVALS = 2 * NUM_EPI_WARPS;

constexpr int P_EPI_BYTES = 16 * 64;          // staging block: 16 rows x 32 bf16 (64-byte swizzle)

// Per tile width kN: B rows per CTA (kN / 2), B scale bytes (all kN rows x 8
// blocks), stage bytes, pipeline depth (about 1.6 us of MMA work either way)
// and tensor-memory columns of the scale buffers (after the accumulator).
template <int kN>
struct PairTile {
  static_assert(kN == 256 || kN == 384, "pair tile width");
  static constexpr int kBBytes = (kN / 2) * KT_BYTES;
  static constexpr int kSfbBytes = (kN / 128) * 1024;
  static constexpr int kStageBytes = P_A_BYTES + kBBytes + P_SFA_BYTES + kSfbBytes;
  static constexpr int kStages = kN == 256 ? 6 : 4;
  static constexpr int kSfaCol = kN;                 // 2 atoms x 4 columns
  static constexpr int kSfbCol = kN + 8;             // 2 atoms x 8 columns (first 256 rows)
  static constexpr int kSfb2Col = kN + 24;           // 2 atoms x 4 columns (rows 256..383)
  static constexpr int kSfBuf = kN == 256 ? 32 : 48; // scale buffers alternate by K tile
  static_assert(kSfb2Col + 8 + kSfBuf <= TMEM_COLS, "tensor memory columns");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

// The plain kernel: PairTile stages, a 1 KB Y staging block per epilogue
// warp.  The fused FFN kernel (kN = 256): 5 stages, a 2 KB block per warp
// (its 32 rows x 64 code bytes of one tile half) and the GELU table.
template <bool kAct, int kN>
struct PairSmem {
  static_assert(!kAct || kN == 256, "the fused epilogue runs on 256-wide tiles");
  static constexpr int kStages = kAct ? 5 : PairTile<kN>::kStages;
  static constexpr int kEpiBytes = kAct ? 32 * 64 : P_EPI_BYTES;
  uint8_t stage[kStages][PairTile<kN>::kStageBytes];
  alignas(1024) uint8_t epi[NUM_EPI_WARPS][kEpiBytes];
  alignas(16) uint16_t gelu_tab[kAct ? kGeluTabEntries : 8];
  uint64_t full[kStages];      // leader's counts the bytes of both CTAs
  uint64_t empty[kStages];     // both CTAs: MMA commit, multicast
  uint64_t acc_full;           // both CTAs: MMA commit, multicast
  uint64_t acc_empty;          // leader: epilogue warps of both CTAs
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

template <bool kAct, int kN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_dual_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_ao, const __grid_constant__ CUtensorMap tm_bo,
                          const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                          const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ GemmArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  using Smem = PairSmem<kAct, kN>;
  using Tile = PairTile<kN>;
  constexpr int NST = Smem::kStages;
  constexpr int P_B_BYTES = Tile::kBBytes;
  constexpr int P_STAGE_BYTES = Tile::kStageBytes;
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile uint32_t* abort_flag = &sm.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int ntiles = args.tiles_m * args.tiles_n;   // 256 x kN tiles
  const int nkt = args.kt_o + args.kt_j;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, P_EPI_ARRIVALS);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0u;
    fence_barrier_init();
    if (args.kt_j > 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_sfa);
      prefetch_tmap(&tm_sfb);
    }
    if (args.kt_o > 0) {
      prefetch_tmap(&tm_ao);
      prefetch_tmap(&tm_bo);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // barriers of both CTAs are initialised
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();                  // barrier and tensor-memory setup overlap the previous kernel
  pdl_launch_dependents();

  if (warp == 0) {
    // ============================ TMA producer (both CTAs) ================
    // The whole warp runs the loop and waits; one elected lane issues.
    uint32_t issued = 0;
    bool ok = true;
    const int atoms_k = args.nblk >> 2;
    uint32_t it = 0, s = 0, ph = 0;
    for (int t = pair; t < ntiles && ok; t += npairs) {
      int tm, tn;
      tile_coords<kN == 384 ? GROUP_M_384 : GROUP_M>(t, args.tiles_m, args.tiles_n, tm, tn);
      const int m_rows = tm * 256 + 128 * static_cast<int>(rank);
      const int n_rows = tn * kN + 128 * static_cast<int>(rank);
      const int n_rows2 = tn * kN + 256 + 64 * static_cast<int>(rank);   // kN = 384 only
      for (int kt = 0; kt < nkt; ++kt, ++it) {
        if (it >= NST &&
            !warp_wait_bounded(&sm.empty[s], ph ^ 1u, abort_flag, DEVERR_TIMEOUT_PRODUCER)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* st = sm.stage[s];
          const uint32_t full_leader = mapa_shared(smem_u32(&sm.full[s]), 0);
          if (kt < args.kt_o) {
            // the leader's barrier expects the bytes of both CTAs
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * (P_A_BYTES + P_B_BYTES));
            tma_load_2d_pair(st, &tm_ao, full_leader, kt * 64, m_rows);
            if constexpr (kN == 256) {
              tma_load_2d_pair(st + P_A_BYTES, &tm_bo, full_leader, kt * 64, n_rows);
            } else {             // B in 64-row boxes: 128 rows, then the 64 of the second MMA
              tma_load_2d_pair(st + P_A_BYTES, &tm_bo, full_leader, kt * 64, n_rows);
              tma_load_2d_pair(st + P_A_BYTES + 64 * KT_BYTES, &tm_bo, full_leader, kt * 64,
                               n_rows + 64);
              tma_load_2d_pair(st + P_A_BYTES + 128 * KT_BYTES, &tm_bo, full_leader, kt * 64,
                               n_rows2);
            }
          } else {
            const int kj = kt - args.kt_o;
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * P_STAGE_BYTES);
            tma_load_2d_pair(st, &tm_a, full_leader, kj * KT_BYTES, m_rows);
            if constexpr (kN == 256) {
              tma_load_2d_pair(st + P_A_BYTES, &tm_b, full_leader, kj * KT_BYTES, n_rows);
            } else {
              tma_load_2d_pair(st + P_A_BYTES, &tm_b, full_leader, kj * KT_BYTES, n_rows);
              tma_load_2d_pair(st + P_A_BYTES + 64 * KT_BYTES, &tm_b, full_leader, kj * KT_BYTES,
                               n_rows + 64);
              tma_load_2d_pair(st + P_A_BYTES + 128 * KT_BYTES, &tm_b, full_leader, kj * KT_BYTES,
                               n_rows2);
            }
            // scale atoms: 256-byte rows of the scale buffers, 4 rows (1 KB) per copy
            const int ya = ((2 * tm + static_cast<int>(rank)) * atoms_k + 2 * kj) * 2;
            tma_load_2d_pair(st + P_A_BYTES + P_B_BYTES, &tm_sfa, full_leader, 0, ya);
            for (int rb = 0; rb < kN / 128; ++rb) {
              const int yb = (((kN / 128) * tn + rb) * atoms_k + 2 * kj) * 2;
              tma_load_2d_pair(st + P_A_BYTES + P_B_BYTES + P_SFA_BYTES + rb * 1024, &tm_sfb,
                               full_leader, 0, yb);
            }
          }
        }
        __syncwarp();
        issued = it + 1;
        if (++s == NST) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      if (rank == 0) {
        // wait for the stages posted in the last ring's worth of K tiles, so
        // no copy lands after teardown (earlier ones were consumed)
        const uint32_t first = issued > NST ? issued - NST : 0;
        for (uint32_t i = first; i < issued; ++i)
          mbar_wait_bounded(&sm.full[i % NST], (i / NST) & 1u, nullptr,
                            DEVERR_TIMEOUT_PRODUCER);
      }
      spin_ns(50000);            // the peer CTA's copies land on the leader's barriers
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer (leader) =====================
    // The whole warp runs the loop and waits; one elected lane issues the
    // tcgen05 instructions.  The issue path is latency-critical, so the loop
    // only adds precomputed deltas: descriptors of stage 0 advanced by
    // STAGE_DESC per stage, K offsets folded into unrolled constants,
    // counters instead of divisions.
    if (rank == 0) {
      constexpr uint64_t STAGE_DESC = P_STAGE_BYTES >> 4;    // descriptor step per stage
      const uint32_t st0 = smem_u32(sm.stage[0]);
      const uint64_t da0 = sdesc_kmajor_sw128(st0);
      const uint64_t db0 = sdesc_kmajor_sw128(st0 + P_A_BYTES);
      const uint64_t dsa0 = sdesc_sf_rows16(st0 + P_A_BYTES + P_B_BYTES);
      const uint64_t dsb0 = sdesc_sf_rows16(st0 + P_A_BYTES + P_B_BYTES + P_SFA_BYTES);
      const uint64_t db1 = sdesc_kmajor_sw128(st0 + P_A_BYTES + 128 * KT_BYTES);   // kN = 384
      constexpr uint32_t ID_O = idesc_bf16(256, 256);
      constexpr uint32_t ID_J0 = idesc_mxf4(256, 256, 0, 0);
      constexpr uint32_t ID_J2 = idesc_mxf4(256, 256, 2, 2);
      constexpr uint32_t ID_O2 = idesc_bf16(256, 128);
      constexpr uint32_t ID_K0 = idesc_mxf4(256, 128, 0, 0);
      constexpr uint32_t ID_K2 = idesc_mxf4(256, 128, 2, 2);
      const uint32_t tsfa = tmem + Tile::kSfaCol;
      const uint32_t tsfb = tmem + Tile::kSfbCol;
      const uint32_t tsfb2 = tmem + Tile::kSfb2Col;
      const uint32_t tacc2 = tmem + 256;
      const int kt_o = args.kt_o, kt_j = args.kt_j;
      const int nk_last_o = (args.k_pad - (kt_o - 1) * 64) / 16;   // K=16 steps in the last bf16 tile
      uint32_t s = 0, ph = 0, buf = 0, tcount = 0;
      uint64_t soff = 0;                 // STAGE_DESC * s
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs, ++tcount) {
        if (!warp_wait_bounded(&sm.acc_empty, (tcount & 1u) ^ 1u, abort_flag, DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t acc = 0;
        for (int kt = 0; kt < kt_o; ++kt) {
          if (!warp_wait_bounded(&sm.full[s], ph, abort_flag, DEVERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const int nk = kt + 1 < kt_o ? 4 : nk_last_o;
            for (int kk = 0; kk < nk; ++kk) {
              mma_bf16_pair(tmem, da0 + soff + 2 * kk, db0 + soff + 2 * kk, ID_O, acc | kk);
              if constexpr (kN == 384)
                mma_bf16_pair(tacc2, da0 + soff + 2 * kk, db1 + soff + 2 * kk, ID_O2, acc | kk);
            }
            tc_commit_pair_multicast(&sm.empty[s], 0x3);
          }
          __syncwarp();
          acc = 1;
          if (++s == NST) {
            s = 0;
            ph ^= 1u;
            soff = 0;
          } else {
            soff += STAGE_DESC;
          }
        }
        for (int kt = 0; kt < kt_j && ok; ++kt) {
          if (!warp_wait_bounded(&sm.full[s], ph, abort_flag, DEVERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            // scale atoms into the buffer the previous K tile's MMAs do not read
            const uint32_t sa = tsfa + buf, sb = tsfb + buf;
            tc_cp_pair_32x128b_warpx4(sa + 0, dsa0 + soff);
            tc_cp_pair_32x128b_warpx4(sa + 4, dsa0 + soff + 32);
            tc_cp_pair_32x128b_warpx4(sb + 0, dsb0 + soff);
            tc_cp_pair_32x128b_warpx4(sb + 8, dsb0 + soff + 32);
            tc_cp_pair_32x128b_warpx4(sb + 4, dsb0 + soff + 64);
            tc_cp_pair_32x128b_warpx4(sb + 12, dsb0 + soff + 96);
            if constexpr (kN == 384) {
              // the third 128-row atom of B scales: K atoms 0 and 1 at +0 / +4
              const uint32_t sc = tsfb2 + buf;
              tc_cp_pair_32x128b_warpx4(sc + 0, dsb0 + soff + 128);
              tc_cp_pair_32x128b_warpx4(sc + 4, dsb0 + soff + 160);
              mma_mxf4_pair(tmem, da0 + soff + 0, db0 + soff + 0, ID_J0, sa, sb, acc);
              mma_mxf4_pair(tacc2, da0 + soff + 0, db1 + soff + 0, ID_K0, sa, sc, acc);
              mma_mxf4_pair(tmem, da0 + soff + 2, db0 + soff + 2, ID_J2, sa | (2u << 30),
                            sb | (2u << 30), 1u);
              mma_mxf4_pair(tacc2, da0 + soff + 2, db1 + soff + 2, ID_K2, sa | (2u << 30),
                            sc | (2u << 30), 1u);
              mma_mxf4_pair(tmem, da0 + soff + 4, db0 + soff + 4, ID_J0, sa + 4, sb + 8, 1u);
              mma_mxf4_pair(tacc2, da0 + soff + 4, db1 + soff + 4, ID_K0, sa + 4, sc + 4, 1u);
              mma_mxf4_pair(tmem, da0 + soff + 6, db0 + soff + 6, ID_J2, (sa + 4) | (2u << 30),
                            (sb + 8) | (2u << 30), 1u);
              mma_mxf4_pair(tacc2, da0 + soff + 6, db1 + soff + 6, ID_K2, (sa + 4) | (2u << 30),
                            (sc + 4) | (2u << 30), 1u);
            } else {
              mma_mxf4_pair(tmem, da0 + soff + 0, db0 + soff + 0, ID_J0, sa, sb, acc);
              mma_mxf4_pair(tmem, da0 + soff + 2, db0 + soff + 2, ID_J2, sa | (2u << 30),
                            sb | (2u << 30), 1u);
              mma_mxf4_pair(tmem, da0 + soff + 4, db0 + soff + 4, ID_J0, sa + 4, sb + 8, 1u);
              mma_mxf4_pair(tmem, da0 + soff + 6, db0 + soff + 6, ID_J2, (sa + 4) | (2u << 30),
                            (sb + 8) | (2u << 30), 1u);
            }
            tc_commit_pair_multicast(&sm.empty[s], 0x3);
          }
          __syncwarp();
          acc = 1;
          buf ^= Tile::kSfBuf;
          if (++s == NST) {
            s = 0;
            ph ^= 1u;
            soff = 0;
          } else {
            soff += STAGE_DESC;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair_multicast(&sm.acc_full, 0x3);
        __syncwarp();
      }
      // wait for every MMA / copy issued before tensor memory is freed (the
      // elected lane is the same one that issued them)
      if (elect_one()) tc_commit_pair(&sm.drain);
      __syncwarp();
      mbar_wait_bounded(&sm.drain, 0u, nullptr, DEVERR_TIMEOUT_MMA);
      __syncwarp();
    }
  } else {
    // ============================ epilogue (both CTAs) ====================
    const int ew = warp - 2;
    const int sp = warp & 3;
    const int half = ew >> 2;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(&sm.acc_empty), 0);
    uint32_t gelu_tab = 0;
    if constexpr (kAct) {
      gelu_table_fill(sm.gelu_tab, ew * 32 + lane, NUM_EPI_WARPS * 32);
      named_bar_sync(1, NUM_EPI_WARPS * 32);
      gelu_tab = smem_u32(sm.gelu_tab);
    }
    uint32_t tcount = 0;
    for (int t = pair; t < ntiles; t += npairs, ++tcount) {
      int tm, tn;
      tile_coords<kN == 384 ? GROUP_M_384 : GROUP_M>(t, args.tiles_m, args.tiles_n, tm, tn);
      int ready = 0;
      if (lane == 0)
        ready = mbar_wait_bounded(&sm.acc_full, tcount & 1u, abort_flag, DEVERR_TIMEOUT_EPILOGUE);
      ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      if constexpr (kN == 384) {
        // this warp's 32 rows x 192 columns, converted to bf16 pairs 16
        // columns at a time so the registers hold 96 words (not 192) plus
        // one 16-column load; the accumulator is released once all are in
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sp) << 16) + 192 * half;
        BfPairs16 yb[6];
#pragma unroll
        for (int h = 0; h < 12; ++h) {
          uint32_t r1[16];
          tmem_ld_32x32b_x16(taddr + 16 * h, r1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __nv_bfloat162 b2 =
                __floats2bfloat162_rn(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
            yb[h >> 1].w[8 * (h & 1) + j] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
        const int row0 = tm * 256 + 128 * static_cast<int>(rank) + 32 * sp;
        const uint32_t stg = smem_u32(sm.epi[ew]);
#pragma unroll
        for (int c = 0; c < 6; ++c) {
          const int col = tn * kN + 192 * half + 32 * c;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (elect_one()) bulk_wait_group_read0();
            __syncwarp();
            if ((lane >> 4) == hh) {
              const uint32_t rl = static_cast<uint32_t>(lane & 15);
              const uint32_t dst = stg + rl * 64u;
#pragma unroll
              for (uint32_t q = 0; q < 4; ++q)
                st_shared_v4(dst + 16u * (q ^ ((rl >> 1) & 3u)), yb[c].w[4 * q], yb[c].w[4 * q + 1],
                             yb[c].w[4 * q + 2], yb[c].w[4 * q + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (elect_one()) {
              tma_store_2d(&tm_y, stg, col, row0 + 16 * hh);
              bulk_commit_group();
            }
            __syncwarp();
          }
        }
        continue;
      }
      uint32_t r[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sp) << 16) + 128 * half;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, r[c]);
      tmem_ld_wait();
      BfPairs16 yb[4];
      if constexpr (kAct) {
#pragma unroll
        for (int c = 0; c < 4; ++c) pack_bf16_pairs(r[c], yb[c]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);

      if constexpr (kAct) {
        // the codes of 4 consecutive MX blocks b0 .. b0+3 (64 bytes per row)
        // go through this warp's staging block, 32 rows x 64 bytes, and leave
        // in one TMA tile store (tm_y maps act_aq here; rows past T clipped)
        const int row0 = tm * 256 + 128 * static_cast<int>(rank) + 32 * sp;
        const int row = row0 + lane;
        const int b0 = (tn * 256 + 128 * half) >> 5;
        const uint32_t stg = smem_u32(sm.epi[ew]);
        if (elect_one()) bulk_wait_group_read0();   // the previous tile's store has read it
        __syncwarp();
        uint32_t codes = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          codes |= act_block(yb[c], row, tn * 256 + 128 * half + 32 * c, &args, gelu_tab, stg) << (8 * c);
        act_store_scales(args, row, b0, codes);
        if (b0 < args.act_nblk) {                   // uniform over the warp
          fence_proxy_async_smem();
          __syncwarp();
          if (elect_one()) {
            tma_store_2d(&tm_y, stg, b0 * 16, row0);
            bulk_commit_group();
          }
          __syncwarp();
        }
        continue;
      }
      // Y through a per-warp staging block, 16 rows x 32 columns at a time:
      // the lanes holding those rows write them (64-byte swizzle: 16-byte
      // chunk j of row r sits at chunk j ^ ((r >> 1) & 3), so the writes hit
      // distinct banks) and one lane stores the block with a TMA tile store,
      // which also clips rows past T and columns past d_out.
      const int row0 = tm * 256 + 128 * static_cast<int>(rank) + 32 * sp;
      const uint32_t stg = smem_u32(sm.epi[ew]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t p[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[c][2 * j]),
                                                          __uint_as_float(r[c][2 * j + 1]));
          p[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        const int col = tn * 256 + 128 * half + 32 * c;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // the previous store from this block must have read it
          if (elect_one()) bulk_wait_group_read0();
          __syncwarp();
          if ((lane >> 4) == hh) {
            const uint32_t rl = static_cast<uint32_t>(lane & 15);
            const uint32_t dst = stg + rl * 64u;
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q)
              st_shared_v4(dst + 16u * (q ^ ((rl >> 1) & 3u)), p[4 * q], p[4 * q + 1], p[4 * q + 2],
                           p[4 * q + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (elect_one()) {
            tma_store_2d(&tm_y, stg, col, row0 + 16 * hh);
            bulk_commit_group();
          }
          __syncwarp();
        }
      }
    }
    if (elect_one()) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();          // the pair's MMAs, copies and remote arrivals are done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
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

// 2-D tile map: inner dimension `inner` elements (row stride `row_bytes`),
// `rows` rows; box = `box_inner` elements x `box_rows`.
static bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                      uint64_t inner, uint64_t rows, uint64_t row_bytes, uint32_t box_rows,
                      uint32_t box_inner = 0, bool swizzle128 = true,
                      CUtensorMapSwizzle swz_other = CU_TENSOR_MAP_SWIZZLE_NONE) {
  PFN_encodeTiled enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner ? box_inner : static_cast<cuuint32_t>(128 / elem_bytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : swz_other,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t gemm_smem_bytes() { return sizeof(GemmSmem) + 1024; }
template <bool kAct, int kN>
size_t gemm_pair_smem_bytes() { return sizeof(PairSmem<kAct, kN>) + 1024; }

template <bool kAct, int kN>
static bool pair_set_smem() {
  return cudaFuncSetAttribute(gemm_dual_pair_kernel<kAct, kN>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(gemm_pair_smem_bytes<kAct, kN>())) == cudaSuccess;
}

template <bool kAct, int kN>
static int pair_clusters(cudaLaunchConfig_t cfg) {
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes<kAct, kN>();
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_dual_pair_kernel<kAct, kN>, &cfg) != cudaSuccess)
    return 0;
  return n;
}

// Number of co-resident CTA pairs of the pair kernel on this device (0 if the
// query fails); cached per device.
static int pair_capacity() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  if (!pair_set_smem<false, 256>() || !pair_set_smem<true, 256>() || !pair_set_smem<false, 384>())
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 148, 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one grid size serves every instantiation: the smallest co-resident count
  int n = pair_clusters<false, 256>(cfg);
  const int n2 = pair_clusters<true, 256>(cfg);
  const int n3 = pair_clusters<false, 384>(cfg);
  if (n2 < n) n = n2;
  if (n3 < n) n = n3;
  if (n <= 0) return 0;
  cached[dev] = n;
  return n;
}

// Output columns per pair tile.  384 where it divides d_out and the epilogue
// stores Y (a third fewer A bytes per FLOP and tile hand-offs); else 256.
// W4A4_PAIR_TILE_N=256 in the environment keeps every launch on 256.
static int pair_tile_n(int64_t d_out, bool act) {
  static int forced = -1;
  if (forced < 0) {
    const char* e = getenv("W4A4_PAIR_TILE_N");
    forced = (e != nullptr && strcmp(e, "256") == 0) ? 1 : 0;
  }
  if (act || forced == 1) return 256;
  return d_out % 384 == 0 ? 384 : 256;
}

// Token counts up to this use the single-CTA kernel (a 256-row pair tile
// would be mostly padding).
constexpr int64_t kPairMinT = 129;

// Host half of a GEMM launch: tile choice, tensor maps and kernel arguments.
// Enqueues nothing, so a composite call can run it before its first launch and
// return an error with nothing enqueued.
cudaError_t plan_gemm(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                      const Geometry& g, const uint8_t* wq, const uint8_t* sfb, const void* w_hp,
                      void* Y, int64_t ldy, const ActOut* act, GemmPlan* p) {
  memset(p, 0, sizeof(*p));
  p->empty = (T == 0 || g.d_out == 0);
  if (p->empty) return cudaSuccess;
  p->act = act != nullptr;
  p->pair = T >= kPairMinT && pair_capacity() > 0;
  p->tile_n = p->pair ? pair_tile_n(g.d_out, p->act) : BN;
  // B box rows: 256 (single CTA), 128 (pair, 256-wide tile), 64 (pair, 384-wide: 3 boxes)
  const uint32_t brows = !p->pair ? BN : (p->tile_n == 384 ? 64 : 128);
  const uint64_t row_j = static_cast<uint64_t>(g.kj_pad / 2);
  if (g.kj_pad > 0) {
    if (!make_tmap(&p->tm_a, aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_j, T, row_j, BM) ||
        !make_tmap(&p->tm_b, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_j, g.d_out, row_j, brows))
      return cudaErrorInvalidValue;
    if (p->pair) {
      // scale buffers seen as rows of 256 bytes; one copy = 4 rows = two 512-byte atoms
      const uint64_t sfa_rows = static_cast<uint64_t>(round_up(T, kSfaRowPad) * g.nblk / 256);
      const uint64_t sfb_rows = static_cast<uint64_t>(g.sfb_rows * g.nblk / 256);
      if (!make_tmap(&p->tm_sfa, sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, sfa_rows, 256, 4, 256,
                     false) ||
          !make_tmap(&p->tm_sfb, sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, sfb_rows, 256, 4, 256,
                     false))
        return cudaErrorInvalidValue;
    }
  }
  if (g.k_pad > 0) {
    const uint64_t row_o = static_cast<uint64_t>(g.k_pad) * 2;
    if (!make_tmap(&p->tm_ao, xo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.k_pad, T, row_o, BM) ||
        !make_tmap(&p->tm_bo, w_hp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.k_pad, g.d_out, row_o,
                   brows))
      return cudaErrorInvalidValue;
  }
  GemmArgs& a = p->a;
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
  a.tiles_m = static_cast<int>((T + (p->pair ? 255 : BM - 1)) / (p->pair ? 256 : BM));
  a.tiles_n = static_cast<int>((g.d_out + p->tile_n - 1) / p->tile_n);
  a.act_inv_s = act ? act->inv_s : nullptr;
  a.act_aq = act ? act->aq : nullptr;
  a.act_sfa = act ? act->sfa : nullptr;
  a.act_xo = act ? static_cast<__nv_bfloat16*>(act->xo) : nullptr;
  a.act_kj = act ? static_cast<int>(act->kj) : 0;
  a.act_nblk = act ? static_cast<int>(act->nblk) : 0;
  a.act_k_pad = act ? static_cast<int>(act->k_pad) : 0;
  const int ntiles = a.tiles_m * a.tiles_n;
  if (p->pair) {
    const int npairs = ntiles < pair_capacity() ? ntiles : pair_capacity();
    p->grid = 2 * npairs;
    p->smem = act ? gemm_pair_smem_bytes<true, 256>()
                  : (p->tile_n == 384 ? gemm_pair_smem_bytes<false, 384>()
                                      : gemm_pair_smem_bytes<false, 256>());
    if (act != nullptr) {
      // the next layer's codes as tiles of 32 rows x 64 bytes, 64-byte swizzle
      if (act->nblk > 0 &&
          !make_tmap(&p->tm_y, act->aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                     static_cast<uint64_t>(act->nblk) * 16, T, static_cast<uint64_t>(act->nblk) * 16,
                     32, 64, false, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    } else if (!make_tmap(&p->tm_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.d_out, T,
                          static_cast<uint64_t>(ldy) * 2, 16, 32, false,
                          CU_TENSOR_MAP_SWIZZLE_64B)) {
      // Y as bf16 tiles of 16 rows x 32 columns, 64-byte swizzle (epilogue staging layout)
      return cudaErrorInvalidValue;
    }
    return cudaSuccess;
  }
  const int sms = device_num_sms();
  p->grid = ntiles < sms ? ntiles : sms;
  p->smem = gemm_smem_bytes();
  cudaError_t e = p->act ? cudaFuncSetAttribute(gemm_dual_kernel<true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(p->smem))
                         : cudaFuncSetAttribute(gemm_dual_kernel<false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(p->smem));
  return e;
}

// Device half: enqueues the planned kernel on `stream`.
cudaError_t run_gemm(const GemmPlan& p, cudaStream_t stream) {
  if (p.empty) return cudaSuccess;
  if (p.pair) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1 + static_cast<unsigned>(pdl_attrs(&attr[1]));
    if (p.act)
      return cudaLaunchKernelEx(&cfg, gemm_dual_pair_kernel<true, 256>, p.tm_a, p.tm_b, p.tm_ao,
                                p.tm_bo, p.tm_sfa, p.tm_sfb, p.tm_y, p.a);
    if (p.tile_n == 384)
      return cudaLaunchKernelEx(&cfg, gemm_dual_pair_kernel<false, 384>, p.tm_a, p.tm_b, p.tm_ao,
                                p.tm_bo, p.tm_sfa, p.tm_sfb, p.tm_y, p.a);
    return cudaLaunchKernelEx(&cfg, gemm_dual_pair_kernel<false, 256>, p.tm_a, p.tm_b, p.tm_ao,
                              p.tm_bo, p.tm_sfa, p.tm_sfb, p.tm_y, p.a);
  }
  if (p.act)
    return launch_pdl(gemm_dual_kernel<true>, dim3(p.grid), dim3(GEMM_THREADS), p.smem, stream, p.tm_a,
                      p.tm_b, p.tm_ao, p.tm_bo, p.a);
  return launch_pdl(gemm_dual_kernel<false>, dim3(p.grid), dim3(GEMM_THREADS), p.smem, stream, p.tm_a,
                    p.tm_b, p.tm_ao, p.tm_bo, p.a);
}

cudaError_t launch_gemm(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                        const Geometry& g, const uint8_t* wq, const uint8_t* sfb, const void* w_hp,
                        void* Y, int64_t ldy, cudaStream_t stream, const ActOut* act) {
  GemmPlan p;
  const cudaError_t e = plan_gemm(aq, sfa, xo, T, g, wq, sfb, w_hp, Y, ldy, act, &p);
  if (e != cudaSuccess) return e;
  return run_gemm(p, stream);
}

}  // namespace w4a4
