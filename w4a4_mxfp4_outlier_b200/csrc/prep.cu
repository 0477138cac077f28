// Online activation preparation: one pass over X that divides by s (as a
// multiply by inv_s), gathers the outlier columns into a dense bf16 matrix
// and MXFP4-encodes the compacted remaining columns, writing E2M1 codes and
// E8M0 scales directly in the layout the block-scaled tensor-core MMA reads.
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.2 ("at inference activations are first divided by s, then
// quantised") and sec. 3.3 (X_J in 4 bits, X_O in high precision).
//
// Rows of at most 480 MX blocks (d_in up to 15360) go to the block-per-lane
// form in prep_block.cu, which needs fewer instructions per element; this
// kernel takes the wider rows (up to d_in = 16384).
//
// Design (HBM-bound in principle: 2 bytes read and ~0.56 bytes written per
// element, so the instruction count per element is what has to stay low):
//  * persistent grid, one CTA per SM; CTA b handles rows b, b+G, b+2G, ...
//  * warp 0 streams whole rows into a ring of kPrepStages shared-memory
//    slots of a fixed kPrepStage bytes with cp.async.bulk (completion counted
//    on an mbarrier per slot);
//  * each consumer thread owns CH chunks of 8 consecutive compacted columns
//    for the whole kernel and keeps the shared-memory address (in slot 0) of
//    each of their 8 source elements, and their inv_s, in registers.  The
//    consumer loop is unrolled over the ring, so the slot offset is an
//    immediate of the load: one load and one shift per element gathered;
//  * four lanes form one 32-element MX block (amax by two xor shuffles);
//    a warp covers 256 columns and stores 128 contiguous code bytes;
//  * the 8 elements of a chunk are gathered pair by pair in an order rotated
//    by (lane / 8) % 4 so the 32 lanes of a warp hit 32 different banks;
//  * padding columns (p >= kj) and padding outlier slots read a zero slot
//    kept at the end of each ring slot, so they encode as +0 with no branch.
#include "w4a4_internal.h"

namespace w4a4 {

constexpr int kPrepStage = 32768 + 128;           // one row of up to 16384 bf16 + zero slot
constexpr int kPrepStages = 6;
constexpr int kPrepZero = kPrepStage - 16;        // offset of the zero slot in a ring slot
constexpr int kPrepMaxD = 16384;

// consumer threads per CTA for CH chunks each, and the register cap that
// lets that many (+ the producer warp) run in one CTA: the state kept per
// chunk is 8 offsets + 8 inv_s registers
// (the warps of a block are spread over the SM's 4 schedulers, each with a
// quarter of the register file: ceil(warps / 4) * 32 * registers <= 16384)
template <int CH> struct PrepCfg;
template <> struct PrepCfg<1> { static constexpr int kMaxConsumers = 992, kMaxRegs = 64; };
template <> struct PrepCfg<2> { static constexpr int kMaxConsumers = 736, kMaxRegs = 80; };
template <> struct PrepCfg<4> { static constexpr int kMaxConsumers = 480, kMaxRegs = 128; };
template <> struct PrepCfg<8> { static constexpr int kMaxConsumers = 256, kMaxRegs = 168; };

// bf16 at byte offset `off` of the ring, widened to the bits of a float
__device__ __forceinline__ uint32_t ring_bf16(const uint8_t* ring, uint32_t off) {
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(ring + off)) << 16;
}

template <int CH>
__global__ void __maxnreg__(PrepCfg<CH>::kMaxRegs) prep_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t ldx, int d_in,
                const float* __restrict__ inv_s, const int32_t* __restrict__ O,
                const int32_t* __restrict__ jmap, int k, int k_pad, int kj, int nchunks, int nblk,
                uint8_t* __restrict__ aq, uint8_t* __restrict__ sfa, uint32_t* __restrict__ xo,
                int stripe4, const int32_t* __restrict__ rows) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(kPrepStages) * kPrepStage);
  uint64_t* empty = full + kPrepStages;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(empty + kPrepStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NT = blockDim.x - 32;           // consumer threads (multiple of 32)

  if (threadIdx.x == 0) {
    for (int u = 0; u < kPrepStages; ++u) {
      mbar_init(&full[u], 1);
      mbar_init(&empty[u], NT / 32);
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  for (int u = threadIdx.x; u < kPrepStages; u += blockDim.x)
    *reinterpret_cast<uint4*>(smem + static_cast<size_t>(u) * kPrepStage + kPrepZero) =
        make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  pdl_wait();                  // the shared-memory setup above overlaps the previous kernel
  pdl_launch_dependents();

  const int64_t nrows = T > blockIdx.x ? (T - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (warp == 0) {
    // ---------------- producer (whole warp; one elected lane issues) ----------------
    const uint32_t bytes = static_cast<uint32_t>(d_in) * 2u;
    const uint16_t* src = X + static_cast<int64_t>(blockIdx.x) * ldx;
    const int64_t src_step = static_cast<int64_t>(gridDim.x) * ldx;
    // failure-detection test hook: no copies at all, the consumers' waits run out
    const bool skip = (g_fault_mask & FAULT_PREP_SKIP_LOADS) != 0u;
    int64_t issued = 0;
    int u = 0;
    uint32_t ph = 0;
    for (int64_t i = 0; i < nrows && !skip; ++i) {
      if (i >= kPrepStages &&
          !warp_wait_bounded(&empty[u], ph ^ 1u, abort_flag, DEVERR_TIMEOUT_PREP))
        break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&full[u], bytes);
        // output row r reads input row rows[r] when a row map is given
        const uint16_t* from =
            rows ? X + static_cast<int64_t>(rows[blockIdx.x + i * gridDim.x]) * ldx : src;
        bulk_load(smem + static_cast<size_t>(u) * kPrepStage, from, bytes, &full[u]);
      }
      __syncwarp();
      src += src_step;
      issued = i + 1;
      if (++u == kPrepStages) {
        u = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0 && *abort_flag) {
      // do not leave bulk copies in flight into shared memory we give back
      const int64_t first = issued > kPrepStages ? issued - kPrepStages : 0;
      for (int64_t i = first; i < issued; ++i)
        mbar_wait_bounded(&full[i % kPrepStages], static_cast<uint32_t>((i / kPrepStages) & 1),
                          nullptr, DEVERR_TIMEOUT_PREP);
    }
    __syncwarp();
    return;
  }

  // ---------------- consumers ----------------
  const int ct = threadIdx.x - 32;
  const int rot = (lane >> 3) & 3;
  uint32_t go[CH][8];      // byte offsets (in ring slot 0) of the 8 gathered elements, rotated pair order
  float2 isv[CH][4];       // their inv_s
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int chunk = ct + c * NT;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int qq = (q + rot) & 3;
      const int p0 = chunk * 8 + 2 * qq;
      uint32_t o0 = kPrepZero, o1 = kPrepZero;
      float i0 = 1.f, i1 = 1.f;
      if (chunk < nchunks && p0 < kj) {
        const int j = jmap[p0];
        o0 = 2u * static_cast<uint32_t>(j);
        i0 = inv_s[j];
      }
      if (chunk < nchunks && p0 + 1 < kj) {
        const int j = jmap[p0 + 1];
        o1 = 2u * static_cast<uint32_t>(j);
        i1 = inv_s[j];
      }
      go[c][2 * q] = o0;
      go[c][2 * q + 1] = o1;
      isv[c][q] = make_float2(i0, i1);
    }
  }
  // the outlier pair this thread gathers on every row (more pairs than
  // threads only when k > 2 * NT; those run through the loop below)
  const int xo_row = k_pad >> 1;                            // bf16 pairs per row of X_O
  uint32_t oo0 = kPrepZero, oo1 = kPrepZero;
  float2 oinv = make_float2(1.f, 1.f);
  if (ct < xo_row) {
    const int o0 = 2 * ct;
    if (o0 < k) {
      oo0 = 2u * static_cast<uint32_t>(O[o0]);
      oinv.x = inv_s[O[o0]];
    }
    if (o0 + 1 < k) {
      oo1 = 2u * static_cast<uint32_t>(O[o0 + 1]);
      oinv.y = inv_s[O[o0 + 1]];
    }
  }
  const int64_t aq_row = static_cast<int64_t>(nblk) * 16;   // bytes per row of codes
  const int64_t atoms_k = nblk >> 2;
  const int64_t rstep = gridDim.x;
  uint8_t* aq_p = aq + static_cast<int64_t>(blockIdx.x) * aq_row;
  uint32_t* xo_p = xo + static_cast<int64_t>(blockIdx.x) * xo_row;
  int64_t r = blockIdx.x;
  uint32_t ph = 0;
  bool ok = true;

  for (int64_t i0 = 0; i0 < nrows && ok; i0 += kPrepStages) {
#pragma unroll
    for (int u = 0; u < kPrepStages; ++u) {
      if (i0 + u >= nrows) break;
      if (!warp_wait_bounded(&full[u], ph, abort_flag, DEVERR_TIMEOUT_PREP)) {
        ok = false;
        break;
      }
      const uint8_t* ring = smem + u * kPrepStage;          // compile-time offset
      // scale byte offset of (row r, block 0) in the MMA layout
      const int64_t sf_row = (((r >> 7) * atoms_k) << 9) + ((r & 31) << 4) + (((r & 127) >> 5) << 2);
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int chunk = ct + c * NT;
        if (chunk < nchunks) {                // uniform per warp (nchunks % 32 == 0)
          float2 v[4];
          float amax = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float x0 = __uint_as_float(ring_bf16(ring, go[c][2 * q]));
            const float x1 = __uint_as_float(ring_bf16(ring, go[c][2 * q + 1]));
            v[q] = __fmul2_rn(make_float2(x0, x1), isv[c][q]);
            amax = max3_nan(amax, fabsf(v[q].x), fabsf(v[q].y));   // NaN-propagating
          }
          amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
          amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
          if (stripe4) {                      // 128x1 stripes: 16 lanes, 4 blocks
            amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
            amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 8));
          }
          const uint32_t code = mx_scale_code(amax);
          const float inv = mx_inv_scale(code);
          const float2 inv2 = make_float2(inv, inv);
          float2 qv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) qv[q] = __fmul2_rn(v[q], inv2);
          uint32_t w = cvt_e2m1x8(qv[0].x, qv[0].y, qv[1].x, qv[1].y, qv[2].x, qv[2].y, qv[3].x,
                                  qv[3].y) & mx_nan_block_mask(code);
          w = __funnelshift_l(w, w, 8 * rot);   // undo the pair rotation
          *reinterpret_cast<uint32_t*>(aq_p + 4 * chunk) = w;
          const uint32_t c4 = __shfl_down_sync(0xFFFFFFFFu, code, 4);
          const uint32_t c8 = __shfl_down_sync(0xFFFFFFFFu, code, 8);
          const uint32_t c12 = __shfl_down_sync(0xFFFFFFFFu, code, 12);
          if ((lane & 15) == 0) {
            // blocks chunk/4 .. chunk/4 + 3 of row r: one 4-byte word of an atom
            *reinterpret_cast<uint32_t*>(sfa + sf_row + ((static_cast<int64_t>(chunk) >> 4) << 9)) =
                code | (c4 << 8) | (c8 << 16) | (c12 << 24);
          }
        }
      }
      if (ct < xo_row) {
        const float x0 = __uint_as_float(ring_bf16(ring, oo0));
        const float x1 = __uint_as_float(ring_bf16(ring, oo1));
        const float2 v = __fmul2_rn(make_float2(x0, x1), oinv);
        xo_p[ct] = bf16_rn_bits(v.x) | (bf16_rn_bits(v.y) << 16);
        for (int i2 = ct + NT; i2 < xo_row; i2 += NT) {
          const int o0 = 2 * i2;
          const uint32_t a0 = o0 < k ? 2u * static_cast<uint32_t>(O[o0]) : kPrepZero;
          const uint32_t a1 = o0 + 1 < k ? 2u * static_cast<uint32_t>(O[o0 + 1]) : kPrepZero;
          const float y0 = __fmul_rn(__uint_as_float(ring_bf16(ring, a0)), o0 < k ? inv_s[O[o0]] : 1.f);
          const float y1 =
              __fmul_rn(__uint_as_float(ring_bf16(ring, a1)), o0 + 1 < k ? inv_s[O[o0 + 1]] : 1.f);
          xo_p[i2] = bf16_rn_bits(y0) | (bf16_rn_bits(y1) << 16);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[u]);
      r += rstep;
      aq_p += rstep * aq_row;
      xo_p += rstep * xo_row;
    }
    ph ^= 1u;
  }
}

struct PrepPlan {
  int ch, nt;
};

static PrepPlan plan_prep(const Geometry& g) {
  const int nchunks = static_cast<int>(g.kj_pad / 8);
  PrepPlan p{1, 0};
  if (nchunks > PrepCfg<1>::kMaxConsumers) p.ch = 2;
  if (nchunks > 2 * PrepCfg<2>::kMaxConsumers) p.ch = 4;
  if (nchunks > 4 * PrepCfg<4>::kMaxConsumers) p.ch = 8;
  int nt = (nchunks + p.ch - 1) / p.ch;
  nt = static_cast<int>(round_up(nt < 32 ? 32 : nt, 32));
  p.nt = nt;
  return p;
}

static constexpr size_t kPrepSmem =
    static_cast<size_t>(kPrepStages) * kPrepStage + 2 * kPrepStages * 8 + 16;

bool prep_supported(const Geometry& g) {
  if (g.d_in > kPrepMaxD) return false;
  const int nchunks = static_cast<int>(g.kj_pad / 8);
  return nchunks <= 8 * PrepCfg<8>::kMaxConsumers;
}

template <int CH>
static cudaError_t launch_prep_ch(const PrepPlan& p, int grid, const void* X, int64_t T,
                                  int64_t ldx, const float* inv_s, const int32_t* O,
                                  const int32_t* jmap, const Geometry& g, uint8_t* aq,
                                  uint8_t* sfa, void* xo, cudaStream_t stream, bool stripe4,
                                  const int32_t* rows) {
  cudaError_t e = cudaFuncSetAttribute(prep_kernel<CH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kPrepSmem));
  if (e != cudaSuccess) return e;
  return launch_pdl(prep_kernel<CH>, dim3(grid), dim3(p.nt + 32), kPrepSmem, stream,
                    static_cast<const uint16_t*>(X), T, ldx, static_cast<int>(g.d_in), inv_s, O, jmap,
                    static_cast<int>(g.k), static_cast<int>(g.k_pad), static_cast<int>(g.kj),
                    static_cast<int>(g.kj_pad / 8), static_cast<int>(g.nblk), aq, sfa,
                    static_cast<uint32_t*>(xo), stripe4 ? 1 : 0, rows);
}

cudaError_t launch_prep(const void* X, int64_t T, int64_t ldx, const float* inv_s,
                        const int32_t* O, const int32_t* jmap, const Geometry& g, uint8_t* aq,
                        uint8_t* sfa, void* xo, cudaStream_t stream, bool stripe4,
                        const int32_t* rows) {
  if (T == 0) return cudaSuccess;
  if (prep_block_supported(g))
    return launch_prep_block(X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
  const PrepPlan p = plan_prep(g);
  const int sms = device_num_sms();
  const int grid = static_cast<int>(T < sms ? T : sms);
  switch (p.ch) {
    case 1: return launch_prep_ch<1>(p, grid, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    case 2: return launch_prep_ch<2>(p, grid, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    case 4: return launch_prep_ch<4>(p, grid, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    default: return launch_prep_ch<8>(p, grid, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
  }
}


template <int CH>
constexpr bool prep_regs_fit() {
  return ((PrepCfg<CH>::kMaxConsumers + 32) / 32 + 3) / 4 * 32 * PrepCfg<CH>::kMaxRegs <= 16384;
}
static_assert(prep_regs_fit<1>(), "CH=1 registers");
static_assert(prep_regs_fit<2>(), "CH=2 registers");
static_assert(prep_regs_fit<4>(), "CH=4 registers");
static_assert(prep_regs_fit<8>(), "CH=8 registers");

}  // namespace w4a4
