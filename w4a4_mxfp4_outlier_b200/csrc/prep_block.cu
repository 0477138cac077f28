// Online activation preparation, block-per-lane form: the same computation as
// prep_kernel (prep.cu) -- X times inv_s, outlier columns gathered to bf16,
// the compacted remaining columns MXFP4-encoded into the MMA layout -- with
// each consumer lane owning one whole 32-element MX block of the row.
//
// Method: paper review "W4A4 Quantization for Inference on Wan2.2-I2V-A14B",
// sec. 3.2 (divide by s, then quantise) and sec. 3.3 (X_J in 4 bits, X_O in
// high precision).
//
// Design (the kernel is issue-bound, so the point is fewer instructions per
// element than prep_kernel's 8-elements-per-lane form):
//  * a ring of rows in shared memory filled by a producer warp with bulk
//    copies of whole rows, as in prep_kernel (its 6 slots of 32.9 KB, or 18
//    slots of 11 KB for rows of up to 5480 elements).  With several thread
//    groups the producer refills whichever group's next slot is free (a
//    non-blocking check per group) instead of waiting on the slots in ring
//    order, where one group running behind held back the refills of the
//    others and left them waiting for rows (up layer 0.140 -> 0.126 ms);
//  * a group of `ntg` consumer threads handles one row, thread t the MX block
//    t: its amax, scale and 16 code bytes need no shuffles (128x1 stripes
//    take two, over the 4 lanes of a stripe);
//  * G = slots / S groups (1, 2, 3 or 6) work on different ring slots, group g
//    owning the S consecutive slots g*S .. g*S + S - 1, so narrow rows still
//    fill the SM.  The group's slot base is folded into its lanes' gather
//    offsets and the loop over its S slots is unrolled, so every group runs
//    the same S copies of the loop body with the slot offset as the loads'
//    immediate (owning every G-th slot instead made the groups run different
//    copies and stall on instruction fetch);
//  * each lane keeps the shared-memory offsets and inv_s of its 32 gathered
//    elements in registers, in an order rotated by 2 * (lane / 2) elements:
//    lanes of a warp then read 32 different banks although their blocks lie
//    64 bytes apart; the 16 code bytes are rotated back before the store.
#include "w4a4_internal.h"

namespace w4a4 {

// up to 480 consumers + the producer warp: 16 warps, 4 per scheduler, so each
// thread may hold 128 registers (the 32 gather offsets and 32 inv_s of its
// block, its 32 products, and the rest)
constexpr int kPbMaxThreads = 512;

// The ring: NSLOT slots of SLOT bytes, a row plus a 16-byte zero slot each.
// Wide rows use prep_kernel's 6 x 32.9 KB; rows of up to 5480 elements use
// 18 x 11 KB (the same shared memory), so three times as many rows are in
// flight where a row is short.
template <int NSLOT, int SLOT>
struct PbRing {
  static constexpr int kSlots = NSLOT, kSlot = SLOT, kZero = SLOT - 16;
  static constexpr size_t kSmem = static_cast<size_t>(NSLOT) * SLOT + 2 * NSLOT * 8 + 16;
};
using PbWide = PbRing<kPrepStages, kPrepStage>;
using PbNarrow = PbRing<18, 10976>;

// bf16 at byte offset `off` of the ring, widened to the bits of a float
__device__ __forceinline__ float pb_ring_f32(const uint8_t* ring, uint32_t off) {
  return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(ring + off)) << 16);
}

template <int S, class R>
__global__ void __launch_bounds__(kPbMaxThreads, 1)
    prep_block_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t ldx, int d_in,
                      const float* __restrict__ inv_s, const int32_t* __restrict__ O,
                      const int32_t* __restrict__ jmap, int k, int k_pad, int kj, int nblk,
                      int ntg, uint8_t* __restrict__ aq, uint8_t* __restrict__ sfa,
                      uint32_t* __restrict__ xo, int stripe4, const int32_t* __restrict__ rows) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(R::kSlots) * R::kSlot);
  uint64_t* empty = full + R::kSlots;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(empty + R::kSlots);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int u = 0; u < R::kSlots; ++u) {
      mbar_init(&full[u], 1);
      // + the producer's outlier gather in the one-group form
      mbar_init(&empty[u], ntg / 32 + ((R::kSlots / S == 1 && k > 0) ? 1 : 0));
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  for (int u = threadIdx.x; u < R::kSlots; u += blockDim.x)
    *reinterpret_cast<uint4*>(smem + static_cast<size_t>(u) * R::kSlot + R::kZero) =
        make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  pdl_wait();                  // the shared-memory setup above overlaps the previous kernel
  pdl_launch_dependents();

  const int64_t nrows = T > blockIdx.x ? (T - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (warp == 0) {
    // ---------------- producer (whole warp; one elected lane issues) ----------------
    // The outlier columns of a row (X_O, k_pad / 2 bf16 pairs) are extra
    // work on top of the blocks; done always by the same consumer warp they
    // made it slower than the others, and every slot's refill waited for it.
    // With one thread group the producer gathers them (it waits for the row
    // to land, writes X_O, then arrives on the slot's "empty" barrier with the
    // consumer warps): down layer 0.350 -> 0.310 ms.  With several groups the
    // producer polls and must stay light, so the group's consumer warps take
    // the rows' outliers in turn (row i: warp i mod warps-per-group).
    const uint32_t bytes = static_cast<uint32_t>(d_in) * 2u;
    const int xo_pairs = k_pad >> 1;                        // bf16 pairs per row of X_O
    // the first two pairs of this lane (p = lane, lane + 32) from registers,
    // any further ones (k > 128) read O and inv_s again
    uint32_t po[4];
    float2 pinv[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int p2 = 2 * (lane + 32 * q);
      po[2 * q] = p2 < k ? 2u * static_cast<uint32_t>(O[p2]) : R::kZero;
      po[2 * q + 1] = p2 + 1 < k ? 2u * static_cast<uint32_t>(O[p2 + 1]) : R::kZero;
      pinv[q] = make_float2(p2 < k ? inv_s[O[p2]] : 1.f, p2 + 1 < k ? inv_s[O[p2 + 1]] : 1.f);
    }
    // X_O of ring row i (slot i mod kSlots, fill cycle i / kSlots); false if
    // the wait for the row gave up
    auto gather_outliers = [&](int64_t i) -> bool {
      const int uu = static_cast<int>(i % R::kSlots);
      if (!warp_wait_bounded(&full[uu], static_cast<uint32_t>((i / R::kSlots) & 1), abort_flag,
                             DEVERR_TIMEOUT_PREP))
        return false;
      const uint8_t* slot = smem + static_cast<size_t>(uu) * R::kSlot;
      uint32_t* xo_p = xo + (static_cast<int64_t>(blockIdx.x) + i * gridDim.x) * xo_pairs;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int pp = lane + 32 * q;
        if (pp < xo_pairs) {
          const float2 vv = __fmul2_rn(make_float2(pb_ring_f32(slot, po[2 * q]), pb_ring_f32(slot, po[2 * q + 1])),
                                       pinv[q]);
          xo_p[pp] = bf16_rn_bits(vv.x) | (bf16_rn_bits(vv.y) << 16);
        }
      }
      for (int pp = lane + 64; pp < xo_pairs; pp += 32) {
        const int o0 = 2 * pp;
        const uint32_t a0 = o0 < k ? 2u * static_cast<uint32_t>(O[o0]) : R::kZero;
        const uint32_t a1 = o0 + 1 < k ? 2u * static_cast<uint32_t>(O[o0 + 1]) : R::kZero;
        const float y0 = __fmul_rn(pb_ring_f32(slot, a0), o0 < k ? inv_s[O[o0]] : 1.f);
        const float y1 = __fmul_rn(pb_ring_f32(slot, a1), o0 + 1 < k ? inv_s[O[o0 + 1]] : 1.f);
        xo_p[pp] = bf16_rn_bits(y0) | (bf16_rn_bits(y1) << 16);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[uu]);
      return true;
    };
    // failure-detection test hook: no copies at all, the consumers' waits run out
    const bool skip = (g_fault_mask & FAULT_PREP_SKIP_LOADS) != 0u;
    constexpr int G = R::kSlots / S;
    if constexpr (G == 1) {
      // one group owns every slot: refill them in order, blocking on each
      int64_t issued = 0;
      int u = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int64_t i = 0; i < nrows && !skip; ++i) {
        if (i >= R::kSlots) {
          // the slot's previous row: its outliers, then the consumers' release
          if (k > 0 && !gather_outliers(i - R::kSlots)) {
            failed = true;
            break;
          }
          if (!warp_wait_bounded(&empty[u], ph ^ 1u, abort_flag, DEVERR_TIMEOUT_PREP)) {
            failed = true;
            break;
          }
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[u], bytes);
          const int64_t r = blockIdx.x + i * gridDim.x;
          // output row r reads input row rows[r] when a row map is given
          const uint16_t* from = X + (rows ? static_cast<int64_t>(rows[r]) : r) * ldx;
          bulk_load(smem + static_cast<size_t>(u) * R::kSlot, from, bytes, &full[u]);
        }
        __syncwarp();
        issued = i + 1;
        if (++u == R::kSlots) {
          u = 0;
          ph ^= 1u;
        }
      }
      // the outliers of the last rows in the ring
      for (int64_t i = issued > R::kSlots ? issued - R::kSlots : 0; k > 0 && !failed && i < issued; ++i)
        failed = !gather_outliers(i);
      if (lane == 0 && *abort_flag) {
        // do not leave bulk copies in flight into shared memory we give back
        const int64_t first = issued > R::kSlots ? issued - R::kSlots : 0;
        for (int64_t i = first; i < issued; ++i)
          mbar_wait_bounded(&full[i % R::kSlots], static_cast<uint32_t>((i / R::kSlots) & 1),
                            nullptr, DEVERR_TIMEOUT_PREP);
      }
    } else {
      // Rows go to the groups' slots in a fixed pattern (row i to group
      // i mod G, which owns slots g*S .. g*S + S - 1 and takes its rows in
      // turn -- groups' row counts differ by one at most), and each group
      // consumes its rows in order.  The producer refills whichever group's next slot is
      // free, so one slow group does not hold back the others' refills.
      int gc[G], gj[G];                       // per group: ring cycle and slot of its next row
#pragma unroll
      for (int q = 0; q < G; ++q) {
        gc[q] = 0;
        gj[q] = 0;
      }
      uint64_t idle_since = 0;
      bool failed = false;
      while (!skip) {
        bool left = false, progress = false;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const int64_t i = (static_cast<int64_t>(gc[q]) * S + gj[q]) * G + q;
          if (i >= nrows) continue;
          left = true;
          const int u = q * S + gj[q];
          bool free_slot = true;
          if (gc[q] > 0) {
            const uint32_t parity = static_cast<uint32_t>(gc[q] - 1) & 1u;
            free_slot = __shfl_sync(0xFFFFFFFFu, mbar_test_wait(smem_u32(&empty[u]), parity) ? 1 : 0, 0) != 0;
          }
          if (!free_slot) continue;
          if (elect_one()) {
            mbar_arrive_expect_tx(&full[u], bytes);
            const int64_t r = blockIdx.x + i * gridDim.x;
            // output row r reads input row rows[r] when a row map is given
            const uint16_t* from = X + (rows ? static_cast<int64_t>(rows[r]) : r) * ldx;
            bulk_load(smem + static_cast<size_t>(u) * R::kSlot, from, bytes, &full[u]);
          }
          __syncwarp();
          if (++gj[q] == S) {
            gj[q] = 0;
            ++gc[q];
          }
          progress = true;
        }
        if (!left) break;
        if (progress) {
          idle_since = 0;
          continue;
        }
        __nanosleep(32);
        if (*abort_flag) {
          failed = true;
          break;
        }
        const uint64_t now = globaltimer_ns();
        if (idle_since == 0) {
          idle_since = now;
        } else if (now - idle_since > *static_cast<volatile uint64_t*>(&g_wait_limit_ns)) {
          if (lane == 0) {
            atomicOr(&g_device_error, DEVERR_TIMEOUT_PREP);
            *abort_flag = 1u;
          }
          failed = true;
          break;
        }
      }
      if (lane == 0 && (failed || *abort_flag)) {
        // do not leave bulk copies in flight into shared memory we give back:
        // the latest fill of every slot
#pragma unroll
        for (int q = 0; q < G; ++q)
          for (int j = 0; j < S; ++j) {
            const int fills = gc[q] + (j < gj[q] ? 1 : 0);
            if (fills > 0)
              mbar_wait_bounded(&full[q * S + j], static_cast<uint32_t>(fills - 1) & 1u, nullptr,
                                DEVERR_TIMEOUT_PREP);
          }
      }
    }
    __syncwarp();
    return;
  }

  // ---------------- consumers ----------------
  const int ct = threadIdx.x - 32;
  const int g = ct / ntg;                   // group (uniform per warp: ntg % 32 == 0)
  const int t = ct - g * ntg;               // MX block of the row this thread encodes
  const bool enc = t < nblk;
  const int m = lane >> 1;
  const int rot = 2 * m;                    // processing order: element e reads (e + rot) mod 32
  const uint32_t gbase = static_cast<uint32_t>(g * S * R::kSlot);   // this group's first slot
  uint32_t go[32];
  float2 isv[16];
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    uint32_t o0 = R::kZero, o1 = R::kZero;
    float i0 = 1.f, i1 = 1.f;
    const int p0 = 32 * t + ((e + rot) & 31);
    const int p1 = 32 * t + ((e + 1 + rot) & 31);
    if (enc && p0 < kj) {
      const int j = jmap[p0];
      o0 = 2u * static_cast<uint32_t>(j);
      i0 = inv_s[j];
    }
    if (enc && p1 < kj) {
      const int j = jmap[p1];
      o1 = 2u * static_cast<uint32_t>(j);
      i1 = inv_s[j];
    }
    go[e] = gbase + o0;
    go[e + 1] = gbase + o1;
    isv[e >> 1] = make_float2(i0, i1);
  }
  // with several groups the group's warps gather the rows' outliers in turn:
  // this lane's pairs p = lane, lane + 32 (further ones read O and inv_s again)
  constexpr bool kConsumerXo = R::kSlots / S > 1;
  const int xo_pairs = k_pad >> 1;
  const int gwarp = t >> 5, gwarps = ntg >> 5;              // warp within the group, warps per group
  uint32_t po[4];
  float2 pinv[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int p2 = 2 * (lane + 32 * q);
    po[2 * q] = gbase + (p2 < k ? 2u * static_cast<uint32_t>(O[p2]) : R::kZero);
    po[2 * q + 1] = gbase + (p2 + 1 < k ? 2u * static_cast<uint32_t>(O[p2 + 1]) : R::kZero);
    pinv[q] = make_float2(p2 < k ? inv_s[O[p2]] : 1.f, p2 + 1 < k ? inv_s[O[p2 + 1]] : 1.f);
  }
  const int64_t aq_row = static_cast<int64_t>(nblk) * 16;   // bytes per row of codes
  // this lane's block in row 0 of the codes and of the scale atoms
  uint8_t* const aq_lane = aq + 16 * t;
  uint8_t* const sfa_lane = sfa + ((t >> 2) << 9) + (t & 3);
  const uint32_t atom_row = static_cast<uint32_t>(nblk >> 2) << 9;   // bytes per 128-row atom row
  const uint32_t ws = static_cast<uint32_t>(m) >> 2;        // the rotation back: whole words ...
  const uint32_t bs = 8u * (static_cast<uint32_t>(m) & 3u);  // ... then bits
  uint32_t ph = 0;
  bool ok = true;
  int xo_turn = 0;                                          // the group's warp that takes this row's outliers


  // this group's rows: g, g + G, g + 2G, ... (CTA-local), in its slots g*S + j
  constexpr int G = R::kSlots / S;
  for (int64_t n0 = 0; ok; n0 += S) {
#pragma unroll
    for (int j = 0; j < S; ++j) {
      const int u = g * S + j;
      const int64_t i = (n0 + j) * G + g;
      if (i >= nrows) {
        ok = false;                         // no rows left (not an error)
        break;
      }
      if (!warp_wait_bounded(&full[u], ph, abort_flag, DEVERR_TIMEOUT_PREP)) {
        ok = false;
        break;
      }
      const uint8_t* ring = smem + j * R::kSlot;          // compile-time offset (+ gbase in go)
      const int r = static_cast<int>(blockIdx.x + i * gridDim.x);   // T < 2^31
      float2 v[16];
      float amax = 0.f;
      if (enc) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          v[e] = __fmul2_rn(make_float2(pb_ring_f32(ring, go[2 * e]), pb_ring_f32(ring, go[2 * e + 1])),
                            isv[e]);
        amax = block_absmax32(v);            // NaN if any element is NaN
      }
      if (stripe4) {                        // 128x1 stripes: the 4 lanes of 4 consecutive blocks
        amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = max_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      }
      if (enc) {
        const uint32_t code = mx_scale_code(amax);
        const float inv = mx_inv_scale(code);
        const float2 inv2 = make_float2(inv, inv);
        const uint32_t keep = mx_nan_block_mask(code);
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 a0 = __fmul2_rn(v[4 * q], inv2), a1 = __fmul2_rn(v[4 * q + 1], inv2);
          const float2 a2 = __fmul2_rn(v[4 * q + 2], inv2), a3 = __fmul2_rn(v[4 * q + 3], inv2);
          w[q] = cvt_e2m1x8(a0.x, a0.y, a1.x, a1.y, a2.x, a2.y, a3.x, a3.y) & keep;
        }
        // nibble e holds element (e + rot) mod 32: rotate the 128 bits left by
        // 4 * rot = 32 * ws + bs bits
        uint32_t a0 = w[0], a1 = w[1], a2 = w[2], a3 = w[3];
        if (ws & 1u) {
          const uint32_t tmp = a3;
          a3 = a2;
          a2 = a1;
          a1 = a0;
          a0 = tmp;
        }
        if (ws & 2u) {
          uint32_t tmp = a0;
          a0 = a2;
          a2 = tmp;
          tmp = a1;
          a1 = a3;
          a3 = tmp;
        }
        const uint4 out = make_uint4(__funnelshift_l(a3, a0, bs), __funnelshift_l(a0, a1, bs),
                                     __funnelshift_l(a1, a2, bs), __funnelshift_l(a2, a3, bs));
        *reinterpret_cast<uint4*>(aq_lane + static_cast<int64_t>(r) * aq_row) = out;
        const uint32_t rl = static_cast<uint32_t>(r) & 127u;
        sfa_lane[static_cast<int64_t>(static_cast<uint32_t>(r) >> 7) * atom_row +
                 (((rl & 31u) << 4) | ((rl >> 5) << 2))] = static_cast<uint8_t>(code);
      }
      const bool my_turn = xo_turn == gwarp;
      if (++xo_turn == gwarps) xo_turn = 0;
      if (kConsumerXo && k > 0 && my_turn) {
        uint32_t* xo_p = xo + static_cast<int64_t>(r) * xo_pairs;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int pp = lane + 32 * q;
          if (pp < xo_pairs) {
            const float2 vv = __fmul2_rn(make_float2(pb_ring_f32(ring, po[2 * q]), pb_ring_f32(ring, po[2 * q + 1])),
                                         pinv[q]);
            xo_p[pp] = bf16_rn_bits(vv.x) | (bf16_rn_bits(vv.y) << 16);
          }
        }
        for (int pp = lane + 64; pp < xo_pairs; pp += 32) {
          const int o0 = 2 * pp;
          const uint32_t a0 = gbase + (o0 < k ? 2u * static_cast<uint32_t>(O[o0]) : R::kZero);
          const uint32_t a1 = gbase + (o0 + 1 < k ? 2u * static_cast<uint32_t>(O[o0 + 1]) : R::kZero);
          const float y0 = __fmul_rn(pb_ring_f32(ring, a0), o0 < k ? inv_s[O[o0]] : 1.f);
          const float y1 = __fmul_rn(pb_ring_f32(ring, a1), o0 + 1 < k ? inv_s[O[o0 + 1]] : 1.f);
          xo_p[pp] = bf16_rn_bits(y0) | (bf16_rn_bits(y1) << 16);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[u]);
    }
    ph ^= 1u;
  }
}

struct PrepBlockPlan {
  int groups, ntg;
};

// Threads per group: one per MX block (and at least one per outlier pair up
// to 512), rounded to warps; groups: the most of 6, 3, 2, 1 (divisors of the
// ring's slot count) that fit the thread limit.  ntg == 0: not supported.
static PrepBlockPlan plan_prep_block(const Geometry& g) {
  const int nblk = static_cast<int>(g.nblk);
  const int xo_pairs = static_cast<int>(g.k_pad / 2);
  int need = nblk > 0 ? nblk : 1;
  if (xo_pairs > need) need = xo_pairs < kPbMaxThreads - 32 ? xo_pairs : kPbMaxThreads - 32;
  const int ntg = static_cast<int>(round_up(need, 32));
  if (nblk > kPbMaxThreads - 32) return {0, 0};
  const int cand[4] = {6, 3, 2, 1};
  for (int c : cand)
    if (c * ntg + 32 <= kPbMaxThreads) return {c, ntg};
  return {0, 0};
}

template <int S, class R>
static cudaError_t launch_prep_block_s(const PrepBlockPlan& p, const void* X, int64_t T, int64_t ldx,
                                       const float* inv_s, const int32_t* O, const int32_t* jmap,
                                       const Geometry& g, uint8_t* aq, uint8_t* sfa, void* xo,
                                       cudaStream_t stream, bool stripe4, const int32_t* rows) {
  static_assert(R::kSlots % S == 0, "groups own whole blocks of ring slots");
  cudaError_t e = cudaFuncSetAttribute(prep_block_kernel<S, R>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(R::kSmem));
  if (e != cudaSuccess) return e;
  const int sms = device_num_sms();
  const int grid = static_cast<int>(T < sms ? T : sms);
  return launch_pdl(prep_block_kernel<S, R>, dim3(grid), dim3(p.groups * p.ntg + 32), R::kSmem, stream,
                    static_cast<const uint16_t*>(X), T, ldx, static_cast<int>(g.d_in), inv_s, O, jmap,
                    static_cast<int>(g.k), static_cast<int>(g.k_pad), static_cast<int>(g.kj),
                    static_cast<int>(g.nblk), p.ntg, aq, sfa, static_cast<uint32_t*>(xo),
                    stripe4 ? 1 : 0, rows);
}

bool prep_block_supported(const Geometry& g) {
  return g.d_in <= kPrepMaxD && plan_prep_block(g).ntg > 0;
}

cudaError_t launch_prep_block(const void* X, int64_t T, int64_t ldx, const float* inv_s,
                              const int32_t* O, const int32_t* jmap, const Geometry& g,
                              uint8_t* aq, uint8_t* sfa, void* xo, cudaStream_t stream,
                              bool stripe4, const int32_t* rows) {
  if (T == 0) return cudaSuccess;
  const PrepBlockPlan p = plan_prep_block(g);
  if (p.ntg == 0) return cudaErrorInvalidValue;
  // short rows: the 18-slot ring unless a single group would have to unroll
  // all 18 slots
  if (2 * g.d_in + 16 <= PbNarrow::kSlot && p.groups > 1) {
    switch (p.groups) {
      case 2: return launch_prep_block_s<9, PbNarrow>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
      case 3: return launch_prep_block_s<6, PbNarrow>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
      default: return launch_prep_block_s<3, PbNarrow>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    }
  }
  switch (p.groups) {
    case 1: return launch_prep_block_s<6, PbWide>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    case 2: return launch_prep_block_s<3, PbWide>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    case 3: return launch_prep_block_s<2, PbWide>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
    default: return launch_prep_block_s<1, PbWide>(p, X, T, ldx, inv_s, O, jmap, g, aq, sfa, xo, stream, stripe4, rows);
  }
}

}  // namespace w4a4
