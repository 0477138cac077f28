/*
 * libw4a4 -- W4A4 dual-branch linear layer for NVIDIA B200 (sm_100a).
 *
 * The method (paper review "W4A4 Quantization for Inference on
 * Wan2.2-I2V-A14B (ICME 2026 Challenge)", sections 3.2-3.4):
 *
 *   s_j  = act_scale_j^alpha / weight_scale_j^(1-alpha)          (sec. 3.2, eq. s_j)
 *   Y    = (X / s)(s * W)                                          (sec. 3.2, fold eq.)
 *   score_j = max_t |x_tj| on the smoothed X; O = top-k columns    (sec. 3.3, eq. score_j)
 *   Y    = X_J W^(q)_J + X_O W^(hp)_O                              (sec. 3.3, eq. Y)
 *
 * with the J branch in MXFP4 (OCP E2M1 elements, one E8M0 scale per 32
 * K-elements, shared exponent floor(log2 amax) - 2, round-half-to-even,
 * saturation at +-6) and the O branch in bfloat16.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers owned by the caller unless a parameter
 *    says "host".  The library never allocates device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream unless stated.
 *  - Matrices are row-major.  X is [T, d_in] bf16 with row stride ldx
 *    elements; W is [d_out, d_in] bf16 (row n = output channel n; this is the
 *    transpose of the pages' d_in x d_out W); Y is [T, d_out] bf16.
 *  - Arguments are validated before anything is launched.  On a non-OK
 *    return nothing was enqueued and outputs are untouched.  Calls that
 *    enqueue several steps (w4a4_linear, w4a4_linear_host,
 *    w4a4_linear_noalloc, w4a4_gemm_dual_act) check the arguments of every
 *    step, and build the GEMM's tensor maps, before the first one; only a
 *    failing launch itself (W4A4_ERR_CUDA) can leave earlier steps enqueued.
 *  - Supported shapes: d_in % 8 == 0, d_out % 16 == 0, row strides % 8 == 0,
 *    all pointers 16-byte aligned, d_in <= 16384.
 *    Anything else returns W4A4_ERR_UNSUPPORTED_SHAPE.
 *  - Device-side failures (a pipeline wait that runs out, about 2 s) are
 *    recorded in a device error word; w4a4_last_error() reads it.  No kernel
 *    traps.
 *  - The calibration, prep and GEMM kernels are launched with programmatic
 *    dependent launch: they may start their on-chip setup while the previous
 *    kernel in the stream finishes and wait for it before touching memory,
 *    so stream order holds as usual.  W4A4_NO_PDL=1 in the environment
 *    launches them plainly (read once per process).
 */
#ifndef W4A4_H
#define W4A4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4A4_ABI_VERSION 1

typedef enum w4a4_status {
  W4A4_OK = 0,
  W4A4_ERR_INVALID_ARG = 1,      /* null pointer, negative size, alpha outside (0,1), k > d_in */
  W4A4_ERR_UNSUPPORTED_SHAPE = 2,/* alignment or size outside the supported set above */
  W4A4_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed */
  W4A4_ERR_TIMEOUT = 4,          /* a device pipeline wait ran out (see w4a4_last_error) */
  W4A4_ERR_SCRATCH_LIMIT = 5,    /* the problem needs more scratch than w4a4_linear_noalloc has */
  W4A4_ERR_BAD_IMAGE = 6,        /* a packed-weight image failed its magic, version, size or checksum check */
  W4A4_ERR_NONFINITE_CALIB = 7   /* a calibration magnitude was inf or NaN (see w4a4_calib_finalize) */
} w4a4_status;

/* Weight scale layouts of the block packing (review sec. 3.4: "32x32 tiles"
 * and "128x1 K-major stripes"; 32x1 is the plain MXFP4 block).  All three
 * are stored in the same per-block MMA layout, so the GEMM reads them alike. */
typedef enum w4a4_wlayout {
  W4A4_SF_32x1_KMAJOR = 0,  /* one E8M0 per 32 consecutive compacted K of one output row */
  W4A4_SF_32x32_TILE = 1,   /* one E8M0 per 32 output rows x 32 compacted K, stored on each row */
  W4A4_SF_128x1_KMAJOR = 2  /* one E8M0 per 128 consecutive compacted K of one output row,
                               stored on each of its 4 blocks */
} w4a4_wlayout;

int w4a4_abi_version(void);
const char* w4a4_status_string(w4a4_status s);

/* ------------------------------------------------------------------------
 * Geometry.  kj = d_in - k columns go to the 4-bit branch after compaction
 * (O columns removed, review sec. 3.3); they are padded with zeros to kj_pad
 * = round_up(kj, 256) so the GEMM runs whole 256-element K tiles.  nblk =
 * kj_pad / 32 MX blocks per row.  k_pad = round_up(k, 16) bf16 columns per
 * row of X_O and W_hp (zero padded).  sfa_rows(T) = round_up(T, 128);
 * sfb_rows = round_up(d_out, 256).
 *
 * Scale-factor buffers use the block-scaled MMA layout: 512-byte atoms of
 * 128 rows x 4 blocks, atoms ordered K-fastest; inside an atom row r, block
 * b sits at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4).  The byte of
 * (row r, block b) is therefore
 *   ((r / 128) * (nblk / 4) + b / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + b % 4.
 * ------------------------------------------------------------------------ */
typedef struct w4a4_dims {
  int64_t d_in, d_out, k;
  int64_t kj;       /* d_in - k */
  int64_t kj_pad;   /* round_up(kj, 256) */
  int64_t nblk;     /* kj_pad / 32 */
  int64_t k_pad;    /* round_up(k, 16) */
  int64_t sfb_rows; /* round_up(d_out, 256) */
} w4a4_dims;

/* Fills *out.  INVALID_ARG if out is NULL, a size is negative or k > d_in. */
w4a4_status w4a4_get_dims(int64_t d_in, int64_t d_out, int64_t k, w4a4_dims* out);

/* ------------------------------------------------------------------------
 * Calibration (offline).  Review sec. 3.1-3.2: per-channel magnitudes of
 * activations and weights; read here as the per-column absolute maximum.
 * ------------------------------------------------------------------------ */

/* absmax[j] = max(absmax[j], max_r |A[r, j]|) for j < cols (absmax zeroed
 * first when reset != 0).  A: bf16 [rows, cols] with row stride lda.  Used
 * for activation batches X [T, d_in] (act_scale) and for W [d_out, d_in]
 * (weight_scale).  absmax: float32 [cols].  rows may be 0.  NaN inputs make
 * the column NaN. */
w4a4_status w4a4_calib_observe(const void* A, int64_t rows, int64_t cols, int64_t lda,
                               float* absmax, int reset, void* stream);

/* One layer's magnitudes from one batch in one launch: the column absmax of
 * X [T, d_in] (row stride ldx) into act_absmax and of W [d_out, d_in] (row
 * stride ldw) into w_absmax, both float32 [d_in] -- the values of
 * w4a4_calib_observe on X and on W (reset applies to both).  T or d_out may
 * be 0.  Further activation batches go through w4a4_calib_observe with
 * reset = 0.  Errors: INVALID_ARG for null or negative arguments, strides
 * below d_in or act_absmax == w_absmax; UNSUPPORTED_SHAPE unless d_in, ldx
 * and ldw are multiples of 8 and X and W are 16-byte aligned. */
w4a4_status w4a4_calib_observe_layer(const void* X, int64_t T, int64_t ldx, const void* W,
                                     int64_t d_out, int64_t ldw, int64_t d_in, float* act_absmax,
                                     float* w_absmax, int reset, void* stream);

/* From act_scale and w_scale (float32 [d_in]) compute, on the device:
 *   s[j]     = fl32( max(a,1e-5)^alpha / max(w,1e-5)^(1-alpha) )  in float64
 *   inv_s[j] = fl32( 1 / s[j] )
 *   score[j] = fl32( act_scale[j] * inv_s[j] )  (= max_t |fl32(x_tj inv_s_j)|,
 *              the score on the smoothed activations; review sec. 3.3, 3.5)
 *   O        = the k columns of largest score, ties to the lower index,
 *              ascending (int32 [k]);  jmap = the other d_in - k columns
 *              ascending (int32 [d_in - k]).
 * Requires 0 < alpha < 1, 0 <= k <= d_in, d_in >= 1 (else INVALID_ARG);
 * d_in > 16384 returns UNSUPPORTED_SHAPE.  O may be NULL when k == 0 and
 * jmap may be NULL when k == d_in.
 * s is defined for finite magnitudes only: if act_scale or w_scale holds an
 * inf or a NaN (calibration data that were not finite), the kernel records it
 * in the device error word -- w4a4_last_error then returns
 * W4A4_ERR_NONFINITE_CALIB -- and s, inv_s, score, O and jmap are
 * unspecified. */
w4a4_status w4a4_calib_finalize(const float* act_scale, const float* w_scale, int64_t d_in,
                                double alpha, int64_t k, float* s, float* inv_s, float* score,
                                int32_t* O, int32_t* jmap, void* stream);

/* ------------------------------------------------------------------------
 * Packed weight (offline).  Review sec. 3.2 (fold s into W), 3.3 (drop the O
 * channels into the bf16 branch, static O kept as a sparse index list), 3.4
 * (block-wise 4-bit packing with the exponent stored beside the payload).
 * ------------------------------------------------------------------------ */
typedef struct w4a4_weight_bytes {
  size_t wq;    /* d_out * kj_pad / 2           E2M1 codes, row n: kj_pad/2 bytes */
  size_t sfb;   /* sfb_rows * nblk               E8M0 codes, MMA layout            */
  size_t w_hp;  /* d_out * k_pad * 2             bf16                              */
} w4a4_weight_bytes;

w4a4_status w4a4_weight_sizes(int64_t d_in, int64_t d_out, int64_t k, w4a4_weight_bytes* out);

/* The per-layer record the online path reads.  All pointers are caller-owned
 * device memory; the record itself lives on the host and is only read. */
typedef struct w4a4_packed_weight {
  int64_t d_in, d_out, k;
  int32_t layout;        /* w4a4_wlayout */
  int32_t reserved;
  uint8_t* wq;           /* [d_out, kj_pad/2]: code of folded W[n, jmap[p]] at p (low nibble = even p) */
  uint8_t* sfb;          /* MMA layout, sfb_rows x nblk; rows >= d_out hold code 0 */
  void* w_hp;            /* bf16 [d_out, k_pad]: bf16_rn(fl32(W[n, O[i]] * s[O[i]])) */
  const float* inv_s;    /* float32 [d_in] from w4a4_calib_finalize */
  const int32_t* O;      /* int32 [k] ascending (NULL if k == 0) */
  const int32_t* jmap;   /* int32 [d_in - k] ascending (NULL if k == d_in) */
} w4a4_packed_weight;

/* Fold and pack.  W: bf16 [d_out, d_in] with row stride ldw.  s, O, jmap from
 * w4a4_calib_finalize.  Fills pw->wq, pw->sfb, pw->w_hp (which must point to
 * buffers of the sizes w4a4_weight_sizes reports) and reads pw->d_in,
 * d_out, k, layout.  Every element of wq/sfb/w_hp, padding included, is
 * written.  Row n, compacted position p: v = fl32(W[n, jmap[p]] * s[jmap[p]]);
 * MX blocks are p = 32b .. 32b+31 (zeros beyond kj). */
w4a4_status w4a4_pack_weight(const void* W, int64_t ldw, const float* s,
                             const w4a4_packed_weight* pw, void* stream);

/* ------------------------------------------------------------------------
 * Online path.  Review sec. 3.2 (activations divided by s, then quantised)
 * and sec. 3.3 (dual-branch GEMM).
 * ------------------------------------------------------------------------ */

/* Bytes of device workspace w4a4_linear needs for T tokens: Aq
 * (T * kj_pad / 2), SFA (round_up(T,128) * nblk) and X_O (T * k_pad * 2),
 * each 1024-byte aligned. */
w4a4_status w4a4_workspace_size(int64_t T, int64_t d_in, int64_t d_out, int64_t k, size_t* bytes);

/* Activation preparation (one pass over X).  For row t and column j,
 * v = fl32(X[t, j] * inv_s[j]) (one IEEE multiply).  Writes
 *   xo  bf16 [T, k_pad]       xo[t, i] = bf16_rn(v at j = O[i]), zeros for i >= k
 *   aq  u8   [T, kj_pad/2]    E2M1 codes of v at j = jmap[p] (zeros for p >= kj)
 *   sfa u8   MMA layout, round_up(T,128) x nblk; rows >= T are not written
 * Each 32-element block takes e = clamp(floor(log2 amax) - 2, -127, 127),
 * code = e + 127 (0 for an all-zero block), elements v * 2^-e rounded to
 * E2M1 (nearest, ties to even, saturating at 6, sign kept).
 * Non-finite values (inf or NaN in X, or a product x * inv_s beyond the
 * float32 range, which is +-inf) follow IEEE float32 arithmetic: amax is the
 * NaN-propagating maximum of |v|; a block holding a NaN gets scale code 0xFF
 * (E8M0's NaN) and all-zero element codes; a block holding an infinity (and
 * no NaN) gets e = 127 (code 254), its infinities saturate to +-6 and its
 * finite elements are v * 2^-127 on the E2M1 grid; an outlier column takes
 * bf16_rn(v): +-inf stays +-inf and every NaN is written as 0x7FC0.
 * aq, sfa, xo may be NULL when their size is zero. */
w4a4_status w4a4_prep_act(const void* X, int64_t T, int64_t ldx, const w4a4_packed_weight* pw,
                          uint8_t* aq, uint8_t* sfa, void* xo, void* stream);

/* Dual-branch product Y[t, n] = sum_p deq(aq)[t,p] deq(wq)[n,p]
 *                              + sum_i xo[t,i] w_hp[n,i]
 * accumulated in float32 in tensor memory (tcgen05 kind::mxf4 block-scaled
 * tiles and kind::f16 tiles into the same accumulator), rounded to bf16.
 * Y: bf16 [T, d_out] with row stride ldy.
 * Tiles: T <= 128 runs one CTA per 128 x 256 tile; larger T a CTA pair per
 * 256 x 384 tile where 384 divides d_out, else per 256 x 256 tile.  The
 * environment variable W4A4_PAIR_TILE_N=256 keeps every pair launch on the
 * 256-wide tile (read once per process); both widths gave bit-identical Y
 * on every shape tested. */
w4a4_status w4a4_gemm_dual(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                           const w4a4_packed_weight* pw, void* Y, int64_t ldy, void* stream);

/* The online layer: w4a4_prep_act into the workspace, then w4a4_gemm_dual.
 * ws_bytes must be at least w4a4_workspace_size(T, ...). */
w4a4_status w4a4_linear(const void* X, int64_t T, int64_t ldx, const w4a4_packed_weight* pw,
                        void* workspace, size_t ws_bytes, void* Y, int64_t ldy, void* stream);

/* The online layer from and to HOST memory: copies X_host (bf16 [T, d_in],
 * dense rows; pinned memory gives an asynchronous copy) to X_dev, runs
 * w4a4_linear, copies Y_dev back to Y_host (bf16 [T, d_out], dense rows), all
 * on `stream`.  X_dev / Y_dev are caller-owned device buffers of those sizes.
 * Returns once the work is enqueued; synchronise the stream before reading
 * Y_host. */
w4a4_status w4a4_linear_host(const void* X_host, int64_t T, const w4a4_packed_weight* pw,
                             void* X_dev, void* workspace, size_t ws_bytes, void* Y_dev,
                             void* Y_host, void* stream);

/* ------------------------------------------------------------------------
 * Packed-weight images (checkpoints).  The offline result of a layer --
 * Wq, SFB, W_hp, s, inv_s, O, jmap -- as one host byte image: a 256-byte
 * header (magic "W4A4PKW1", format version, layout, d_in, d_out, k, the
 * section sizes, an FNV-1a 64 checksum of the section bytes) followed by the
 * sections in that order, each padded to 64 bytes.  The review's static O and
 * offline fold (sec. 3.3, 3.5) make this record the complete state of a
 * quantised layer.  Host buffers are caller-owned; pinned memory makes the
 * copies faster.  Each call synchronises `stream`.
 * ------------------------------------------------------------------------ */

/* Bytes of the image of *pw. */
w4a4_status w4a4_packed_image_size(const w4a4_packed_weight* pw, size_t* bytes);

/* Writes the image of *pw (device buffers named in the record, plus s, a
 * float32 [d_in] device array) to host[0 .. bytes).  INVALID_ARG if bytes is
 * below w4a4_packed_image_size or a needed pointer is NULL. */
w4a4_status w4a4_packed_save(const w4a4_packed_weight* pw, const float* s, void* host,
                             size_t bytes, void* stream);

/* Reads the header of an image: d_in, d_out, k, layout (any output pointer
 * may be NULL), so a caller can allocate the buffers before loading.
 * BAD_IMAGE on a wrong magic or version, inconsistent sizes, a short buffer
 * or a checksum mismatch. */
w4a4_status w4a4_packed_image_info(const void* host, size_t bytes, int64_t* d_in, int64_t* d_out,
                                   int64_t* k, int32_t* layout);

/* Copies an image into the device buffers the record *pw names (its inv_s,
 * O and jmap arrays are written too) and into s.  The record's d_in, d_out,
 * k and layout must equal the image's (else INVALID_ARG); BAD_IMAGE as for
 * w4a4_packed_image_info. */
w4a4_status w4a4_packed_load(const void* host, size_t bytes, const w4a4_packed_weight* pw,
                             float* s, void* stream);

/* ------------------------------------------------------------------------
 * The FFN pair (review sec. 3.1, 3.5: both FFN projections, ffn.0 up and
 * ffn.2 down, take the same W4A4 recipe).  Between them the Wan2.2 FFN
 * applies GELU, which the pages do not write out; here X_down[t, c] is the
 * bf16 value nearest (ties to even) the exact GELU in tanh form,
 * gelu(y) = 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), of the bf16
 * value y = bf16_rn(Y_up[t, c]): a function of the 16-bit input, the same
 * whether fused or not.  +inf maps to +inf, -inf and NaN to NaN.
 *
 * Fused use: calibrate and pack the down layer, w4a4_ffn_link it, pack the up
 * weight in its natural channel order and reorder that pack with
 * w4a4_permute_packed_rows(rows = perm), then per batch
 * w4a4_prep_act (up) -> w4a4_gemm_dual_act (up, writing the down layer's Aq,
 * SFA, X_O) -> w4a4_gemm_dual (down).
 * ------------------------------------------------------------------------ */

/* X[t, j] = bf16_rn(gelu(Y[t, j])) for a bf16 [T, d] matrix (row strides
 * ldy, ldx elements; X may be Y); the unfused activation, e.g. to calibrate
 * the down layer.  Errors: INVALID_ARG for negative sizes, ld < d or a null
 * pointer with T, d > 0. */
w4a4_status w4a4_gelu_bf16(const void* Y, int64_t T, int64_t d, int64_t ldy, void* X, int64_t ldx,
                           void* stream);

/* For a packed down layer `next`: perm[c] (int32 [d_in]) = jmap[c] for
 * c < kj, O[c - kj] after, and inv_s_perm[c] = inv_s[perm[c]] (float32
 * [d_in]): the up layer's output-channel order under which the down layer's
 * compacted input is contiguous. */
w4a4_status w4a4_ffn_link(const w4a4_packed_weight* next, int32_t* perm, float* inv_s_perm,
                          void* stream);

/* w4a4_pack_weight with the rows of W permuted: packed output channel n is
 * W row rows[n] (rows: int32 [d_out] device array).  This packs the permuted
 * matrix: with 32x32 tiles, a tile groups 32 consecutive permuted rows, so
 * the result differs from a reordered natural pack; for the fused FFN use
 * w4a4_permute_packed_rows. */
w4a4_status w4a4_pack_weight_rows(const void* W, int64_t ldw, const float* s, const int32_t* rows,
                                  const w4a4_packed_weight* pw, void* stream);

/* dst = src with its output channels reordered: packed row r of dst is packed
 * row rows[r] of src (rows: int32 [d_out] device array, a permutation) -- the
 * E2M1 codes, the E8M0 scales (each row keeps its scale from src, so 32x32
 * tiles stay the tiles of src's channel order) and the bf16 outlier rows.
 * src and dst: same d_in, d_out, k and layout, distinct buffers; dst's
 * input-side arrays (s, inv_s, O, jmap) are not written (the caller shares
 * or copies them).  Asynchronous on `stream`.  Errors: INVALID_ARG for
 * mismatched shapes, a null `rows` or shared output buffers. */
w4a4_status w4a4_permute_packed_rows(const w4a4_packed_weight* src, const int32_t* rows,
                                     const w4a4_packed_weight* dst, void* stream);

/* The up projection with the fused FFN epilogue: computes the dual-branch
 * product of (aq, sfa, xo) with pw (packed with rows = perm) and, instead of
 * storing Y, writes the down layer's activation buffers as w4a4_prep_act
 * would for X = bf16_rn(gelu(bf16 Y)) in its original channel order:
 * aq_next [T, kj_pad/2], sfa_next (MMA layout), xo_next bf16 [T, k_pad].
 * next->d_in must equal pw->d_out.  inv_s_perm from w4a4_ffn_link. */
w4a4_status w4a4_gemm_dual_act(const uint8_t* aq, const uint8_t* sfa, const void* xo, int64_t T,
                               const w4a4_packed_weight* pw, const w4a4_packed_weight* next,
                               const float* inv_s_perm, uint8_t* aq_next, uint8_t* sfa_next,
                               void* xo_next, void* stream);

/* Size of the fixed device scratch array behind w4a4_linear_noalloc. */
#define W4A4_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* The online layer (w4a4_prep_act then w4a4_gemm_dual, exactly as
 * w4a4_linear) without a caller workspace and without allocating anything.
 * The paper has no counterpart to this call: it is a service for callers that
 * cannot hand the library device memory at the point where the layer runs --
 * a host framework or plugin that owns every device allocation and passes
 * only inputs and outputs, or a serving loop whose device memory is fixed at
 * start-up, where allocating (and the synchronisation cudaMalloc / cudaFree
 * may imply) is not allowed per call.
 *   Scratch: a static device array of W4A4_NOALLOC_SCRATCH_BYTES (32 MiB) in
 *   the library, held on every device the library is used on until the
 *   process exits.  A problem whose w4a4_workspace_size exceeds it returns
 *   W4A4_ERR_SCRATCH_LIMIT before anything is enqueued (at d_in = 5120,
 *   k = 32 about 12000 tokens fit; use w4a4_linear for larger T).
 *   Sharing: every call on a device uses the same array, which keeps what the
 *   previous call left there.  No byte needs clearing -- the scale rows past T
 *   that a call reads without writing reach only output rows past T, which
 *   are never stored -- but calls whose GPU work overlaps (other streams,
 *   other host threads) race on the array and must be serialised by the
 *   caller.
 *   Set-up: the first call in each CUDA context looks up the array's device
 *   address in that context (a host-side query with the device current;
 *   nothing is allocated) -- normally once per device, in its primary
 *   context.  The lookup is cached by the context's unique id, so a caller's
 *   own driver-API context, or a new primary context after cudaDeviceReset,
 *   gets its own address.  Make the first call in a context before any stream
 *   capture.
 * Arguments, layouts and the other errors are those of w4a4_linear. */
w4a4_status w4a4_linear_noalloc(const void* X, int64_t T, int64_t ldx,
                                const w4a4_packed_weight* pw, void* Y, int64_t ldy,
                                void* stream);

/* Layer-wise parameter choice (review sec. 4 table and sec. 6: alpha and k
 * per layer are the next step; the pages give no procedure).  Sums over a
 * T x d_out block, in float64: sums[0] = sum (Y - Yref)^2, sums[1] =
 * sum Yref^2, with Y bf16 (row stride ldy) and Yref float32 (row stride ldr);
 * sums is a device array of 2 doubles, zeroed by the call.  A search scores a
 * candidate (alpha, k, layout) by sqrt(sums[0] / sums[1]). */
w4a4_status w4a4_error_sums(const void* Y, int64_t ldy, const float* Yref, int64_t ldr, int64_t T,
                            int64_t d_out, double* sums, void* stream);

/* Synchronises `stream` and reports device-side failures recorded since the
 * last clear: W4A4_OK, W4A4_ERR_TIMEOUT if a bounded wait ran out (the
 * affected output is incomplete; reported first), or W4A4_ERR_NONFINITE_CALIB
 * if w4a4_calib_finalize met an inf or NaN magnitude.  *bits (may be NULL) receives the raw
 * error word.  clear != 0 resets the word. */
w4a4_status w4a4_last_error(void* stream, int clear, uint32_t* bits);

/* Failure-detection test hook, not for production use.  Sets, on the current
 * device, how long a device pipeline wait may last before it is abandoned
 * (wait_limit_ns; 0 restores the default of about 2 s; at most the default)
 * and a fault mask: W4A4_FAULT_PREP_SKIP_LOADS makes the activation-prep
 * kernel's producer issue no row copies, so every consumer wait of the next
 * prep launches runs out -- the kernel records W4A4_ERR_TIMEOUT in the device
 * error word and returns, leaving its outputs incomplete, with no trap and the
 * context usable.  Synchronises the device first.  Call with (0, 0) to
 * restore normal operation.  INVALID_ARG for an unknown mask bit or a limit
 * above the default. */
#define W4A4_FAULT_PREP_SKIP_LOADS 1u
w4a4_status w4a4_test_fault(uint32_t mask, uint64_t wait_limit_ns);

/* Number of streaming multiprocessors of the current device (used to size
 * persistent grids); 0 on error. */
int w4a4_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A4_H */
