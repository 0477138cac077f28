// Packed-weight images: the offline result of one layer (codes, scales, the
// bf16 outlier columns, s / inv_s and the O / J index lists) copied to a host
// byte buffer and back, so a calibrated and packed layer can be stored and
// reloaded without recalibrating.  The review's deterministic inference
// graph (static O, offline fold) is what makes the packed record a complete,
// reusable artefact.
//
// Image layout (little-endian, every section 64-byte aligned):
//   header   ImageHeader (magic "W4A4PKW1", format version, layout, d_in,
//            d_out, k, section sizes, FNV-1a 64 of all section bytes)
//   wq       d_out * kj_pad / 2 bytes
//   sfb      sfb_rows * nblk bytes
//   w_hp     d_out * k_pad * 2 bytes
//   s        d_in float32
//   inv_s    d_in float32
//   O        k int32
//   jmap     (d_in - k) int32
#include <cstring>

#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {

constexpr char kImageMagic[8] = {'W', '4', 'A', '4', 'P', 'K', 'W', '1'};
constexpr uint32_t kImageVersion = 1;
constexpr int kImageSections = 7;
constexpr size_t kImageAlign = 64;

struct ImageHeader {
  char magic[8];
  uint32_t version;
  int32_t layout;
  int64_t d_in, d_out, k;
  uint64_t size[kImageSections];
  uint64_t fnv;
};
static_assert(sizeof(ImageHeader) <= 256, "header fits its 256-byte slot");
constexpr size_t kHeaderSlot = 256;

static size_t align_up(size_t a) { return (a + kImageAlign - 1) / kImageAlign * kImageAlign; }

static void section_sizes(const Geometry& g, uint64_t size[kImageSections]) {
  size[0] = static_cast<uint64_t>(g.d_out * g.kj_pad / 2);      // wq
  size[1] = static_cast<uint64_t>(g.sfb_rows * g.nblk);          // sfb
  size[2] = static_cast<uint64_t>(g.d_out * g.k_pad * 2);        // w_hp
  size[3] = static_cast<uint64_t>(g.d_in * 4);                   // s
  size[4] = static_cast<uint64_t>(g.d_in * 4);                   // inv_s
  size[5] = static_cast<uint64_t>(g.k * 4);                      // O
  size[6] = static_cast<uint64_t>((g.d_in - g.k) * 4);           // jmap
}

static size_t image_total(const uint64_t size[kImageSections]) {
  size_t t = kHeaderSlot;
  for (int i = 0; i < kImageSections; ++i) t += align_up(size[i]);
  return t;
}

// FNV-1a, 64 bit, over the section bytes in order
static uint64_t fnv1a(const uint8_t* base, const uint64_t size[kImageSections]) {
  uint64_t h = 1469598103934665603ull;
  size_t off = kHeaderSlot;
  for (int i = 0; i < kImageSections; ++i) {
    const uint8_t* p = base + off;
    for (uint64_t j = 0; j < size[i]; ++j) {
      h ^= p[j];
      h *= 1099511628211ull;
    }
    off += align_up(size[i]);
  }
  return h;
}

}  // namespace w4a4

using namespace w4a4;

// The packed record's device pointers for the sections, with the record's
// s pointer taken from `s` (the record itself carries inv_s only).
static void section_ptrs(const w4a4_packed_weight* pw, const float* s, const void* p[kImageSections]) {
  p[0] = pw->wq;
  p[1] = pw->sfb;
  p[2] = pw->w_hp;
  p[3] = s;
  p[4] = pw->inv_s;
  p[5] = pw->O;
  p[6] = pw->jmap;
}

extern "C" w4a4_status w4a4_packed_image_size(const w4a4_packed_weight* pw, size_t* bytes) {
  Geometry g;
  const w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (bytes == nullptr) return W4A4_ERR_INVALID_ARG;
  uint64_t size[kImageSections];
  section_sizes(g, size);
  *bytes = image_total(size);
  return W4A4_OK;
}

extern "C" w4a4_status w4a4_packed_save(const w4a4_packed_weight* pw, const float* s, void* host,
                                        size_t bytes, void* stream) {
  Geometry g;
  w4a4_status st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (host == nullptr || s == nullptr) return W4A4_ERR_INVALID_ARG;
  uint64_t size[kImageSections];
  section_sizes(g, size);
  if (bytes < image_total(size)) return W4A4_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(host);
  memset(base, 0, image_total(size));
  const void* src[kImageSections];
  section_ptrs(pw, s, src);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  size_t off = kHeaderSlot;
  for (int i = 0; i < kImageSections; ++i) {
    if (size[i] > 0) {
      if (src[i] == nullptr) return W4A4_ERR_INVALID_ARG;
      const cudaError_t e =
          cudaMemcpyAsync(base + off, src[i], size[i], cudaMemcpyDeviceToHost, strm);
      if (e != cudaSuccess) return W4A4_ERR_CUDA;
    }
    off += align_up(size[i]);
  }
  if (cudaStreamSynchronize(strm) != cudaSuccess) return W4A4_ERR_CUDA;
  ImageHeader h;
  memset(&h, 0, sizeof(h));
  memcpy(h.magic, kImageMagic, sizeof(h.magic));
  h.version = kImageVersion;
  h.layout = pw->layout;
  h.d_in = pw->d_in;
  h.d_out = pw->d_out;
  h.k = pw->k;
  for (int i = 0; i < kImageSections; ++i) h.size[i] = size[i];
  h.fnv = fnv1a(base, size);
  memcpy(base, &h, sizeof(h));
  return W4A4_OK;
}

// Header checks shared by info and load: magic, version, sizes consistent
// with the dims, image long enough, checksum.
static w4a4_status read_header(const void* host, size_t bytes, ImageHeader* h, Geometry* g) {
  if (host == nullptr || bytes < kHeaderSlot) return W4A4_ERR_BAD_IMAGE;
  memcpy(h, host, sizeof(*h));
  if (memcmp(h->magic, kImageMagic, sizeof(h->magic)) != 0 || h->version != kImageVersion)
    return W4A4_ERR_BAD_IMAGE;
  w4a4_dims d;
  if (w4a4_get_dims(h->d_in, h->d_out, h->k, &d) != W4A4_OK) return W4A4_ERR_BAD_IMAGE;
  *g = make_geometry(h->d_in, h->d_out, h->k);
  uint64_t size[kImageSections];
  section_sizes(*g, size);
  for (int i = 0; i < kImageSections; ++i)
    if (h->size[i] != size[i]) return W4A4_ERR_BAD_IMAGE;
  if (bytes < image_total(size)) return W4A4_ERR_BAD_IMAGE;
  if (fnv1a(static_cast<const uint8_t*>(host), size) != h->fnv) return W4A4_ERR_BAD_IMAGE;
  return W4A4_OK;
}

extern "C" w4a4_status w4a4_packed_image_info(const void* host, size_t bytes, int64_t* d_in,
                                              int64_t* d_out, int64_t* k, int32_t* layout) {
  ImageHeader h;
  Geometry g;
  const w4a4_status st = read_header(host, bytes, &h, &g);
  if (st != W4A4_OK) return st;
  if (d_in) *d_in = h.d_in;
  if (d_out) *d_out = h.d_out;
  if (k) *k = h.k;
  if (layout) *layout = h.layout;
  return W4A4_OK;
}

extern "C" w4a4_status w4a4_packed_load(const void* host, size_t bytes, const w4a4_packed_weight* pw,
                                        float* s, void* stream) {
  ImageHeader h;
  Geometry gi;
  w4a4_status st = read_header(host, bytes, &h, &gi);
  if (st != W4A4_OK) return st;
  Geometry g;
  st = check_pw(pw, &g);
  if (st != W4A4_OK) return st;
  if (pw->d_in != h.d_in || pw->d_out != h.d_out || pw->k != h.k || pw->layout != h.layout)
    return W4A4_ERR_INVALID_ARG;
  if (s == nullptr) return W4A4_ERR_INVALID_ARG;
  const void* dst_c[kImageSections];
  section_ptrs(pw, s, dst_c);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  const uint8_t* base = static_cast<const uint8_t*>(host);
  size_t off = kHeaderSlot;
  for (int i = 0; i < kImageSections; ++i) {
    if (h.size[i] > 0) {
      if (dst_c[i] == nullptr) return W4A4_ERR_INVALID_ARG;
      const cudaError_t e = cudaMemcpyAsync(const_cast<void*>(dst_c[i]), base + off, h.size[i],
                                            cudaMemcpyHostToDevice, strm);
      if (e != cudaSuccess) return W4A4_ERR_CUDA;
    }
    off += align_up(h.size[i]);
  }
  return cudaStreamSynchronize(strm) == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}
