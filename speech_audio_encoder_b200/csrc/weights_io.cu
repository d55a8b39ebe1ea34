// The flat weight file: sal_weights_file_info reads and checks its header;
// sal_weights_file_load streams its tensors into one device buffer and fills the
// sal_weights record that points into it.
//
// Layout (little-endian; include/sal.h states it in full): a 256-byte header, then every
// tensor as row-major bf16, each starting on a 256-byte boundary (zero padding between),
// in the order w_proj, b_proj, lnf_g, lnf_b, then per layer ln1_g, ln1_b, w_qkv, b_qkv,
// qn_g, kn_g, w_o, b_o, ln2_g, ln2_b, w1, b1, w2, b2. The data region is byte for byte the
// device buffer, so loading is one stream of host-to-device copies and the record is a
// table of offsets.
//
// The copy goes through two pinned staging buffers: while chunk i is being copied to the
// device from one, chunk i + 1 is read from the file into the other.
#include <stdio.h>
#include <string.h>
#include <sys/stat.h>

#include <cstdint>

#include "sal_internal.h"

namespace sal {
namespace {

constexpr char kMagic[8] = {'S', 'A', 'L', 'E', 'N', 'C', 'W', '1'};
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 256;
constexpr uint32_t kDtypeBf16 = 1;
constexpr uint32_t kAlign = 256;
constexpr size_t kStageBytes = size_t(32) << 20;
constexpr int kLayerTensors = 14;

struct Header {
  char magic[8];
  uint32_t version, header_bytes, dtype;
  uint32_t width, heads, head_dim, ffn, stack_dim, n_layers, align;
  uint64_t data_bytes;
};
static_assert(sizeof(Header) == 56, "header layout");

uint64_t padded(uint64_t elems) { return (elems * 2 + kAlign - 1) / kAlign * kAlign; }

// Elements of each global tensor (w_proj, b_proj, lnf_g, lnf_b) and of each layer tensor,
// in file order.
constexpr uint64_t kGlobalElems[4] = {uint64_t(kWidth) * kStack * kMels, kWidth, kWidth, kWidth};
constexpr uint64_t kLayerElems[kLayerTensors] = {
    kWidth, kWidth, uint64_t(3) * kWidth * kWidth, 3 * kWidth, kHeadDim, kHeadDim, uint64_t(kWidth) * kWidth,
    kWidth, kWidth, kWidth, uint64_t(kFfn) * kWidth, kFfn, uint64_t(kWidth) * kFfn, kWidth};

uint64_t data_bytes_for(uint64_t n_layers) {
  uint64_t b = 0, per_layer = 0;
  for (uint64_t e : kGlobalElems) b += padded(e);
  for (uint64_t e : kLayerElems) per_layer += padded(e);
  return b + n_layers * per_layer;
}

// Reads and checks the header of `f` (opened for reading) against the library's sizes
// and the file's length.
sal_status read_header(FILE* f, Header* h) {
  unsigned char raw[kHeaderBytes];
  if (fread(raw, 1, kHeaderBytes, f) != kHeaderBytes) return SAL_EINVAL;  // shorter than a header
  memcpy(h, raw, sizeof(Header));
  if (memcmp(h->magic, kMagic, sizeof(kMagic)) != 0 || h->version != kVersion || h->header_bytes != kHeaderBytes ||
      h->dtype != kDtypeBf16 || h->align != kAlign)
    return SAL_EINVAL;
  for (size_t i = sizeof(Header); i < kHeaderBytes; ++i)
    if (raw[i] != 0) return SAL_EINVAL;  // reserved bytes
  if (h->width != kWidth || h->heads != kHeads || h->head_dim != kHeadDim || h->ffn != kFfn ||
      h->stack_dim != kStack * kMels)
    return SAL_ESHAPE;
  if (h->n_layers > 4096 || h->data_bytes != data_bytes_for(h->n_layers)) return SAL_EINVAL;
  struct stat st;
  if (fstat(fileno(f), &st) != 0) return SAL_EIO;
  if (static_cast<uint64_t>(st.st_size) != kHeaderBytes + h->data_bytes) return SAL_EINVAL;
  return SAL_OK;
}

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f) fclose(f);
  }
};

struct Staging {
  void* buf[2] = {nullptr, nullptr};
  cudaEvent_t done[2] = {nullptr, nullptr};
  ~Staging() {
    for (int i = 0; i < 2; ++i) {
      if (done[i]) {
        cudaEventSynchronize(done[i]);
        cudaEventDestroy(done[i]);
      }
      if (buf[i]) cudaFreeHost(buf[i]);
    }
  }
};

}  // namespace
}  // namespace sal

using namespace sal;

extern "C" sal_status sal_weights_file_info(const char* path, int* n_layers, size_t* device_bytes) {
  if (!path || !n_layers || !device_bytes) return SAL_EINVAL;
  *n_layers = 0;
  *device_bytes = 0;
  File file;
  file.f = fopen(path, "rb");
  if (!file.f) return SAL_EIO;
  Header h;
  const sal_status st = read_header(file.f, &h);
  if (st != SAL_OK) return st;
  *n_layers = static_cast<int>(h.n_layers);
  *device_bytes = static_cast<size_t>(h.data_bytes);
  return SAL_OK;
}

extern "C" sal_status sal_weights_file_load(const char* path, void* device_buffer, size_t buffer_bytes,
                                            sal_layer* layers, int max_layers, sal_weights* w, void* stream) {
  const NvtxRange nvtx_("sal_weights_file_load");
  if (!path || !device_buffer || !w || max_layers < 0 || (max_layers > 0 && !layers) ||
      (reinterpret_cast<uintptr_t>(device_buffer) & (kAlign - 1)))
    return SAL_EINVAL;
  File file;
  file.f = fopen(path, "rb");
  if (!file.f) return SAL_EIO;
  Header h;
  const sal_status st = read_header(file.f, &h);
  if (st != SAL_OK) return st;
  if (buffer_bytes < h.data_bytes || static_cast<uint64_t>(max_layers) < h.n_layers) return SAL_EWORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* dst = static_cast<char*>(device_buffer);
  {
    Staging stg;
    for (int i = 0; i < 2; ++i)
      if (cudaHostAlloc(&stg.buf[i], kStageBytes, cudaHostAllocDefault) != cudaSuccess ||
          cudaEventCreateWithFlags(&stg.done[i], cudaEventDisableTiming) != cudaSuccess)
        return SAL_ECUDA;
    bool recorded[2] = {false, false};
    uint64_t off = 0;
    for (int i = 0; off < h.data_bytes; ++i) {
      const int b = i & 1;
      const size_t n = static_cast<size_t>(h.data_bytes - off < kStageBytes ? h.data_bytes - off : kStageBytes);
      if (recorded[b] && cudaEventSynchronize(stg.done[b]) != cudaSuccess) return SAL_ECUDA;  // buffer b free
      if (fread(stg.buf[b], 1, n, file.f) != n) return SAL_EIO;
      if (cudaMemcpyAsync(dst + off, stg.buf[b], n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
          cudaEventRecord(stg.done[b], s) != cudaSuccess)
        return SAL_ECUDA;
      recorded[b] = true;
      off += n;
    }
    if (cudaStreamSynchronize(s) != cudaSuccess) return SAL_ECUDA;
  }

  // the record: offsets in file order
  uint64_t off = 0;
  const void* g[4];
  for (int i = 0; i < 4; ++i) {
    g[i] = dst + off;
    off += padded(kGlobalElems[i]);
  }
  for (uint32_t l = 0; l < h.n_layers; ++l) {
    const void* p[kLayerTensors];
    for (int i = 0; i < kLayerTensors; ++i) {
      p[i] = dst + off;
      off += padded(kLayerElems[i]);
    }
    layers[l] = sal_layer{p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7], p[8], p[9], p[10], p[11], p[12], p[13]};
  }
  w->w_proj = g[0];
  w->b_proj = g[1];
  w->lnf_g = g[2];
  w->lnf_b = g[3];
  w->layers = layers;
  w->n_layers = static_cast<int>(h.n_layers);
  return SAL_OK;
}
