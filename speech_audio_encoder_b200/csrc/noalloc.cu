// sal_qkv_rope_noalloc: the QKV projection with QK-norm and RoPE, for callers that must
// not allocate device memory.
//
// Some callers cannot call cudaMalloc (or have torch allocate for them) at the moment
// they run this step: a real-time audio callback or a serving loop must not stall on an
// allocation (cudaMalloc can synchronise the device and can fail under memory pressure),
// a plugin host may forbid device allocations after start-up, and a framework that owns
// the device memory pool may not hand out a scratch buffer for one call. sal_qkv_rope
// needs such a buffer for its rotation table; this variant keeps that table in a fixed
// array compiled into the library instead.
//
// The array is file-scope device memory of kMaxT * 64 * 2 floats (2 MiB). Every GPU that
// loads the library holds it until the process exits. Every call shares it and it keeps
// the last call's table; the table is rewritten in full (all t < T) before it is read, so
// nothing needs clearing. Calls whose kernels overlap on the GPU (two streams, say) race
// on the array and must not be issued that way.
//
// The first call on a device looks up the array's device address (cudaGetSymbolAddress)
// with that device current; make that first call before any stream capture begins.
#include <mutex>

#include "sal_internal.h"

namespace sal {
namespace {

constexpr int64_t kMaxT = 4096;  // positions per clip this entry point accepts

static __device__ __align__(256) float g_rope_scratch[kMaxT * 64 * 2];

std::mutex g_mu;
float* g_scratch_ptr[64] = {};

// Device address of the scratch array on the current device; nullptr on failure.
float* scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rope_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace sal

using namespace sal;

extern "C" sal_status sal_qkv_rope_noalloc(const void* h, int batch, int64_t T, const sal_layer* layer, void* q,
                                           void* k, void* v, void* stream) {
  const NvtxRange nvtx_("sal_qkv_rope_noalloc");
  if (batch < 0 || T < 0 || !layer) return SAL_EINVAL;
  if (T > kMaxT) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (!h || !q || !k || !v || !aligned16(h) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !layer->w_qkv || !layer->b_qkv || !layer->qn_g || !layer->kn_g || !aligned16(layer->w_qkv) ||
      !aligned16(layer->b_qkv) || !aligned16(layer->qn_g) || !aligned16(layer->kn_g))
    return SAL_EINVAL;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return SAL_ECUDA;
  if (major != 10) return SAL_EDEVICE;
  float* cs = scratch_ptr();
  if (!cs) return SAL_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const sal_status st = rope_table_launch(cs, T, s);
  if (st != SAL_OK) return st;
  QkvOut qo{q, k, v, layer->qn_g, layer->kn_g, cs, T, 0};
  return gemm_launch(kEpiQkv, h, static_cast<int64_t>(batch) * T, kWidth, layer->w_qkv, 3 * kWidth,
                     layer->b_qkv, nullptr, &qo, s);
}
