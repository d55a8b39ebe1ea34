// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <utility>

#include "../../include/sal.h"
#include "sal_check.cuh"

namespace sal {

constexpr int kWin = 400;
constexpr int kHop = 160;
constexpr int kNfft = 512;
constexpr int kBins = 257;
constexpr int kMels = SAL_N_MELS;
constexpr int kStack = SAL_STACK;
constexpr int kWidth = SAL_WIDTH;
constexpr int kHeads = SAL_HEADS;
constexpr int kHeadDim = SAL_HEAD_DIM;
constexpr int kFfn = SAL_FFN;

// Serving windows over recordings of `total` positions: cores of `core` consecutive
// positions from 0 (the last may be shorter), each window its core extended by up to `ctx`
// positions on each side inside the recording. A windowed batch holds `count` windows per
// recording, each left-aligned in `slot` positions (the longest window); window w of a
// recording covers [max(0, w core - ctx), min(total, (w + 1) core + ctx)).
struct Windows {
  int count = 0;
  int core = 0, ctx = 0;
  int64_t total = 0;
  int64_t slot = 0;
};
Windows make_windows(int64_t total, int64_t core, int64_t ctx);  // sal_api.cu

// An NVTX range for the lifetime of the object: every compute entry point, every encoder
// layer and every stage of a layer is one, so a profiler that reads NVTX (Nsight Compute's
// --nvtx filters, Nsight Systems) can attribute kernels to them. Without such a tool
// attached a push or pop costs a few nanoseconds of host time.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

uint64_t wait_limit_ns();
bool pdl_enabled();  // programmatic dependent launch (env SAL_PDL=0 turns it off)
void count_launch();  // one kernel enqueued
unsigned int* device_status_ptr();  // device address of the status word (current device)

// frontend.cu
sal_status frontend_launch(const float* wave, int64_t n_samples, int batch, int64_t frames,
                           int64_t positions, float* logmel, void* stacked, cudaStream_t s);

// rowops.cu
sal_status layernorm_launch(const float* x, int64_t rows, const void* g, const void* b, void* y,
                            cudaStream_t s, int width = kWidth);  // width 1280 or 1024
sal_status rope_table_launch(float* cs, int64_t T, cudaStream_t s);
// x [batch * total, 1280] f32 -> xw [batch * count * slot, 1280] f32, each window's
// positions left-aligned in its slots and the slots past its length zeroed.
sal_status window_gather_launch(const float* x, int batch, const Windows& win, float* xw, cudaStream_t s);
// The core rows back: emb [batch * total, 1280] bf16 from embw, and (when xw and x are
// not null) the same rows of the fp32 stream from xw into x.
sal_status window_scatter_launch(const void* embw, const float* xw, int batch, const Windows& win, void* emb,
                                 float* x, cudaStream_t s);
sal_status speaker_fuse_launch(const void* H, const float* P, int64_t rows, const void* g, const void* b, void* out,
                               cudaStream_t s);

// gemm.cu
struct QkvOut {
  void *q, *k, *v;
  const void *qn_g, *kn_g;
  const float* rope_cs;  // [min(T, chunk)][64] cos then the same rows of sin
  int64_t T;
  int64_t chunk;         // positions restart every `chunk` positions (<= 0: whole clip)
};
// n_valid (0: N) < N runs the column tiles over N but reads only n_valid rows of W and
// entries of the bias; the columns past n_valid come out as 0 (for an N that is not a
// multiple of 64, into an output N columns wide).
sal_status gemm_launch(int epilogue, const void* A, int64_t M, int K, const void* W, int N,
                       const void* bias, void* out, const QkvOut* qkv, cudaStream_t s, int n_valid = 0);
constexpr int kEpiQkv = 100;  // internal epilogue id: QK-norm + RoPE scatter

// attention.cu
sal_status attention_launch(const void* q, const void* k, const void* v, int batch, int64_t T,
                            int64_t chunk, void* o, cudaStream_t s, const Windows* win = nullptr);
// Test hook of sal_attention_withhold: the kernel to run alone (1 one-tile, 2 two-tile) and
// the key/value tile (counted from each CTA's first) whose loads are never issued.
struct AttnWithhold {
  int kernel;
  int tile;
};
// Any number of heads of width 64 or 128 (o is [batch, T, heads * head_dim]); head_dim 64
// always runs the one-tile kernel.
sal_status attention_launch_heads(const void* q, const void* k, const void* v, int batch, int64_t T,
                                  int64_t chunk, int heads, int head_dim, void* o, cudaStream_t s,
                                  const AttnWithhold* hold = nullptr, const Windows* win = nullptr);

// ctc.cu
sal_status ctc_qk_norm_rope_launch(const float* qkv, int64_t rows, int64_t T, const void* qn_g, const void* kn_g,
                                   const float* cs, void* q, void* k, void* v, cudaStream_t s);
sal_status log_softmax_launch(const float* z, int64_t rows, int n, int64_t ld, float* out, cudaStream_t s);

// tensor maps (sal_api.cu)
bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer);
bool make_tmap_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t b0, uint32_t b1, uint32_t b2);

// The launch helpers have internal linkage: in the bounds-checked build each one writes
// the range table of the translation unit that holds the kernel.
namespace {

// Launches `kernel` on `s` with programmatic dependent launch allowed: the kernel may be
// scheduled while its predecessor on the stream is still running, runs its prologue, and
// waits in griddepcontrol.wait (every kernel of this library does so before touching
// global memory) until the predecessor has completed.
// cluster_x > 1: thread-block clusters of cluster_x CTAs along x (grid.x a multiple of it).
// Bounds-checked build: the ranges declared since the previous launch are copied into
// this unit's table first (stream-ordered, so the previous launch has finished with it).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  unsigned cluster_x, Args&&... args) {
#if defined(SAL_CHECKED) && defined(__CUDACC__)
  {
    CkTable t;
    if (!ck_take(&t)) return cudaErrorMemoryAllocation;
    const cudaError_t e = cudaMemcpyToSymbolAsync(sal_ck_table, &t, sizeof(t), 0, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
  }
#endif
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  return launch_kernel_cluster(kernel, grid, block, smem, s, 1u, std::forward<Args>(args)...);
}

}  // namespace

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace sal
