// Row kernels of the encoder: the pre-norm / final LayerNorm, and the RoPE table.
//
// LayerNorm (eps 1e-5, affine) normalises each fp32 row of the residual stream (1280
// wide in the encoder, 1024 in the CTC adapter) and writes it as bf16, the operand of the
// next tensor-core GEMM. One warp per row: width / 32 values per lane held in registers,
// two-pass mean and variance.
//
// RoPE table: cos and sin of t * 10000^(-2 i / 128), i < 64, t < T. The angle reaches
// 4.5e4 rad at one hour, where fp32 would lose ~3 digits, so it is formed and reduced in
// fp64 before the fp32 table entry is written.
//
// Speaker-activity fusion (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset
// Audits", section "How audio and speakers reach the language model", the paragraph on
// Sortformer activity): per position, the eight slot activities are thresholded at 0.5,
// normalised by a LayerNorm over the slots, mapped to width 1280 by the fixed sinusoidal
// speaker kernel K[s, 2i] = sin(s w_i), K[s, 2i+1] = cos(s w_i), w_i = 10000^(-2i/1280)
// (scale 1), and added to the encoder state. One warp per position; K (40 KB, built in
// fp64 on the host) sits in shared memory.
//
// Serving windows (section "Local encoder windows, recording-wide language context", the
// paragraph on the serving path): the gather copies each context-extended window of a
// recording's residual stream into its own left-aligned slot range of a windowed batch
// (zeroing the slots past the window's length); the scatter copies every window's core
// rows back in order, dropping the context rows. One warp per row, 16-byte accesses.
#define SAL_CK_FILE 2
#include <cuda_bf16.h>
#include <math.h>

#include <cmath>
#include <mutex>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

constexpr int kLnWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// kVec float4 per lane: the row width is 128 kVec.
template <int kVec>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ x, int64_t rows,
                                                        const __nv_bfloat16* __restrict__ g,
                                                        const __nv_bfloat16* __restrict__ b,
                                                        __nv_bfloat16* __restrict__ y) {
  constexpr int kW = 128 * kVec;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kLnWarps + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + row * kW);
  float4 v[kVec];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    v[i] = *SAL_CK_LD(xr + lane + 32 * i, 16);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
  const float mean = warp_sum(s) * (1.0f / kW);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const float a = v[i].x - mean, bb = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    q += (a * a + bb * bb) + (c * c + d * d);
  }
  const float rstd = 1.0f / sqrtf(warp_sum(q) * (1.0f / kW) + 1e-5f);
  const uint2* g2 = reinterpret_cast<const uint2*>(g);
  const uint2* b2 = reinterpret_cast<const uint2*>(b);
  uint2* yr = reinterpret_cast<uint2*>(y + row * kW);
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int c4 = lane + 32 * i;
    const uint2 gg = __ldg(SAL_CK_LD(g2 + c4, 8)), bb = __ldg(SAL_CK_LD(b2 + c4, 8));
    const float o0 = (v[i].x - mean) * rstd * __uint_as_float(gg.x << 16) + __uint_as_float(bb.x << 16);
    const float o1 = (v[i].y - mean) * rstd * __uint_as_float(gg.x & 0xFFFF0000u) + __uint_as_float(bb.x & 0xFFFF0000u);
    const float o2 = (v[i].z - mean) * rstd * __uint_as_float(gg.y << 16) + __uint_as_float(bb.y << 16);
    const float o3 = (v[i].w - mean) * rstd * __uint_as_float(gg.y & 0xFFFF0000u) + __uint_as_float(bb.y & 0xFFFF0000u);
    __nv_bfloat162 p0 = __floats2bfloat162_rn(o0, o1), p1 = __floats2bfloat162_rn(o2, o3);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&p0);
    out.y = *reinterpret_cast<uint32_t*>(&p1);
    *SAL_CK_ST(yr + c4, 8) = out;
  }
}

__global__ void rope_table_kernel(float* __restrict__ cs, int64_t T) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (idx >= T * 64) return;
  const int64_t t = idx >> 6;
  const int i = static_cast<int>(idx & 63);
  const double inv = pow(10000.0, -static_cast<double>(2 * i) / 128.0);
  double s, c;
  sincos(static_cast<double>(t) * inv, &s, &c);
  *SAL_CK_ST(cs + idx, 4) = static_cast<float>(c);
  *SAL_CK_ST(cs + T * 64 + idx, 4) = static_cast<float>(s);
}

constexpr int kSlots = 8;
struct SpeakerKernel {
  float k[kSlots][kWidth];
};
__device__ SpeakerKernel g_speaker_kernel;

__global__ void __launch_bounds__(256) speaker_fuse_kernel(const __nv_bfloat16* __restrict__ H,
                                                           const float* __restrict__ P, int64_t rows,
                                                           const __nv_bfloat16* __restrict__ g,
                                                           const __nv_bfloat16* __restrict__ b,
                                                           __nv_bfloat16* __restrict__ out) {
  extern __shared__ __align__(16) float sk[];  // [8][1280]
  {
    const float4* src = reinterpret_cast<const float4*>(&g_speaker_kernel);
    float4* dst = reinterpret_cast<float4*>(sk);
    for (int i = threadIdx.x; i < kSlots * kWidth / 4; i += blockDim.x) dst[i] = *SAL_CK_LD(src + i, 16);
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int s = lane & 7;
  const float gs = __bfloat162float(*SAL_CK_LD(g + s, 2)), bs = __bfloat162float(*SAL_CK_LD(b + s, 2));
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    // every group of 8 lanes holds the 8 slots of this position
    const float a = *SAL_CK_LD(P + row * kSlots + s, 4) > 0.5f ? 1.f : 0.f;
    float sum = a;
#pragma unroll
    for (int o = 1; o < kSlots; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mu = sum * (1.0f / kSlots);
    float q = (a - mu) * (a - mu);
#pragma unroll
    for (int o = 1; o < kSlots; o <<= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float ah = (a - mu) / sqrtf(q * (1.0f / kSlots) + 1e-5f) * gs + bs;
    float w[kSlots];
#pragma unroll
    for (int t = 0; t < kSlots; ++t) w[t] = __shfl_sync(0xffffffffu, ah, t);
    const uint2* hr = reinterpret_cast<const uint2*>(H + row * kWidth);
    uint2* orow = reinterpret_cast<uint2*>(out + row * kWidth);
#pragma unroll
    for (int i = 0; i < kWidth / 128; ++i) {
      const int c4 = lane + 32 * i;  // columns 4 c4 .. 4 c4 + 3
      const uint2 hv = *SAL_CK_LD(hr + c4, 8);
      float o0 = __uint_as_float(hv.x << 16), o1 = __uint_as_float(hv.x & 0xFFFF0000u);
      float o2 = __uint_as_float(hv.y << 16), o3 = __uint_as_float(hv.y & 0xFFFF0000u);
#pragma unroll
      for (int t = 0; t < kSlots; ++t) {
        const float4 kv = reinterpret_cast<const float4*>(sk + t * kWidth)[c4];
        o0 = fmaf(w[t], kv.x, o0);
        o1 = fmaf(w[t], kv.y, o1);
        o2 = fmaf(w[t], kv.z, o2);
        o3 = fmaf(w[t], kv.w, o3);
      }
      __nv_bfloat162 p0 = __floats2bfloat162_rn(o0, o1), p1 = __floats2bfloat162_rn(o2, o3);
      uint2 ov;
      ov.x = *reinterpret_cast<uint32_t*>(&p0);
      ov.y = *reinterpret_cast<uint32_t*>(&p1);
      *SAL_CK_ST(orow + c4, 8) = ov;
    }
  }
}

// First position of window w of a recording.
__device__ __forceinline__ int64_t window_lo(const Windows& wn, int64_t w) {
  const int64_t lo = w * wn.core - wn.ctx;
  return lo > 0 ? lo : 0;
}

__global__ void __launch_bounds__(256) window_gather_kernel(const float* __restrict__ x, int batch, Windows wn,
                                                            float* __restrict__ xw) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(batch) * wn.count * wn.slot;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row >= rows) return;
  const int64_t clip = row / wn.slot, i = row - clip * wn.slot;
  const int64_t b = clip / wn.count, w = clip - b * wn.count;
  const int64_t lo = window_lo(wn, w);
  int64_t hi = (w + 1) * wn.core + wn.ctx;
  if (hi > wn.total) hi = wn.total;
  float4* dst = reinterpret_cast<float4*>(xw + row * kWidth);
  if (lo + i < hi) {
    const float4* src = reinterpret_cast<const float4*>(x + (b * wn.total + lo + i) * kWidth);
#pragma unroll
    for (int c = 0; c < kWidth / 128; ++c) *SAL_CK_ST(dst + lane + 32 * c, 16) = *SAL_CK_LD(src + lane + 32 * c, 16);
  } else {
#pragma unroll
    for (int c = 0; c < kWidth / 128; ++c) *SAL_CK_ST(dst + lane + 32 * c, 16) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__global__ void __launch_bounds__(256) window_scatter_kernel(const __nv_bfloat16* __restrict__ embw,
                                                             const float* __restrict__ xw, int batch, Windows wn,
                                                             __nv_bfloat16* __restrict__ emb, float* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(batch) * wn.total;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row >= rows) return;
  const int64_t b = row / wn.total, t = row - b * wn.total;
  const int64_t w = t / wn.core;  // the window whose core holds position t
  const int64_t src_row = (b * wn.count + w) * wn.slot + (t - window_lo(wn, w));
  const uint4* se = reinterpret_cast<const uint4*>(embw + src_row * kWidth);
  uint4* de = reinterpret_cast<uint4*>(emb + row * kWidth);
  for (int c = lane; c < kWidth / 8; c += 32) *SAL_CK_ST(de + c, 16) = *SAL_CK_LD(se + c, 16);
  if (x) {
    const float4* sx = reinterpret_cast<const float4*>(xw + src_row * kWidth);
    float4* dx = reinterpret_cast<float4*>(x + row * kWidth);
#pragma unroll
    for (int c = 0; c < kWidth / 128; ++c) *SAL_CK_ST(dx + lane + 32 * c, 16) = *SAL_CK_LD(sx + lane + 32 * c, 16);
  }
}

std::mutex g_spk_mu;
bool g_spk_done[64] = {};
const void* g_spk_addr[64] = {};  // device address of the speaker kernel table

sal_status ensure_speaker_kernel() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SAL_ECUDA;
  std::lock_guard<std::mutex> lk(g_spk_mu);
  if (g_spk_done[dev]) return SAL_OK;
  static SpeakerKernel host;
  for (int s = 0; s < kSlots; ++s)
    for (int i = 0; i < kWidth / 2; ++i) {
      const double w = std::pow(10000.0, -2.0 * i / kWidth);
      host.k[s][2 * i] = static_cast<float>(std::sin(s * w));
      host.k[s][2 * i + 1] = static_cast<float>(std::cos(s * w));
    }
  if (cudaMemcpyToSymbol(g_speaker_kernel, &host, sizeof(host)) != cudaSuccess) return SAL_ECUDA;
  if (cudaFuncSetAttribute(speaker_fuse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sizeof(SpeakerKernel))) != cudaSuccess)
    return SAL_ECUDA;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_speaker_kernel) != cudaSuccess) return SAL_ECUDA;
  g_spk_addr[dev] = addr;
  g_spk_done[dev] = true;
  return SAL_OK;
}

}  // namespace

sal_status speaker_fuse_launch(const void* H, const float* P, int64_t rows, const void* g, const void* b, void* out,
                               cudaStream_t s) {
  if (rows == 0) return SAL_OK;
  const sal_status st = ensure_speaker_kernel();
  if (st != SAL_OK) return st;
  int sms = 148;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (rows + 7) / 8;
  const unsigned grid = static_cast<unsigned>(want < 4 * sms ? want : 4 * sms);
  ck_declare(H, rows * kWidth * 2, false);
  ck_declare(P, rows * kSlots * 4, false);
  ck_declare(g, kSlots * 2, false);
  ck_declare(b, kSlots * 2, false);
  ck_declare(out, rows * kWidth * 2, true);
  ck_declare(g_spk_addr[dev], sizeof(SpeakerKernel), false);
  return launch_kernel(speaker_fuse_kernel, dim3(grid), dim3(256), sizeof(SpeakerKernel), s,
                       static_cast<const __nv_bfloat16*>(H), P, rows, static_cast<const __nv_bfloat16*>(g),
                       static_cast<const __nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(out)) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

sal_status layernorm_launch(const float* x, int64_t rows, const void* g, const void* b, void* y,
                            cudaStream_t s, int width) {
  if (rows == 0) return SAL_OK;
  const unsigned grid = static_cast<unsigned>((rows + kLnWarps - 1) / kLnWarps);
  const auto gg = static_cast<const __nv_bfloat16*>(g);
  const auto bb = static_cast<const __nv_bfloat16*>(b);
  const auto yy = static_cast<__nv_bfloat16*>(y);
  if (width != kWidth && width != 1024) return SAL_ESHAPE;
  ck_declare(x, rows * width * 4, false);
  ck_declare(g, width * 2, false);
  ck_declare(b, width * 2, false);
  ck_declare(y, rows * width * 2, true);
  cudaError_t e;
  if (width == kWidth)
    e = launch_kernel(layernorm_kernel<kWidth / 128>, dim3(grid), dim3(32 * kLnWarps), 0, s, x, rows, gg, bb, yy);
  else if (width == 1024)
    e = launch_kernel(layernorm_kernel<8>, dim3(grid), dim3(32 * kLnWarps), 0, s, x, rows, gg, bb, yy);
  else
    return SAL_ESHAPE;
  return e == cudaSuccess ? SAL_OK : SAL_ECUDA;
}

sal_status window_gather_launch(const float* x, int batch, const Windows& win, float* xw, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(batch) * win.count * win.slot;
  if (rows == 0) return SAL_OK;
  ck_declare(x, batch * win.total * kWidth * 4, false);
  ck_declare(xw, rows * kWidth * 4, true);
  return launch_kernel(window_gather_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, s, x, batch,
                       win, xw) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

sal_status window_scatter_launch(const void* embw, const float* xw, int batch, const Windows& win, void* emb,
                                 float* x, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(batch) * win.total;
  if (rows == 0) return SAL_OK;
  const int64_t wrows = static_cast<int64_t>(batch) * win.count * win.slot;
  ck_declare(embw, wrows * kWidth * 2, false);
  ck_declare(emb, rows * kWidth * 2, true);
  if (x) {
    ck_declare(xw, wrows * kWidth * 4, false);
    ck_declare(x, rows * kWidth * 4, true);
  }
  return launch_kernel(window_scatter_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, s,
                       static_cast<const __nv_bfloat16*>(embw), xw, batch, win, static_cast<__nv_bfloat16*>(emb),
                       x) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

sal_status rope_table_launch(float* cs, int64_t T, cudaStream_t s) {
  if (T == 0) return SAL_OK;
  const int64_t n = T * 64;
  ck_declare(cs, 2 * n * 4, true);
  return launch_kernel(rope_table_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, cs, T) ==
                 cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

}  // namespace sal
