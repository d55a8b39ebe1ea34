// Row kernels of the CTC timestamp adapter (page "Nemotron 3.5 Transcribe: From Recorded
// Speech to Dataset Audits", section "Use alignment and audio questions as supporting
// evidence": the unfused width-1,280 ASR states, upsampled from the 80 ms to a 40 ms grid
// by a stride-two transposed convolution, two Transformer layers with 16 heads, and a
// projection to 23,862 tokens plus the CTC blank). The adapter runs at width 1,024 with
// 16 heads of 64 and the encoder's layer recipe; its GEMMs, LayerNorms and attention are
// the encoder's kernels at those sizes. Two steps are its own:
//
//   * QK-norm + RoPE + head split for head dim 64. The QKV GEMM writes fp32 rows
//     [q | k | v] of 3 x 1024 (bias included). One warp per position: for each head, lane
//     l holds elements l and l + 32, which are exactly the rotate-half pair (l, l + 32).
//     The RMS factor is one warp sum; the rotation angle t * 10000^(-2 l / 64) equals the
//     encoder table's angle t * 10000^(-2 (2 l) / 128), so the adapter reads column 2 l
//     of the same fp64-built table. q, k, v go out as bf16 [batch, 16, T, 64].
//   * log-softmax over the 23,863 classes of each 40 ms position: one CTA per row, an
//     online maximum and sum of exponentials in one pass over the fp32 scores, then
//     z - max - log(sum) written out.
#define SAL_CK_FILE 5
#include <cuda_bf16.h>
#include <math.h>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

constexpr int kW = 1024, kH = 16, kHd = 64;

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(256) ctc_qk_norm_rope_kernel(const float* __restrict__ qkv, int64_t rows, int64_t T,
                                                               const __nv_bfloat16* __restrict__ qn_g,
                                                               const __nv_bfloat16* __restrict__ kn_g,
                                                               const float* __restrict__ cs,
                                                               __nv_bfloat16* __restrict__ q,
                                                               __nv_bfloat16* __restrict__ k,
                                                               __nv_bfloat16* __restrict__ v) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row >= rows) return;
  const int64_t b = row / T, t = row - b * T;
  const float c = *SAL_CK_LD(cs + t * 64 + 2 * lane, 4), s = *SAL_CK_LD(cs + T * 64 + t * 64 + 2 * lane, 4);
  const float gq0 = __bfloat162float(*SAL_CK_LD(qn_g + lane, 2));
  const float gq1 = __bfloat162float(*SAL_CK_LD(qn_g + lane + 32, 2));
  const float gk0 = __bfloat162float(*SAL_CK_LD(kn_g + lane, 2));
  const float gk1 = __bfloat162float(*SAL_CK_LD(kn_g + lane + 32, 2));
  const float* src = qkv + row * (3 * kW);
#pragma unroll 4
  for (int h = 0; h < kH; ++h) {
    const int64_t dst = ((b * kH + h) * T + t) * kHd;
    {  // q
      float x0 = *SAL_CK_LD(src + h * kHd + lane, 4), x1 = *SAL_CK_LD(src + h * kHd + 32 + lane, 4);
      const float r = rsqrtf(warp_sum32(x0 * x0 + x1 * x1) * (1.0f / kHd) + 1e-6f);
      x0 *= r * gq0;
      x1 *= r * gq1;
      *SAL_CK_ST(q + dst + lane, 2) = __float2bfloat16_rn(x0 * c - x1 * s);
      *SAL_CK_ST(q + dst + 32 + lane, 2) = __float2bfloat16_rn(x1 * c + x0 * s);
    }
    {  // k
      float x0 = *SAL_CK_LD(src + kW + h * kHd + lane, 4), x1 = *SAL_CK_LD(src + kW + h * kHd + 32 + lane, 4);
      const float r = rsqrtf(warp_sum32(x0 * x0 + x1 * x1) * (1.0f / kHd) + 1e-6f);
      x0 *= r * gk0;
      x1 *= r * gk1;
      *SAL_CK_ST(k + dst + lane, 2) = __float2bfloat16_rn(x0 * c - x1 * s);
      *SAL_CK_ST(k + dst + 32 + lane, 2) = __float2bfloat16_rn(x1 * c + x0 * s);
    }
    *SAL_CK_ST(v + dst + lane, 2) = __float2bfloat16_rn(*SAL_CK_LD(src + 2 * kW + h * kHd + lane, 4));
    *SAL_CK_ST(v + dst + 32 + lane, 2) = __float2bfloat16_rn(*SAL_CK_LD(src + 2 * kW + h * kHd + 32 + lane, 4));
  }
}

// (m, s) pairs of an online log-sum-exp: s = sum exp(z - m).
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * __expf(m - mm) + s2 * __expf(m2 - mm);
  m = mm;
}

constexpr int kLsThreads = 512;

__global__ void __launch_bounds__(kLsThreads) log_softmax_kernel(const float* __restrict__ z, int64_t rows, int n,
                                                                 int64_t ld, float* __restrict__ out) {
  __shared__ float sm[kLsThreads / 32], ss[kLsThreads / 32];
  const int64_t row = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (row >= rows) return;
  const float* zr = z + row * ld;
  float m = -INFINITY, s = 0.f;
  for (int i = threadIdx.x; i < n; i += kLsThreads) {
    const float a = *SAL_CK_LD(zr + i, 4);  // kept in L2 for the second pass
    if (a > m) {
      s = s * __expf(m - a) + 1.f;
      m = a;
    } else {
      s += __expf(a - m);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, m2, s2);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sm[warp] = m;
    ss[warp] = s;
  }
  __syncthreads();
  if (warp == 0) {
    m = lane < kLsThreads / 32 ? sm[lane] : -INFINITY;
    s = lane < kLsThreads / 32 ? ss[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
      lse_merge(m, s, m2, s2);
    }
    if (lane == 0) sm[0] = m + logf(s);
  }
  __syncthreads();
  const float lse = sm[0];
  float* orow = out + row * static_cast<int64_t>(n);
  for (int i = threadIdx.x; i < n; i += kLsThreads) __stcs(SAL_CK_ST(orow + i, 4), __ldcs(SAL_CK_LD(zr + i, 4)) - lse);
}

}  // namespace

sal_status ctc_qk_norm_rope_launch(const float* qkv, int64_t rows, int64_t T, const void* qn_g, const void* kn_g,
                                   const float* cs, void* q, void* k, void* v, cudaStream_t s) {
  if (rows == 0) return SAL_OK;
  ck_declare(qkv, rows * 3 * kW * 4, false);
  ck_declare(qn_g, kHd * 2, false);
  ck_declare(kn_g, kHd * 2, false);
  ck_declare(cs, 2 * T * 64 * 4, false);
  ck_declare(q, rows * kW * 2, true);
  ck_declare(k, rows * kW * 2, true);
  ck_declare(v, rows * kW * 2, true);
  return launch_kernel(ctc_qk_norm_rope_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, s, qkv,
                       rows, T, static_cast<const __nv_bfloat16*>(qn_g), static_cast<const __nv_bfloat16*>(kn_g), cs,
                       static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
                       static_cast<__nv_bfloat16*>(v)) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

sal_status log_softmax_launch(const float* z, int64_t rows, int n, int64_t ld, float* out, cudaStream_t s) {
  if (rows == 0 || n == 0) return SAL_OK;
  if (rows > 0x7fffffff) return SAL_ESHAPE;
  ck_declare(z, ((rows - 1) * ld + n) * 4, false);
  ck_declare(out, rows * n * 4, true);
  return launch_kernel(log_softmax_kernel, dim3(static_cast<unsigned>(rows)), dim3(kLsThreads), 0, s, z, rows, n, ld,
                       out) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

}  // namespace sal
