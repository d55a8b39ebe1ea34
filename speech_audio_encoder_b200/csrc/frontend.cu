// Front end: 16 kHz float32 waveform -> 128 natural-log Slaney mel energies per 10 ms
// frame (25 ms periodic Hann window, 512-point FFT), plus the bf16 copy of the first
// 8 T frames that, read as [T, 1024], is the frame-major stack of eight frames.
// (Page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits", section
// "How audio and speakers reach the language model", exported-frontend paragraph.)
//
// One CTA of 8 warps covers 32 consecutive frames of one clip. Their 160*31 + 400
// samples are staged in shared memory once (overlapping windows are never re-read from
// HBM). Each warp then takes one frame at a time:
//   1. the 400 windowed samples, zero-padded to 512, are packed as 256 complex values
//      z[m] = y[2m] + i y[2m+1];
//   2. a 256-point complex FFT, factored 8 x 8 x 4 (two radix-8 passes in registers
//      with twiddles, one radix-4 pass), with two shared-memory exchanges;
//   3. the split step X[k] = E[k] + e^{-2 pi i k/512} O[k], E and O the transforms of
//      the even and odd samples recovered from Z[k] and conj(Z[256-k]); power |X[k]|^2;
//   4. 128 sparse triangular filters (504 non-zero weights), ln(max(e, 1e-10)).
// The FFT, power and filter sums run in fp64: a bin 60 dB under the frame's strongest
// component (the noise floor of a clean tone) carries an fp32 FFT error of ~1e-6 of the
// frame norm, i.e. a few 1e-4 in its log, above the 1e-4 budget; B200's fp64 rate is half
// its fp32 rate, so the whole transform stays in double. The twiddle, window and filter
// tables are computed once on the host in double precision and read through L1.
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>
#include <vector>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

constexpr int kFramesPerCta = 32;
constexpr int kWarps = 8;
constexpr int kFramesPerWarp = kFramesPerCta / kWarps;
constexpr int kTileSamples = kHop * (kFramesPerCta - 1) + kWin;  // 5360
constexpr int kMelNnz = 504;

struct FrontTables {
  double2 tw256[256];  // e^{-2 pi i j / 256}
  double2 tw512[258];  // e^{-2 pi i k / 512}, k = 0..256 (+1 pad)
  double hann[400];
  double mel_w[kMelNnz];
  int mel_meta[128];   // first bin | count << 9 | weight offset << 13
};

__device__ FrontTables g_front_tables;

// Per-warp scratch (doubles): exchange A is 2 x (8 rows x 36), exchange B is 2 x (64 x 5).
// The spectrum Z (2 x 256) reuses A; the power spectrum (257) reuses B.
constexpr int kAStride = 36;
constexpr int kAElems = 2 * 8 * kAStride;  // 576
constexpr int kBElems = 2 * 64 * 5;        // 640
constexpr int kWarpElems = kAElems + kBElems;

constexpr size_t kSmemBytes = sizeof(float) * kTileSamples + sizeof(double) * kWarps * kWarpElems;

struct C2 {
  double x, y;
};
__device__ __forceinline__ C2 cadd(C2 a, C2 b) { return {a.x + b.x, a.y + b.y}; }
__device__ __forceinline__ C2 csub(C2 a, C2 b) { return {a.x - b.x, a.y - b.y}; }
__device__ __forceinline__ C2 cmul(C2 a, double2 w) {
  return {fma(a.x, w.x, -a.y * w.y), fma(a.x, w.y, a.y * w.x)};
}
__device__ __forceinline__ C2 mul_neg_i(C2 a) { return {a.y, -a.x}; }  // a * (-i)
__device__ __forceinline__ C2 mul_pos_i(C2 a) { return {-a.y, a.x}; }  // a * (+i)

// X[k] = sum_n x[n] e^{-2 pi i n k / 4}
__device__ __forceinline__ void dft4(C2 a, C2 b, C2 c, C2 d, C2& y0, C2& y1, C2& y2, C2& y3) {
  const C2 s0 = cadd(a, c), d0 = csub(a, c);
  const C2 s1 = cadd(b, d), d1 = csub(b, d);
  y0 = cadd(s0, s1);
  y2 = csub(s0, s1);
  y1 = cadd(d0, mul_neg_i(d1));
  y3 = cadd(d0, mul_pos_i(d1));
}

// X[k] = sum_n x[n] e^{-2 pi i n k / 8}, in place.
__device__ __forceinline__ void dft8(C2 (&v)[8]) {
  C2 e0, e1, e2, e3, o0, o1, o2, o3;
  dft4(v[0], v[2], v[4], v[6], e0, e1, e2, e3);
  dft4(v[1], v[3], v[5], v[7], o0, o1, o2, o3);
  const double r = 0.70710678118654752440;
  // twiddles e^{-2 pi i k / 8}, k = 1, 2, 3
  o1 = {(o1.x + o1.y) * r, (o1.y - o1.x) * r};
  o2 = mul_neg_i(o2);
  o3 = {(o3.y - o3.x) * r, -(o3.x + o3.y) * r};
  v[0] = cadd(e0, o0);
  v[4] = csub(e0, o0);
  v[1] = cadd(e1, o1);
  v[5] = csub(e1, o1);
  v[2] = cadd(e2, o2);
  v[6] = csub(e2, o2);
  v[3] = cadd(e3, o3);
  v[7] = csub(e3, o3);
}

__global__ void __launch_bounds__(256, 2)
    frontend_kernel(const float* __restrict__ wave, int64_t n_samples, int64_t F, int64_t n_stack,
                    float* __restrict__ logmel, __nv_bfloat16* __restrict__ stacked) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* wbuf = reinterpret_cast<double*>(smem_raw);
  float* tile = reinterpret_cast<float*>(smem_raw + sizeof(double) * kWarps * kWarpElems);
  const FrontTables& tab = g_front_tables;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t clip = blockIdx.y;
  const int64_t f0 = static_cast<int64_t>(blockIdx.x) * kFramesPerCta;
  const int nf = static_cast<int>(F - f0 < kFramesPerCta ? F - f0 : kFramesPerCta);
  const int nsamp = kHop * (nf - 1) + kWin;  // a multiple of 4
  pdl_wait();
  pdl_trigger();

  {  // samples [160 f0, 160 f0 + nsamp) of this clip, read once
    const int64_t g0 = clip * n_samples + kHop * f0;
    const float* src = wave + g0;
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
      const float4* s4 = reinterpret_cast<const float4*>(src);
      float4* d4 = reinterpret_cast<float4*>(tile);
      for (int i = tid; i < nsamp / 4; i += blockDim.x) d4[i] = __ldcs(s4 + i);
    } else {
      for (int i = tid; i < nsamp; i += blockDim.x) tile[i] = __ldcs(src + i);
    }
  }
  __syncthreads();

  double* are = wbuf + warp * kWarpElems;
  double* aim = are + 8 * kAStride;
  double* bre = are + kAElems;
  double* bim = bre + 64 * 5;
  double* zre = are;        // Z[k], k < 256 (reuses exchange A)
  double* zim = are + 256;
  double* pw = bre;         // |X[k]|^2, k <= 256 (reuses exchange B)

  for (int i = 0; i < kFramesPerWarp; ++i) {
    const int fl = warp * kFramesPerWarp + i;
    if (fl >= nf) break;
    const float* x = tile + kHop * fl;

    // ---- pass 1: lane = n2; 8-point DFT over n1 of z[32 n1 + n2], twiddle W256^(n2 k1)
    C2 v[8];
#pragma unroll
    for (int n1 = 0; n1 < 8; ++n1) {
      const int s = 64 * n1 + 2 * lane;  // sample index of the real part
      if (s < kWin) {
        const float2 xx = *reinterpret_cast<const float2*>(x + s);
        const double2 ww = __ldg(reinterpret_cast<const double2*>(tab.hann + s));
        v[n1] = {static_cast<double>(xx.x) * ww.x, static_cast<double>(xx.y) * ww.y};
      } else {
        v[n1] = {0.0, 0.0};
      }
    }
    dft8(v);
#pragma unroll
    for (int k1 = 0; k1 < 8; ++k1) {
      const C2 t = k1 ? cmul(v[k1], __ldg(tab.tw256 + lane * k1)) : v[0];
      are[k1 * kAStride + lane] = t.x;
      aim[k1 * kAStride + lane] = t.y;
    }
    __syncwarp();

    // ---- pass 2: lane = (k1, b); 8-point DFT over a of A[k1][4a + b], twiddle W32^(b c)
    {
      const int k1 = lane >> 2, b = lane & 3;
#pragma unroll
      for (int a = 0; a < 8; ++a) v[a] = {are[k1 * kAStride + 4 * a + b], aim[k1 * kAStride + 4 * a + b]};
      dft8(v);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const C2 t = (b && c) ? cmul(v[c], __ldg(tab.tw256 + 8 * b * c)) : v[c];
        const int p = 8 * c + k1;
        bre[p * 5 + b] = t.x;
        bim[p * 5 + b] = t.y;
      }
    }
    __syncwarp();

    // ---- pass 3: lane takes p = 8 c + k1 in {lane, lane + 32}; 4-point DFT over b
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = lane + 32 * h;
      C2 y0, y1, y2, y3;
      dft4({bre[p * 5 + 0], bim[p * 5 + 0]}, {bre[p * 5 + 1], bim[p * 5 + 1]},
           {bre[p * 5 + 2], bim[p * 5 + 2]}, {bre[p * 5 + 3], bim[p * 5 + 3]}, y0, y1, y2, y3);
      zre[p] = y0.x;        zim[p] = y0.y;
      zre[p + 64] = y1.x;   zim[p + 64] = y1.y;
      zre[p + 128] = y2.x;  zim[p + 128] = y2.y;
      zre[p + 192] = y3.x;  zim[p + 192] = y3.y;
    }
    __syncwarp();

    // ---- split into the real 512-point spectrum; power
#pragma unroll
    for (int h = 0; h < 9; ++h) {
      const int k = lane + 32 * h;
      if (k > 256) break;
      const int kk = k & 255, kr = (256 - k) & 255;
      const double ar = zre[kk], ai = zim[kk], br = zre[kr], bi = -zim[kr];  // b = conj(Z[256-k])
      const C2 e = {0.5 * (ar + br), 0.5 * (ai + bi)};
      // o = (Z[k] - conj(Z[256-k])) / (2 i)
      const C2 o = {0.5 * (ai - bi), -0.5 * (ar - br)};
      const C2 xo = cmul(o, __ldg(tab.tw512 + k));
      const double xr = e.x + xo.x, xi = e.y + xo.y;
      pw[k] = fma(xr, xr, xi * xi);
    }
    __syncwarp();

    // ---- mel filters, log, stores
    const int64_t f = f0 + fl;
    float* out = logmel + (clip * F + f) * kMels;
    __nv_bfloat16* sout = (f < n_stack) ? stacked + (clip * n_stack + f) * kMels : nullptr;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int m = lane + 32 * h;
      const int meta = __ldg(tab.mel_meta + m);
      const int k0 = meta & 511, cnt = (meta >> 9) & 15, off = meta >> 13;
      double e = 0.0;
      for (int j = 0; j < cnt; ++j) e = fma(__ldg(tab.mel_w + off + j), pw[k0 + j], e);
      const float lm = static_cast<float>(log(fmax(e, 1e-10)));
      __stcs(out + m, lm);
      if (sout) sout[m] = __float2bfloat16_rn(lm);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------- host tables

double hz_to_mel_slaney(double f) {
  const double logstep = std::log(6.4) / 27.0;
  return f >= 1000.0 ? 15.0 + std::log(f / 1000.0) / logstep : f * 3.0 / 200.0;
}

double mel_to_hz_slaney(double m) {
  const double logstep = std::log(6.4) / 27.0;
  return m >= 15.0 ? 1000.0 * std::exp(logstep * (m - 15.0)) : m * 200.0 / 3.0;
}

bool build_tables(FrontTables* t) {
  const double pi = 3.14159265358979323846;
  for (int j = 0; j < 256; ++j) t->tw256[j] = make_double2(std::cos(2 * pi * j / 256.0), -std::sin(2 * pi * j / 256.0));
  for (int k = 0; k < 258; ++k) t->tw512[k] = make_double2(std::cos(2 * pi * k / 512.0), -std::sin(2 * pi * k / 512.0));
  for (int n = 0; n < 400; ++n) t->hann[n] = 0.5 - 0.5 * std::cos(2 * pi * n / 400.0);
  // Slaney filters: 130 points equally spaced in mel over 0..8000 Hz.
  double pts[kMels + 2];
  const double mmax = hz_to_mel_slaney(8000.0);
  for (int i = 0; i < kMels + 2; ++i) pts[i] = mel_to_hz_slaney(mmax * i / (kMels + 1));
  int off = 0;
  for (int m = 0; m < kMels; ++m) {
    const double norm = 2.0 / (pts[m + 2] - pts[m]);
    int first = -1, cnt = 0;
    for (int k = 0; k < kBins; ++k) {
      const double fk = 31.25 * k;
      const double rise = (fk - pts[m]) / (pts[m + 1] - pts[m]);
      const double fall = (pts[m + 2] - fk) / (pts[m + 2] - pts[m + 1]);
      const double w = std::fmax(0.0, std::fmin(rise, fall)) * norm;
      if (w > 0.0) {
        if (first < 0) first = k;
        if (k != first + cnt || off + cnt >= kMelNnz || cnt >= 15) return false;  // must be contiguous
        t->mel_w[off + cnt] = w;
        ++cnt;
      }
    }
    if (first < 0) return false;
    t->mel_meta[m] = first | (cnt << 9) | (off << 13);
    off += cnt;
  }
  return off == kMelNnz;
}

std::mutex g_init_mu;
bool g_init_done[64] = {};

sal_status ensure_tables() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SAL_ECUDA;
  std::lock_guard<std::mutex> lk(g_init_mu);
  if (g_init_done[dev]) return SAL_OK;
  static FrontTables host;
  static bool built = false;
  if (!built) {
    if (!build_tables(&host)) return SAL_ECUDA;
    built = true;
  }
  if (cudaMemcpyToSymbol(g_front_tables, &host, sizeof(FrontTables)) != cudaSuccess) return SAL_ECUDA;
  if (cudaFuncSetAttribute(frontend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess)
    return SAL_ECUDA;
  g_init_done[dev] = true;
  return SAL_OK;
}

}  // namespace

sal_status frontend_launch(const float* wave, int64_t n_samples, int batch, int64_t frames,
                           int64_t positions, float* logmel, void* stacked, cudaStream_t s) {
  if (frames == 0) return SAL_OK;
  const sal_status st = ensure_tables();
  if (st != SAL_OK) return st;
  const dim3 grid(static_cast<unsigned>((frames + kFramesPerCta - 1) / kFramesPerCta),
                  static_cast<unsigned>(batch));
  const int64_t n_stack = stacked ? positions * kStack : 0;
  return launch_kernel(frontend_kernel, grid, dim3(256), kSmemBytes, s, wave, n_samples, frames, n_stack, logmel,
                       static_cast<__nv_bfloat16*>(stacked)) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

}  // namespace sal
