// Front end: 16 kHz float32 waveform -> 128 natural-log Slaney mel energies per 10 ms
// frame (25 ms periodic Hann window, 512-point FFT), plus the bf16 copy of the first
// 8 T frames that, read as [T, 1024], is the frame-major stack of eight frames.
// (Page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits", section
// "How audio and speakers reach the language model", exported-frontend paragraph.)
//
// One CTA of 8 warps covers 32 consecutive frames of one clip. Their 160*31 + 400
// samples are staged in shared memory once (overlapping windows are never re-read from
// HBM). Each half-warp (16 lanes) then takes one frame at a time:
//   1. the 400 windowed samples, zero-padded to 512, are packed as 256 complex values
//      z[m] = y[2m] + i y[2m+1];
//   2. a 256-point complex FFT factored 16 x 16: lane n2 transforms z[16 n1 + n2] over n1
//      in registers and applies the twiddle W256^(n2 k1); one transposing exchange in
//      shared memory; lane k1 transforms over n2, giving Z[k1 + 16 k2];
//   3. the split step for the pair (k, 256 - k) at once: with E = (Z[k] + conj Z[256-k]) / 2
//      and O = (Z[k] - conj Z[256-k]) / 2i, X[k] = E + W512^k O and X[256-k] =
//      conj(E - W512^k O); the powers |X|^2 overwrite the two Z entries in place;
//   4. 128 sparse triangular filters (504 non-zero weights), ln(max(e, 1e-10)).
// The FFT, power and filter sums run in fp64: a bin 60 dB under the frame's strongest
// component (the noise floor of a clean tone) carries an fp32 FFT error of ~1e-6 of the
// frame norm, i.e. a few 1e-4 in its log, above the 1e-4 budget; B200's fp64 rate is half
// its fp32 rate, so the whole transform stays in double (the log of the fp64 energy is
// taken in fp32: its rounding is ~1e-7). The twiddle, window and filter tables are
// computed once on the host in double precision and copied to shared memory per CTA.
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
constexpr int kHalfWarps = 2 * kWarps;
constexpr int kFramesPerHalf = kFramesPerCta / kHalfWarps;  // 2
constexpr int kTileSamples = kHop * (kFramesPerCta - 1) + kWin;  // 5360
constexpr int kMelNnz = 504;

struct FrontTables {
  double2 tw256[256];  // e^{-2 pi i j / 256}
  double2 tw512[130];  // e^{-2 pi i k / 512}, k = 0..128 (+1 pad)
  double hann[400];
  double mel_w[kMelNnz];
  int mel_meta[128];   // first bin | count << 9 | weight offset << 13
};
static_assert(sizeof(FrontTables) % 16 == 0, "table copy uses 16-byte words");

__device__ FrontTables g_front_tables;

// Per half-warp scratch: 16 rows of 17 complex doubles (the transposing exchange), later
// the spectrum Z[0..255] in natural order and the powers written over it.
constexpr int kScratch = 16 * 17;  // double2 entries
constexpr size_t kSmemBytes =
    sizeof(FrontTables) + sizeof(double2) * kHalfWarps * kScratch + sizeof(float) * kTileSamples;

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

// X[k] = sum_n x[n] e^{-2 pi i n k / 16}, in place: n = 4a + b, k = c + 4d; a 4-point
// transform over a for each b, the twiddle e^{-2 pi i b c / 16}, a 4-point transform over b.
__device__ __forceinline__ void dft16(C2 (&v)[16]) {
  const double c1 = 0.92387953251128675613, s1 = 0.38268343236508977173;  // cos, sin of pi/8
  const double r = 0.70710678118654752440;
  C2 y[4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b) dft4(v[b], v[4 + b], v[8 + b], v[12 + b], y[b][0], y[b][1], y[b][2], y[b][3]);
  // twiddles W16^(b c)
  y[1][1] = cmul(y[1][1], make_double2(c1, -s1));                        // W^1
  y[1][2] = {(y[1][2].x + y[1][2].y) * r, (y[1][2].y - y[1][2].x) * r};  // W^2
  y[1][3] = cmul(y[1][3], make_double2(s1, -c1));                        // W^3
  y[2][1] = {(y[2][1].x + y[2][1].y) * r, (y[2][1].y - y[2][1].x) * r};  // W^2
  y[2][2] = mul_neg_i(y[2][2]);                                          // W^4
  y[2][3] = {(y[2][3].y - y[2][3].x) * r, -(y[2][3].x + y[2][3].y) * r}; // W^6
  y[3][1] = cmul(y[3][1], make_double2(s1, -c1));                        // W^3
  y[3][2] = {(y[3][2].y - y[3][2].x) * r, -(y[3][2].x + y[3][2].y) * r}; // W^6
  y[3][3] = cmul(y[3][3], make_double2(-c1, s1));                        // W^9
#pragma unroll
  for (int c = 0; c < 4; ++c) dft4(y[0][c], y[1][c], y[2][c], y[3][c], v[c], v[c + 4], v[c + 8], v[c + 12]);
}

__global__ void __launch_bounds__(256, 2)
    frontend_kernel(const float* __restrict__ wave, int64_t n_samples, int64_t F, int64_t n_stack,
                    float* __restrict__ logmel, __nv_bfloat16* __restrict__ stacked) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FrontTables& tab = *reinterpret_cast<FrontTables*>(smem_raw);
  double2* scratch_all = reinterpret_cast<double2*>(smem_raw + sizeof(FrontTables));
  float* tile = reinterpret_cast<float*>(scratch_all + kHalfWarps * kScratch);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int hl = lane & 15;           // lane within the half-warp
  const int half = tid >> 4;          // half-warp index 0..15
  const int64_t clip = blockIdx.y;
  const int64_t f0 = static_cast<int64_t>(blockIdx.x) * kFramesPerCta;
  const int nf = static_cast<int>(F - f0 < kFramesPerCta ? F - f0 : kFramesPerCta);
  const int nsamp = kHop * (nf - 1) + kWin;  // a multiple of 4

  {  // tables (computed once on the host)
    const int4* src = reinterpret_cast<const int4*>(&g_front_tables);
    int4* dst = reinterpret_cast<int4*>(smem_raw);
    for (int i = tid; i < static_cast<int>(sizeof(FrontTables) / 16); i += blockDim.x) dst[i] = src[i];
  }
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

  double2* scr = scratch_all + half * kScratch;
  double* pw = reinterpret_cast<double*>(scr);  // power P[k] lands at pw[2 k]

  // Both half-warps of a warp run the same number of frames (the masks below keep
  // frames past the clip end from being stored), so __syncwarp covers every lane.
#pragma unroll 1
  for (int i = 0; i < kFramesPerHalf; ++i) {
    const int fl = half * kFramesPerHalf + i;
    const bool live = fl < nf;
    const float* x = tile + kHop * (live ? fl : 0);

    // ---- pass 1: lane n2 = hl transforms z[16 n1 + n2] over n1, then twiddles
    C2 v[16];
#pragma unroll
    for (int n1 = 0; n1 < 16; ++n1) {
      const int s = 32 * n1 + 2 * hl;  // sample index of the real part
      if (n1 < 13 && s < kWin) {
        const float2 xx = *reinterpret_cast<const float2*>(x + s);
        const double2 ww = *reinterpret_cast<const double2*>(tab.hann + s);
        v[n1] = {static_cast<double>(xx.x) * ww.x, static_cast<double>(xx.y) * ww.y};
      } else {
        v[n1] = {0.0, 0.0};
      }
    }
    dft16(v);
#pragma unroll
    for (int k1 = 0; k1 < 16; ++k1) {
      const C2 t = k1 ? cmul(v[k1], tab.tw256[hl * k1]) : v[0];
      scr[hl * 17 + k1] = make_double2(t.x, t.y);
    }
    __syncwarp();

    // ---- pass 2: lane k1 = hl transforms over n2, giving Z[k1 + 16 k2]
#pragma unroll
    for (int n2 = 0; n2 < 16; ++n2) {
      const double2 a = scr[n2 * 17 + hl];
      v[n2] = {a.x, a.y};
    }
    dft16(v);
    __syncwarp();
#pragma unroll
    for (int k2 = 0; k2 < 16; ++k2) scr[hl + 16 * k2] = make_double2(v[k2].x, v[k2].y);
    __syncwarp();

    // ---- split and power for the pairs (k, 256 - k), k = hl + 16 k2 < 128; lane 0 also
    //      takes k = 0 (X[0], X[256] are real) and k = 128 (its own partner)
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2) {
      const int k = hl + 16 * k2;
      const double2 a = scr[k];
      if (k == 0) {
        const double e0 = a.x + a.y, e256 = a.x - a.y;
        const double2 z128 = scr[128];
        pw[0] = e0 * e0;
        pw[2 * 256] = e256 * e256;
        pw[2 * 128] = z128.x * z128.x + z128.y * z128.y;
      } else {
        const double2 bz = scr[256 - k];
        const C2 b = {bz.x, -bz.y};                                  // conj Z[256 - k]
        const C2 e = {0.5 * (a.x + b.x), 0.5 * (a.y + b.y)};
        const C2 o = {0.5 * (a.y - b.y), -0.5 * (a.x - b.x)};       // (a - b) / 2i
        const C2 t = cmul(o, tab.tw512[k]);
        const double pr = e.x + t.x, pi = e.y + t.y, qr = e.x - t.x, qi = e.y - t.y;
        pw[2 * k] = fma(pr, pr, pi * pi);
        pw[2 * (256 - k)] = fma(qr, qr, qi * qi);
      }
    }
    __syncwarp();

    // ---- mel filters, log, stores (16 lanes x 8 filters)
    const int64_t f = f0 + fl;
    if (live) {
      float* out = logmel + (clip * F + f) * kMels;
      __nv_bfloat16* sout = (f < n_stack) ? stacked + (clip * n_stack + f) * kMels : nullptr;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const int m = hl + 16 * h;
        const int meta = tab.mel_meta[m];
        const int k0 = meta & 511, cnt = (meta >> 9) & 15, off = meta >> 13;
        double e = 0.0;
        for (int j = 0; j < cnt; ++j) e = fma(tab.mel_w[off + j], pw[2 * (k0 + j)], e);
        const float lm = logf(static_cast<float>(fmax(e, 1e-10)));
        __stcs(out + m, lm);
        if (sout) sout[m] = __float2bfloat16_rn(lm);
      }
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
  for (int k = 0; k < 130; ++k) t->tw512[k] = make_double2(std::cos(2 * pi * k / 512.0), -std::sin(2 * pi * k / 512.0));
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
