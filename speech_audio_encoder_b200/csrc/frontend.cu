// Front end: 16 kHz float32 waveform -> 128 natural-log Slaney mel energies per 10 ms
// frame (25 ms periodic Hann window, 512-point FFT), plus the bf16 copy of the first
// 8 T frames that, read as [T, 1024], is the frame-major stack of eight frames.
// (Page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits", section
// "How audio and speakers reach the language model", exported-frontend paragraph.)
//
// A persistent kernel: one CTA of 16 warps per SM. Every warp works on its own: it walks
// pairs of consecutive frames (one clip each), and while it transforms one pair, the
// 560 samples of its next pair are on their way into its own shared-memory buffer
// (cp.async, double buffered), so no CTA-wide barrier ties the warps' phases together.
// Each half-warp (16 lanes) takes one frame of the pair:
//   1. the 400 windowed samples, zero-padded to 512, are packed as 256 complex values
//      z[m] = y[2m] + i y[2m+1];
//   2. a 256-point complex FFT factored 16 x 16: lane n2 transforms z[16 n1 + n2] over n1
//      in registers and applies the twiddle W256^(n2 k1) (powers of W256^n2 formed in
//      registers); one transposing exchange in
//      shared memory; lane k1 transforms over n2, giving Z[k1 + 16 k2] in its registers;
//   3. the split step for the pair (k, 256 - k): with E = Z[k] + conj Z[256-k] and
//      O = (Z[k] - conj Z[256-k]) / i, 2 X[k] = E + W512^k O and 2 X[256-k] =
//      conj(E - W512^k O). Z[256-k] sits in lane 16 - k1, so the pairs meet by warp
//      shuffles; the powers 4 |X|^2 go to shared memory in fp32 (a relative rounding of
//      2^-24 per bin);
//   4. 128 sparse triangular filters (504 non-zero weights, scaled by 1/4) summed in fp32
//      (positive terms: relative error below 1e-6) over zero-padded windows of 2 to 12
//      bins, ln(max(e, 1e-10)).
// The window product and the transform run in fp64. A bin 60 dB under the frame's
// strongest component (the noise floor of a clean tone) carries an fp32 error of ~1e-6 of
// the frame norm, a few 1e-4 in its log and above the 1e-4 budget, because every rounding
// of a sample or butterfly scales with the strong component (rounding only the window
// product to fp32 already costs 2e-4 on the 1 s tone clip). The powers and the filter
// sums round each value relative to itself and stay in fp32.
#define SAL_CK_FILE 1
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>
#include <vector>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kHalfWarps = 2 * kWarps;
constexpr int kPairSamples = kHop + kWin;  // 560: two consecutive frames
constexpr int kMelNnz = 504;

// Filter m = lane + 16 h of the half-warp's 8 groups spans at most mel_taps(h) bins (the
// widths of the Slaney filters grow with frequency); every lane of a group runs that many
// taps over a zero-padded window, so the loops unroll completely.
__host__ __device__ constexpr int mel_taps(int h) {
  return h < 3 ? 2 : h == 3 ? 3 : h == 4 ? 4 : h == 5 ? 6 : h == 6 ? 9 : 12;
}
// offset of group h in the padded weight table: 16 x (taps of the groups before it)
__host__ __device__ constexpr int mel_base(int h) {
  return 16 * (h == 0 ? 0 : h == 1 ? 2 : h == 2 ? 4 : h == 3 ? 6 : h == 4 ? 9 : h == 5 ? 13 : h == 6 ? 19 : h == 7 ? 28 : 40);
}
constexpr bool mel_table_consistent() {
  for (int h = 0; h < 8; ++h)
    if (mel_base(h + 1) - mel_base(h) != 16 * mel_taps(h)) return false;
  return true;
}
static_assert(mel_table_consistent(), "mel group offsets");
constexpr int kMelPadded = mel_base(8);  // 640

struct FrontTables {
  double2 tw256[16];       // [n2] = e^{-2 pi i n2 / 256}
  double2 tw512[8 * 16];   // [k2][k1] = e^{-2 pi i k / 512}, k = k1 + 16 k2 < 128
  double hann[kWin];
  float mel_w[kMelPadded];  // [group h][tap j][lane]: weights / 4 of filter 16 h + lane at bin mel_k0 + j
  int mel_k0[kMels];        // first bin of each filter's window
};
static_assert(sizeof(FrontTables) % 16 == 0, "table copy uses 16-byte words");

__device__ FrontTables g_front_tables;

// Per half-warp scratch: 16 rows of 17 complex doubles (the transposing exchange), later
// the 257 fp32 powers. The stride is 16 banks off a multiple of 32 banks so that the two
// half-warps of a warp meet different banks in the 4-byte phases.
constexpr int kScratch = 16 * 17 + 4;  // double2 entries
constexpr size_t kOffSamples = sizeof(FrontTables);  // [warp][2][kPairSamples] floats
constexpr size_t kOffScratch = kOffSamples + sizeof(float) * kWarps * 2 * kPairSamples;
constexpr size_t kSmemBytes = kOffScratch + sizeof(double2) * kHalfWarps * kScratch;
static_assert(kOffSamples % 16 == 0 && kOffScratch % 16 == 0 && (kPairSamples * 4) % 16 == 0, "alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

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
// kTailZero: x[13] = x[14] = x[15] = 0 (the zero padding in pass 1, where the 400 samples
// fill z[0..199] of the 256 packed values), so three of the first 4-point transforms have
// a zero last input and skip two complex additions each.
template <bool kTailZero>
__device__ __forceinline__ void dft16(C2 (&v)[16]) {
  const double c1 = 0.92387953251128675613, s1 = 0.38268343236508977173;  // cos, sin of pi/8
  const double r = 0.70710678118654752440;
  C2 y[4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    if (kTailZero && b > 0) {  // dft4(a, b, c, 0)
      const C2 s0 = cadd(v[b], v[8 + b]), d0 = csub(v[b], v[8 + b]), m = v[4 + b];
      y[b][0] = cadd(s0, m);
      y[b][2] = csub(s0, m);
      y[b][1] = cadd(d0, mul_neg_i(m));
      y[b][3] = cadd(d0, mul_pos_i(m));
    } else {
      dft4(v[b], v[4 + b], v[8 + b], v[12 + b], y[b][0], y[b][1], y[b][2], y[b][3]);
    }
  }
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

__device__ __forceinline__ C2 shfl_c2(C2 a, int src) {
  return {__shfl_sync(0xffffffffu, a.x, src), __shfl_sync(0xffffffffu, a.y, src)};
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// The samples of frame pair `pin` of clip `clip` (frames 2 pin and 2 pin + 1) into `dst`,
// by the 32 lanes of a warp: 400 samples for a pair holding one frame, else 560.
__device__ __forceinline__ void stage_pair(float* dst, const float* __restrict__ wave, int64_t n_samples,
                                           int64_t F, int64_t clip, int64_t pin, bool vec, int lane) {
  const int64_t f = 2 * pin;
  const int n = f + 1 < F ? kPairSamples : kWin;
  const float* src = wave + clip * n_samples + kHop * f;
  if (vec) {
    for (int i = lane; i < n / 4; i += 32) cp_async16(dst + 4 * i, SAL_CK_LD(src + 4 * i, 16));
  } else {
    for (int i = lane; i < n; i += 32) cp_async4(dst + i, SAL_CK_LD(src + i, 4));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    frontend_kernel(const float* __restrict__ wave, int64_t n_samples, int batch, int64_t F, int64_t n_stack,
                    float* __restrict__ logmel, __nv_bfloat16* __restrict__ stacked) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FrontTables& tab = *reinterpret_cast<FrontTables*>(smem_raw);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int hl = lane & 15;    // lane within the half-warp
  const int sub = lane >> 4;   // frame of the pair
  const int half = tid >> 4;   // half-warp index in the CTA
  float* samples = reinterpret_cast<float*>(smem_raw + kOffSamples) + warp * 2 * kPairSamples;
  double2* scr = reinterpret_cast<double2*>(smem_raw + kOffScratch) + half * kScratch;
  float* pw = reinterpret_cast<float*>(scr);  // 4 |X[k]|^2 after the transform
  const int partner = (lane & 16) | ((16 - hl) & 15);

  {  // tables (computed once on the host)
    const int4* src = reinterpret_cast<const int4*>(&g_front_tables);
    int4* dst = reinterpret_cast<int4*>(smem_raw);
    for (int i = tid; i < static_cast<int>(sizeof(FrontTables) / 16); i += kThreads) dst[i] = *SAL_CK_LD(src + i, 16);
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  const int64_t pairs_per_clip = (F + 1) / 2;
  const int64_t n_pairs = pairs_per_clip * batch;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
  // 16-byte copies need 16-byte aligned sources: every pair starts 1280 B into its clip
  const bool vec = (reinterpret_cast<uintptr_t>(wave) & 15u) == 0 && (n_samples & 3) == 0;
  // the warp's pairs: pair, pair + stride, ...; (clip, pair within the clip) advance by
  // (stride_clips, stride_rem) without a division per step
  int64_t pair = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  int64_t clip = pair / pairs_per_clip, pin = pair - clip * pairs_per_clip;
  const int64_t stride_clips = stride / pairs_per_clip, stride_rem = stride - stride_clips * pairs_per_clip;
  if (pair < n_pairs) stage_pair(samples, wave, n_samples, F, clip, pin, vec, lane);
  cp_async_commit();

  for (int it = 0; pair < n_pairs; ++it) {
    float* cur = samples + (it & 1) * kPairSamples;
    int64_t nclip = clip + stride_clips, npin = pin + stride_rem;
    if (npin >= pairs_per_clip) {
      npin -= pairs_per_clip;
      ++nclip;
    }
    if (pair + stride < n_pairs)
      stage_pair(samples + ((it + 1) & 1) * kPairSamples, wave, n_samples, F, nclip, npin, vec, lane);
    cp_async_commit();
    cp_async_wait_one();  // this pair's samples have landed (for this lane's copies)
    __syncwarp();         // ... and for every lane's

    const int64_t f = 2 * pin + sub;
    const bool live = f < F;
    const float* x = cur + (live ? kHop * sub : 0);

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
    dft16<true>(v);
    {
      // twiddles W256^(n2 k1) as running products of W256^n2 in registers (fp64: 14
      // products add a few 1e-16): one table read per frame instead of 15, which measured
      // 8 % faster than reading them all
      scr[hl * 17] = make_double2(v[0].x, v[0].y);
      const double2 w1 = tab.tw256[hl];
      double2 w = w1;
#pragma unroll
      for (int k1 = 1; k1 < 16; ++k1) {
        const C2 t = cmul(v[k1], w);
        scr[hl * 17 + k1] = make_double2(t.x, t.y);
        if (k1 < 15) w = make_double2(fma(w.x, w1.x, -w.y * w1.y), fma(w.x, w1.y, w.y * w1.x));
      }
    }
    __syncwarp();

    // ---- pass 2: lane k1 = hl transforms over n2, giving Z[k1 + 16 k2] in v[k2]
#pragma unroll
    for (int n2 = 0; n2 < 16; ++n2) {
      const double2 a = scr[n2 * 17 + hl];
      v[n2] = {a.x, a.y};
    }
    dft16<false>(v);
    __syncwarp();  // the scratch now takes the powers

    // ---- split and power. Lane k1 owns the pairs (k, 256 - k), k = k1 + 16 k2, k2 < 8;
    //      Z[256 - k] = Z[(16 - k1) + 16 (15 - k2)] is v[15 - k2] of lane 16 - k1. Lane 0
    //      pairs with itself (Z[256 - 16 k2] = its own v[16 - k2]), and also takes k = 0
    //      (X[0], X[256] are real) and k = 128 (X[128] = conj Z[128]).
    if (hl == 0) pw[128] = static_cast<float>(4.0 * fma(v[8].x, v[8].x, v[8].y * v[8].y));
    C2 r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const C2 send = (hl == 0 && i < 7) ? v[9 + i] : v[8 + i];
      r[i] = shfl_c2(send, partner);
    }
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2) {
      const int k = hl + 16 * k2;
      const C2 a = v[k2];
      const C2 b = {r[7 - k2].x, -r[7 - k2].y};  // conj Z[256 - k]
      const C2 e = cadd(a, b);
      const C2 o = mul_neg_i(csub(a, b));
      const C2 t = cmul(o, tab.tw512[k2 * 16 + hl]);
      const double pr = e.x + t.x, pi = e.y + t.y, qr = e.x - t.x, qi = e.y - t.y;
      double p_lo = fma(pr, pr, pi * pi), p_hi = fma(qr, qr, qi * qi);
      if (k2 == 0 && hl == 0) {
        const double x0 = a.x + a.y, x256 = a.x - a.y;
        p_lo = 4.0 * x0 * x0;
        p_hi = 4.0 * x256 * x256;
      }
      pw[k] = static_cast<float>(p_lo);
      pw[256 - k] = static_cast<float>(p_hi);
    }
    __syncwarp();

    // ---- mel filters, log, stores (16 lanes x 8 filters)
    if (live) {
      float* out = logmel + (clip * F + f) * kMels;
      __nv_bfloat16* sout = (f < n_stack) ? stacked + (clip * n_stack + f) * kMels : nullptr;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const int m = hl + 16 * h;
        const float* pk = pw + tab.mel_k0[m];
        const float* wk = tab.mel_w + mel_base(h) + hl;
        float e = 0.f;
#pragma unroll
        for (int j = 0; j < mel_taps(h); ++j) e = fmaf(wk[16 * j], pk[j], e);
        // __logf: absolute error ~1e-6 over the range of e, far inside the 1e-4 budget
        const float lm = __logf(fmaxf(e, 1e-10f));
        __stcs(SAL_CK_ST(out + m, 4), lm);
        if (sout) *SAL_CK_ST(sout + m, 2) = __float2bfloat16_rn(lm);
      }
    }
    __syncwarp();  // the samples buffer and the scratch are free again
    pair += stride;
    clip = nclip;
    pin = npin;
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
  for (int n2 = 0; n2 < 16; ++n2) t->tw256[n2] = make_double2(std::cos(2 * pi * n2 / 256.0), -std::sin(2 * pi * n2 / 256.0));
  for (int k = 0; k < 128; ++k) t->tw512[k] = make_double2(std::cos(2 * pi * k / 512.0), -std::sin(2 * pi * k / 512.0));
  for (int n = 0; n < kWin; ++n) t->hann[n] = 0.5 - 0.5 * std::cos(2 * pi * n / 400.0);
  // Slaney filters: 130 points equally spaced in mel over 0..8000 Hz.
  double pts[kMels + 2];
  const double mmax = hz_to_mel_slaney(8000.0);
  for (int i = 0; i < kMels + 2; ++i) pts[i] = mel_to_hz_slaney(mmax * i / (kMels + 1));
  // dense weights of each filter, then the padded windows
  std::vector<double> dense(static_cast<size_t>(kMels) * kBins, 0.0);
  int nnz = 0;
  for (int m = 0; m < kMels; ++m) {
    const double norm = 2.0 / (pts[m + 2] - pts[m]);
    for (int k = 0; k < kBins; ++k) {
      const double fk = 31.25 * k;
      const double rise = (fk - pts[m]) / (pts[m + 1] - pts[m]);
      const double fall = (pts[m + 2] - fk) / (pts[m + 2] - pts[m + 1]);
      const double w = std::fmax(0.0, std::fmin(rise, fall)) * norm;
      dense[static_cast<size_t>(m) * kBins + k] = w;
      nnz += w > 0.0;
    }
  }
  for (int m = 0; m < kMels; ++m) {
    const int h = m / 16, lane = m % 16, taps = mel_taps(h);
    int first = -1, last = -1;
    for (int k = 0; k < kBins; ++k)
      if (dense[static_cast<size_t>(m) * kBins + k] > 0.0) {
        if (first < 0) first = k;
        last = k;
      }
    if (first < 0) return false;
    const int k0 = first + taps <= kBins ? first : kBins - taps;
    if (last >= k0 + taps) return false;  // the filter must fit its group's window
    t->mel_k0[m] = k0;
    for (int j = 0; j < taps; ++j)
      t->mel_w[mel_base(h) + 16 * j + lane] = static_cast<float>(0.25 * dense[static_cast<size_t>(m) * kBins + k0 + j]);
  }
  return nnz == kMelNnz;
}

std::mutex g_init_mu;
bool g_init_done[64] = {};
int g_sms[64] = {};
const void* g_tables_addr[64] = {};  // device address of the tables

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
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return SAL_ECUDA;
  g_sms[dev] = n;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_front_tables) != cudaSuccess) return SAL_ECUDA;
  g_tables_addr[dev] = addr;
  g_init_done[dev] = true;
  return SAL_OK;
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_init_mu);
  return (dev >= 0 && dev < 64 && g_sms[dev] > 0) ? g_sms[dev] : 1;
}

const void* tables_addr() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_init_mu);
  return (dev >= 0 && dev < 64) ? g_tables_addr[dev] : nullptr;
}

}  // namespace

sal_status frontend_launch(const float* wave, int64_t n_samples, int batch, int64_t frames,
                           int64_t positions, float* logmel, void* stacked, cudaStream_t s) {
  if (frames == 0) return SAL_OK;
  const sal_status st = ensure_tables();
  if (st != SAL_OK) return st;
  const int64_t ctas = ((frames + 1) / 2 * batch + kWarps - 1) / kWarps;
  const int64_t sms = sm_count();
  const dim3 grid(static_cast<unsigned>(ctas < sms ? ctas : sms));
  const int64_t n_stack = stacked ? positions * kStack : 0;
  ck_declare(wave, batch * n_samples * 4, false);
  ck_declare(logmel, batch * frames * kMels * 4, true);
  ck_declare(stacked, batch * n_stack * kMels * 2, true);
  ck_declare(tables_addr(), sizeof(FrontTables), false);
  return launch_kernel(frontend_kernel, grid, dim3(kThreads), kSmemBytes, s, wave, n_samples, batch, frames, n_stack,
                       logmel, static_cast<__nv_bfloat16*>(stacked)) == cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

}  // namespace sal
