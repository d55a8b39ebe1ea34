// fp64 oracle in plain C++: the log-mel front end, 8-frame stacking and the bidirectional
// Transformer encoder, written as textbook loops.
//
// TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU-baseline legs of
// bench.py may load this library (through oracle/__init__.py). It shares no code, table or
// constant generator with the CUDA library; the two meet only through the seeded inputs
// of speech_audio_encoder_b200/synth.py.
//
// Every function is the plain definition of one step, in double precision:
//   * the DFT is the explicit sum X_k = sum_n y[n] e^{-2 pi i k n / 512} (no FFT);
//   * the mel filters are built row by row from the Slaney formulas;
//   * a linear layer is the triple loop C[i][j] = b[j] + sum_k A[i][k] W[j][k];
//   * LayerNorm takes a two-pass mean and variance; softmax subtracts the row maximum;
//   * GELU uses std::erf and RoPE std::cos / std::sin of the fp64 angle.
// The only reordering is what a reader can see at once: the matrix product runs over a
// 4 x 8 block of outputs at a time (each output's sum still runs over k in order), and
// the attention forms a row's scores key by key, each as a dot product in order. Rows,
// frames and heads are independent and are spread over threads (OpenMP).
//
// Sources (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits",
// flozi.net):
//   [ARCH]  section "How audio and speakers reach the language model", the paragraph on
//           the exported frontend: 16 kHz mono audio, 128 log-mel features, 25 ms Hann
//           window, 512-point FFT, 10 ms hop; eight stacked frames projected to width
//           1,280; 32 Transformer layers with ten heads, QK normalisation, feed-forward
//           expansion four and rotary position embeddings.
//   [FUSE]  the same section, the paragraphs on speaker activity and the connector.
//   [CTC]   section "Use alignment and audio questions as supporting evidence".
// The readings where the page is silent are numbered as in oracle/__init__.py.
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <vector>

namespace {

constexpr int kSampleRate = 16000;  // [ARCH]
constexpr int kWin = 400;           // 25 ms [ARCH]
constexpr int kHop = 160;           // 10 ms [ARCH]
constexpr int kNfft = 512;          // [ARCH]
constexpr int kBins = kNfft / 2 + 1;
constexpr int kMels = 128;          // [ARCH]
constexpr double kPi = 3.14159265358979323846;

}  // namespace

extern "C" {

int oc_threads(void) { return omp_get_max_threads(); }

// Frames of 400 samples every 160 (reading 1): none below 400 samples.
int64_t oc_frame_count(int64_t n) { return n < kWin ? 0 : 1 + (n - kWin) / kHop; }

// Periodic Hann window of length 400 (reading 2): w[n] = 0.5 - 0.5 cos(2 pi n / 400).
void oc_hann(double* w) {
  for (int n = 0; n < kWin; ++n) w[n] = 0.5 - 0.5 * std::cos(2.0 * kPi * n / kWin);
}

// Slaney mel scale (reading 4): linear 3 f / 200 below 1 kHz, logarithmic above with
// 27 mels per factor 6.4.
double oc_hz_to_mel(double f) {
  if (f < 1000.0) return 3.0 * f / 200.0;
  return 15.0 + std::log(f / 1000.0) * 27.0 / std::log(6.4);
}

double oc_mel_to_hz(double m) {
  if (m < 15.0) return 200.0 * m / 3.0;
  return 1000.0 * std::exp((m - 15.0) * std::log(6.4) / 27.0);
}

// 128 x 257 filter matrix (reading 4): 130 points equally spaced in mel over 0..8000 Hz;
// row m is the triangle rising from point m to point m + 1 and falling to point m + 2,
// sampled at the bin frequencies 31.25 k Hz, scaled by 2 / (f_{m+2} - f_m).
void oc_mel_filterbank(double* W) {
  double pts[kMels + 2];
  const double top = oc_hz_to_mel(kSampleRate / 2.0);
  for (int i = 0; i < kMels + 2; ++i) pts[i] = oc_mel_to_hz(top * i / (kMels + 1));
  for (int m = 0; m < kMels; ++m) {
    const double lo = pts[m], mid = pts[m + 1], hi = pts[m + 2];
    for (int k = 0; k < kBins; ++k) {
      const double f = static_cast<double>(k) * kSampleRate / kNfft;
      const double rise = (f - lo) / (mid - lo), fall = (hi - f) / (hi - mid);
      const double tri = std::max(0.0, std::min(rise, fall));
      W[m * kBins + k] = tri * 2.0 / (hi - lo);
    }
  }
}

// C [M, N] = A [M, K] B [N, K]^T (+ bias [N] when not null): every output is the sum over
// k = 0, 1, ..., K - 1, in that order, of A[i][k] B[j][k], plus the bias at the end.
// Blocked for the caches only: a 64 x 128 block of outputs is accumulated in a local
// array, k advancing one 256-wide panel at a time (each output's partial sum carries over
// from panel to panel, so its order is that of the plain loop); panels of A and B are
// first copied to contiguous, zero-padded arrays, and the inner loop updates 4 x 8
// outputs per k.
void oc_linear(const double* A, int64_t M, int64_t K, const double* B, int64_t N, const double* bias, double* C) {
  constexpr int MB = 64, NB = 128, KB = 256;
  const int64_t mt = (M + MB - 1) / MB, nt = (N + NB - 1) / NB;
#pragma omp parallel
  {
    std::vector<double> Ap(static_cast<size_t>(MB) * KB), Bp(static_cast<size_t>(KB) * NB),
        Ct(static_cast<size_t>(MB) * NB);
#pragma omp for schedule(dynamic, 1)
    for (int64_t tile = 0; tile < mt * nt; ++tile) {
      const int64_t i0 = (tile / nt) * MB, j0 = (tile % nt) * NB;
      const int64_t mi = std::min<int64_t>(MB, M - i0), nj = std::min<int64_t>(NB, N - j0);
      std::fill(Ct.begin(), Ct.end(), 0.0);
      for (int64_t k0 = 0; k0 < K; k0 += KB) {
        const int64_t kk = std::min<int64_t>(KB, K - k0);
        for (int i = 0; i < MB; ++i)
          for (int k = 0; k < KB; ++k) Ap[i * KB + k] = (i < mi && k < kk) ? A[(i0 + i) * K + k0 + k] : 0.0;
        for (int k = 0; k < KB; ++k)
          for (int j = 0; j < NB; ++j) Bp[k * NB + j] = (j < nj && k < kk) ? B[(j0 + j) * K + k0 + k] : 0.0;
        for (int jb = 0; jb < NB; jb += 8)
          for (int ib = 0; ib < MB; ib += 4) {
            double acc[4][8];
            for (int r = 0; r < 4; ++r)
              for (int c = 0; c < 8; ++c) acc[r][c] = Ct[(ib + r) * NB + jb + c];
            for (int k = 0; k < kk; ++k) {
              const double* __restrict b = &Bp[k * NB + jb];
              for (int r = 0; r < 4; ++r) {
                const double a = Ap[(ib + r) * KB + k];
                for (int c = 0; c < 8; ++c) acc[r][c] += a * b[c];
              }
            }
            for (int r = 0; r < 4; ++r)
              for (int c = 0; c < 8; ++c) Ct[(ib + r) * NB + jb + c] = acc[r][c];
          }
      }
      for (int64_t i = 0; i < mi; ++i)
        for (int64_t j = 0; j < nj; ++j) C[(i0 + i) * N + j0 + j] = Ct[i * NB + j] + (bias ? bias[j0 + j] : 0.0);
    }
  }
}

// |X_k|^2, k = 0..256, of frames y [F, len] (len <= 512) zero-padded to 512 samples
// (reading 3): X_k = sum_{n < len} y[n] (cos(2 pi k n / 512) - i sin(2 pi k n / 512)); the
// padding adds nothing. The cos and sin matrices are the DFT's own, so the sums are one
// matrix product each.
void oc_power_spectrum(const double* y, int64_t F, int64_t len, double* P) {
  std::vector<double> Cm(static_cast<size_t>(kBins) * len), Sm(static_cast<size_t>(kBins) * len);
  for (int k = 0; k < kBins; ++k)
    for (int64_t n = 0; n < len; ++n) {
      const double ang = 2.0 * kPi * static_cast<double>((k * n) % kNfft) / kNfft;
      Cm[k * len + n] = std::cos(ang);
      Sm[k * len + n] = std::sin(ang);
    }
  std::vector<double> re(static_cast<size_t>(F) * kBins), im(static_cast<size_t>(F) * kBins);
  oc_linear(y, F, len, Cm.data(), kBins, nullptr, re.data());
  oc_linear(y, F, len, Sm.data(), kBins, nullptr, im.data());
  for (int64_t i = 0; i < F * kBins; ++i) P[i] = re[i] * re[i] + im[i] * im[i];
}

// [count, 128] natural-log mel energies of frames [first, first + count) of one clip
// (readings 1-5): frame f is w[n] x[160 f + n], n < 400; ln(max(sum_k W[m][k] P[k], 1e-10)).
void oc_log_mel(const float* wave, int64_t n_samples, int64_t first, int64_t count, double* out) {
  (void)n_samples;
  double w[kWin];
  oc_hann(w);
  std::vector<double> W(static_cast<size_t>(kMels) * kBins);
  oc_mel_filterbank(W.data());
  const int64_t chunk = 8192;
  std::vector<double> y, P, E;
  for (int64_t s = 0; s < count; s += chunk) {
    const int64_t c = std::min(chunk, count - s);
    y.assign(static_cast<size_t>(c) * kWin, 0.0);
#pragma omp parallel for schedule(static)
    for (int64_t f = 0; f < c; ++f)
      for (int n = 0; n < kWin; ++n) y[f * kWin + n] = w[n] * static_cast<double>(wave[(first + s + f) * kHop + n]);
    P.assign(static_cast<size_t>(c) * kBins, 0.0);
    oc_power_spectrum(y.data(), c, kWin, P.data());
    E.assign(static_cast<size_t>(c) * kMels, 0.0);
    oc_linear(P.data(), c, kBins, W.data(), kMels, nullptr, E.data());
    for (int64_t i = 0; i < c * kMels; ++i) out[s * kMels + i] = std::log(std::max(E[i], 1e-10));
  }
}

// Per row: (x - mean) / sqrt(var + eps) g + b with a two-pass mean and variance
// (reading 8).
void oc_layer_norm(const double* x, int64_t rows, int64_t width, const double* g, const double* b, double eps,
                   double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * width;
    double mu = 0.0;
    for (int64_t i = 0; i < width; ++i) mu += xr[i];
    mu /= width;
    double var = 0.0;
    for (int64_t i = 0; i < width; ++i) var += (xr[i] - mu) * (xr[i] - mu);
    var /= width;
    const double inv = 1.0 / std::sqrt(var + eps);
    for (int64_t i = 0; i < width; ++i) y[r * width + i] = (xr[i] - mu) * inv * g[i] + b[i];
  }
}

// Per row: x / sqrt(mean(x^2) + eps) g (reading 9).
void oc_rms_norm(const double* x, int64_t rows, int64_t width, const double* g, double eps, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * width;
    double ss = 0.0;
    for (int64_t i = 0; i < width; ++i) ss += xr[i] * xr[i];
    const double inv = 1.0 / std::sqrt(ss / width + eps);
    for (int64_t i = 0; i < width; ++i) y[r * width + i] = xr[i] * inv * g[i];
  }
}

// Rotate the pairs (i, i + hd/2) of each row by the angle pos[row] 10000^(-2 i / hd)
// (reading 10): (a, b) -> (a cos - b sin, b cos + a sin).
void oc_rope(const double* x, int64_t rows, int64_t hd, const double* pos, double* y) {
  const int64_t half = hd / 2;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < half; ++i) {
      const double th = pos[r] * std::pow(10000.0, -2.0 * static_cast<double>(i) / static_cast<double>(hd));
      const double c = std::cos(th), s = std::sin(th);
      const double a = x[r * hd + i], b = x[r * hd + half + i];
      y[r * hd + i] = a * c - b * s;
      y[r * hd + half + i] = b * c + a * s;
    }
}

// softmax(q k^T / sqrt(hd)) of one head: P [Tq, Tk] (reading 11). The scores are the
// matrix product q k^T (oc_linear: each a dot product over d in order), scaled; each row
// then has its maximum subtracted before exponentiating, and is divided by its sum.
void oc_attention_probs(const double* q, int64_t Tq, const double* k, int64_t Tk, int64_t hd, double* P) {
  const double scale = 1.0 / std::sqrt(static_cast<double>(hd));
  oc_linear(q, Tq, hd, k, Tk, nullptr, P);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < Tq; ++t) {
    double* p = P + t * Tk;
    double mx = -INFINITY;
    for (int64_t s = 0; s < Tk; ++s) {
      p[s] *= scale;
      mx = std::max(mx, p[s]);
    }
    double z = 0.0;
    for (int64_t s = 0; s < Tk; ++s) {
      p[s] = std::exp(p[s] - mx);
      z += p[s];
    }
    for (int64_t s = 0; s < Tk; ++s) p[s] /= z;
  }
}

// Per head h: O_h = softmax(q_h k_h^T / sqrt(hd)) v_h (reading 11). q [H, Tq, hd],
// k and v [H, Tk, hd], o [H, Tq, hd]. Query rows are independent, so they are taken 256
// at a time (the probabilities of 256 rows against every key, then their product with v,
// each output a sum over the keys in order).
void oc_attention(const double* q, int64_t H, int64_t Tq, const double* k, const double* v, int64_t Tk, int64_t hd,
                  double* o) {
  constexpr int64_t kRows = 256;
  std::vector<double> vt(static_cast<size_t>(hd) * Tk), P(static_cast<size_t>(std::min(kRows, Tq)) * Tk);
  for (int64_t h = 0; h < H; ++h) {
    const double* vh = v + h * Tk * hd;
#pragma omp parallel for schedule(static)
    for (int64_t d = 0; d < hd; ++d)
      for (int64_t s = 0; s < Tk; ++s) vt[d * Tk + s] = vh[s * hd + d];
    for (int64_t t0 = 0; t0 < Tq; t0 += kRows) {
      const int64_t n = std::min(kRows, Tq - t0);
      oc_attention_probs(q + (h * Tq + t0) * hd, n, k + h * Tk * hd, Tk, hd, P.data());
      oc_linear(P.data(), n, Tk, vt.data(), hd, nullptr, o + (h * Tq + t0) * hd);
    }
  }
}

// Exact GELU 0.5 x (1 + erf(x / sqrt 2)) (reading 12).
void oc_gelu(const double* x, int64_t n, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) y[i] = 0.5 * x[i] * (1.0 + std::erf(x[i] / std::sqrt(2.0)));
}

// Parameters of one encoder layer, float64, weights [out, in].
typedef struct {
  const double *ln1_g, *ln1_b, *w_qkv, *b_qkv, *qn_g, *kn_g, *w_o, *b_o;
  const double *ln2_g, *ln2_b, *w1, *b1, *w2, *b2;
} oc_layer;

// One pre-norm bidirectional Transformer layer on one sequence x [T, width] ([ARCH],
// readings 7-12), evaluated at the positions rows[0..n_rows): keys and values come from
// every position, everything after the attention is per position.
//   h = LN1(x); [q k v] = h Wqkv^T + b; per head q = RoPE(RMS(q) g_q), k likewise (the
//   positions are the sequence indices); o = softmax(q k^T / sqrt(hd)) v;
//   x1 = x + o Wo^T + bo;  out = x1 + W2 GELU(W1 LN2(x1) + b1) + b2.
void oc_encoder_layer_rows(const double* x, int64_t T, int64_t width, int64_t heads, int64_t hd, int64_t ffn,
                           const oc_layer* L, const int64_t* rows, int64_t n_rows, double* out) {
  const int64_t W = width, R = n_rows;
  std::vector<double> h(static_cast<size_t>(T) * W), qkv(static_cast<size_t>(T) * 3 * W);
  oc_layer_norm(x, T, W, L->ln1_g, L->ln1_b, 1e-5, h.data());
  oc_linear(h.data(), T, W, L->w_qkv, 3 * W, L->b_qkv, qkv.data());
  // per head [heads, T, hd] k and v over every position; q over the selected rows
  std::vector<double> q(static_cast<size_t>(heads) * R * hd), k(static_cast<size_t>(heads) * T * hd),
      v(static_cast<size_t>(heads) * T * hd);
  std::vector<double> tmp(static_cast<size_t>(std::max(T, R)) * hd), tmp2(tmp.size()), pos(std::max(T, R));
  for (int64_t hh = 0; hh < heads; ++hh) {
    for (int64_t t = 0; t < T; ++t) pos[t] = static_cast<double>(t);
    for (int64_t t = 0; t < T; ++t)
      for (int64_t d = 0; d < hd; ++d) tmp[t * hd + d] = qkv[t * 3 * W + W + hh * hd + d];
    oc_rms_norm(tmp.data(), T, hd, L->kn_g, 1e-6, tmp2.data());
    oc_rope(tmp2.data(), T, hd, pos.data(), &k[hh * T * hd]);
    for (int64_t t = 0; t < T; ++t)
      for (int64_t d = 0; d < hd; ++d) v[(hh * T + t) * hd + d] = qkv[t * 3 * W + 2 * W + hh * hd + d];
    for (int64_t r = 0; r < R; ++r) {
      pos[r] = static_cast<double>(rows[r]);
      for (int64_t d = 0; d < hd; ++d) tmp[r * hd + d] = qkv[rows[r] * 3 * W + hh * hd + d];
    }
    oc_rms_norm(tmp.data(), R, hd, L->qn_g, 1e-6, tmp2.data());
    oc_rope(tmp2.data(), R, hd, pos.data(), &q[hh * R * hd]);
  }
  std::vector<double> o(static_cast<size_t>(heads) * R * hd);
  oc_attention(q.data(), heads, R, k.data(), v.data(), T, hd, o.data());
  std::vector<double> oc(static_cast<size_t>(R) * W), x1(static_cast<size_t>(R) * W);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t hh = 0; hh < heads; ++hh)
      for (int64_t d = 0; d < hd; ++d) oc[r * W + hh * hd + d] = o[(hh * R + r) * hd + d];
  oc_linear(oc.data(), R, W, L->w_o, W, L->b_o, x1.data());
  for (int64_t r = 0; r < R; ++r)
    for (int64_t i = 0; i < W; ++i) x1[r * W + i] += x[rows[r] * W + i];
  std::vector<double> h2(static_cast<size_t>(R) * W), u(static_cast<size_t>(R) * ffn), ug(u.size());
  oc_layer_norm(x1.data(), R, W, L->ln2_g, L->ln2_b, 1e-5, h2.data());
  oc_linear(h2.data(), R, W, L->w1, ffn, L->b1, u.data());
  oc_gelu(u.data(), R * ffn, ug.data());
  oc_linear(ug.data(), R, ffn, L->w2, W, L->b2, out);
  for (int64_t i = 0; i < R * W; ++i) out[i] += x1[i];
}

}  // extern "C"

extern "C" {

// Fixed sinusoidal speaker kernel K [n_slots, width] (reading 15):
// K[s][2i] = sin(s w_i), K[s][2i + 1] = cos(s w_i), w_i = 10000^(-2 i / width).
void oc_speaker_kernel(int64_t n_slots, int64_t width, double* K) {
  for (int64_t s = 0; s < n_slots; ++s)
    for (int64_t i = 0; i < width / 2; ++i) {
      const double w = std::pow(10000.0, -2.0 * static_cast<double>(i) / static_cast<double>(width));
      K[s * width + 2 * i] = std::sin(static_cast<double>(s) * w);
      K[s * width + 2 * i + 1] = std::cos(static_cast<double>(s) * w);
    }
}

// Per row: z - max - log(sum exp(z - max)) (reading 21).
void oc_log_softmax(const double* z, int64_t rows, int64_t n, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double* zr = z + r * n;
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) mx = std::max(mx, zr[i]);
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += std::exp(zr[i] - mx);
    const double lse = mx + std::log(s);
    for (int64_t i = 0; i < n; ++i) y[r * n + i] = zr[i] - lse;
  }
}

}  // extern "C"
