// The extern "C" entry points of libsal (declared in include/sal.h): argument checks,
// tensor-map construction, workspace layout and the per-layer launch sequence.
//
// Per encoder layer, on the caller's stream (page "Nemotron 3.5 Transcribe: From Recorded
// Speech to Dataset Audits", section "How audio and speakers reach the language model"):
//   1. h = LayerNorm1(x)                                  (row kernel, fp32 -> bf16)
//   2. q, k, v = RoPE(RMSNorm(h Wqkv^T + b))              (GEMM, QK-norm + RoPE epilogue)
//   3. o = softmax(q k^T / sqrt(128)) v                   (attention kernel)
//   4. x += o Wo^T + bo                                   (GEMM, residual epilogue)
//   5. h = LayerNorm2(x)                                  (row kernel)
//   6. u = GELU(h W1^T + b1)                              (GEMM, GELU epilogue)
//   7. x += u W2^T + b2                                   (GEMM, residual epilogue)
// and after the last layer emb = LayerNormF(x).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <mutex>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {

__device__ unsigned int g_status = 0;

namespace {

std::atomic<uint64_t> g_wait_limit_ns{4000000000ull};
std::atomic<uint64_t> g_launches{0};

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode_tiled;
}

std::mutex g_dev_mu;
int g_dev_ok[64] = {};  // 0 unknown, 1 sm_100, 2 other

sal_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAL_ECUDA;
  if (dev < 0 || dev >= 64) return SAL_EDEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev_ok[dev]) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return SAL_ECUDA;
    g_dev_ok[dev] = major == 10 ? 1 : 2;
  }
  return g_dev_ok[dev] == 1 ? SAL_OK : SAL_EDEVICE;
}

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct EncoderWs {
  void* h;      // [M, 1280] bf16
  void *q, *k, *v, *o;  // [M, 1280] bf16 each; u [M, 5120] bf16 overlays all four
  void* u;
  float* rope;  // [2, T, 64] f32
  size_t bytes;
};

EncoderWs encoder_ws_layout(void* base, int batch, int64_t T) {
  const size_t M = static_cast<size_t>(batch) * static_cast<size_t>(T);
  const size_t act = align256(M * kWidth * 2);
  EncoderWs w{};
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.h = p + off;
  off += act;
  w.q = p + off;
  w.k = p + off + act;
  w.v = p + off + 2 * act;
  w.o = p + off + 3 * act;
  w.u = p + off;
  off += std::max(4 * act, align256(M * kFfn * 2));
  w.rope = reinterpret_cast<float*>(p + off);
  off += align256(static_cast<size_t>(T) * 64 * 2 * sizeof(float));
  w.bytes = off;
  return w;
}

// CTC adapter workspace over M2 = batch * 2T positions of width 1024: the fp32 residual
// stream x, the bf16 LN output h, q / k / v / o, one large region that holds in turn the
// fp32 QKV rows, the bf16 FFN hidden rows and the fp32 class scores, the RoPE table of
// the 2T positions, and the upsampling bias repeated for both taps.
constexpr int kCtcClassesPad = (SAL_CTC_CLASSES + 255) / 256 * 256;  // 24,064: 256-wide column tiles

struct CtcWs {
  float* x;
  void *h, *q, *k, *v, *o, *big, *bias2;
  float* rope;
  size_t bytes;
};

CtcWs ctc_ws_layout(void* base, int batch, int64_t T) {
  const size_t M2 = static_cast<size_t>(batch) * static_cast<size_t>(2 * T);
  const size_t W = SAL_CTC_WIDTH;
  char* p = static_cast<char*>(base);
  CtcWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    char* r = p + off;
    off += align256(n);
    return r;
  };
  w.x = reinterpret_cast<float*>(take(M2 * W * 4));
  w.h = take(M2 * W * 2);
  w.q = take(M2 * W * 2);
  w.k = take(M2 * W * 2);
  w.v = take(M2 * W * 2);
  w.o = take(M2 * W * 2);
  w.big = take(M2 * std::max(std::max(3 * W * 4, static_cast<size_t>(SAL_CTC_FFN) * 2),
                             static_cast<size_t>(kCtcClassesPad) * 4));
  w.rope = reinterpret_cast<float*>(take(static_cast<size_t>(2 * T) * 64 * 2 * sizeof(float)));
  w.bias2 = take(2 * W * 2);
  w.bytes = off;
  return w;
}

bool layer_ok(const sal_layer& L) {
  const void* ps[] = {L.ln1_g, L.ln1_b, L.w_qkv, L.b_qkv, L.qn_g, L.kn_g, L.w_o,
                      L.b_o,   L.ln2_g, L.ln2_b, L.w1,    L.b1,    L.w2,   L.b2};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return false;
  return true;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

Windows make_windows(int64_t total, int64_t core, int64_t ctx) {
  Windows wn;
  if (total <= 0 || core <= 0) return wn;
  if (core > total) core = total;  // one window: the whole clip
  if (ctx > total) ctx = total;    // context past the clip ends is clipped anyway
  if (ctx < 0) ctx = 0;
  wn.count = static_cast<int>((total + core - 1) / core);
  wn.core = static_cast<int>(core);
  wn.ctx = static_cast<int>(ctx);
  wn.total = total;
  for (int64_t w = 0; w < wn.count; ++w) {
    const int64_t lo = std::max<int64_t>(0, w * core - ctx), hi = std::min<int64_t>(total, (w + 1) * core + ctx);
    wn.slot = std::max(wn.slot, hi - lo);
  }
  return wn;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SAL_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

unsigned int* device_status_ptr() {
  static std::mutex mu;
  static unsigned int* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned int*>(p);
  }
  return ptrs[dev];
}

#ifdef SAL_CHECKED
// Bounds-checked build: the ranges declared on this thread since its last launch, the
// test hook's shortening of writable ranges, and per device the report and the sink.
namespace {
struct CkPending {
  CkTable t{};
  bool overflow = false;
};
thread_local CkPending g_ck;
std::atomic<uint64_t> g_ck_shrink{0};
struct CkDevice {
  CkReport* report = nullptr;
  void* sink = nullptr;
};
CkDevice g_ck_dev[64];
std::mutex g_ck_mu;
constexpr CkReport kCkClear = {0ull, ~0ull, ~0ull};

CkDevice* ck_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_ck_mu);
  CkDevice& d = g_ck_dev[dev];
  if (!d.report) {
    void *r = nullptr, *k = nullptr;
    if (cudaMalloc(&r, sizeof(CkReport)) != cudaSuccess) return nullptr;
    if (cudaMalloc(&k, kCkSinkBytes) != cudaSuccess ||
        cudaMemcpy(r, &kCkClear, sizeof(CkReport), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(r);
      if (k) cudaFree(k);
      return nullptr;
    }
    d.report = static_cast<CkReport*>(r);
    d.sink = k;
  }
  return &d;
}
}  // namespace

void ck_declare(const void* p, uint64_t bytes, bool writable) {
  if (!p) return;
  CkPending& pnd = g_ck;
  if (pnd.t.n >= kCkSpans) {
    pnd.overflow = true;
    return;
  }
  if (writable) {
    const uint64_t sh = g_ck_shrink.load();
    bytes = bytes > sh ? bytes - sh : 0;
  }
  const int i = pnd.t.n++;
  pnd.t.lo[i] = reinterpret_cast<uintptr_t>(p);
  pnd.t.hi[i] = pnd.t.lo[i] + bytes;
  if (writable) pnd.t.writable |= 1u << i;
}

bool ck_take(CkTable* t) {
  CkPending& pnd = g_ck;
  CkDevice* d = ck_device();
  const bool ok = d && !pnd.overflow;
  *t = pnd.t;
  t->seq = g_launches.load();
  t->report = d ? d->report : nullptr;
  t->sink = d ? d->sink : nullptr;
  pnd = CkPending{};
  return ok;
}
#endif

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sal

using namespace sal;

#define SAL_TRY(expr)                 \
  do {                                \
    const sal_status st_ = (expr);    \
    if (st_ != SAL_OK) return st_;    \
  } while (0)

namespace {
// Stage names, indexed by the SAL_KIND_* values.
const char* const kKindNames[SAL_KIND_COUNT] = {"rope_table", "layernorm", "qkv", "attention",
                                                "out_proj", "ffn_up", "ffn_down"};
}  // namespace

extern "C" {

int64_t sal_frame_count(int64_t n) { return n < kWin ? 0 : 1 + (n - kWin) / kHop; }

int64_t sal_position_count(int64_t n) { return sal_frame_count(n) / kStack; }

const char* sal_status_string(int status) {
  switch (status) {
    case SAL_OK: return "ok";
    case SAL_EINVAL: return "invalid argument (null or misaligned pointer, bad value)";
    case SAL_ESHAPE: return "unsupported shape";
    case SAL_EWORKSPACE: return "workspace too small";
    case SAL_ECUDA: return "CUDA runtime error";
    case SAL_ETIMEOUT: return "a bounded device wait gave up";
    case SAL_EDEVICE: return "device is not an sm_100 GPU";
    case SAL_EIO: return "a file could not be opened or read";
    default: return "unknown status";
  }
}

void sal_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 1); }

int sal_checked_build(void) {
#ifdef SAL_CHECKED
  return 1;
#else
  return 0;
#endif
}

sal_status sal_check_report(uint64_t* count, uint64_t* first_address, int* file, int* line, uint64_t* first_launch) {
  if (!count || !first_address || !file || !line || !first_launch) return SAL_EINVAL;
  *count = *first_address = *first_launch = 0;
  *file = *line = 0;
#ifdef SAL_CHECKED
  CkDevice* d = ck_device();
  if (!d) return SAL_ECUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SAL_ECUDA;
  CkReport r;
  if (cudaMemcpy(&r, d->report, sizeof(r), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(d->report, &kCkClear, sizeof(r), cudaMemcpyHostToDevice) != cudaSuccess)
    return SAL_ECUDA;
  *count = r.count;
  if (r.count) {
    *first_address = r.min_key >> 16;
    *file = static_cast<int>((r.min_key >> 12) & 15u);
    *line = static_cast<int>(r.min_key & 4095u);
    *first_launch = r.min_seq;
  }
  return SAL_OK;
#else
  return SAL_EINVAL;
#endif
}

void sal_check_shrink_writable(uint64_t bytes) {
#ifdef SAL_CHECKED
  g_ck_shrink.store(bytes);
#else
  (void)bytes;
#endif
}

sal_status sal_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAL_ECUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return SAL_ECUDA;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return SAL_ECUDA;
  return (v & kStatusTimeout) ? SAL_ETIMEOUT : SAL_OK;
}

sal_status sal_frontend(const float* wave, int64_t n_samples, int batch, float* logmel, void* stacked,
                        void* stream) {
  const NvtxRange nvtx_("sal_frontend");
  if (batch < 0 || n_samples < 0) return SAL_EINVAL;
  const int64_t F = sal_frame_count(n_samples), T = F / kStack;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || F == 0) return SAL_OK;
  if (batch > 65535) return SAL_ESHAPE;
  if (!wave || !logmel || !aligned16(wave) || !aligned16(logmel)) return SAL_EINVAL;
  if (stacked && !aligned16(stacked)) return SAL_EINVAL;
  SAL_TRY(check_device());
  return frontend_launch(wave, n_samples, batch, F, T, logmel, stacked, static_cast<cudaStream_t>(stream));
}

sal_status sal_stack_project(const void* stacked, int batch, int64_t T, const sal_weights* w, float* x,
                             void* stream) {
  const NvtxRange nvtx_("sal_stack_project");
  if (batch < 0 || T < 0 || !w) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (!stacked || !x || !w->w_proj || !w->b_proj || !aligned16(stacked) || !aligned16(x) ||
      !aligned16(w->w_proj) || !aligned16(w->b_proj))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return gemm_launch(SAL_EPI_STORE_F32, stacked, static_cast<int64_t>(batch) * T, SAL_STACK_DIM, w->w_proj,
                     kWidth, w->b_proj, x, nullptr, static_cast<cudaStream_t>(stream));
}

size_t sal_encoder_workspace_bytes(int batch, int64_t T) {
  if (batch <= 0 || T <= 0) return 0;
  return encoder_ws_layout(nullptr, batch, T).bytes;
}

namespace {
bool windowed(const sal_forward_options* o) { return o && o->window_core > 0; }

// Workspace of a windowed forward: the windowed fp32 stream and bf16 embeddings, then the
// encoder workspace of the windowed batch.
size_t windowed_ws_bytes(int batch, const Windows& wn) {
  const size_t rows = static_cast<size_t>(batch) * wn.count * static_cast<size_t>(wn.slot);
  return align256(rows * kWidth * 4) + align256(rows * kWidth * 2) +
         encoder_ws_layout(nullptr, batch * wn.count, wn.slot).bytes;
}
}  // namespace

size_t sal_encoder_workspace_bytes_ex(int batch, int64_t T, const sal_forward_options* opts) {
  if (batch <= 0 || T <= 0) return 0;
  if (!windowed(opts)) return sal_encoder_workspace_bytes(batch, T);
  return windowed_ws_bytes(batch, make_windows(T, opts->window_core, opts->window_context));
}

sal_status sal_encoder_forward(float* x, int batch, int64_t T, const sal_weights* w, int n_layers, void* emb,
                               void* workspace, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_("sal_encoder_forward");
  return sal_encoder_forward_ex(x, batch, T, w, n_layers, emb, workspace, ws_bytes, stream, nullptr);
}

namespace {
// Records trace events around the launches of one kind (as event-record nodes when the
// stream is being captured into a CUDA graph).
struct Tracer {
  const sal_trace* tr;
  cudaStream_t s;
  int seen = 0;
  bool before(int kind) {
    if (!tr || tr->kind != kind || 2 * seen + 1 >= tr->n_events) return true;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(tr->events[2 * seen]), s, cudaEventRecordExternal) ==
           cudaSuccess;
  }
  bool after(int kind) {
    if (!tr || tr->kind != kind || 2 * seen + 1 >= tr->n_events) return true;
    const bool ok = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(tr->events[2 * seen + 1]), s,
                                            cudaEventRecordExternal) == cudaSuccess;
    ++seen;
    return ok;
  }
};
}  // namespace

#define SAL_TRACED(kind, expr)                              \
  do {                                                      \
    const NvtxRange stage_(kKindNames[kind]);               \
    if (!tr.before(kind)) return SAL_ECUDA;                 \
    SAL_TRY(expr);                                          \
    if (!tr.after(kind)) return SAL_ECUDA;                  \
  } while (0)

namespace {
// The layer sequence over `batch` clips of T positions, then the final LayerNorm into emb.
// `win`: the clips are serving windows (attention only over each window's own length).
sal_status run_layers(float* x, int batch, int64_t T, const sal_weights* w, int n_layers, void* emb,
                      const EncoderWs& ws, int64_t chunk, const Windows* win, Tracer& tr, cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(batch) * T;
  if (n_layers > 0) SAL_TRACED(SAL_KIND_ROPE_TABLE, rope_table_launch(ws.rope, chunk, s));
  for (int i = 0; i < n_layers; ++i) {
    char name[16];
    snprintf(name, sizeof(name), "layer %d", i);
    const NvtxRange layer(name);
    const sal_layer& L = w->layers[i];
    SAL_TRACED(SAL_KIND_LAYERNORM, layernorm_launch(x, M, L.ln1_g, L.ln1_b, ws.h, s));
    QkvOut qo{ws.q, ws.k, ws.v, L.qn_g, L.kn_g, ws.rope, T, chunk};
    SAL_TRACED(SAL_KIND_QKV, gemm_launch(kEpiQkv, ws.h, M, kWidth, L.w_qkv, 3 * kWidth, L.b_qkv, nullptr, &qo, s));
    SAL_TRACED(SAL_KIND_ATTENTION, attention_launch(ws.q, ws.k, ws.v, batch, T, chunk, ws.o, s, win));
    SAL_TRACED(SAL_KIND_OUT_PROJ,
               gemm_launch(SAL_EPI_RESID_F32, ws.o, M, kWidth, L.w_o, kWidth, L.b_o, x, nullptr, s));
    SAL_TRACED(SAL_KIND_LAYERNORM, layernorm_launch(x, M, L.ln2_g, L.ln2_b, ws.h, s));
    SAL_TRACED(SAL_KIND_FFN_UP, gemm_launch(SAL_EPI_GELU_BF16, ws.h, M, kWidth, L.w1, kFfn, L.b1, ws.u, nullptr, s));
    SAL_TRACED(SAL_KIND_FFN_DOWN,
               gemm_launch(SAL_EPI_RESID_F32, ws.u, M, kFfn, L.w2, kWidth, L.b2, x, nullptr, s));
  }
  SAL_TRACED(SAL_KIND_LAYERNORM, layernorm_launch(x, M, w->lnf_g, w->lnf_b, emb, s));
  return SAL_OK;
}
}  // namespace

sal_status sal_encoder_forward_ex(float* x, int batch, int64_t T, const sal_weights* w, int n_layers, void* emb,
                                  void* workspace, size_t ws_bytes, void* stream, const sal_forward_options* opts) {
  const NvtxRange nvtx_("sal_encoder_forward_ex");
  const sal_trace* trace = opts ? opts->trace : nullptr;
  const int64_t chunk = (opts && opts->chunk > 0 && opts->chunk < T) ? opts->chunk : T;
  if (batch < 0 || T < 0 || !w || n_layers < 0 || n_layers > w->n_layers) return SAL_EINVAL;
  if (windowed(opts) && (opts->chunk > 0 || opts->window_context < 0)) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (batch > 6553) return SAL_ESHAPE;  // attention grid.y = 10 * batch
  if (!x || !emb || !aligned16(x) || !aligned16(emb)) return SAL_EINVAL;
  if (!w->lnf_g || !w->lnf_b || !aligned16(w->lnf_g) || !aligned16(w->lnf_b)) return SAL_EINVAL;
  if (n_layers > 0 && !w->layers) return SAL_EINVAL;
  for (int i = 0; i < n_layers; ++i)
    if (!layer_ok(w->layers[i])) return SAL_EINVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SAL_EINVAL;
  if (trace && (trace->kind < 0 || trace->kind >= SAL_KIND_COUNT || trace->n_events < 0 ||
                (trace->n_events > 0 && !trace->events)))
    return SAL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Tracer tr{trace, s};
  if (!windowed(opts)) {
    const EncoderWs ws = encoder_ws_layout(workspace, batch, T);
    if (ws_bytes < ws.bytes) return SAL_EWORKSPACE;
    SAL_TRY(check_device());
    return run_layers(x, batch, T, w, n_layers, emb, ws, chunk, nullptr, tr, s);
  }
  // Serving windows: gather every window into its own slots of a windowed batch, run the
  // layers on it as independent sequences, scatter the core rows back.
  const Windows wn = make_windows(T, opts->window_core, opts->window_context);
  const int64_t bw = static_cast<int64_t>(batch) * wn.count;
  if (bw > 6553) return SAL_ESHAPE;  // attention grid.y = 10 * windows
  if (ws_bytes < windowed_ws_bytes(batch, wn)) return SAL_EWORKSPACE;
  SAL_TRY(check_device());
  const size_t rows = static_cast<size_t>(bw) * static_cast<size_t>(wn.slot);
  char* p = static_cast<char*>(workspace);
  float* xw = reinterpret_cast<float*>(p);
  p += align256(rows * kWidth * 4);
  void* embw = p;
  p += align256(rows * kWidth * 2);
  const EncoderWs ws = encoder_ws_layout(p, static_cast<int>(bw), wn.slot);
  SAL_TRY(window_gather_launch(x, batch, wn, xw, s));
  SAL_TRY(run_layers(xw, static_cast<int>(bw), wn.slot, w, n_layers, embw, ws, wn.slot, &wn, tr, s));
  return window_scatter_launch(embw, xw, batch, wn, emb, x, s);
}

uint64_t sal_launch_count(void) { return g_launches.load(); }

size_t sal_encode_workspace_bytes(int batch, int64_t n_samples) {
  if (batch <= 0 || n_samples < 0) return 0;
  const int64_t F = sal_frame_count(n_samples), T = F / kStack;
  const size_t M = static_cast<size_t>(batch) * static_cast<size_t>(T);
  size_t b = align256(static_cast<size_t>(batch) * n_samples * 4);          // staged wave
  b += align256(static_cast<size_t>(batch) * F * kMels * 4);                // log-mel
  b += align256(M * SAL_STACK_DIM * 2);                                     // stacked
  b += align256(M * kWidth * 4);                                            // x
  b += align256(M * kWidth * 2);                                            // staged emb
  b += T > 0 ? encoder_ws_layout(nullptr, batch, T).bytes : 0;
  return b;
}

sal_status sal_encode(const float* wave, int64_t n_samples, int batch, const sal_weights* w, int n_layers,
                      void* emb, void* workspace, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_("sal_encode");
  if (batch < 0 || n_samples < 0 || !w) return SAL_EINVAL;
  const int64_t F = sal_frame_count(n_samples), T = F / kStack;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (!wave || !emb || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SAL_EINVAL;
  if (ws_bytes < sal_encode_workspace_bytes(batch, n_samples)) return SAL_EWORKSPACE;
  SAL_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t M = static_cast<size_t>(batch) * static_cast<size_t>(T);
  char* p = static_cast<char*>(workspace);
  float* wave_d = reinterpret_cast<float*>(p);
  p += align256(static_cast<size_t>(batch) * n_samples * 4);
  float* logmel = reinterpret_cast<float*>(p);
  p += align256(static_cast<size_t>(batch) * F * kMels * 4);
  void* stacked = p;
  p += align256(M * SAL_STACK_DIM * 2);
  float* x = reinterpret_cast<float*>(p);
  p += align256(M * kWidth * 4);
  void* emb_d = p;
  p += align256(M * kWidth * 2);
  const size_t enc_bytes = encoder_ws_layout(nullptr, batch, T).bytes;

  const bool wave_host = !is_device_ptr(wave);
  const bool emb_host = !is_device_ptr(emb);
  if (wave_host) {
    if (cudaMemcpyAsync(wave_d, wave, static_cast<size_t>(batch) * n_samples * 4, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return SAL_ECUDA;
  } else {
    wave_d = const_cast<float*>(wave);
  }
  SAL_TRY(sal_frontend(wave_d, n_samples, batch, logmel, stacked, stream));
  SAL_TRY(sal_stack_project(stacked, batch, T, w, x, stream));
  SAL_TRY(sal_encoder_forward(x, batch, T, w, n_layers, emb_host ? emb_d : emb, p, enc_bytes, stream));
  if (emb_host &&
      cudaMemcpyAsync(emb, emb_d, M * kWidth * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SAL_ECUDA;
  return SAL_OK;
}

sal_status sal_layernorm(const float* x, int64_t rows, const void* g, const void* b, void* y, void* stream) {
  const NvtxRange nvtx_("sal_layernorm");
  if (rows < 0) return SAL_EINVAL;
  if (rows == 0) return SAL_OK;
  if (!x || !g || !b || !y || !aligned16(x) || !aligned16(g) || !aligned16(b) || !aligned16(y)) return SAL_EINVAL;
  SAL_TRY(check_device());
  return layernorm_launch(x, rows, g, b, y, static_cast<cudaStream_t>(stream));
}

sal_status sal_linear(int epilogue, const void* A, int64_t M, int K, const void* W, int N, const void* bias,
                      void* out, void* stream) {
  const NvtxRange nvtx_("sal_linear");
  if (epilogue < SAL_EPI_STORE_F32 || epilogue > SAL_EPI_RESID_F32 || M < 0) return SAL_EINVAL;
  if (M == 0) return SAL_OK;
  if (!A || !W || !bias || !out || !aligned16(A) || !aligned16(W) || !aligned16(bias) || !aligned16(out))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return gemm_launch(epilogue, A, M, K, W, N, bias, out, nullptr, static_cast<cudaStream_t>(stream));
}

sal_status sal_qkv_rope(const void* h, int batch, int64_t T, const sal_layer* layer, void* q, void* k, void* v,
                        float* rope_cs, void* stream) {
  const NvtxRange nvtx_("sal_qkv_rope");
  if (batch < 0 || T < 0 || !layer) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (!h || !q || !k || !v || !rope_cs || !aligned16(h) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(rope_cs) || !layer->w_qkv || !layer->b_qkv || !layer->qn_g || !layer->kn_g ||
      !aligned16(layer->w_qkv) || !aligned16(layer->b_qkv) || !aligned16(layer->qn_g) || !aligned16(layer->kn_g))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SAL_TRY(rope_table_launch(rope_cs, T, s));
  QkvOut qo{q, k, v, layer->qn_g, layer->kn_g, rope_cs, T, 0};
  return gemm_launch(kEpiQkv, h, static_cast<int64_t>(batch) * T, kWidth, layer->w_qkv, 3 * kWidth,
                     layer->b_qkv, nullptr, &qo, s);
}

sal_status sal_speaker_fuse(const void* H, const float* P, int64_t rows, const void* g, const void* b, void* out,
                            void* stream) {
  const NvtxRange nvtx_("sal_speaker_fuse");
  if (rows < 0) return SAL_EINVAL;
  if (rows == 0) return SAL_OK;
  if (!H || !P || !g || !b || !out || !aligned16(H) || !aligned16(P) || !aligned16(g) || !aligned16(b) ||
      !aligned16(out))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return speaker_fuse_launch(H, P, rows, g, b, out, static_cast<cudaStream_t>(stream));
}

sal_status sal_connector(const void* x, int64_t rows, const void* W, const void* bias, void* out, void* stream) {
  const NvtxRange nvtx_("sal_connector");
  if (rows < 0) return SAL_EINVAL;
  if (rows == 0) return SAL_OK;
  if (!x || !W || !bias || !out || !aligned16(x) || !aligned16(W) || !aligned16(bias) || !aligned16(out))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return gemm_launch(SAL_EPI_STORE_BF16, x, rows, kWidth, W, SAL_LLM_WIDTH, bias, out, nullptr,
                     static_cast<cudaStream_t>(stream));
}

sal_status sal_attention(const void* q, const void* k, const void* v, int batch, int64_t T, void* o,
                         void* stream) {
  const NvtxRange nvtx_("sal_attention");
  return sal_attention_chunked(q, k, v, batch, T, 0, o, stream);
}

sal_status sal_attention_chunked(const void* q, const void* k, const void* v, int batch, int64_t T,
                                 int64_t chunk, void* o, void* stream) {
  const NvtxRange nvtx_("sal_attention_chunked");
  if (batch < 0 || T < 0) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (batch > 6553) return SAL_ESHAPE;  // grid.y = 10 * batch
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return attention_launch(q, k, v, batch, T, chunk, o, static_cast<cudaStream_t>(stream));
}

sal_status sal_attention_heads(const void* q, const void* k, const void* v, int batch, int64_t T, int heads,
                               int head_dim, void* o, void* stream) {
  const NvtxRange nvtx_("sal_attention_heads");
  if (batch < 0 || T < 0 || heads < 0) return SAL_EINVAL;
  if (head_dim != 64 && head_dim != 128) return SAL_ESHAPE;
  if (T > 2 * SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0 || heads == 0) return SAL_OK;
  if (static_cast<int64_t>(batch) * heads > 65535) return SAL_ESHAPE;  // grid.y
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SAL_EINVAL;
  SAL_TRY(check_device());
  return attention_launch_heads(q, k, v, batch, T, 0, heads, head_dim, o, static_cast<cudaStream_t>(stream));
}

sal_status sal_log_softmax(const float* z, int64_t rows, int n, int64_t ld, float* out, void* stream) {
  const NvtxRange nvtx_("sal_log_softmax");
  if (rows < 0 || n < 0 || ld < n) return SAL_EINVAL;
  if (rows == 0 || n == 0) return SAL_OK;
  if (!z || !out) return SAL_EINVAL;
  SAL_TRY(check_device());
  return log_softmax_launch(z, rows, n, ld, out, static_cast<cudaStream_t>(stream));
}

size_t sal_ctc_workspace_bytes(int batch, int64_t T) {
  if (batch <= 0 || T <= 0) return 0;
  return ctc_ws_layout(nullptr, batch, T).bytes;
}

sal_status sal_ctc_adapter(const void* h, int batch, int64_t T, const sal_ctc_weights* w, float* logp,
                           void* workspace, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_("sal_ctc_adapter");
  if (batch < 0 || T < 0 || !w || w->n_layers < 0) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS || batch > 4095) return SAL_ESHAPE;  // attention grid.y = 16 * batch
  if (batch == 0 || T == 0) return SAL_OK;
  if (!h || !logp || !aligned16(h) || !aligned16(logp)) return SAL_EINVAL;
  const void* ps[] = {w->w_up, w->b_up, w->lnf_g, w->lnf_b, w->w_out, w->b_out};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return SAL_EINVAL;
  if (w->n_layers > 0 && !w->layers) return SAL_EINVAL;
  for (int i = 0; i < w->n_layers; ++i)
    if (!layer_ok(w->layers[i])) return SAL_EINVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SAL_EINVAL;
  const CtcWs ws = ctc_ws_layout(workspace, batch, T);
  if (ws_bytes < ws.bytes) return SAL_EWORKSPACE;
  SAL_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  constexpr int W = SAL_CTC_WIDTH, F = SAL_CTC_FFN;
  const int64_t T2 = 2 * T, M2 = static_cast<int64_t>(batch) * T2;
  // the transposed convolution as one GEMM: [B T, 1280] x [2048, 1280]^T -> [B T, 2048],
  // which read row-major is [B 2T, 1024] (tap j of input t lands on row 2t + j); the bias
  // of an output channel is the same for both taps
  if (cudaMemcpyAsync(ws.bias2, w->b_up, W * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(static_cast<char*>(ws.bias2) + W * 2, w->b_up, W * 2, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return SAL_ECUDA;
  SAL_TRY(gemm_launch(SAL_EPI_STORE_F32, h, static_cast<int64_t>(batch) * T, kWidth, w->w_up, 2 * W, ws.bias2,
                      ws.x, nullptr, s));
  if (w->n_layers > 0) SAL_TRY(rope_table_launch(ws.rope, T2, s));
  for (int i = 0; i < w->n_layers; ++i) {
    const sal_layer& L = w->layers[i];
    SAL_TRY(layernorm_launch(ws.x, M2, L.ln1_g, L.ln1_b, ws.h, s, W));
    SAL_TRY(gemm_launch(SAL_EPI_STORE_F32, ws.h, M2, W, L.w_qkv, 3 * W, L.b_qkv, ws.big, nullptr, s));
    SAL_TRY(ctc_qk_norm_rope_launch(static_cast<const float*>(ws.big), M2, T2, L.qn_g, L.kn_g, ws.rope, ws.q, ws.k,
                                    ws.v, s));
    SAL_TRY(attention_launch_heads(ws.q, ws.k, ws.v, batch, T2, 0, SAL_CTC_HEADS, SAL_CTC_HEAD_DIM, ws.o, s));
    SAL_TRY(gemm_launch(SAL_EPI_RESID_F32, ws.o, M2, W, L.w_o, W, L.b_o, ws.x, nullptr, s));
    SAL_TRY(layernorm_launch(ws.x, M2, L.ln2_g, L.ln2_b, ws.h, s, W));
    SAL_TRY(gemm_launch(SAL_EPI_GELU_BF16, ws.h, M2, W, L.w1, F, L.b1, ws.big, nullptr, s));
    SAL_TRY(gemm_launch(SAL_EPI_RESID_F32, ws.big, M2, F, L.w2, W, L.b2, ws.x, nullptr, s));
  }
  SAL_TRY(layernorm_launch(ws.x, M2, w->lnf_g, w->lnf_b, ws.h, s, W));
  // class scores over a width padded to a multiple of 256 (the rows of w_out past 23,863
  // read as zero), then the log-softmax of the 23,863 real ones
  SAL_TRY(gemm_launch(SAL_EPI_STORE_F32, ws.h, M2, W, w->w_out, kCtcClassesPad, w->b_out, ws.big, nullptr, s,
                      SAL_CTC_CLASSES));
  return log_softmax_launch(static_cast<const float*>(ws.big), M2, SAL_CTC_CLASSES, kCtcClassesPad, logp, s);
}

}  // extern "C"
