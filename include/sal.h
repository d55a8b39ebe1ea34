/*
 * sal.h - C-ABI of libsal: the speech front end and ASR encoder of Nemotron 3.5
 * Transcribe on one NVIDIA B200 (sm_100a).
 *
 * What the library computes is fixed by the page "Nemotron 3.5 Transcribe: From
 * Recorded Speech to Dataset Audits" (flozi.net), section "How audio and speakers
 * reach the language model", paragraph on the exported frontend: 16 kHz mono audio,
 * 128 log-mel features from a 25 ms Hann window, a 512-point FFT and a 10 ms hop;
 * eight successive frames stacked and projected to width 1,280; 32 Transformer layers
 * with ten heads, QK normalisation, feed-forward expansion four and rotary position
 * embeddings; 12.5 embeddings per second of audio. Where that paragraph is silent the
 * library takes these readings:
 *   frames F = N < 400 ? 0 : 1 + (N - 400) / 160, positions T = F / 8 (integer division,
 *   no padding, remainder frames dropped); periodic Hann; power spectrum |X_k|^2;
 *   Slaney mel filters over 0..8 kHz with Slaney area normalisation; natural log with a
 *   clamp at 1e-10; frame-major stacking S[t][128 j + m] = M[8 t + j][m]; pre-norm
 *   LayerNorm (eps 1e-5) with a final LayerNorm; RMS QK-norm over head_dim 128
 *   (eps 1e-6, one gain vector for q and one for k, shared by heads) before RoPE;
 *   rotate-half RoPE, base 10000, positions 0..T-1 per clip; full bidirectional
 *   softmax attention scaled by 1/sqrt(128); exact-erf GELU; two-matrix FFN 1280 ->
 *   5120 -> 1280; every linear layer has a bias.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless a call says otherwise. The caller owns every
 *     buffer and keeps it alive until the stream has passed the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls are asynchronous: they validate arguments on the host, enqueue kernels and
 *     return.
 *   - Errors come back as a sal_status code; nothing is thrown across the ABI. A
 *     bounded device-side wait that gave up is reported by sal_last_device_status().
 *   - Every pointer must be 16-byte aligned (SAL_EINVAL otherwise); a clip batch is
 *     `batch` clips of equal length stored back to back.
 *   - bf16 tensors are IEEE bfloat16 bit patterns (uint16_t); parameters are bf16.
 *   - T > 45000 (more than one hour of audio per clip) is SAL_ESHAPE; N < 400 samples
 *     or T = 0 is a valid empty problem that launches nothing and returns SAL_OK.
 *   - The library allocates no device memory (the bounds-checked build excepted: a few
 *     hundred bytes per device for its report). Scratch space is the caller's
 *     `workspace`; sal_encoder_workspace_bytes() gives its size. sal_weights_file_load
 *     allocates pinned host memory for its staging buffers while it runs.
 *   - Thread safety: calls on different streams may run concurrently.
 */
#ifndef SAL_H_
#define SAL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAL_OK = 0,
    SAL_EINVAL = 1,     /* null or misaligned pointer, bad enum value, bad count */
    SAL_ESHAPE = 2,     /* a size outside what the library supports */
    SAL_EWORKSPACE = 3, /* workspace smaller than sal_encoder_workspace_bytes() */
    SAL_ECUDA = 4,      /* a CUDA runtime call or kernel launch failed */
    SAL_ETIMEOUT = 5,   /* a bounded device wait gave up (see sal_last_device_status) */
    SAL_EDEVICE = 6,    /* the current device is not a B200-class sm_100 GPU */
    SAL_EIO = 7         /* a file could not be opened or read */
} sal_status;

#define SAL_N_MELS 128
#define SAL_STACK 8
#define SAL_STACK_DIM 1024
#define SAL_WIDTH 1280
#define SAL_HEADS 10
#define SAL_HEAD_DIM 128
#define SAL_FFN 5120
#define SAL_MAX_POSITIONS 45000

/* Frames of a clip of n_samples samples: n < 400 ? 0 : 1 + (n - 400) / 160.
 * (Exported-frontend paragraph: 25 ms window, 10 ms hop at 16 kHz.) */
int64_t sal_frame_count(int64_t n_samples);

/* Encoder positions: sal_frame_count(n) / 8 (eight stacked frames per position,
 * 12.5 per second). */
int64_t sal_position_count(int64_t n_samples);

/* Static English text for a status code. Never NULL. */
const char* sal_status_string(int status);

/* Per-layer parameters, all DEVICE pointers to bf16 arrays (row-major, [out, in]):
 *   ln1_g, ln1_b [1280]      pre-attention LayerNorm gain and bias
 *   w_qkv [3840, 1280]       rows 0..1279 = q, 1280..2559 = k, 2560..3839 = v; head h of
 *   b_qkv [3840]             each uses rows 128 h .. 128 h + 127 of its block
 *   qn_g, kn_g [128]         RMS QK-norm gains (shared by the ten heads)
 *   w_o [1280, 1280], b_o [1280]     attention output projection
 *   ln2_g, ln2_b [1280]      pre-FFN LayerNorm
 *   w1 [5120, 1280], b1 [5120]       FFN up (GELU)
 *   w2 [1280, 5120], b2 [1280]       FFN down
 * Weight matrices must be 16-byte aligned (they are read by TMA). */
typedef struct {
    const void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *qn_g, *kn_g, *w_o, *b_o;
    const void *ln2_g, *ln2_b, *w1, *b1, *w2, *b2;
} sal_layer;

/* Whole-encoder parameters. w_proj [1280, 1024] and b_proj [1280] are the stack
 * projection; lnf_g, lnf_b [1280] the final LayerNorm; `layers` is a HOST array of
 * n_layers sal_layer records (read during the call only). */
typedef struct {
    const void *w_proj, *b_proj;
    const sal_layer* layers;
    int n_layers;
    const void *lnf_g, *lnf_b;
} sal_weights;

/* ---------------------------------------------------------------------------------
 * Flat weight file: this library's own format for the encoder's parameters (the pages'
 * models ship in a third-party container format, which is not read here). Little-endian:
 *   bytes [0, 8)    magic "SALENCW1"
 *         [8, 12)   version 1            [12, 16) header bytes 256
 *         [16, 20)  dtype 1 (bf16)       [20, 24) width 1280
 *         [24, 28)  heads 10             [28, 32) head dim 128
 *         [32, 36)  FFN width 5120       [36, 40) stack width 1024
 *         [40, 44)  n_layers             [44, 48) alignment 256
 *         [48, 56)  data bytes D (uint64)
 *         [56, 256) zero
 *   then D bytes: every tensor as row-major bf16 starting on a 256-byte boundary (zero
 *   padding), in the order w_proj [1280, 1024], b_proj, lnf_g, lnf_b [1280], then for
 *   each layer ln1_g, ln1_b [1280], w_qkv [3840, 1280], b_qkv [3840], qn_g, kn_g [128],
 *   w_o [1280, 1280], b_o, ln2_g, ln2_b [1280], w1 [5120, 1280], b1 [5120],
 *   w2 [1280, 5120], b2 [1280]. The file is exactly 256 + D bytes long.
 * --------------------------------------------------------------------------------- */

/* Reads the header of the file at `path` (host only, no CUDA call): *n_layers and the
 * device buffer size *device_bytes (= D). Errors: SAL_EINVAL (null argument; bad magic,
 * version, dtype, alignment, reserved bytes, data size or file length), SAL_ESHAPE (sizes
 * other than this library's), SAL_EIO (cannot open or read); outputs 0 on error. */
sal_status sal_weights_file_info(const char* path, int* n_layers, size_t* device_bytes);

/* Loads the file into device_buffer (device memory, 256-byte aligned, >= D bytes: the
 * tensors keep the file's layout) through pinned staging buffers on `stream`, and returns
 * after the copies have completed. Fills layers[0 .. n_layers) (a host array of at least
 * n_layers records, owned by the caller) and *w, whose pointers address device_buffer;
 * w->layers = layers. Errors: as sal_weights_file_info, plus SAL_EINVAL (null buffer or
 * record, misaligned buffer), SAL_EWORKSPACE (buffer_bytes < D or max_layers < n_layers),
 * SAL_ECUDA; on error the contents of device_buffer are unspecified. */
sal_status sal_weights_file_load(const char* path, void* device_buffer, size_t buffer_bytes,
                                 sal_layer* layers, int max_layers, sal_weights* w, void* stream);

/* Front end (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits",
 * section "How audio and speakers reach the language model", exported-frontend
 * paragraph: 16 kHz mono, 128 log-mel features, 25 ms Hann window, 512-point FFT, 10 ms
 * hop, eight stacked frames): wave [batch, n_samples] float32 at 16 kHz ->
 *   logmel  [batch, F, 128] float32, natural-log mel energies (required), and
 *   stacked [batch, T, 1024] bf16, the frame-major stack of the first 8 T frames
 *           (the projection's input; may be NULL).
 * One kernel: framing, Hann window, 512-point real FFT, power, 128 Slaney mel filters,
 * log and the bf16 stacked copy. Errors: SAL_EINVAL (negative sizes, null or misaligned
 * pointer), SAL_ESHAPE (T > 45,000 or batch > 65,535), SAL_EDEVICE, SAL_ECUDA. */
sal_status sal_frontend(const float* wave, int64_t n_samples, int batch, float* logmel,
                        void* stacked, void* stream);

/* Stack projection (same paragraph: the eight stacked frames are projected to width
 * 1,280) x0 = S P^T + p: stacked [batch * T, 1024] bf16 -> x [batch * T, 1280] float32
 * (the encoder's residual stream); w->w_proj [1280, 1024] and w->b_proj [1280] bf16.
 * Errors: SAL_EINVAL, SAL_ESHAPE (T > 45,000), SAL_EDEVICE, SAL_ECUDA. */
sal_status sal_stack_project(const void* stacked, int batch, int64_t T, const sal_weights* w,
                             float* x, void* stream);

/* Bytes of scratch that sal_encoder_forward needs for `batch` clips of T positions. */
size_t sal_encoder_workspace_bytes(int batch, int64_t T);

/* Encoder (same paragraph: 32 Transformer layers at width 1,280 with ten heads, QK
 * normalisation, feed-forward expansion four and rotary position embeddings; the
 * readings above for what it leaves open): x [batch * T, 1280] float32 holds x0 on
 * entry and the residual stream after n_layers layers on return (clobbered); emb
 * [batch * T, 1280] bf16 receives the final LayerNorm of it. n_layers may be
 * 0..w->n_layers. Positions restart at 0 in each clip and attention never crosses clips.
 * `workspace` is device scratch of ws_bytes >= sal_encoder_workspace_bytes(batch, T),
 * 256-byte aligned. Errors: SAL_EINVAL (bad count, null or misaligned pointer, a layer
 * with a null or misaligned parameter), SAL_ESHAPE (T > 45,000 or batch > 6,553),
 * SAL_EWORKSPACE, SAL_EDEVICE, SAL_ECUDA. */
sal_status sal_encoder_forward(float* x, int batch, int64_t T, const sal_weights* w, int n_layers,
                               void* emb, void* workspace, size_t ws_bytes, void* stream);

/* Whole path: wave -> log-mel -> stack -> projection -> n_layers layers -> final LN.
 * `wave` [batch, n_samples] float32 and `emb` [batch, T, 1280] bf16 may each be HOST or
 * DEVICE memory (host buffers are copied through the workspace on `stream`; pinned host
 * memory makes the copies asynchronous). `workspace` must hold
 * sal_encode_workspace_bytes(batch, n_samples) bytes of device memory. */
size_t sal_encode_workspace_bytes(int batch, int64_t n_samples);
sal_status sal_encode(const float* wave, int64_t n_samples, int batch, const sal_weights* w,
                      int n_layers, void* emb, void* workspace, size_t ws_bytes, void* stream);

/* Kinds of kernel launch, for the event trace of sal_encoder_forward_ex. */
typedef enum {
    SAL_KIND_ROPE_TABLE = 0,
    SAL_KIND_LAYERNORM = 1, /* LN1, LN2 and the final LN */
    SAL_KIND_QKV = 2,       /* QKV GEMM + QK-norm + RoPE epilogue */
    SAL_KIND_ATTENTION = 3,
    SAL_KIND_OUT_PROJ = 4,  /* attention output projection + residual */
    SAL_KIND_FFN_UP = 5,    /* FFN up + GELU */
    SAL_KIND_FFN_DOWN = 6,  /* FFN down + residual */
    SAL_KIND_COUNT = 7
} sal_kernel_kind;

/* Event trace: for the i-th launch of kind `kind` inside the call (i < n_events / 2),
 * events[2 i] is recorded on the stream just before it and events[2 i + 1] just after.
 * Events are cudaEvent_t handles created (and recorded at least once) by the caller. */
typedef struct {
    int kind;
    void* const* events;
    int n_events;
} sal_trace;

/* Options of sal_encoder_forward_ex.
 *   chunk: attention and RoPE positions work per chunk of `chunk` positions of each clip
 *          (the last chunk of a clip may be shorter); no attention crosses a chunk border
 *          and positions restart at 0 in every chunk, so every chunk is encoded as an
 *          independent sequence and the outputs come out concatenated in order. This is
 *          the training-time scheme of the page "Nemotron 3.5 Transcribe: From Recorded
 *          Speech to Dataset Audits", section "Local encoder windows, recording-wide
 *          language context" (independent 30-second post-feature chunks = 375 positions).
 *          chunk <= 0 or chunk >= T: attention over the whole clip (sal_encoder_forward).
 *   trace: optional event trace (may be NULL).
 *   window_core, window_context: serving windows (the serving-path paragraph of the same
 *          section: context-extended windows, overlap outputs discarded, core outputs
 *          concatenated; its defaults are SAL_WINDOW_CORE = 500 core positions and
 *          SAL_WINDOW_CONTEXT = 50 context positions on each side). With window_core > 0
 *          each clip is cut into cores of window_core consecutive positions from 0 (the
 *          last may be shorter); window w is its core extended by up to window_context
 *          positions on each side inside the clip. Every window runs the n_layers layers
 *          and the final LayerNorm as an independent sequence (attention inside the
 *          window, positions from 0 at its start), and emb receives each position's
 *          output from the window whose core holds it; x receives, at each position, the
 *          residual stream of that same window. window_core <= 0: no windows. Windows
 *          and chunk > 0 together are SAL_EINVAL; window_context must be >= 0. The
 *          workspace must hold sal_encoder_workspace_bytes_ex(batch, T, opts). */
typedef struct {
    int64_t chunk;
    const sal_trace* trace;
    int64_t window_core;
    int64_t window_context;
} sal_forward_options;

#define SAL_WINDOW_CORE 500
#define SAL_WINDOW_CONTEXT 50

/* Workspace bytes of sal_encoder_forward_ex with these options (opts may be NULL; 0 when
 * batch or T is <= 0). Equal to sal_encoder_workspace_bytes without serving windows. */
size_t sal_encoder_workspace_bytes_ex(int batch, int64_t T, const sal_forward_options* opts);

/* sal_encoder_forward with options (opts may be NULL: whole-clip attention, no trace). */
sal_status sal_encoder_forward_ex(float* x, int batch, int64_t T, const sal_weights* w,
                                  int n_layers, void* emb, void* workspace, size_t ws_bytes,
                                  void* stream, const sal_forward_options* opts);

/* Kernel launches this library has enqueued since the process started (all devices and
 * streams; a launch captured into a CUDA graph counts once, at capture). */
uint64_t sal_launch_count(void);

/* Synchronises `stream` and reports (then clears) the device status word that bounded
 * waits set when they give up: SAL_OK or SAL_ETIMEOUT. */
sal_status sal_last_device_status(void* stream);

/* Upper bound in nanoseconds of every mbarrier wait inside the kernels (default 4e9; 0 is
 * taken as 1). A wait that exceeds it sets the device status word and the kernel winds
 * down: each CTA waits for its own TMA loads and MMAs still in flight, with a fixed bound
 * of 4 s that this limit does not shorten, then frees its tensor memory and returns. */
void sal_set_wait_limit_ns(uint64_t ns);

/* ---------------------------------------------------------------------------------
 * Bounds-checked build. libsal_checked.so is this library compiled with SAL_CHECKED:
 * the same entry points, in which every plain global load and store of every kernel is
 * tested against the byte ranges of the buffers that launch was given (inputs read-only,
 * outputs and workspace writable). An access outside them is not made: it is counted,
 * the lowest such address is kept with the file and line of the access, and the kernel
 * carries on (its outputs are then unspecified). TMA copies are clipped by the hardware
 * to their tensor maps and are not counted. The checked build serialises every launch
 * behind a small host-to-device copy, must be driven from one host thread and one stream
 * at a time, and cannot be captured into a CUDA graph. Both libraries export these calls.
 * --------------------------------------------------------------------------------- */

/* 1 in libsal_checked.so, 0 in libsal.so. */
int sal_checked_build(void);

/* Synchronises the current device and reports, then clears, the accesses the checked
 * build refused on it since the last report: their count, the lowest address, the source
 * file of that access (1 frontend.cu, 2 rowops.cu, 3 gemm.cu, 4 attention.cu, 5 ctc.cu)
 * and line, and the smallest sal_launch_count value before a launch that made one. All
 * outputs are 0 when count is 0. SAL_EINVAL (outputs 0) from libsal.so or on a null
 * pointer; SAL_ECUDA if the device cannot be reached. */
sal_status sal_check_report(uint64_t* count, uint64_t* first_address, int* file, int* line,
                            uint64_t* first_launch);

/* Test hook of the checked build (no effect in libsal.so): every writable range declared
 * from now on is taken `bytes` shorter at its end (0 restores the exact ranges), so the
 * stores a kernel makes there are refused and reported instead of made. */
void sal_check_shrink_writable(uint64_t bytes);

/* ---------------------------------------------------------------------------------
 * Single-step entry points (the stages sal_encoder_forward chains; for tests and
 * per-kernel timing). Layouts as above; M = batch * T rows.
 * --------------------------------------------------------------------------------- */

/* y = LayerNorm(x) * g + b over rows of 1280 (eps 1e-5): x float32 -> y bf16. */
sal_status sal_layernorm(const float* x, int64_t rows, const void* g, const void* b, void* y,
                         void* stream);

typedef enum {
    SAL_EPI_STORE_F32 = 0,  /* out f32 [M, N] = A W^T + bias                 */
    SAL_EPI_STORE_BF16 = 1, /* out bf16 [M, N] = A W^T + bias                */
    SAL_EPI_GELU_BF16 = 2,  /* out bf16 [M, N] = GELU_erf(A W^T + bias)      */
    SAL_EPI_RESID_F32 = 3   /* out f32 [M, N] += A W^T + bias (residual add) */
} sal_epilogue;

/* Linear layer on the tensor cores: A [M, K] bf16 (row-major), W [N, K] bf16, bias [N]
 * bf16. K and N must be multiples of 64 (SAL_ESHAPE otherwise). */
sal_status sal_linear(int epilogue, const void* A, int64_t M, int K, const void* W, int N,
                      const void* bias, void* out, void* stream);

/* QKV projection with the QK-norm and RoPE epilogue: h [batch * T, 1280] bf16 ->
 * q, k, v [batch, 10, T, 128] bf16 (q and k RMS-normalised with qn_g / kn_g, then
 * rotated by RoPE at position t of their clip). rope_cs is device scratch of
 * 2 * T * 64 float32 that the call fills with the rotation table. */
sal_status sal_qkv_rope(const void* h, int batch, int64_t T, const sal_layer* layer, void* q,
                        void* k, void* v, float* rope_cs, void* stream);

/* Bidirectional attention per (clip, head): q, k, v [batch, 10, T, 128] bf16 ->
 * o [batch * T, 1280] bf16, o[b*T + t][128 h + d] = softmax(q k^T / sqrt(128)) v. */
sal_status sal_attention(const void* q, const void* k, const void* v, int batch, int64_t T,
                         void* o, void* stream);

/* sal_attention restricted to chunks of `chunk` positions of each clip (block-diagonal:
 * row t attends to the keys of its own chunk only; chunk <= 0 or >= T: whole clip). */
sal_status sal_attention_chunked(const void* q, const void* k, const void* v, int batch, int64_t T,
                                 int64_t chunk, void* o, void* stream);

/* ---------------------------------------------------------------------------------
 * After the encoder (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset
 * Audits", section "How audio and speakers reach the language model"): speaker-activity
 * fusion into the encoder states, then the identity connector to the language width.
 * --------------------------------------------------------------------------------- */

#define SAL_SPEAKER_SLOTS 8
#define SAL_LLM_WIDTH 2688

/* out = H + LN_8(P > 0.5) K, per position: P [rows, 8] float32 slot activities already on
 * the 80 ms ASR grid; the indicators P > 0.5 are normalised over the 8 slots (LayerNorm,
 * eps 1e-5, gain g [8] and bias b [8] bf16) and mapped to width 1280 by the fixed
 * sinusoidal speaker kernel K[s, 2i] = sin(s w_i), K[s, 2i+1] = cos(s w_i),
 * w_i = 10000^(-2i/1280), scale 1. H and out are [rows, 1280] bf16 (may alias). The page
 * states the steps but its equation is missing from the text; this is the reading. */
sal_status sal_speaker_fuse(const void* H, const float* P, int64_t rows, const void* g, const void* b,
                            void* out, void* stream);

/* The identity connector: out [rows, 2688] bf16 = x [rows, 1280] bf16 W^T + bias, with
 * W [2688, 1280] and bias [2688] bf16 (one learned linear projection, no downsampling). */
sal_status sal_connector(const void* x, int64_t rows, const void* W, const void* bias, void* out,
                         void* stream);

/* sal_qkv_rope without a caller-supplied scratch buffer, for callers that cannot allocate
 * device memory when they run this step (a real-time audio callback or serving loop that
 * must not stall or fail on cudaMalloc, a plugin host that forbids device allocations
 * after start-up, a framework that owns the memory pool). The pages describe nothing like
 * it: it is a deployment convenience with no counterpart in the method.
 * Same inputs and outputs as sal_qkv_rope; the rotation table lives in a fixed 2 MiB
 * array inside the library (held by every GPU that loads it, until exit), so T must be
 * at most 4096 (SAL_ESHAPE otherwise). No allocation of any kind. Every call shares that
 * array and fully rewrites the part it reads; calls whose kernels overlap on the GPU
 * (e.g. on two streams) race on it. The first call on a device looks up the array's
 * address; make it before any stream capture. */
sal_status sal_qkv_rope_noalloc(const void* h, int batch, int64_t T, const sal_layer* layer,
                                void* q, void* k, void* v, void* stream);

/* ---------------------------------------------------------------------------------
 * CTC timestamp adapter (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset
 * Audits", section "Use alignment and audio questions as supporting evidence"): about 50M
 * parameters on the unfused ASR states (width 1,280); a stride-two transposed
 * convolution from the 80 ms to a 40 ms grid, two Transformer layers with 16 heads, and a
 * projection to a 23,862-token vocabulary plus the CTC blank. The page gives no widths.
 * This library reads the adapter as:
 *   - width 1,024 (16 heads of 64, FFN 4,096): the width that gives about 50M parameters
 *     with the encoder's layer recipe (pre-norm LN, RMS QK-norm, RoPE over 40 ms steps,
 *     exact-erf GELU);
 *   - a transposed-convolution kernel of 2 (each 80 ms state gives two 40 ms states);
 *   - a final LayerNorm before the projection;
 *   - log-softmax over the 23,863 classes (blank last) as the output.
 * --------------------------------------------------------------------------------- */

#define SAL_CTC_WIDTH 1024
#define SAL_CTC_HEADS 16
#define SAL_CTC_HEAD_DIM 64
#define SAL_CTC_FFN 4096
#define SAL_CTC_LAYERS 2
#define SAL_CTC_CLASSES 23863

/* Device pointers, bf16, 16-byte aligned (the layer array itself is host memory). */
typedef struct {
  const void* w_up;         /* [2 * 1024, 1280]: row 1024 j + c is tap j of output channel c */
  const void* b_up;         /* [1024], shared by both taps */
  const sal_layer* layers;  /* n_layers layers at width 1024: ln* [1024], w_qkv [3072, 1024], b_qkv [3072],
                               qn_g / kn_g [64], w_o [1024, 1024], w1 [4096, 1024], b1 [4096],
                               w2 [1024, 4096], other biases [1024] */
  int n_layers;             /* SAL_CTC_LAYERS */
  const void *lnf_g, *lnf_b;  /* [1024] */
  const void *w_out, *b_out;  /* [23863, 1024], [23863] */
} sal_ctc_weights;

/* Workspace bytes for sal_ctc_adapter over batch clips of T encoder positions (0 when
 * either is <= 0). About 110 KB per 40 ms position, most of it the fp32 class scores. */
size_t sal_ctc_workspace_bytes(int batch, int64_t T);

/* Frame log-probabilities of the adapter. h: [batch * T, 1280] bf16, the unfused encoder
 * states (sal_encoder_forward's output); logp: [batch * 2T, 23863] float32, row
 * 2 T b + u holding 40 ms position u of clip b. workspace: >= sal_ctc_workspace_bytes,
 * 256-byte aligned, owned by the caller. Errors: SAL_EINVAL (null or misaligned pointer,
 * n_layers out of range), SAL_ESHAPE (T > 45,000 or batch > 4095), SAL_EWORKSPACE. */
sal_status sal_ctc_adapter(const void* h, int batch, int64_t T, const sal_ctc_weights* w, float* logp,
                           void* workspace, size_t ws_bytes, void* stream);

/* Attention for heads of width 64 or 128 (the encoder: 10 x 128; the CTC adapter:
 * 16 x 64): q, k, v [batch, heads, T, head_dim] bf16; o [batch, T, heads * head_dim] bf16.
 * SAL_ESHAPE for another head width, T > 90,000 or batch * heads > 65535. */
sal_status sal_attention_heads(const void* q, const void* k, const void* v, int batch, int64_t T, int heads,
                               int head_dim, void* o, void* stream);

/* The kernels sal_attention would launch for 128-wide heads on a GPU with `sms` SMs:
 * *pairs query-tile pairs (of 128 rows) per (clip, head) go to the two-tile kernel, out of
 * *query_tiles tiles. P is the
 * count among none, all and the largest filling whole waves whose greedy schedule ends
 * first (a two-tile CTA counted as 1.35 one-tile CTAs); splits are tried from 16 query
 * tiles up. The tiles past the pairs go to split-mode CTAs of the same launch (a tile's keys
 * split between the CTA's two warpgroups), counted as 0.75 one-tile CTAs; with no pairs
 * the one-tile kernel takes every tile. For head_dim 64 every pair goes to the two-tile
 * kernel and an odd last tile to a split-mode CTA. SAL_ATTN_PP=0/1 in the environment
 * forces none/all; SAL_ATTN_PAIRS=n forces n pairs and split mode for the rest. Host
 * arithmetic only: no device is needed. */
sal_status sal_attention_plan(int batch, int64_t T, int heads, int head_dim, int sms, int* pairs, int* query_tiles);
/* (sal_attention_plan returns SAL_ESHAPE for T > 90,000, as sal_attention_heads does.) */

/* Test hook for the bounded waits (no counterpart on the pages). One launch of the
 * attention kernel `kernel` (1: one query tile per CTA; 2: two query tiles per CTA) over
 * 10 heads of width 128, as sal_attention, except that every CTA's producer never issues
 * the loads of its key/value tile number `tile` (counted from the CTA's first key tile).
 * The wait for that tile gives up after the limit of sal_set_wait_limit_ns, the kernel
 * winds down, and sal_last_device_status then reports SAL_ETIMEOUT; o is unspecified.
 * A CTA with `tile` or fewer key tiles is unaffected. Errors: SAL_EINVAL (kernel not 1 or
 * 2, tile < 0, null or misaligned pointer), SAL_ESHAPE as sal_attention, SAL_EDEVICE
 * (not an sm_100 GPU, or kernel 2 unavailable on it). */
sal_status sal_attention_withhold(const void* q, const void* k, const void* v, int batch, int64_t T, int kernel,
                                  int tile, void* o, void* stream);

/* Row log-softmax (the adapter's last step): out[r, i] = z[r, i] - log sum_j exp z[r, j]
 * for i < n. z rows are ld floats apart (ld >= n), out rows n floats apart; float32. */
sal_status sal_log_softmax(const float* z, int64_t rows, int n, int64_t ld, float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAL_H_ */
