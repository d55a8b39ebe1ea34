// Tensor-core linear layers of the encoder: C = A W^T (+ bias, + fused epilogue), with
// A [M, K] bf16 activations and W [N, K] bf16 weights, both K-contiguous.
//
// Used for the stack projection (1024 -> 1280), the QKV projection (1280 -> 3840), the
// attention output projection (1280 -> 1280) and the two FFN matrices (1280 -> 5120 ->
// 1280) of every layer (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset
// Audits", section "How audio and speakers reach the language model": width 1,280,
// ten heads, feed-forward expansion four).
//
// Design (sm_100a):
//   * persistent CTAs, one per SM, walking 128 x BN output tiles (optionally split along K);
//   * warp 0 issues TMA loads of 128 x 64 A and BN x 64 W tiles (128-byte swizzle) into a
//     multi-stage shared-memory ring guarded by mbarriers;
//   * warp 1 (one thread) issues tcgen05.mma (M = 128, N = BN, K = 16) into one of two
//     TMEM accumulators, so the epilogue of tile i overlaps the main loop of tile i + 1;
//   * warps 2-5 (one TMEM lane = one output row per thread) read the accumulator with
//     tcgen05.ld and apply the fused epilogue: bias; bias + exact-erf GELU; bias +
//     residual add into the fp32 stream; or, for QKV, bias + per-head RMS QK-norm + RoPE
//     with the q / k / v heads scattered to [batch, head, T, 128].
// Every mbarrier wait is bounded; a wait that gives up flags the device status word
// and the CTA winds down (waiting, bounded, for its own TMA loads and MMAs in flight)
// before it frees its TMEM and exits.
#define SAL_CK_FILE 3
#include <cuda_bf16.h>
#include <math.h>

#include <cstdlib>
#include <mutex>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

struct GemmArgs {
  int64_t M;
  int N, K, splits;
  int n_valid;  // rows of W and entries of the bias that exist (<= N; the rest read as 0)
  const __nv_bfloat16* bias;
  void* out;
  // QKV epilogue
  __nv_bfloat16 *q, *k, *v;
  const __nv_bfloat16 *qn_g, *kn_g;
  const float* rope_cs;  // [2][rope_rows][64]: cos rows, then sin rows
  int64_t T;
  int64_t chunk;         // positions restart every `chunk` positions of a clip
  int64_t rope_rows;     // rows of the table = min(T, chunk)
  uint64_t limit_ns;
  unsigned int* status;
};

// PAIR: a cluster of two CTAs computes a 256 x BN tile with tcgen05.mma.cta_group::2. Each
// CTA loads its own 128 rows of A and its own BN / 2 rows of W (no multicast), holds its 128
// rows of the accumulator in its TMEM and runs the epilogue on them; the even CTA issues
// the MMAs. Per SM this reads half of the W tile of the one-CTA form for the same MMA work.
template <int BN, int EPI, bool PAIR = false>
struct Cfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr bool QKV = EPI == kEpiQkv;
  static constexpr bool F32_OUT = EPI == SAL_EPI_STORE_F32 || EPI == SAL_EPI_RESID_F32;
  // epilogue shared memory: QKV stages a whole head per warp (32 rows x 128 fp32); the
  // other kinds stage 128-byte-wide output boxes for TMA, two per warp
  static constexpr int CW = F32_OUT ? 32 : 64;  // output columns per 128-byte box row
  static constexpr int EPW = 4;  // epilogue warps, one per TMEM lane quarter
  static constexpr int THREADS = 64 + 32 * EPW;
  static constexpr int SCR_BYTES = QKV ? 4 * 32 * 128 * 4 + 4 * 32 * 4 : 4 * 2 * 4096;
  static constexpr int BNL = PAIR ? BN / 2 : BN;  // rows of W this CTA loads per tile
  static constexpr int STAGES = PAIR ? (QKV ? 5 : 6)
                                     : (QKV ? (BN == 256 ? 3 : 4) : (BN == 256 ? 4 : (BN == 128 ? 6 : 8)));
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BNL * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + SCR_BYTES + 256;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!PAIR || BN == 256, "CTA pairs use 256-wide tiles");
};

// Exact-erf GELU 0.5 x (1 + erf(x / sqrt 2)), with erf from the rational approximation of
// Abramowitz and Stegun, Handbook of Mathematical Functions, formula 7.1.26 (after
// Hastings): for z >= 0, erf z = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) e^(-z^2),
// t = 1 / (1 + p z), |error| <= 1.5e-7; odd in z. Evaluated in fp32 (reciprocal and
// exponential on the SFU) it stays within 6e-7 of erf over the whole line, branch-free;
// the GELU output is then rounded to bf16 (2^-9 relative).
__device__ __forceinline__ float gelu_erf(float x) {
  const float z = fabsf(x) * 0.70710678118654752f;
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, z, 1.0f)));
  float q = fmaf(1.061405429f, t, -1.453152027f);
  q = fmaf(q, t, 1.421413741f);
  q = fmaf(q, t, -0.284496736f);
  q = fmaf(q, t, 0.254829592f);
  q *= t;
  const float e = fast_exp2(-1.4426950408889634f * z * z);
  const float erf_z = copysignf(fmaf(-q, e, 1.0f), x);  // erf(x / sqrt 2)
  const float h = 0.5f * x;
  return fmaf(h, erf_z, h);
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, int i) { return __bfloat162float(*SAL_CK_LD(p + i, 2)); }

// Warp scratch: 32 rows x W fp32 columns, row r at r * W floats; the 16-byte chunk j of a
// row sits at chunk position (j & ~7) | ((j ^ r) & 7), so a thread-per-row store of 8
// consecutive chunks and a row read by the whole warp are both free of bank conflicts.
template <int W>
__device__ __forceinline__ int scr_chunk(int r, int j) {
  return r * (W / 4) + ((j & ~7) | ((j ^ r) & 7));
}

// Thread `lane` (= row) copies 32 accumulator columns [32 cc, 32 cc + 32) of its TMEM lane
// into the warp scratch.
template <int W>
__device__ __forceinline__ void stage_chunk(float4* scr, int lane, int cc, const uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    scr[scr_chunk<W>(lane, cc * 8 + i)] =
        make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]), __uint_as_float(r[4 * i + 2]),
                    __uint_as_float(r[4 * i + 3]));
}

template <int BN, int EPI, bool PAIR>
__global__ void __launch_bounds__(Cfg<BN, EPI, PAIR>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
  using C = Cfg<BN, EPI, PAIR>;
  extern __shared__ unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  float4* scratch = reinterpret_cast<float4*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scratch) + C::SCR_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* bye = drain + 1;  // pairs: the peer has finished every access to this CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bye + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // pairs: this CTA's rank; the even CTA (rank 0) issues the MMAs and owns the barriers
  // that both CTAs' loads and epilogues report to
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      // one arrival per epilogue thread; pairs: one per epilogue warp of both CTAs
      mbar_init(&tempty[a], PAIR ? 2 * C::EPW : 32 * C::EPW);
    }
    mbar_init(drain, 1);
    mbar_init(bye, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if constexpr (!C::QKV) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // both CTAs' barriers are initialised before either CTA touches the other's
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  }
  tc_fence_after();
  // Programmatic dependent launch: the roles that read or write what earlier kernels
  // produce (the A loads, the epilogue) wait for them below; the weight loads of the
  // first tile and the MMA warp (shared and tensor memory only) do not.
  pdl_trigger();
  const uint32_t tmem_base = *tmem_slot;
  const WaitGuard guard{abort_flag, args.limit_ns, args.status};

  // a work unit is one (row block, column tile, K split); a row block is 128 rows, or
  // 256 for a CTA pair (this CTA's rows are the half given by its rank)
  const int ROWS = PAIR ? 2 * C::BM : C::BM;
  const int num_m = static_cast<int>((args.M + ROWS - 1) / ROWS);
  const int num_n = args.N / BN;
  const int kb_per = (args.K / C::BK) / args.splits;
  const int num_tiles = num_m * num_n * args.splits;
  const int first_tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // the producer's record of the stages it loaded and their phases (for the wind-down)
  uint32_t issued = 0, issued_par = 0;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      // A stage's barrier expects the bytes of every load into it: this CTA's, or for a
      // pair both CTAs' (only the even CTA's barrier is armed; the odd CTA's loads report
      // to it).
      auto expect = [&](int st) {
        if (!PAIR || rank == 0) mbar_arrive_expect_tx(&full[st], PAIR ? 2 * C::STAGE_BYTES : C::STAGE_BYTES);
      };
      auto load_a = [&](int st, int kb, int mrow) {
        if constexpr (PAIR)
          tma_load_2d_pair(sA + st * C::A_BYTES, &tmA, mapa_shared(smem_u32(&full[st]), 0), kb * C::BK, mrow);
        else
          tma_load_2d(sA + st * C::A_BYTES, &tmA, &full[st], kb * C::BK, mrow);
      };
      auto load_b = [&](int st, int kb, int n) {
        if constexpr (PAIR)
          tma_load_2d_pair(sB + st * C::B_BYTES, &tmB, mapa_shared(smem_u32(&full[st]), 0), kb * C::BK,
                           n * BN + static_cast<int>(rank) * C::BNL);
        else
          tma_load_2d(sB + st * C::B_BYTES, &tmB, &full[st], kb * C::BK, n * BN);
      };
      // The weights do not depend on the previous kernel: the W tiles of the first stages
      // of this CTA's first tile go out before the wait (the stages start empty), their
      // A tiles after it, completing the same barriers.
      const int tile0 = first_tile;
      int pre = 0;
      if (tile0 < num_tiles) {
        const int sp0 = tile0 % args.splits, n0 = (tile0 / args.splits) % num_n;
        pre = kb_per < C::STAGES ? kb_per : C::STAGES;
        for (int i = 0; i < pre; ++i) {
          expect(i);
          load_b(i, sp0 * kb_per + i, n0);
        }
      }
      pdl_wait();
      for (int tile = first_tile; tile < num_tiles; tile += tile_step) {
        const int sp = tile % args.splits;
        const int rest = tile / args.splits;
        const int n = rest % num_n, m = rest / num_n;
        const int mrow = PAIR ? (2 * m + static_cast<int>(rank)) * C::BM : m * C::BM;
        for (int i = 0; i < kb_per; ++i) {
          const int kb = sp * kb_per + i;
          if (tile == tile0 && i < pre) {  // stage i already expects its bytes; W is in flight
            load_a(stage, kb, mrow);
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1, guard)) goto producer_done;
            expect(stage);
            load_a(stage, kb, mrow);
            load_b(stage, kb, n);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {  // pairs: the even CTA issues for both
      constexpr uint32_t IDESC = idesc_bf16(PAIR ? 256 : 128, BN, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool any_mma = false;
      for (int tile = first_tile; tile < num_tiles; tile += tile_step) {
        if (!mbar_wait<PAIR>(&tempty[acc], acc_phase ^ 1, guard)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        bool ok = true;
        for (int i = 0; i < kb_per; ++i) {
          if (!mbar_wait(&full[stage], phase, guard)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            if constexpr (PAIR)
              umma_ss_pair(d, sdesc_kmajor_sw128(a0 + kk * 32), sdesc_kmajor_sw128(b0 + kk * 32), IDESC,
                           (i | kk) != 0);
            else
              umma_ss(d, sdesc_kmajor_sw128(a0 + kk * 32), sdesc_kmajor_sw128(b0 + kk * 32), IDESC,
                      (i | kk) != 0);
          }
          if constexpr (PAIR)
            umma_commit_pair(&empty[stage]);  // frees the stage in both CTAs
          else
            umma_commit(&empty[stage]);
          any_mma = true;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (PAIR)
          umma_commit_pair(&tfull[acc]);  // both CTAs' epilogues
        else
          umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (*abort_flag && any_mma) {  // one more commit covers every MMA issued so far
        if constexpr (PAIR)
          umma_commit_pair(drain);
        else
          umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    // Each warp owns TMEM lanes (= tile rows) 32 q .. 32 q + 31, one row per thread.
    pdl_wait();  // outputs (and the RoPE table) are shared with earlier kernels
    const int quarter = warp & 3;
    uint32_t acc = 0, acc_phase = 0;
    // This warp has read its lanes of accumulator a: every thread arrives (one CTA), or
    // for a pair one lane per warp arrives on the even CTA's barrier.
    auto release_acc = [&](uint32_t a) {
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[a]), 0));
      } else {
        mbar_arrive(&tempty[a]);
      }
    };
    if constexpr (C::QKV) {
      // Per head: stage the 32 x 128 accumulator block in shared memory, then walk its
      // rows with the lanes across the columns (lane l holds columns 4l .. 4l + 3): the
      // RMS norm is a warp sum, the RoPE partner column i +- 64 sits 16 lanes away, and
      // cos / sin of t * theta_i advance row by row by one rotation through theta_i, so
      // the loop issues no global load besides one table row per 32-row block.
      float4* scr = scratch + (warp - 2) * (32 * 128 / 4);
      float* inv_row = reinterpret_cast<float*>(scratch + 4 * (32 * 128 / 4)) + (warp - 2) * 32;
      const int q4 = lane & 15;
      const float sg = lane >= 16 ? 1.f : -1.f;  // i < 64: a c - b s;  i >= 64: b c + a s
      float4 c1 = make_float4(1.f, 1.f, 1.f, 1.f), s1 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (args.rope_rows > 1) {  // table row 1 holds cos / sin of theta_i itself
        c1 = __ldg(SAL_CK_LD(reinterpret_cast<const float4*>(args.rope_cs + 64) + q4, 16));
        s1 = __ldg(SAL_CK_LD(reinterpret_cast<const float4*>(args.rope_cs + (args.rope_rows + 1) * 64) + q4, 16));
      }
      for (int tile = first_tile; tile < num_tiles; tile += tile_step) {
        const int rest = tile / args.splits;
        const int n = rest % num_n, m = PAIR ? 2 * (rest / num_n) + static_cast<int>(rank) : rest / num_n;
        if (!mbar_wait_warp(&tfull[acc], acc_phase, guard)) break;
        tc_fence_after();
        const int64_t row0 = static_cast<int64_t>(m) * C::BM + quarter * 32;
        const int nrows = static_cast<int>(args.M - row0 < 32 ? (args.M - row0 > 0 ? args.M - row0 : 0) : 32);
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
#pragma unroll 1
        for (int hb = 0; hb < BN / 128; ++hb) {
          const int col0 = n * BN + hb * 128;
          const int sec = col0 / kWidth;
          const int head = (col0 % kWidth) / kHeadDim;
          // thread-per-row: add the bias, stage the row, and (q, k) take its RMS factor
          float ss = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t r[32];
            tmem_ld32(taddr + hb * 128 + cc * 32, r);
            tmem_wait_ld();
            const uint4* b8 = reinterpret_cast<const uint4*>(args.bias + col0 + cc * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 bb = __ldg(SAL_CK_LD(b8 + j, 16));
              const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(r[8 * j + 2 * e]) + bf16_lo(bw[e]);
                const float hi = __uint_as_float(r[8 * j + 2 * e + 1]) + bf16_hi(bw[e]);
                ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                r[8 * j + 2 * e] = __float_as_uint(lo);
                r[8 * j + 2 * e + 1] = __float_as_uint(hi);
              }
            }
            stage_chunk<128>(scr, lane, cc, r);
          }
          if (hb == BN / 128 - 1) release_acc(acc);  // accumulator no longer needed
          inv_row[lane] = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + 1e-6f);
          __syncwarp();
          __nv_bfloat16* base = sec == 0 ? args.q : (sec == 1 ? args.k : args.v);
          if (nrows > 0) {
            int64_t b = row0 / args.T, t = row0 - b * args.T;
            int64_t pos = t % args.chunk;  // RoPE position: restarts at every chunk
            __nv_bfloat16* dst = base + ((b * kHeads + head) * args.T + t) * kHeadDim;
            if (sec == 2) {
#pragma unroll 4
              for (int r = 0; r < nrows; ++r) {
                const float4 v = scr[scr_chunk<128>(r, lane)];
                uint2 o;
                o.x = pack_bf16x2(v.x, v.y);
                o.y = pack_bf16x2(v.z, v.w);
                *SAL_CK_ST(reinterpret_cast<uint2*>(dst) + lane, 8) = o;
                dst += kHeadDim;
                if (++t == args.T) {  // next clip
                  t = 0;
                  ++b;
                  dst = base + (b * kHeads + head) * args.T * kHeadDim;
                }
              }
            } else {
              const __nv_bfloat16* gp = (sec == 0 ? args.qn_g : args.kn_g) + 4 * lane;
              const float4 g4 = make_float4(bf16_at(gp, 0), bf16_at(gp, 1), bf16_at(gp, 2), bf16_at(gp, 3));
              float4 c = __ldg(SAL_CK_LD(reinterpret_cast<const float4*>(args.rope_cs + pos * 64) + q4, 16));
              float4 sn =
                  __ldg(SAL_CK_LD(reinterpret_cast<const float4*>(args.rope_cs + (args.rope_rows + pos) * 64) + q4, 16));
#pragma unroll 4
              for (int r = 0; r < nrows; ++r) {
                float4 v = scr[scr_chunk<128>(r, lane)];
                const float inv = inv_row[r];
                v.x *= inv * g4.x; v.y *= inv * g4.y; v.z *= inv * g4.z; v.w *= inv * g4.w;
                float4 p;  // the partner half: column i +- 64
                p.x = __shfl_xor_sync(0xffffffffu, v.x, 16);
                p.y = __shfl_xor_sync(0xffffffffu, v.y, 16);
                p.z = __shfl_xor_sync(0xffffffffu, v.z, 16);
                p.w = __shfl_xor_sync(0xffffffffu, v.w, 16);
                uint2 o;
                o.x = pack_bf16x2(fmaf(sg * p.x, sn.x, v.x * c.x), fmaf(sg * p.y, sn.y, v.y * c.y));
                o.y = pack_bf16x2(fmaf(sg * p.z, sn.z, v.z * c.z), fmaf(sg * p.w, sn.w, v.w * c.w));
                *SAL_CK_ST(reinterpret_cast<uint2*>(dst) + lane, 8) = o;
                dst += kHeadDim;
                ++pos;
                if (++t == args.T) {  // next clip: positions restart at 0
                  t = 0;
                  pos = 0;
                  ++b;
                  dst = base + (b * kHeads + head) * args.T * kHeadDim;
                }
                if (pos == args.chunk || pos == 0) {  // a new clip or chunk starts at position 0
                  pos = 0;
                  c = make_float4(1.f, 1.f, 1.f, 1.f);
                  sn = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {  // rotate by theta_i: angle (pos + 1) theta_i
                  const float4 cc = c;
                  c.x = fmaf(cc.x, c1.x, -sn.x * s1.x); sn.x = fmaf(sn.x, c1.x, cc.x * s1.x);
                  c.y = fmaf(cc.y, c1.y, -sn.y * s1.y); sn.y = fmaf(sn.y, c1.y, cc.y * s1.y);
                  c.z = fmaf(cc.z, c1.z, -sn.z * s1.z); sn.z = fmaf(sn.z, c1.z, cc.z * s1.z);
                  c.w = fmaf(cc.w, c1.w, -sn.w * s1.w); sn.w = fmaf(sn.w, c1.w, cc.w * s1.w);
                }
              }
            }
          }
          __syncwarp();
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    } else {
      // Per 128-byte-wide column chunk: each thread converts its row's values and writes
      // them into a 128B-swizzled 32-row box in shared memory (two boxes per warp, used in
      // turn); one lane then issues a TMA store of the box, or a TMA reduce-add into the
      // fp32 residual stream, while the warp moves on to the next chunk.
      uint8_t* stg = reinterpret_cast<uint8_t*>(scratch) + (warp - 2) * 8192;
      uint32_t kbuf = 0;
      for (int tile = first_tile; tile < num_tiles; tile += tile_step) {
        const int sp = tile % args.splits;
        const int rest = tile / args.splits;
        const int n = rest % num_n, m = PAIR ? 2 * (rest / num_n) + static_cast<int>(rank) : rest / num_n;
        if (!mbar_wait_warp(&tfull[acc], acc_phase, guard)) break;
        tc_fence_after();
        const int y = m * C::BM + quarter * 32;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += C::CW) {
          uint8_t* buf = stg + (kbuf & 1) * 4096;
          if (kbuf >= 2) {  // the store issued from this box two chunks ago has read it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          uint32_t r[C::CW];
          tmem_ld32(taddr + c, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          if constexpr (C::CW == 64) tmem_ld32(taddr + c + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
          if (c + C::CW == BN) release_acc(acc);  // accumulator no longer needed
          const int col0 = n * BN + c;
          const bool add_bias = !(EPI == SAL_EPI_RESID_F32 && sp != 0);
          const uint4* bias8 = reinterpret_cast<const uint4*>(args.bias + col0);
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // 16-byte chunk j of this row
            uint4 word;
            if constexpr (C::F32_OUT) {
              float v[4];
              uint2 bb = make_uint2(0, 0);
              if (add_bias) {
                const int cb = col0 + 4 * j;
                if (cb + 4 <= args.n_valid) {
                  bb = __ldg(SAL_CK_LD(reinterpret_cast<const uint2*>(bias8) + j, 8));
                } else {  // the last, partial bias chunk
                  const uint16_t* bu = reinterpret_cast<const uint16_t*>(args.bias);
                  uint32_t e[4];
#pragma unroll
                  for (int q = 0; q < 4; ++q) e[q] = cb + q < args.n_valid ? *SAL_CK_LD(bu + cb + q, 2) : 0u;
                  bb = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
                }
              }
              v[0] = __uint_as_float(r[4 * j + 0]) + bf16_lo(bb.x);
              v[1] = __uint_as_float(r[4 * j + 1]) + bf16_hi(bb.x);
              v[2] = __uint_as_float(r[4 * j + 2]) + bf16_lo(bb.y);
              v[3] = __uint_as_float(r[4 * j + 3]) + bf16_hi(bb.y);
              word = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                                __float_as_uint(v[3]));
            } else {
              uint4 bb;
              const int cb = col0 + 8 * j;
              if (cb + 8 <= args.n_valid) {
                bb = __ldg(SAL_CK_LD(bias8 + j, 16));
              } else {  // the last, partial bias chunk
                const uint16_t* bu = reinterpret_cast<const uint16_t*>(args.bias);
                uint32_t e[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) e[q] = cb + q < args.n_valid ? *SAL_CK_LD(bu + cb + q, 2) : 0u;
                bb = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
              }
              const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float lo = __uint_as_float(r[8 * j + 2 * e]) + bf16_lo(bw[e]);
                float hi = __uint_as_float(r[8 * j + 2 * e + 1]) + bf16_hi(bw[e]);
                if constexpr (EPI == SAL_EPI_GELU_BF16) {
                  lo = gelu_erf(lo);
                  hi = gelu_erf(hi);
                }
                o[e] = pack_bf16x2(lo, hi);
              }
              word = make_uint4(o[0], o[1], o[2], o[3]);
            }
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = word;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if constexpr (EPI == SAL_EPI_RESID_F32)
              tma_reduce_add_2d(&tmC, buf, col0, y);
            else
              tma_store_2d(&tmC, buf, col0, y);
            bulk_commit();
          }
          ++kbuf;
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (lane == 0) bulk_wait_all();  // every store of this warp has landed
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  // Every role has finished, so the abort flag is final. After an abort some loads may
  // have been issued that no consumer waited for: let each land before the CTA, and its
  // shared memory, goes away. Thread 0 is the producer thread.
  if constexpr (PAIR) {
    // Neither CTA of a pair frees its TMEM or leaves while the other may still reach it.
    // The odd CTA's loads and epilogue arrivals report to the even CTA; the even CTA's MMAs
    // read the odd CTA's shared memory and write its TMEM (drained by the MMA thread before
    // the barrier above). So: the odd CTA says it is done, the even CTA waits for that,
    // drains the loads it armed (both CTAs' bytes), says goodbye, and only then does the
    // odd CTA free its TMEM and leave. Every wait is bounded; the odd CTA's outlasts the
    // even CTA's drains.
    if (threadIdx.x == 0) {
      if (rank == 1) {
        mbar_arrive_cluster(mapa_shared(smem_u32(bye), 0));
        drain_wait(bye, 0, (C::STAGES + 2) * kDrainLimitNs);
      } else {
        drain_wait(bye, 0);
        if (*abort_flag)
          for (int s = 0; s < C::STAGES; ++s)
            if (issued & (1u << s)) drain_wait(&full[s], (issued_par >> s) & 1);
        mbar_arrive_cluster(mapa_shared(smem_u32(bye), 1));
      }
    }
    __syncthreads();
  } else if (threadIdx.x == 0 && *abort_flag) {
    for (int s = 0; s < C::STAGES; ++s)
      if (issued & (1u << s)) drain_wait(&full[s], (issued_par >> s) & 1);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

int g_num_sms[64] = {};
std::mutex g_mu;

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_num_sms[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms[dev] = n > 0 ? n : 148;
  }
  return g_num_sms[dev];
}

template <int BN, int EPI, bool PAIR = false>
sal_status launch_bn(const GemmArgs& a, const void* A, const void* W, cudaStream_t s) {
  using C = Cfg<BN, EPI, PAIR>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
      if (cudaFuncSetAttribute(gemm_kernel<BN, EPI, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(C::SMEM)) != cudaSuccess)
        return SAL_ECUDA;
      attr_done[dev] = true;
    }
  }
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d_bf16(&ta, A, a.K, a.M, C::BK, C::BM)) return SAL_ECUDA;
  // rows >= n_valid read as zeros; a pair's CTAs each load BN / 2 rows
  if (!make_tmap_2d_bf16(&tb, W, a.K, a.n_valid, C::BK, C::BNL)) return SAL_ECUDA;
  if constexpr (C::QKV) {
    tc = ta;  // unused
  } else if constexpr (C::F32_OUT) {
    if (!make_tmap_2d_f32(&tc, a.out, a.N, a.M, C::CW, 32)) return SAL_ECUDA;
  } else {
    if (!make_tmap_2d_bf16(&tc, a.out, a.N, a.M, C::CW, 32)) return SAL_ECUDA;
  }
  // bounds-checked build: the buffers this launch may touch (after the last early return)
  ck_declare(A, a.M * a.K * 2, false);
  ck_declare(W, static_cast<int64_t>(a.n_valid) * a.K * 2, false);
  ck_declare(a.bias, static_cast<int64_t>(a.n_valid) * 2, false);
  if constexpr (C::QKV) {
    ck_declare(a.q, a.M * kWidth * 2, true);
    ck_declare(a.k, a.M * kWidth * 2, true);
    ck_declare(a.v, a.M * kWidth * 2, true);
    ck_declare(a.qn_g, kHeadDim * 2, false);
    ck_declare(a.kn_g, kHeadDim * 2, false);
    ck_declare(a.rope_cs, a.rope_rows * 2 * 64 * 4, false);
  } else {
    ck_declare(a.out, a.M * a.N * (C::F32_OUT ? 4 : 2), true);
  }
  if constexpr (PAIR) {
    // one cluster of two CTAs per pair of SMs, walking 256-row work units
    const int units = static_cast<int>((a.M + 2 * C::BM - 1) / (2 * C::BM)) * (a.N / BN) * a.splits;
    const int pairs = units < num_sms() / 2 ? units : num_sms() / 2;
    return launch_kernel_cluster(gemm_kernel<BN, EPI, true>, dim3(2 * pairs), dim3(C::THREADS), C::SMEM, s, 2u, ta,
                                 tb, tc, a) == cudaSuccess
               ? SAL_OK
               : SAL_ECUDA;
  } else {
    const int tiles = static_cast<int>((a.M + C::BM - 1) / C::BM) * (a.N / BN) * a.splits;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_kernel(gemm_kernel<BN, EPI, false>, dim3(grid), dim3(C::THREADS), C::SMEM, s, ta, tb, tc, a) ==
                   cudaSuccess
               ? SAL_OK
               : SAL_ECUDA;
  }
}

template <int EPI>
sal_status launch_epi(int BN, bool pair, const GemmArgs& a, const void* A, const void* W, cudaStream_t s) {
  if (pair) return BN == 256 ? launch_bn<256, EPI, true>(a, A, W, s) : SAL_ESHAPE;
  if constexpr (EPI == kEpiQkv) {  // one or two heads per tile
    return BN == 256 ? launch_bn<256, EPI>(a, A, W, s) : (BN == 128 ? launch_bn<128, EPI>(a, A, W, s) : SAL_ESHAPE);
  } else {
    switch (BN) {
      case 256: return launch_bn<256, EPI>(a, A, W, s);
      case 128: return launch_bn<128, EPI>(a, A, W, s);
      default: return launch_bn<64, EPI>(a, A, W, s);
    }
  }
}

// Tile width: 256 when those tiles alone fill the GPU; otherwise 128. At small M (a 30 s
// clip is 374 rows) every GEMM is one short wave bound by the L2 -> SM traffic of
// re-reading A for every column tile and W for every row tile; measured at M = 374,
// 128-wide tiles beat 64 (fewer A re-reads) and 256 (too few CTAs).
int pick_bn(int64_t M, int N, bool qkv) {
  const int64_t mt = (M + 127) / 128;
  // QKV: two heads per tile once those tiles fill the SMs (a 256-wide tile never straddles
  // the q / k / v sections: 1280 and 2560 are multiples of 256)
  if (qkv) return mt * (N / 256) >= num_sms() ? 256 : 128;
  if (N % 256 == 0 && mt * (N / 256) >= num_sms()) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

// CTA pairs (256 x 256 work units over two SMs) for 256-wide tiles without a K split, once
// the pairs' units alone fill every pair of SMs, for the plain epilogues. (Measured at
// 11,984 and 44,999 rows: +5 to +12 % for FFN up, FFN down and the output projection;
// the QKV epilogue, which stages a whole head per warp, runs 8 % slower at 11,984 rows and
// even at 44,999, so it keeps one CTA per tile.) SAL_GEMM_PAIR=0 / 1 in the environment
// forces pairs off / on where the shape allows them, for measurement.
bool use_pair(int64_t M, int N, int BN, int splits, bool qkv) {
  static const int mode = [] {
    const char* e = std::getenv("SAL_GEMM_PAIR");
    return e && e[0] == '0' ? 0 : (e && e[0] == '1' ? 1 : -1);
  }();
  if (mode == 0 || BN != 256 || splits != 1 || N % 256) return false;
  if (mode == 1) return true;
  return !qkv && (M + 255) / 256 * (N / 256) >= num_sms() / 2;
}

}  // namespace

sal_status gemm_launch(int epilogue, const void* A, int64_t M, int K, const void* W, int N,
                       const void* bias, void* out, const QkvOut* qkv, cudaStream_t s, int n_valid) {
  if (M == 0) return SAL_OK;
  if (K <= 0 || K % 64 || N <= 0 || N % 64) return SAL_ESHAPE;
  if (n_valid <= 0) n_valid = N;
  if (n_valid > N || (epilogue == kEpiQkv && n_valid != N)) return SAL_EINVAL;
  if (M > (int64_t(1) << 31) - 1) return SAL_ESHAPE;
  const bool is_qkv = epilogue == kEpiQkv;
  if (is_qkv && (N != 3 * kWidth || !qkv)) return SAL_EINVAL;
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.splits = 1;
  a.n_valid = n_valid;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.out = out;
  a.limit_ns = wait_limit_ns();
  a.status = device_status_ptr();
  if (!a.status) return SAL_ECUDA;
  if (is_qkv) {
    a.q = static_cast<__nv_bfloat16*>(qkv->q);
    a.k = static_cast<__nv_bfloat16*>(qkv->k);
    a.v = static_cast<__nv_bfloat16*>(qkv->v);
    a.qn_g = static_cast<const __nv_bfloat16*>(qkv->qn_g);
    a.kn_g = static_cast<const __nv_bfloat16*>(qkv->kn_g);
    a.rope_cs = qkv->rope_cs;
    a.T = qkv->T;
    a.chunk = qkv->chunk > 0 && qkv->chunk < qkv->T ? qkv->chunk : qkv->T;
    a.rope_rows = a.chunk;
  }
  const int BN = pick_bn(M, N, is_qkv);
  if (epilogue == SAL_EPI_RESID_F32) {
    // split K when the output tiles alone leave most SMs idle: up to 8 splits while the
    // work units stay within two waves and each split keeps >= 4 k-blocks (partial sums
    // are reduced into the residual stream by the TMA reduce-add; the bias goes in with
    // split 0)
    const int64_t tiles = (M + 127) / 128 * (N / BN);
    const int kb = K / 64;
    while (tiles * a.splits * 2 <= 2 * num_sms() && kb % (a.splits * 2) == 0 && kb / (a.splits * 2) >= 4 &&
           a.splits < 8)
      a.splits *= 2;
  }
  const bool pair = use_pair(M, N, BN, a.splits, is_qkv);
  switch (epilogue) {
    case SAL_EPI_STORE_F32: return launch_epi<SAL_EPI_STORE_F32>(BN, pair, a, A, W, s);
    case SAL_EPI_STORE_BF16: return launch_epi<SAL_EPI_STORE_BF16>(BN, pair, a, A, W, s);
    case SAL_EPI_GELU_BF16: return launch_epi<SAL_EPI_GELU_BF16>(BN, pair, a, A, W, s);
    case SAL_EPI_RESID_F32: return launch_epi<SAL_EPI_RESID_F32>(BN, pair, a, A, W, s);
    case kEpiQkv: return launch_epi<kEpiQkv>(BN, pair, a, A, W, s);
    default: return SAL_EINVAL;
  }
}

}  // namespace sal
