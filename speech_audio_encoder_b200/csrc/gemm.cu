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
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

struct GemmArgs {
  int64_t M;
  int N, K, splits;
  const __nv_bfloat16* bias;
  void* out;
  // QKV epilogue
  __nv_bfloat16 *q, *k, *v;
  const __nv_bfloat16 *qn_g, *kn_g;
  const float* rope_cs;
  int64_t T;
  uint64_t limit_ns;
  unsigned int* status;
};

template <int BN>
struct Cfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + 256;
};

__device__ __forceinline__ void load_bias32(const __nv_bfloat16* p, float (&b)[32]) {
  const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(p4 + i);
    b[8 * i + 0] = bf16_lo(u.x); b[8 * i + 1] = bf16_hi(u.x);
    b[8 * i + 2] = bf16_lo(u.y); b[8 * i + 3] = bf16_hi(u.y);
    b[8 * i + 4] = bf16_lo(u.z); b[8 * i + 5] = bf16_hi(u.z);
    b[8 * i + 6] = bf16_lo(u.w); b[8 * i + 7] = bf16_hi(u.w);
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    u.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    u.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    u.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d4[i] = u;
  }
}

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs args) {
  using C = Cfg<BN>;
  extern __shared__ unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitGuard guard{abort_flag, args.limit_ns, args.status};

  const int num_m = static_cast<int>((args.M + C::BM - 1) / C::BM);
  const int num_n = args.N / BN;
  const int kb_per = (args.K / C::BK) / args.splits;
  const int num_tiles = num_m * num_n * args.splits;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int sp = tile % args.splits;
        const int rest = tile / args.splits;
        const int n = rest % num_n, m = rest / num_n;
        for (int i = 0; i < kb_per; ++i) {
          const int kb = sp * kb_per + i;
          if (!mbar_wait(&empty[stage], phase ^ 1, guard)) goto producer_done;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * C::BK, m * C::BM);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * C::BK, n * BN);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:
      if (*abort_flag) {  // let every load this CTA issued land before the CTA exits
        for (int s = 0; s < C::STAGES; ++s)
          if (issued & (1u << s)) drain_wait(&full[s], (issued_par >> s) & 1, args.limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, BN, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool any_mma = false;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, guard)) break;
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
          for (int kk = 0; kk < C::BK / 16; ++kk)
            umma_ss(d, sdesc_kmajor_sw128(a0 + kk * 32), sdesc_kmajor_sw128(b0 + kk * 32), IDESC,
                    (i | kk) != 0);
          umma_commit(&empty[stage]);
          any_mma = true;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (*abort_flag && any_mma) {  // one more commit covers every MMA issued so far
        umma_commit(drain);
        drain_wait(drain, 0, args.limit_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int sp = tile % args.splits;
      const int rest = tile / args.splits;
      const int n = rest % num_n, m = rest / num_n;
      if (!mbar_wait_warp(&tfull[acc], acc_phase, guard)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(m) * C::BM + row_in_tile;
      const bool valid = row < args.M;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;

      if constexpr (EPI == kEpiQkv) {
        const int64_t b = valid ? row / args.T : 0;
        const int64_t t = valid ? row - b * args.T : 0;
#pragma unroll 1
        for (int hb = 0; hb < BN / 128; ++hb) {
          const int col0 = n * BN + hb * 128;
          const int sec = col0 / kWidth;
          const int head = (col0 % kWidth) / kHeadDim;
          __nv_bfloat16* base = sec == 0 ? args.q : (sec == 1 ? args.k : args.v);
          __nv_bfloat16* dst = base + ((b * kHeads + head) * args.T + t) * kHeadDim;
          const uint32_t ta = taddr + hb * 128;
          if (sec == 2) {
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
              uint32_t r[32];
              float bias[32], vv[32];
              tmem_ld32(ta + c, r);
              tmem_wait_ld();
              load_bias32(args.bias + col0 + c, bias);
#pragma unroll
              for (int j = 0; j < 32; ++j) vv[j] = __uint_as_float(r[j]) + bias[j];
              if (valid) store_bf16x32(dst + c, vv);
            }
          } else {
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
              uint32_t r[32];
              float bias[32];
              tmem_ld32(ta + c, r);
              tmem_wait_ld();
              load_bias32(args.bias + col0 + c, bias);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float x = __uint_as_float(r[j]) + bias[j];
                ss = fmaf(x, x, ss);
              }
            }
            const float inv = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + 1e-6f);
            const __nv_bfloat16* g = sec == 0 ? args.qn_g : args.kn_g;
            const float* cosr = args.rope_cs + t * 64;
            const float* sinr = args.rope_cs + args.T * 64 + t * 64;
#pragma unroll 1
            for (int i0 = 0; i0 < 64; i0 += 32) {
              uint32_t ra[32], rb[32];
              float ba[32], bb[32], ga[32], gb[32], oa[32], ob[32];
              tmem_ld32(ta + i0, ra);
              tmem_ld32(ta + i0 + 64, rb);
              tmem_wait_ld();
              load_bias32(args.bias + col0 + i0, ba);
              load_bias32(args.bias + col0 + i0 + 64, bb);
              load_bias32(g + i0, ga);
              load_bias32(g + i0 + 64, gb);
              if (valid) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  const float av = (__uint_as_float(ra[j]) + ba[j]) * inv * ga[j];
                  const float bv = (__uint_as_float(rb[j]) + bb[j]) * inv * gb[j];
                  const float cs = __ldg(cosr + i0 + j), sn = __ldg(sinr + i0 + j);
                  oa[j] = av * cs - bv * sn;
                  ob[j] = bv * cs + av * sn;
                }
                store_bf16x32(dst + i0, oa);
                store_bf16x32(dst + i0 + 64, ob);
              }
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          float bias[32], vv[32];
          tmem_ld32(taddr + c, r);
          tmem_wait_ld();
          const int col0 = n * BN + c;
          if (EPI == SAL_EPI_RESID_F32 && sp != 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) bias[j] = 0.f;
          } else {
            load_bias32(args.bias + col0, bias);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) vv[j] = __uint_as_float(r[j]) + bias[j];
          if (valid) {
            if constexpr (EPI == SAL_EPI_STORE_F32) {
              float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(args.out) + row * args.N + col0);
#pragma unroll
              for (int i = 0; i < 8; ++i) o4[i] = make_float4(vv[4 * i], vv[4 * i + 1], vv[4 * i + 2], vv[4 * i + 3]);
            } else if constexpr (EPI == SAL_EPI_STORE_BF16) {
              store_bf16x32(static_cast<__nv_bfloat16*>(args.out) + row * args.N + col0, vv);
            } else if constexpr (EPI == SAL_EPI_GELU_BF16) {
#pragma unroll
              for (int j = 0; j < 32; ++j) vv[j] = gelu_erf(vv[j]);
              store_bf16x32(static_cast<__nv_bfloat16*>(args.out) + row * args.N + col0, vv);
            } else {  // residual add into the fp32 stream
              float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(args.out) + row * args.N + col0);
              if (args.splits == 1) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  float4 x = o4[i];
                  x.x += vv[4 * i]; x.y += vv[4 * i + 1]; x.z += vv[4 * i + 2]; x.w += vv[4 * i + 3];
                  o4[i] = x;
                }
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  atomicAdd(o4 + i, make_float4(vv[4 * i], vv[4 * i + 1], vv[4 * i + 2], vv[4 * i + 3]));
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
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

template <int BN, int EPI>
sal_status launch_bn(const GemmArgs& a, const void* A, const void* W, cudaStream_t s) {
  using C = Cfg<BN>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
      if (cudaFuncSetAttribute(gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(C::SMEM)) != cudaSuccess)
        return SAL_ECUDA;
      attr_done[dev] = true;
    }
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, A, a.K, a.M, C::BK, C::BM)) return SAL_ECUDA;
  if (!make_tmap_2d_bf16(&tb, W, a.K, a.N, C::BK, BN)) return SAL_ECUDA;
  const int tiles = static_cast<int>((a.M + C::BM - 1) / C::BM) * (a.N / BN) * a.splits;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  count_launch();
  gemm_kernel<BN, EPI><<<grid, 192, C::SMEM, s>>>(ta, tb, a);
  return cudaGetLastError() == cudaSuccess ? SAL_OK : SAL_ECUDA;
}

template <int EPI>
sal_status launch_epi(int BN, const GemmArgs& a, const void* A, const void* W, cudaStream_t s) {
  switch (BN) {
    case 256: return launch_bn<256, EPI>(a, A, W, s);
    case 128: return launch_bn<128, EPI>(a, A, W, s);
    default:
      if constexpr (EPI == kEpiQkv) return SAL_ESHAPE;
      else return launch_bn<64, EPI>(a, A, W, s);
  }
}

// Largest tile width whose tile count fills the GPU; the narrowest otherwise.
int pick_bn(int64_t M, int N, bool qkv) {
  const int64_t mt = (M + 127) / 128;
  const int sms = num_sms();
  if (N % 256 == 0 && mt * (N / 256) >= sms) return 256;
  if (N % 128 == 0 && (qkv || mt * (N / 128) >= sms)) return 128;
  return qkv ? 128 : 64;
}

}  // namespace

sal_status gemm_launch(int epilogue, const void* A, int64_t M, int K, const void* W, int N,
                       const void* bias, void* out, const QkvOut* qkv, cudaStream_t s) {
  if (M == 0) return SAL_OK;
  if (K <= 0 || K % 64 || N <= 0 || N % 64) return SAL_ESHAPE;
  if (M > (int64_t(1) << 31) - 1) return SAL_ESHAPE;
  const bool is_qkv = epilogue == kEpiQkv;
  if (is_qkv && (N != 3 * kWidth || !qkv)) return SAL_EINVAL;
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.splits = 1;
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
  }
  const int BN = pick_bn(M, N, is_qkv);
  if (epilogue == SAL_EPI_RESID_F32) {
    // split K when the output tiles alone leave most SMs idle (partial sums are added
    // atomically into the residual stream; the bias goes in with split 0)
    const int64_t tiles = (M + 127) / 128 * (N / BN);
    const int kb = K / 64;
    while (tiles * a.splits * 2 <= num_sms() && kb % (a.splits * 2) == 0 && a.splits < 8)
      a.splits *= 2;
  }
  switch (epilogue) {
    case SAL_EPI_STORE_F32: return launch_epi<SAL_EPI_STORE_F32>(BN, a, A, W, s);
    case SAL_EPI_STORE_BF16: return launch_epi<SAL_EPI_STORE_BF16>(BN, a, A, W, s);
    case SAL_EPI_GELU_BF16: return launch_epi<SAL_EPI_GELU_BF16>(BN, a, A, W, s);
    case SAL_EPI_RESID_F32: return launch_epi<SAL_EPI_RESID_F32>(BN, a, A, W, s);
    case kEpiQkv: return launch_epi<kEpiQkv>(BN, a, A, W, s);
    default: return SAL_EINVAL;
  }
}

}  // namespace sal
