// Bidirectional multi-head attention of the encoder on the tensor cores:
//   O[b, t, 128 h + :] = softmax(q_h k_h^T / sqrt(128)) v_h   over all T positions of clip b
// (page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits", section "How
// audio and speakers reach the language model": ten heads over width 1,280; full-clip
// bidirectional attention, no mask).
//
// Flash-style streaming: the T x T score matrix is never stored. One CTA owns a tile of
// 128 query rows of one (clip, head) and walks the keys 128 at a time:
//   * warp 0 loads Q once and K / V tiles through a two-stage TMA ring (128-byte swizzle);
//   * warp 1 (one thread) issues S_j = Q K_j^T (tcgen05.mma, both operands in shared
//     memory) into one of two TMEM score buffers, then O += P_j V_j with P_j read from TMEM
//     (A operand) and V_j from shared memory (MN-major B operand);
//   * warps 2-5 own one query row per thread: read S_j from TMEM, online softmax in the
//     log2 domain (exp2 on the SFU), write P_j back to TMEM as bf16 pairs, and rescale the
//     TMEM accumulator O only when the running maximum grew by more than 2^8 (otherwise
//     the stale maximum keeps every p <= 256, exact in fp32 and bf16 range);
//   * S_{j+1} is computed while the softmax of S_j runs.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384), P0 [384,448), P1 [448,512).
#define SAL_CK_FILE 4
#include <cuda_bf16.h>
#include <math.h>

#include <cstdlib>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "sal_internal.h"
#include "sal_ptx.cuh"

namespace sal {
namespace {

constexpr int kTile = 128;
constexpr int kBox = kTile * 64 * 2;       // one 64-column half of a 128 x 128 bf16 tile
constexpr uint32_t kColO = 256;
__device__ __forceinline__ uint32_t col_s(int s) { return s ? 128u : 0u; }    // score buffers
__device__ __forceinline__ uint32_t col_p(int s) { return s ? 448u : 384u; }  // bf16 P buffers
__host__ __device__ constexpr int tile_bytes(int hd) { return kTile * hd * 2; }  // a 128-row tile of Q, K or V
__host__ __device__ constexpr size_t smem_one_tile(int hd) { return 1024 + 5 * tile_bytes(hd) + 256; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// The choice between the one-tile and two-tile kernels can be forced with SAL_ATTN_PP.
// SAL_ATTN_PP: unset = choose by the wave model below, 0 = never the two-tile kernel,
// 1 = always (where its grid has at least one query-tile pair); for measuring the choice.
int attention_pp_mode() {
  static const int mode = [] {
    const char* e = std::getenv("SAL_ATTN_PP");
    return e && e[0] == '0' ? 0 : (e && e[0] == '1' ? 1 : -1);
  }();
  return mode;
}

// SAL_ATTN_PAIRS=n (n >= 0) in the environment forces the two-tile kernel with n pairs per
// (clip, head), clamped to all of them, and every other tile in split mode (n = 0: every
// tile split). For measuring the split cost; -1 when unset.
int attention_pairs_forced() {
  static const int n = [] {
    const char* e = std::getenv("SAL_ATTN_PAIRS");
    return e && e[0] >= '0' && e[0] <= '9' ? std::atoi(e) : -1;
  }();
  return n;
}

struct AttnArgs {
  // two-tile kernel: CTAs x < pairs take the query-tile pair (2x, 2x + 1); each CTA past
  // them takes one query tile, 2 pairs + (x - pairs), split over the keys between its two
  // warpgroups (key tiles 0, 2, 4, ... and 1, 3, 5, ...) and merged at the end
  int pairs = 0;
  int64_t T;
  int64_t chunk;  // attention stays inside chunks of this many positions (T: whole clip)
  int heads;
  __nv_bfloat16* o;
  float scale_log2;
  uint64_t limit_ns;
  unsigned int* status;
  // Test hook (sal_attention_withhold): the key/value tile at this index (relative to the
  // CTA's first key tile) is never loaded, so the wait for it gives up at limit_ns. -1: off.
  int withhold = -1;
  // Serving windows (win_count > 0): clip c of the batch is window c % win_count of a
  // recording of win_total positions, left-aligned in its T slots; only its first
  // window_len(c) positions are keys (see valid_len).
  int win_count = 0, win_core = 0, win_ctx = 0;
  int64_t win_total = 0;
};

// Positions of clip `clip` that are keys: T, or for serving windows the window's own
// length (its core extended by up to win_ctx positions on each side inside the recording).
__device__ __forceinline__ int64_t valid_len(const AttnArgs& a, int clip) {
  if (a.win_count <= 0) return a.T;
  const int64_t w = clip % a.win_count;
  const int64_t lo = w * a.win_core - a.win_ctx, hi = (w + 1) * a.win_core + a.win_ctx;
  return (hi < a.win_total ? hi : a.win_total) - (lo > 0 ? lo : 0);
}

// Key tiles [j0, j0 + n) that the query rows [q_lo, q_hi) can see: the union of their
// chunks [floor(t / chunk) chunk, next chunk start) clipped to the T key positions. Rows
// at or past T (padding slots of a serving window) see the chunk of row T - 1.
__device__ __forceinline__ void kv_tile_range(int64_t q_lo, int64_t q_hi, int64_t T, int64_t chunk, int& j0,
                                              int& n) {
  if (q_hi > T) q_hi = T;
  if (q_lo > T - 1) q_lo = T - 1;
  if (q_hi <= q_lo) q_hi = q_lo + 1;
  const int64_t kv_lo = (q_lo / chunk) * chunk;
  int64_t kv_hi = ((q_hi - 1) / chunk + 1) * chunk;
  if (kv_hi > T) kv_hi = T;
  j0 = static_cast<int>(kv_lo / 128);
  n = static_cast<int>((kv_hi + 127) / 128) - j0;
}

// Keys [lo, hi) that row t may attend to: its own chunk among the Tk key positions; empty
// for rows t >= T (past the tensor), the chunk of row Tk - 1 for rows Tk <= t < T (padding
// slots of a serving window, computed but never used). Positions fit in 32 bits.
__device__ __forceinline__ void row_range(int t, int T, int Tk, int chunk, int& lo, int& hi) {
  if (t >= T) {
    lo = hi = 0;
    return;
  }
  if (t >= Tk) t = Tk - 1;
  lo = (t / chunk) * chunk;
  hi = lo + chunk < Tk ? lo + chunk : Tk;
}

// Columns [c_lo, c_hi) of key tile jt inside [lo, hi).
__device__ __forceinline__ void tile_cols(int lo, int hi, int jt, int& c_lo, int& c_hi) {
  const int base = jt * 128;
  c_lo = min(max(lo - base, 0), 128);
  c_hi = min(max(hi - base, 0), 128);
}

// Maximum of a row of 128 scores held as raw fp32 bits: eight independent chains of
// three-input max over 16 scores each, then merged, so the longest dependent chain is 10
// instructions instead of 64.
__device__ __forceinline__ float row_max128(const uint32_t (&r)[4][32]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t* v = &r[k >> 1][(k & 1) * 16];
    m[k] = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
    for (int i = 2; i < 16; i += 2) m[k] = max3f(m[k], __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
  }
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Scores outside [c_lo, c_hi) of this 32-column chunk become -inf, so the unmasked softmax
// that follows gives them weight 0 (run only on tiles that need a mask).
__device__ __forceinline__ void mask_chunk(uint32_t (&r)[32], int col0, int c_lo, int c_hi) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (col0 + i < c_lo || col0 + i >= c_hi) r[i] = 0xff800000u;  // -inf
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  extern __shared__ unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int TB = tile_bytes(HD);
  uint8_t* sQ = smem;
  uint8_t* sK[2] = {smem + TB, smem + 2 * TB};
  uint8_t* sV[2] = {smem + 3 * TB, smem + 4 * TB};
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 5 * TB);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* o_done = bars + 10;
  uint64_t* drain = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t T = args.T;
  const int bh = blockIdx.y;
  const int qt = blockIdx.x;
  const int64_t Tk = valid_len(args, bh / args.heads);  // key positions of this clip
  int j0, n_kv;
  kv_tile_range(static_cast<int64_t>(qt) * kTile, static_cast<int64_t>(qt) * kTile + kTile, Tk, args.chunk, j0,
                n_kv);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard guard{abort_flag, args.limit_ns, args.status};
  // the producer's record of the stages it loaded and their phases (for the wind-down)
  uint32_t issued_q = 0, issued = 0, par_k = 0;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, TB);
#pragma unroll
      for (int b = 0; b < HD / 64; ++b) tma_load_3d(sQ + b * kBox, &tmQ, q_full, 64 * b, qt * kTile, bh);
      issued_q = 1;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j & 1;
        const uint32_t use_par = (j >> 1) & 1;
        if (!mbar_wait(&kv_empty[s], use_par ^ 1, guard)) break;
        if (j == args.withhold) continue;  // nothing issued: stage s keeps its last tracked load
        mbar_arrive_expect_tx(&k_full[s], TB);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) tma_load_3d(sK[s] + b * kBox, &tmK, &k_full[s], 64 * b, (j0 + j) * kTile, bh);
        mbar_arrive_expect_tx(&v_full[s], TB);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) tma_load_3d(sV[s] + b * kBox, &tmV, &v_full[s], 64 * b, (j0 + j) * kTile, bh);
        issued |= 1u << s;
        par_k = (par_k & ~(1u << s)) | (use_par << s);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, HD, false, true);
      bool ok = mbar_wait(q_full, 0, guard);
      bool any_mma = false;
      const uint32_t q0 = smem_u32(sQ);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(&k_full[s], (j >> 1) & 1, guard)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK[s]);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
          umma_ss(tmem + col_s(s), sdesc_kmajor_sw128(q0 + off), sdesc_kmajor_sw128(k0 + off), IDESC_S,
                  kk > 0);
        }
        umma_commit(&s_full[s]);
        any_mma = true;
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j & 1;
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, guard)) break;
        if (!mbar_wait(&v_full[s], (j >> 1) & 1, guard)) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV[s]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + kColO, tmem + col_p(s) + kk * 8, sdesc_mnmajor_sw128(v0 + kk * 2048, kBox), IDESC_O,
                  (j > 0 || kk > 0));
        umma_commit(&kv_empty[s]);
        umma_commit(o_done);
      }
      if (*abort_flag && any_mma) {
        // every MMA issued so far is covered by one more commit
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 2..5
    const int quarter = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int row = quarter * 32 + lane;
    const float sl2 = args.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    int row_lo, row_hi;
    row_range(qt * kTile + row, static_cast<int>(T), static_cast<int>(Tk), static_cast<int>(args.chunk), row_lo,
              row_hi);
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!mbar_wait_warp(&s_full[s], (j >> 1) & 1, guard)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + col_s(s) + 32 * c, r[c]);
      tmem_wait_ld();
      int c_lo, c_hi;
      tile_cols(row_lo, row_hi, j0 + j, c_lo, c_hi);
      if (!__all_sync(0xffffffffu, c_lo == 0 && c_hi == kTile)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) mask_chunk(r[c], 32 * c, c_lo, c_hi);
      }
      float mx = row_max128(r) * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        rescale = true;
      }
      // a row that has seen no key yet keeps m_ref = -inf; its masked scores still give 0
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      // two scores per instruction: x = s * scale - m (packed fma), the row sum (packed add)
      const uint64_t sl2_2 = f2_pack(sl2, sl2), negm_2 = f2_pack(-m_use, -m_use);
      uint64_t sum2[4];  // one running pair sum per 32-column chunk: four short chains
      uint32_t p[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float x0, x1, e0, e1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])), sl2_2, negm_2), x0, x1);
          if (HD == 64 && ((i >> 1) & 7) < 3) {
            // head dim 64: the MMAs of a tile take half the SFU's exponential time, so 6 of
            // every 16 pairs go to the FMA pipe
            exp2_pair_poly(x0, x1, e0, e1);
          } else {
            e0 = fast_exp2(x0);
            e1 = fast_exp2(x1);
          }
          sum2[c] = i == 0 ? f2_pack(e0, e1) : f2_add(sum2[c], f2_pack(e0, e1));
          p[c >> 1][(c & 1) * 16 + (i >> 1)] = pack_bf16x2(e0, e1);
        }
      float sum_lo, sum_hi;
      f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sum_lo, sum_hi);
      const float sum = sum_lo + sum_hi;
      if (j > 0) {
        // PV_{j-1} must be complete before O is rescaled or P buffer s is overwritten
        if (!mbar_wait_warp(o_done, (j - 1) & 1, guard)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + kColO + 32 * c, o);
          }
        }
      }
      l = l * alpha + sum;
      tmem_st32(tmem + lane_base + col_p(s), p[0]);
      tmem_st32(tmem + lane_base + col_p(s) + 32, p[1]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait_warp(o_done, (n_kv - 1) & 1, guard)) {
      tc_fence_after();
      const int64_t t = static_cast<int64_t>(qt) * kTile + row;
      const int b = bh / args.heads, h = bh % args.heads;
      const float inv_l = 1.0f / l;
      __nv_bfloat16* dst = args.o + (static_cast<int64_t>(b) * T + t) * (args.heads * HD) + h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
        tmem_wait_ld();
        if (t < T) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
            u.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
            u.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
            u.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
            *SAL_CK_ST(d4 + i, 16) = u;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // Every role has finished, so the abort flag is final. After an abort some loads may
  // have been issued that no consumer waited for: let each land before the CTA, and its
  // shared memory, goes away.
  if (warp == 0 && lane == 0 && *abort_flag) {
    if (issued_q) drain_wait(q_full, 0);
    for (int s = 0; s < 2; ++s)
      if (issued & (1u << s)) {
        drain_wait(&k_full[s], (par_k >> s) & 1);
        drain_wait(&v_full[s], (par_k >> s) & 1);
      }
  }
}

// ---------------------------------------------------------------------------------
// Two-tile variant for long clips: one CTA owns TWO 128-row query tiles of one
// (clip, head), so each K / V tile loaded serves 256 queries, and two softmax warpgroups
// take turns with the tensor core. CTAs past args.pairs take one query tile in split mode:
// both warpgroups work on it, on alternate key tiles, and merge their results at the end.
//   warp 0: TMA loads of Q0 and Q1 once and of K_j through a two-stage ring, released
//           after the S products that read it
//   warp 3: TMA loads of V_j through a two-stage ring, released after its P V products
//   warp 1: issues the S products, S0_0 S1_0 S0_1 S1_1 ..., each as soon as its score
//           buffer is free
//   warp 2: issues the P V products, P_i(j) V_j once P_i(j) is stored and S_i(j+1) has
//           been issued (the tensor core runs MMAs in issue order: an S product, on the
//           critical path, never waits behind a P V product). Two issuing threads,
//           because one thread takes nearly as long to issue a 128 x 128 x 16 MMA as the
//           tensor core takes to run it.
//   warps 4-7 / 8-11: softmax of query tile 0 / 1, one row per thread
// TMEM at head dim 128: S [0,128) O0 [128,256) O1 [256,384) P0 [384,448) P1 [448,512).
// The one score buffer S is shared by the two query tiles: a warpgroup copies its S_i(j)
// into registers and hands the buffer back at once, so the next product (the other tile's
// S, then its own S_i(j+1)) runs on the tensor core while its exponentials are computed.
// P_i (bf16 pairs) has a region of its own, so S_i(j+1) does not wait for P_i(j) V_j. The
// warpgroup waits for P_i(j-1) V_{j-1} to complete before it rescales O_i or overwrites
// P_i. At head dim 64 each query tile has a score buffer of its own (PPLayout).
// Warpgroup 0 (loads, MMA issue) shrinks to kRegsCtrl registers per thread and the two
// softmax warpgroups grow to kRegsSoftmax, so each softmax thread holds its whole row of
// S (128 scores) and reads it from TMEM in one round trip per tile.
// Of every 16 score pairs of a row chunk, this many take their exponentials on the FMA
// pipe (exp2_pair_poly) instead of the SFU. Head dim 128: none, since the polynomial's
// extra instructions slow the MMA-issuing threads that share the softmax warps' SM
// sub-partitions (measured 3-5 % slower at 2 of 16). Head dim 64 (the MMAs of a tile take
// half the time, the softmax is the bound): SAL_PP_POLY_PAIRS_HD64 of 16.
#ifndef SAL_PP_POLY_PAIRS
#define SAL_PP_POLY_PAIRS 0
#endif
#ifndef SAL_PP_POLY_PAIRS_HD64
#define SAL_PP_POLY_PAIRS_HD64 6
#endif
// Layout of the two-tile kernel per head dim. At 128 the TMEM holds one score buffer
// shared by the two query tiles: S [0,128) O0 [128,256) O1 [256,384) P0 [384,448)
// P1 [448,512). At 64 the accumulators are half as wide and each query tile has a score
// buffer of its own: S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384) P0 P1 as above.
template <int HD>
struct PPLayout {
  static constexpr int kTileB = kTile * HD * 2;  // a 128-row tile of Q, K or V
  static constexpr int kBoxes = HD / 64;         // 64-column boxes of a tile
  static constexpr bool kSharedS = HD == 128;
  static constexpr size_t kSmem = 1024 + 6 * static_cast<size_t>(kTileB) + 256 + 2048;  // + split-mode merge
  static constexpr int kPoly = HD == 64 ? SAL_PP_POLY_PAIRS_HD64 : SAL_PP_POLY_PAIRS;
  __device__ static uint32_t col_s(int i) { return kSharedS ? 0u : 128u * i; }
  __device__ static uint32_t col_o(int i) { return kSharedS ? 128u + 128u * i : 256u + 64u * i; }
  __device__ static uint32_t col_p(int i) { return 384u + 64u * i; }
};
static_assert(PPLayout<128>::kSmem <= 227 * 1024 && PPLayout<64>::kSmem <= 227 * 1024, "shared memory");

// 32 consecutive output columns of one row: bf16(a * x[i] + b * y[i]), 64 bytes.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&x)[32], float a, float b,
                                            const uint32_t (&y)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = fmaf(__uint_as_float(y[8 * i + e]), b, __uint_as_float(x[8 * i + e]) * a);
    *SAL_CK_ST(d4 + i, 16) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                        pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
}

constexpr int kThreadsPP = 384;
constexpr int kRegsCtrl = 104, kRegsSoftmax = 200;
constexpr int kRegsNeededPP = kRegsCtrl * 128 + kRegsSoftmax * 256;  // <= launch regs x 384

// SPLIT: the launch may hold split-mode CTAs. A launch of pairs only runs the form without
// the split-mode code, whose registers and branches it would otherwise carry.
template <int HD, bool SPLIT>
__global__ void __launch_bounds__(kThreadsPP, 1)
    attention_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  using L = PPLayout<HD>;
  constexpr int kTileBytes = L::kTileB;
  extern __shared__ unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // Q0, Q1
  uint8_t* sK = smem + 2 * kTileBytes;      // K stage 0, 1
  uint8_t* sV = smem + 4 * kTileBytes;      // V stage 0, 1
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * kTileBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* k_empty = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2] S_i(j) is in the score buffer
  uint64_t* p_full = bars + 11;   // [2] P_i(j) is in its region (O_i rescaled if needed)
  uint64_t* pv_done = bars + 13;  // [2] P_i(j) V_j has completed
  // a score buffer has been read (one phase per S product in it): [0] is the shared
  // buffer (head dim 128), [i] the buffer of query tile i (head dim 64)
  uint64_t* s_free[2] = {bars + 15, bars + 20};
  uint64_t* drain = bars + 16;     // wind-down of the S issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* drain_pv = bars + 18;  // wind-down of the P V issuer
  volatile int* s_issued = reinterpret_cast<volatile int*>(bars + 19);  // S products issued so far
  uint64_t* merge_bar = bars + 21;  // split mode: both warpgroups' final (m, l) are written
  float* merge_ml = reinterpret_cast<float*>(smem + 6 * kTileBytes + 256);  // [2][128][2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t T = args.T;
  const int bh = blockIdx.y;
  const bool split = SPLIT && static_cast<int>(blockIdx.x) >= args.pairs;
  const int qt2 = blockIdx.x;                                    // pair mode: 256-row query block
  const int qt1 = 2 * args.pairs + (static_cast<int>(blockIdx.x) - args.pairs);  // split mode: query tile
  const int64_t Tk = valid_len(args, bh / args.heads);  // key positions of this clip
  int j0, n_kv;
  {
    const int64_t q_lo = split ? static_cast<int64_t>(qt1) * kTile : static_cast<int64_t>(qt2) * 2 * kTile;
    kv_tile_range(q_lo, q_lo + (split ? kTile : 2 * kTile), Tk, args.chunk, j0, n_kv);
  }
  // S products (and P V products) of the CTA, q = 2 x + i for warpgroup i's x-th: over
  // key tile x (pair mode) or key tile q (split mode)
  const int n_prod = split ? n_kv : 2 * n_kv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(s_free[0], 4);  // one arrival per warp of the warpgroup that read S
    mbar_init(s_free[1], 4);
    mbar_init(drain, 1);
    mbar_init(drain_pv, 1);
    mbar_init(merge_bar, 256);
    *s_issued = 0;
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard guard{abort_flag, args.limit_ns, args.status};
  // the producer's record of the stages it loaded and their phases (for the wind-down)
  uint32_t issued_k = 0, issued_v = 0, par_k = 0, par_v = 0;
  // Each role runs inside the branch that set its register limit, so the compiler
  // allocates it against that limit.
  if (warp < 4) {
    setmaxnreg_dec<kRegsCtrl>();
    if (warp == 0) {
      if (lane == 0) {
        const int nq = split ? 1 : 2;  // split mode: both warpgroups use Q0
        mbar_arrive_expect_tx(q_full, nq * kTileBytes);
        for (int i = 0; i < nq; ++i)
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sQ + i * kTileBytes + b * kBox, &tmQ, q_full, 64 * b, (split ? qt1 : 2 * qt2 + i) * kTile,
                        bh);
        for (int j = 0; j < n_kv; ++j) {
          const int s = j & 1;
          const uint32_t use_par = (j >> 1) & 1;
          if (!mbar_wait(&k_empty[s], use_par ^ 1, guard)) break;
          if (j == args.withhold) continue;  // nothing issued: stage s keeps its last tracked loads
          mbar_arrive_expect_tx(&k_full[s], kTileBytes);
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sK + s * kTileBytes + b * kBox, &tmK, &k_full[s], 64 * b, (j0 + j) * kTile, bh);
          issued_k |= 1u << s;
          par_k = (par_k & ~(1u << s)) | (use_par << s);
          if constexpr (!SPLIT) {  // pairs only: V_j right behind K_j from the same thread
            if (!mbar_wait(&v_empty[s], use_par ^ 1, guard)) break;
            mbar_arrive_expect_tx(&v_full[s], kTileBytes);
            for (int b = 0; b < L::kBoxes; ++b)
              tma_load_3d(sV + s * kTileBytes + b * kBox, &tmV, &v_full[s], 64 * b, (j0 + j) * kTile, bh);
            issued_v |= 1u << s;
            par_v = (par_v & ~(1u << s)) | (use_par << s);
          }
        }
      }
    } else if (warp == 3) {
      // With split-mode CTAs in the launch, V loads come from a thread of their own: a V
      // stage frees up only after its P V product, which must not hold back the next K tile
      // (in split mode each stage serves one warpgroup, and V_j's stage is free only after
      // that warpgroup's P V of tile j - 2). Without them a second polling thread costs the
      // softmax warps that share its SM sub-partition more than it gains.
      if (SPLIT && lane == 0) {
        for (int j = 0; j < n_kv; ++j) {
          const int s = j & 1;
          const uint32_t use_par = (j >> 1) & 1;
          if (!mbar_wait(&v_empty[s], use_par ^ 1, guard)) break;
          if (j == args.withhold) continue;  // nothing issued: stage s keeps its last tracked load
          mbar_arrive_expect_tx(&v_full[s], kTileBytes);
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sV + s * kTileBytes + b * kBox, &tmV, &v_full[s], 64 * b, (j0 + j) * kTile, bh);
          issued_v |= 1u << s;
          par_v = (par_v & ~(1u << s)) | (use_par << s);
        }
      }
    } else if (warp == 1) {
      // S issue: S_i(x) into its score buffer, in the order S0_0 S1_0 S0_1 S1_1 ...
      if (lane == 0) {
        constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
        bool any_mma = false;
        bool ok = mbar_wait(q_full, 0, guard);
        for (int q = 0; ok && q < n_prod; ++q) {
          const int i = q & 1, x = q >> 1;
          const int jk = split ? q : x;  // key tile (from j0), in stage jk & 1
          const int s = jk & 1;
          // the previous S product in the same buffer has been read out of it (the shared
          // buffer: the previous product; own buffers: this tile's previous one), and K_x
          // has landed
          const bool reuse = L::kSharedS ? q > 0 : x > 0;
          const uint32_t par = L::kSharedS ? (q - 1) & 1 : (x - 1) & 1;
          ok = (!reuse || mbar_wait(s_free[L::kSharedS ? 0 : i], par, guard)) &&
               mbar_wait(&k_full[s], (jk >> 1) & 1, guard);
          if (!ok) break;
          tc_fence_after();
          const uint32_t q0 = smem_u32(sQ + (split ? 0 : i) * kTileBytes), k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            umma_ss(tmem + L::col_s(i), sdesc_kmajor_sw128(q0 + off), sdesc_kmajor_sw128(k0 + off), IDESC_S,
                    kk > 0);
          }
          umma_commit(&s_full[i]);
          if (split || i == 1) umma_commit(&k_empty[s]);  // every product with this K tile issued
          any_mma = true;
          *s_issued = q + 1;
        }
        if (*abort_flag && any_mma) {
          umma_commit(drain);
          drain_wait(drain, 0);
        }
      }
    } else if (warp == 2) {
      // P V issue: O_i += P_i(j) V_j. A second issuing thread, because one thread alone
      // spends longer issuing the 32 MMAs of a key tile than the tensor core takes to run
      // them. The tensor core runs MMAs in issue order, and an S product is on the
      // critical path (the score buffer is shared), so P_i(j) V_j waits until S_i(j+1)
      // has been issued and then runs while warpgroup i reads S_i(j+1).
      if (lane == 0) {
        constexpr uint32_t IDESC_O = idesc_bf16(128, HD, false, true);
        bool any_mma = false, ok = true;
        if constexpr (!SPLIT && HD == 64) {
          // head dim 64, pairs only: per key tile, P0 V then P1 V. A P V MMA is 32 cycles of
          // tensor work here, and this nested form issues faster than the flat loop below
          // (measured 10.1 against 11.2 ms at 44,999 positions); at head dim 128 the flat
          // loop measured faster.
          for (int j = 0; ok && j < n_kv; ++j) {
            const int s = j & 1;
            for (int i = 0; i < 2; ++i) {
              ok = mbar_wait(&p_full[i], j & 1, guard) && mbar_wait(&v_full[s], (j >> 1) & 1, guard);
              if (!ok) break;
              if (j + 1 < n_kv) {
                // a plain spin (the wait is short and its end is on the critical path); the
                // bound is checked every 64 polls
                const int need = 2 * (j + 1) + i + 1;
                uint64_t t0 = 0;
                for (uint32_t spin = 1; *s_issued < need; ++spin) {
                  if ((spin & 63) != 0) continue;
                  if (*abort_flag) {
                    ok = false;
                    break;
                  }
                  const uint64_t now = globaltimer_ns();
                  if (t0 == 0) {
                    t0 = now;
                  } else if (now - t0 > args.limit_ns) {
                    *abort_flag = 1;
                    atomicOr(args.status, kStatusTimeout);
                    ok = false;
                    break;
                  }
                }
                if (!ok) break;
              }
              tc_fence_after();
              const uint32_t v0 = smem_u32(sV + s * kTileBytes);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                umma_ts(tmem + L::col_o(i), tmem + L::col_p(i) + kk * 8, sdesc_mnmajor_sw128(v0 + kk * 2048, kBox),
                        IDESC_O, (j > 0 || kk > 0));
              umma_commit(&pv_done[i]);
              any_mma = true;
            }
            if (ok) umma_commit(&v_empty[s]);
          }
        } else {
          for (int q = 0; ok && q < n_prod; ++q) {
            const int i = q & 1, x = q >> 1;
            const int jk = split ? q : x;  // key tile (from j0), in stage jk & 1
            const int s = jk & 1;
            ok = mbar_wait(&p_full[i], x & 1, guard) && mbar_wait(&v_full[s], (jk >> 1) & 1, guard);
            if (!ok) break;
            if (q + 2 < n_prod) {
              // S_i(x+1) (product q + 2) must have been issued; a plain spin (the wait is short
              // and its end is on the critical path), the bound checked every 64 polls
              const int need = q + 3;
              uint64_t t0 = 0;
              for (uint32_t spin = 1; *s_issued < need; ++spin) {
                if ((spin & 63) != 0) continue;
                if (*abort_flag) {
                  ok = false;
                  break;
                }
                const uint64_t now = globaltimer_ns();
                if (t0 == 0) {
                  t0 = now;
                } else if (now - t0 > args.limit_ns) {
                  *abort_flag = 1;
                  atomicOr(args.status, kStatusTimeout);
                  ok = false;
                  break;
                }
              }
              if (!ok) break;
            }
            tc_fence_after();
            const uint32_t v0 = smem_u32(sV + s * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tmem + L::col_o(i), tmem + L::col_p(i) + kk * 8, sdesc_mnmajor_sw128(v0 + kk * 2048, kBox),
                      IDESC_O, (x > 0 || kk > 0));
            umma_commit(&pv_done[i]);
            if (split || i == 1) umma_commit(&v_empty[s]);  // every product with this V tile issued
            any_mma = true;
          }
        }
        if (*abort_flag && any_mma) {
          umma_commit(drain_pv);
          drain_wait(drain_pv, 0);
        }
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 4) >> 2;  // query tile 0 or 1
    const int quarter = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t colS = L::col_s(wg), colO = L::col_o(wg), colP = L::col_p(wg);
    const int row = quarter * 32 + lane;
    const float sl2 = args.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    int row_lo, row_hi;
    row_range((split ? qt1 : 2 * qt2 + wg) * kTile + row, static_cast<int>(T), static_cast<int>(Tk),
              static_cast<int>(args.chunk), row_lo, row_hi);
    // this warpgroup's key tiles: all n_kv (pair mode), or every other one from wg (split)
    const int n_my = split ? (n_kv + 1 - wg) / 2 : n_kv;
    for (int j = 0; j < n_my; ++j) {
      const int jk = split ? 2 * j + wg : j;  // key tile (from j0)
      if (!mbar_wait_warp(&s_full[wg], j & 1, guard)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the whole row of S in registers (one wait for four loads), then the buffer goes
      // back to the tensor core for the next product
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + colS + 32 * c, r[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free[L::kSharedS ? 0 : wg]);
      int c_lo, c_hi;
      tile_cols(row_lo, row_hi, j0 + jk, c_lo, c_hi);
      if (!__all_sync(0xffffffffu, c_lo == 0 && c_hi == kTile)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) mask_chunk(r[c], 32 * c, c_lo, c_hi);
      }
      float mx = row_max128(r) * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        rescale = true;
      }
      // exponentials, row sum, bf16 P packed in place over the scores already consumed
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;  // a row with no key seen yet
      const uint64_t sl2_2 = f2_pack(sl2, sl2), negm_2 = f2_pack(-m_use, -m_use);
      uint64_t sum2[4];  // one running pair sum per 32-column chunk: four short chains
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])), sl2_2, negm_2), x0, x1);
          float e0, e1;
          if (L::kPoly > 0 && ((i >> 1) & 15) < L::kPoly) {
            exp2_pair_poly(x0, x1, e0, e1);  // on the FMA pipe, leaving the SFU to the others
          } else {
            e0 = fast_exp2(x0);
            e1 = fast_exp2(x1);
          }
          sum2[c] = i == 0 ? f2_pack(e0, e1) : f2_add(sum2[c], f2_pack(e0, e1));
          r[c >> 1][(c & 1) * 16 + (i >> 1)] = pack_bf16x2(e0, e1);
        }
      }
      if (j > 0) {
        // P_i(j-1) V_{j-1} must be complete before O_i is rescaled or P_i overwritten
        if (!mbar_wait_warp(&pv_done[wg], (j - 1) & 1, guard)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32(tmem + lane_base + colP, r[0]);
      tmem_st32(tmem + lane_base + colP + 32, r[1]);
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + colO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + colO + 32 * c, o);
        }
      }
      float sum_lo, sum_hi;
      f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sum_lo, sum_hi);
      l = l * alpha + (sum_lo + sum_hi);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
    }
    const int b = bh / args.heads, h = bh % args.heads;
    if (!split) {
      if (ok && mbar_wait_warp(&pv_done[wg], (n_my - 1) & 1, guard)) {
        tc_fence_after();
        const int64_t t = static_cast<int64_t>(2 * qt2 + wg) * kTile + row;
        const float inv_l = 1.0f / l;
        __nv_bfloat16* dst = args.o + (static_cast<int64_t>(b) * T + t) * (args.heads * HD) + h * HD;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + colO + 32 * c, o);
          tmem_wait_ld();
          if (t < T) store_row32(dst + 32 * c, o, inv_l, 0.f, o);
        }
      }
    } else {
      // Both warpgroups hold a partial result for the same rows (the keys split between
      // them). Once both are final, each writes half of the columns of
      //   O = (O0 2^(m0 - m) + O1 2^(m1 - m)) / (l0 2^(m0 - m) + l1 2^(m1 - m)), m = max(m0, m1),
      // reading both accumulators (every warp reaches both regions in its lane quarter).
      // Every softmax thread arrives on merge_bar once, aborted or not.
      const bool mine = ok && (n_my == 0 || mbar_wait_warp(&pv_done[wg], (n_my - 1) & 1, guard));
      merge_ml[(wg * 128 + row) * 2 + 0] = m_ref;
      merge_ml[(wg * 128 + row) * 2 + 1] = mine ? l : 0.f;
      mbar_arrive(merge_bar);
      if (mine && mbar_wait_warp(merge_bar, 0, guard) && !*abort_flag) {
        tc_fence_after();
        const float m0 = merge_ml[row * 2], l0 = merge_ml[row * 2 + 1];
        const float m1 = merge_ml[(128 + row) * 2], l1 = merge_ml[(128 + row) * 2 + 1];
        const float m = fmaxf(m0, m1);
        // a part that saw no key has l = 0 (and m = -inf): its weight is 0
        const float a0 = l0 > 0.f ? fast_exp2(m0 - m) : 0.f, a1 = l1 > 0.f ? fast_exp2(m1 - m) : 0.f;
        const float lsum = l0 * a0 + l1 * a1;
        const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
        const int64_t t = static_cast<int64_t>(qt1) * kTile + row;
        __nv_bfloat16* dst = args.o + (static_cast<int64_t>(b) * T + t) * (args.heads * HD) + h * HD;
#pragma unroll 1
        for (int c = 0; c < HD / 64; ++c) {
          const uint32_t col = static_cast<uint32_t>(wg * (HD / 2) + 32 * c);
          uint32_t o0[32], o1[32];
          tmem_ld32(tmem + lane_base + L::col_o(0) + col, o0);
          tmem_ld32(tmem + lane_base + L::col_o(1) + col, o1);
          tmem_wait_ld();
          if (t < T) store_row32(dst + col, o0, a0 * inv, a1 * inv, o1);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // Every role has finished, so the abort flag is final: let every load this CTA issued
  // land before the CTA, and its shared memory, goes away.
  if (lane == 0 && (warp == 0 || warp == 3) && *abort_flag) {  // each producer drains its own loads
    if (warp == 0) drain_wait(q_full, 0);
    for (int s = 0; s < 2; ++s) {
      if (issued_k & (1u << s)) drain_wait(&k_full[s], (par_k >> s) & 1);
      if (issued_v & (1u << s)) drain_wait(&v_full[s], (par_v >> s) & 1);
    }
  }
}

std::mutex g_mu;
bool g_attr[64] = {};
bool g_pp_ok[64] = {};    // the two-tile kernel's launch registers cover its warpgroup split
bool g_pp_ok64[64] = {};  // the same for its head-dim-64 forms

template <int HD, bool SPLIT>
bool pp_attr() {
  return cudaFuncSetAttribute(attention_pp_kernel<HD, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(PPLayout<HD>::kSmem)) == cudaSuccess;
}
// Adds 1 to `ok_count` when this form's launch registers cover its warpgroup split; false
// if the attributes cannot be read.
template <int HD, bool SPLIT>
bool pp_regs_ok(int& ok_count) {
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, attention_pp_kernel<HD, SPLIT>) != cudaSuccess) return false;
  ok_count += fa.numRegs * kThreadsPP >= kRegsNeededPP && fa.numRegs <= 168;
  return true;
}

// Makespan, in units of one one-tile CTA over the same keys, of the launch the library
// makes: for every (clip, head) in launch order, P two-tile CTAs (cost kPairCost each) and
// then its R = n_qt - 2P split-mode CTAs (split_cost), each placed on the first free SM;
// with P = -1, n_qt one-tile CTAs per (clip, head).
constexpr double kPairCost = 1.35;  // measured: 1.20 - 1.39 over 12,000 - 44,999 positions
constexpr int kMinSplitTiles = 16;  // query tiles per clip below which no mix is tried
// A split CTA walks half of a pair's keys, plus a fixed part (its start and the merge) that
// weighs more on short clips: fitted to 0.757 at 59 query tiles (7,499 positions, every
// tile split against all pairs) and 0.92 at 6 (16 clips of 749).
double split_cost(int n_qt) { return 0.74 + 1.09 / (n_qt > 0 ? n_qt : 1); }

double makespan(int n_qt, int P, uint64_t bh, int sms) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < sms; ++i) free_at.push(0.0);
  double end = 0.0;
  auto place = [&](int n, double cost) {
    for (int i = 0; i < n; ++i) {
      const double t = free_at.top() + cost;
      free_at.pop();
      free_at.push(t);
      end = t > end ? t : end;
    }
  };
  const int R = n_qt - 2 * P > 0 ? n_qt - 2 * P : 0;
  for (uint64_t c = 0; c < bh; ++c) {
    if (P < 0) {
      place(n_qt, 1.0);
    } else {
      place(P, kPairCost);
      place(R, split_cost(n_qt));
    }
  }
  return end;
}

// Pairs per (clip, head) for the two-tile kernel, the rest of the tiles in split mode, or
// -1 for the one-tile kernel: whichever of one-tile only, all pairs, no pairs (every tile
// split) and (from kMinSplitTiles query tiles up) the largest counts of pairs filling
// whole waves schedules shortest. Cached per shape.
int choose_pairs(int n_qt, uint64_t bh, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, uint64_t, int>, int> cache;
  const auto key = std::make_tuple(n_qt, bh, sms);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int all = (n_qt + 1) / 2;
  int best = -1;
  double best_t = makespan(n_qt, -1, bh, sms);
  std::vector<int> cands{all, 0};
  // The pair cost was measured on 24 - 352 key tiles per CTA; on shorter clips (6 tiles
  // for 16 clips of 60 s) a mix of pairs and one-tile CTAs ran slower than all pairs.
  if (n_qt >= kMinSplitTiles)
    for (uint64_t w = 1; w * sms <= static_cast<uint64_t>(all) * bh; ++w)
      cands.push_back(static_cast<int>(w * sms / bh));
  for (int P : cands) {
    if (P > 0 && static_cast<uint64_t>(P) * bh < 120) continue;  // too few CTAs to pair tiles
    const double t = makespan(n_qt, P, bh, sms);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = P;
    }
  }
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = best;
  return best;
}

}  // namespace

sal_status attention_launch_heads(const void* q, const void* k, const void* v, int batch, int64_t T,
                                  int64_t chunk, int heads, int head_dim, void* o, cudaStream_t s,
                                  const AttnWithhold* hold, const Windows* win) {
  if (T == 0 || batch == 0) return SAL_OK;
  if (head_dim != 64 && head_dim != 128) return SAL_ESHAPE;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev >= 0 && dev < 64 && !g_attr[dev]) {
      if (cudaFuncSetAttribute(attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_one_tile(128))) != cudaSuccess ||
          cudaFuncSetAttribute(attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_one_tile(64))) != cudaSuccess ||
          !pp_attr<128, false>() || !pp_attr<128, true>() || !pp_attr<64, false>() || !pp_attr<64, true>())
        return SAL_ECUDA;
      // setmaxnreg.inc waits until the registers it asks for are free: run the kernel only
      // if what warpgroup 0 gives back covers what the softmax warpgroups take (and the
      // launch count is one that 384 threads can get at all: at most 168)
      int r128 = 0, r64 = 0;
      if (!pp_regs_ok<128, false>(r128) || !pp_regs_ok<128, true>(r128) || !pp_regs_ok<64, false>(r64) ||
          !pp_regs_ok<64, true>(r64))
        return SAL_ECUDA;
      g_pp_ok[dev] = r128 == 2;
      g_pp_ok64[dev] = r64 == 2;
      g_attr[dev] = true;
    }
  }
  const uint64_t bh = static_cast<uint64_t>(batch) * heads;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d_bf16(&tq, q, head_dim, T, bh, 64, kTile, 1)) return SAL_ECUDA;
  if (!make_tmap_3d_bf16(&tk, k, head_dim, T, bh, 64, kTile, 1)) return SAL_ECUDA;
  if (!make_tmap_3d_bf16(&tv, v, head_dim, T, bh, 64, kTile, 1)) return SAL_ECUDA;
  AttnArgs a;
  a.T = T;
  a.chunk = chunk > 0 && chunk < T ? chunk : T;
  a.heads = heads;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  a.limit_ns = wait_limit_ns();
  a.status = device_status_ptr();
  if (!a.status) return SAL_ECUDA;
  if (hold) a.withhold = hold->tile;
  if (win && win->count > 0) {
    a.win_count = win->count;
    a.win_core = win->core;
    a.win_ctx = win->ctx;
    a.win_total = win->total;
  }
  const dim3 grid1(static_cast<unsigned>((T + kTile - 1) / kTile), static_cast<unsigned>(bh));
  // bounds-checked build: the buffers a launch may touch, declared right before it
  auto declare = [&] {
    const int64_t bytes = static_cast<int64_t>(bh) * T * head_dim * 2;  // each of q, k, v and o
    ck_declare(q, bytes, false);
    ck_declare(k, bytes, false);
    ck_declare(v, bytes, false);
    ck_declare(o, bytes, true);
  };
  if (head_dim == 64) {
    // the CTC adapter's heads: every query-tile pair to the two-tile kernel and an odd last
    // tile to a split-mode CTA of the same launch, unless it is unavailable or switched off
    bool pp64 = false;
    {
      std::lock_guard<std::mutex> lk(g_mu);
      pp64 = dev >= 0 && dev < 64 && g_pp_ok64[dev];
    }
    if (pp64 && attention_pp_mode() != 0) {
      const int n_qt = static_cast<int>((T + kTile - 1) / kTile);
      a.pairs = n_qt / 2;
      const dim3 grid(static_cast<unsigned>(n_qt / 2 + n_qt % 2), static_cast<unsigned>(bh));
      declare();
      const cudaError_t e =
          n_qt % 2 ? launch_kernel(attention_pp_kernel<64, true>, grid, dim3(kThreadsPP), PPLayout<64>::kSmem, s,
                                   tq, tk, tv, a)
                   : launch_kernel(attention_pp_kernel<64, false>, grid, dim3(kThreadsPP), PPLayout<64>::kSmem, s,
                                   tq, tk, tv, a);
      return e == cudaSuccess ? SAL_OK : SAL_ECUDA;
    }
    declare();
    return launch_kernel(attention_kernel<64>, grid1, dim3(192), smem_one_tile(64), s, tq, tk, tv, a) ==
                   cudaSuccess
               ? SAL_OK
               : SAL_ECUDA;
  }
  // The two-tile kernel takes the first P query-tile pairs of every (clip, head) and the
  // remaining tiles one CTA each in split mode (the keys split between its warpgroups),
  // all in one launch; with P = 0 the one-tile kernel takes every tile. P is chosen by
  // list scheduling (choose_pairs).
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_qt = static_cast<int>((T + kTile - 1) / kTile);
  bool pp_ok = false;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    pp_ok = dev >= 0 && dev < 64 && g_pp_ok[dev];
  }
  const int mode = attention_pp_mode();
  int P = -1;  // query-tile pairs per (clip, head) for the two-tile kernel; -1: the one-tile kernel
  if (hold) {
    if (hold->kernel == 2 && !pp_ok) return SAL_EDEVICE;
    P = hold->kernel == 2 ? (n_qt + 1) / 2 : -1;
  } else if (pp_ok && mode == 1) {
    P = (n_qt + 1) / 2;
  } else if (pp_ok && mode != 0) {
    P = choose_pairs(n_qt, bh, sms);
  }
  const int forced = hold || !pp_ok ? -1 : attention_pairs_forced();
  if (forced >= 0) P = forced < (n_qt + 1) / 2 ? forced : (n_qt + 1) / 2;
  if (P >= 0) {
    const int rest = n_qt - 2 * P > 0 ? n_qt - 2 * P : 0;
    a.pairs = P;
    const dim3 grid(static_cast<unsigned>(P + rest), static_cast<unsigned>(bh));
    declare();
    const cudaError_t e =
        rest > 0 ? launch_kernel(attention_pp_kernel<128, true>, grid, dim3(kThreadsPP), PPLayout<128>::kSmem, s,
                                 tq, tk, tv, a)
                 : launch_kernel(attention_pp_kernel<128, false>, grid, dim3(kThreadsPP), PPLayout<128>::kSmem, s,
                                 tq, tk, tv, a);
    return e == cudaSuccess ? SAL_OK : SAL_ECUDA;
  }
  declare();
  return launch_kernel(attention_kernel<128>, grid1, dim3(192), smem_one_tile(128), s, tq, tk, tv, a) ==
                 cudaSuccess
             ? SAL_OK
             : SAL_ECUDA;
}

sal_status attention_launch(const void* q, const void* k, const void* v, int batch, int64_t T,
                            int64_t chunk, void* o, cudaStream_t s, const Windows* win) {
  return attention_launch_heads(q, k, v, batch, T, chunk, kHeads, kHeadDim, o, s, nullptr, win);
}

}  // namespace sal

// Test hook: one attention launch in which every CTA's producer withholds one key/value
// tile, so that a bounded wait gives up (see sal.h).
extern "C" sal_status sal_attention_withhold(const void* q, const void* k, const void* v, int batch, int64_t T,
                                             int kernel, int tile, void* o, void* stream) {
  using namespace sal;
  const NvtxRange nvtx_("sal_attention_withhold");
  if (batch < 0 || T < 0 || tile < 0 || (kernel != 1 && kernel != 2)) return SAL_EINVAL;
  if (T > SAL_MAX_POSITIONS) return SAL_ESHAPE;
  if (batch == 0 || T == 0) return SAL_OK;
  if (batch > 6553) return SAL_ESHAPE;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SAL_EINVAL;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return SAL_ECUDA;
  if (major != 10) return SAL_EDEVICE;
  const AttnWithhold hold{kernel, tile};
  return attention_launch_heads(q, k, v, batch, T, 0, kHeads, kHeadDim, o, static_cast<cudaStream_t>(stream),
                                &hold);
}

// The split attention_launch_heads makes for 128-wide heads when the two-tile kernel is
// available (host arithmetic only; no device is touched).
extern "C" sal_status sal_attention_plan(int batch, int64_t T, int heads, int head_dim, int sms, int* pairs,
                                         int* query_tiles) {
  using namespace sal;
  if (batch < 0 || T < 0 || heads < 0 || sms <= 0 || !pairs || !query_tiles) return SAL_EINVAL;
  if (T > 2 * SAL_MAX_POSITIONS) return SAL_ESHAPE;  // the longest sequence sal_attention_heads takes
  const int n_qt = static_cast<int>((T + kTile - 1) / kTile);
  *query_tiles = n_qt;
  *pairs = 0;
  if ((head_dim != 128 && head_dim != 64) || batch == 0 || T == 0 || heads == 0) return SAL_OK;
  const uint64_t bh = static_cast<uint64_t>(batch) * heads;
  const int mode = attention_pp_mode();
  if (head_dim == 64) {  // every pair to the two-tile kernel, an odd last tile split
    *pairs = mode == 0 ? 0 : n_qt / 2;
    return SAL_OK;
  }
  int P = mode == 0 ? -1 : (mode == 1 ? (n_qt + 1) / 2 : choose_pairs(n_qt, bh, sms));
  const int forced = attention_pairs_forced();
  if (forced >= 0) P = forced < (n_qt + 1) / 2 ? forced : (n_qt + 1) / 2;
  *pairs = P > 0 ? P : 0;
  return SAL_OK;
}
