// Chunk forms of the prefill hand-off and the helpers of the tensor-memory
// kernels that run them (prefill_chunk_tc.cuh): each prompt's final state
// written as its slot's base, log entries cleared, for bf16-input handles.
//
// GDN.  Within a chunk of C tokens the delta rule unrolls into dense products (the
// WY form of a product of Householder-like factors).  With Gamma_t the
// cumulative log-decay inside the chunk, S the state at the chunk start, and
// row t of K, Q, V the chunk's keys, queries and values:
//   A[t][s] = beta_t e^{Gamma_t - Gamma_s} (k_t . k_s)      for s < t
//   (I + A) W = diag(beta e^{Gamma}) K,   (I + A) U = diag(beta) V
//   B = U - W S                        (rows: the delta-corrected b_t)
//   O = diag(e^{Gamma}) Q S + (Q K^T (.) [e^{Gamma_t - Gamma_s}]_{s<=t}) B
//   S <- e^{Gamma_end} S + (diag(e^{Gamma_end - Gamma}) K)^T B
// Every exponent is <= 0, so no cumulative decay is ever divided by.  This
// restates the recurrence of the eager step over C tokens at once; the
// tokens' b_t and o_t are those of the recurrence (same arithmetic, other
// summation order).
//
// KDA and RWKV6.  With Gamma_t in R^{d_k} the cumulative log-decay inside a chunk, S the state
// at the chunk start and rows t of K, Q (r for RWKV6) and V the chunk's keys,
// queries and values, the C tokens unroll into dense products.
//
// KDA (per-key gated delta rule), for s < t:
//   A[t][s] = beta_t sum_j k_tj k_sj e^{Gamma_tj - Gamma_sj}
//   (I + A) W = diag(beta) (e^{Gamma} (.) K),   (I + A) U = diag(beta) V
//   B = U - W S                                 (rows: the delta-corrected b_t)
//   P[t][s] = sum_j q_tj k_sj e^{Gamma_tj - Gamma_sj}          (s <= t)
//   O = (e^{Gamma} (.) Q) S + P B
//   S <- diag(e^{Gamma_end}) S + (e^{Gamma_end - Gamma} (.) K)^T B
// RWKV6 (raw update, output from the state before the token):
//   P[t][s] = sum_j r_tj k_sj e^{Gamma_{t-1,j} - Gamma_sj}      (s < t)
//   P[t][t] = (u (.) k_t) . r_t
//   O = (e^{Gamma_{t-1}} (.) R) S + P V
//   S <- diag(e^{Gamma_end}) S + (e^{Gamma_end - Gamma} (.) K)^T V
// These restate the per-token recurrences of the eager step over C tokens at
// once (same values, other summation order).
//
// Every exponent is <= 0.  The pair weights e^{Gamma_t - Gamma_s} differ per
// key, so they cannot be split into a row factor and a column factor without
// dividing by a cumulative decay (which overflows fp32 for strongly decaying
// keys).  A and P are therefore formed pair by pair on the SIMT lanes, one
// exp2 per (pair, key), shared by A and P for KDA; only the products with the
// state, W and B run on the tensor cores (tf32 operands, fp32 accumulation).
#pragma once

#include <cuda_bf16.h>
#include <mma.h>

#include <type_traits>

#include "prefill.cuh"

namespace dl {

namespace wm = nvcuda::wmma;

// Output tiles (i, j) of an (M x N) product, 16 x 16 each, spread over the
// CTA's warps.
template <int M, int N, typename F>
__device__ __forceinline__ void for_tiles(F tile_fn) {
  constexpr int TN = N / 16, TILES = (M / 16) * TN;
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int tile = warp; tile < TILES; tile += nw) tile_fn(tile / TN, tile % TN);
}

using AccBf = wm::fragment<wm::accumulator, 16, 16, 16, float>;   // of bf16 products
using BfA = wm::fragment<wm::matrix_a, 16, 16, 16, __nv_bfloat16, wm::row_major>;
using BfBc = wm::fragment<wm::matrix_b, 16, 16, 16, __nv_bfloat16, wm::col_major>;

// X Y^T of two bf16 row-major [C][LDK] blocks (rows 16i.. of X, 16j.. of Y)
// into an fp32 [C][LDA] block; tiles above the diagonal are zero.
template <int C, int DK, int LDK, int LDA>
__device__ __forceinline__ void lower_xyt(const __nv_bfloat16* X, const __nv_bfloat16* Y, float* out) {
  for_tiles<C, C>([&](int i, int j) {
    AccBf acc;
    wm::fill_fragment(acc, 0.f);
    if (j <= i) {
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        BfA fa;
        BfBc fb;
        wm::load_matrix_sync(fa, X + (16 * i) * LDK + kk, LDK);
        wm::load_matrix_sync(fb, Y + (16 * j) * LDK + kk, LDK);
        wm::mma_sync(acc, fa, fb, acc);
      }
    }
    wm::store_matrix_sync(out + (16 * i) * LDA + 16 * j, acc, LDA, wm::mem_row_major);
  });
}

__device__ __forceinline__ bool aligned_to(const void* p, unsigned bytes) {
  return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) == 0;
}

// 16-byte asynchronous global -> shared copy; bytes < 16 zero-fills the rest
// (0: the destination becomes zeros and nothing is read).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(gmem_u64(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 2^x on the SFU (ex2.approx, flushes subnormal results to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Eight bf16 of a 16-byte-aligned shared row as floats.
__device__ __forceinline__ void bf16x8_to_f32(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Four bf16 of an 8-byte-aligned shared row as floats.
__device__ __forceinline__ void bf16x4_to_f32(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
}

// (t, s) of strict lower-triangle pair p = t (t - 1) / 2 + s, 0 <= s < t.
__device__ __forceinline__ void strict_pair(int p, int& t, int& s) {
  t = static_cast<int>((1.f + sqrtf(8.f * static_cast<float>(p) + 1.f)) * 0.5f);
  while (t * (t - 1) / 2 > p) --t;
  while ((t + 1) * t / 2 <= p) ++t;
  s = p - t * (t - 1) / 2;
}

// tf32 warp-MMA fragments (16 x 16 x 8) for the split-precision products
using TfA = wm::fragment<wm::matrix_a, 16, 16, 8, wm::precision::tf32, wm::row_major>;
using TfBc = wm::fragment<wm::matrix_b, 16, 16, 8, wm::precision::tf32, wm::col_major>;
using AccTf = wm::fragment<wm::accumulator, 16, 16, 8, float>;

// x = hi + lo with hi and lo both tf32 (hi the rounding of x)
template <typename Frag>
__device__ __forceinline__ void split_tf32(Frag& hi, Frag& lo) {
#pragma unroll
  for (int i = 0; i < hi.num_elements; ++i) {
    const float x = hi.x[i];
    hi.x[i] = wm::__float_to_tf32(x);
    lo.x[i] = wm::__float_to_tf32(x - hi.x[i]);
  }
}

// acc = X Y^T over columns [k0, k0 + KN) of fp32 X, Y [16][ldm], on one
// warp, to about fp32 accuracy: with X = Xh + Xl and Y = Yh + Yl split into
// tf32 parts, the sum Xl Yh + Xh Yl + Xh Yh (the Xl Yl term is below fp32
// rounding).
template <int KN>
__device__ __forceinline__ void xyt_split_tf32(const float* X, const float* Y, int ldm, int k0, AccTf& acc) {
  wm::fill_fragment(acc, 0.f);
#pragma unroll
  for (int k = k0; k < k0 + KN; k += 8) {
    TfA xh, xl;
    TfBc yh, yl;
    wm::load_matrix_sync(xh, X + k, ldm);
    wm::load_matrix_sync(yh, Y + k, ldm);
    split_tf32(xh, xl);
    split_tf32(yh, yl);
    wm::mma_sync(acc, xl, yh, acc);
    wm::mma_sync(acc, xh, yl, acc);
    wm::mma_sync(acc, xh, yh, acc);
  }
}

// A (KDA: beta_t-weighted, strictly lower) and P (lower; RWKV6: strictly
// lower plus the bonus diagonal) of one 32-token chunk, Gamma in log2 units;
// the upper triangles zero, P tf32-rounded.
//
// A pair (t, s) with a token r between them (s <= r < t) factors as
// 2^{Gamma_t - Gamma_s} = 2^{Gamma_t - Gamma_r} 2^{Gamma_r - Gamma_s}, both
// exponents <= 0 (Gamma_{t-1} in place of Gamma_t for RWKV6's P, with
// r <= t - 1), so a block of such pairs is a product of rows each scaled once
// and no cumulative decay is divided by.  Blocks, by level:
//   1. t >= 16 > s through token 15 (a 16 x 16 block);
//   2. (256 threads) inside each half, t in its second quarter and s in its
//      first, through token 7 or 23 (two 8 x 8 blocks, the diagonal blocks
//      of one 16 x 16 product).
// Each level's rows (Ks: keys s; Kt: beta_t-weighted keys t, KDA; Qt:
// queries t; fp32 [16][LDX]) are products on warp MMAs in split tf32, four
// warps a product (KDA: warps 0-3 A, 4-7 P; RWKV6: warps 0-3 P), each over a
// quarter of the keys, with partial blocks in sXA and sXP (fp32 [4][16][16]).
// The strict pairs left inside the quarters (112; 240 inside the halves at
// 512 threads) and the 32 diagonal pairs take one exp2 per (pair, key) on the
// SIMT lanes, a strict pair split over two adjacent lanes by keys: one item a
// thread.  The second level pays at two CTAs an SM (B=64 L=512 on B200: KDA
// +8%, RWKV6 +9% at d = 64 and +15% at d = 128) and costs 4% at one
// 512-thread CTA an SM, whose threads the first level's items already fill.
// Two block barriers inside (four with the second level); the caller
// synchronises after the call.
template <int OP, int DK, int C, int NT, int LDK, int LDG, int LDA, int LDX>
__device__ __forceinline__ void key_pair_phase(const __nv_bfloat16* sK, const __nv_bfloat16* sQ, const float* sG,
                                               const float* sBeta, const float* sBonus, float* sKs, float* sKt,
                                               float* sQt, float* sXA, float* sXP, float* sA, float* sP) {
  static_assert(C == 32, "halves of 16 tokens, quarters of 8");
  static_assert(LDX % 4 == 0 && LDA % 4 == 0, "warp-MMA leading dimensions");
  static_assert(NT == 256 || NT == 512, "eight or sixteen warps");
  constexpr bool DELTA = OP == OP_KDA;
  const int tid = threadIdx.x, warp = tid >> 5;

  // the rows of one level: row i pairs key s, token t and reference r
  auto scale_rows = [&](int level) {
    for (int idx = tid; idx < 16 * DK / 4; idx += NT) {
      const int i = idx / (DK / 4), j = 4 * (idx % (DK / 4));
      const int s = level == 1 ? i : 16 * (i >> 3) + (i & 7);
      const int t = level == 1 ? 16 + i : s + 8;
      const int r = level == 1 ? 15 : 16 * (i >> 3) + 7;
      const float4 gm = *reinterpret_cast<const float4*>(sG + r * LDG + j);
      const float4 gs = *reinterpret_cast<const float4*>(sG + s * LDG + j);
      const float4 gt = *reinterpret_cast<const float4*>(sG + (DELTA ? t : t - 1) * LDG + j);
      const float es[4] = {ex2_approx(gm.x - gs.x), ex2_approx(gm.y - gs.y), ex2_approx(gm.z - gs.z),
                           ex2_approx(gm.w - gs.w)};
      const float et[4] = {ex2_approx(gt.x - gm.x), ex2_approx(gt.y - gm.y), ex2_approx(gt.z - gm.z),
                           ex2_approx(gt.w - gm.w)};
      float ks[4], kt[4], qt[4];
      bf16x4_to_f32(sK + s * LDK + j, ks);
      bf16x4_to_f32(sQ + t * LDK + j, qt);
      *reinterpret_cast<float4*>(sKs + i * LDX + j) =
          make_float4(ks[0] * es[0], ks[1] * es[1], ks[2] * es[2], ks[3] * es[3]);
      *reinterpret_cast<float4*>(sQt + i * LDX + j) =
          make_float4(qt[0] * et[0], qt[1] * et[1], qt[2] * et[2], qt[3] * et[3]);
      if (DELTA) {
        bf16x4_to_f32(sK + t * LDK + j, kt);
        const float bt = sBeta[t];
        *reinterpret_cast<float4*>(sKt + i * LDX + j) =
            make_float4(bt * kt[0] * et[0], bt * kt[1] * et[1], bt * kt[2] * et[2], bt * kt[3] * et[3]);
      }
    }
  };
  // the level's 16 x 16 products, partial sums a quarter of the keys each
  auto products = [&]() {
    if (warp < (DELTA ? 8 : 4)) {
      const bool isA = DELTA && warp < 4;
      const int w4 = warp & 3;
      AccTf acc;
      xyt_split_tf32<DK / 4>(isA ? sKt : sQt, sKs, LDX, w4 * (DK / 4), acc);
      wm::store_matrix_sync((isA ? sXA : sXP) + w4 * 256, acc, 16, wm::mem_row_major);
    }
  };
  // entry e of the 16 x 16 product into (t, s)
  auto sum_entry = [&](int e, int t, int s) {
    sP[t * LDA + s] = wm::__float_to_tf32((sXP[e] + sXP[256 + e]) + (sXP[512 + e] + sXP[768 + e]));
    if (DELTA) sA[t * LDA + s] = (sXA[e] + sXA[256 + e]) + (sXA[512 + e] + sXA[768 + e]);
  };

  constexpr bool TWO = NT == 256;             // the second level of blocks
  scale_rows(1);
  __syncthreads();
  products();
  if (TWO) {
    __syncthreads();
    for (int idx = tid; idx < 256; idx += NT) sum_entry(idx, 16 + (idx >> 4), idx & 15);
    scale_rows(2);
    __syncthreads();
    products();
  }

  // the strict pairs left (two lanes each) and the diagonal, one item a thread
  constexpr int BS = TWO ? 8 : 16;              // the blocks they sit in
  constexpr int NPB = BS * (BS - 1) / 2, KS = 2;
  constexpr int NSPLIT = (C / BS) * NPB * KS, NI = NSPLIT + C;
  static_assert(NI == NT && NSPLIT % 32 == 0, "one round, warp-uniform kinds");
  {
    const int p = tid;
    float accA = 0.f, accP = 0.f;
    int t = 0, s = 0;
    const bool split = p < NSPLIT;
    if (split) {   // strict pair inside a block, keys [j0, j0 + DK / KS)
      const int q = p / KS, b = q / NPB;
      strict_pair(q - NPB * b, t, s);
      t += BS * b;
      s += BS * b;
      const int j0 = (p % KS) * (DK / KS);
      const __nv_bfloat16* kt = sK + t * LDK;
      const __nv_bfloat16* ks = sK + s * LDK;
      const __nv_bfloat16* qt = sQ + t * LDK;
      const float* gt = sG + (OP == OP_RWKV6 ? t - 1 : t) * LDG;
      const float* gs = sG + s * LDG;
#pragma unroll 2
      for (int j = j0; j < j0 + DK / KS; j += 8) {
        float fks[8], fqt[8], fkt[8];
        bf16x8_to_f32(ks + j, fks);
        bf16x8_to_f32(qt + j, fqt);
        if (DELTA) bf16x8_to_f32(kt + j, fkt);
        const float4 gt0 = *reinterpret_cast<const float4*>(gt + j);
        const float4 gt1 = *reinterpret_cast<const float4*>(gt + j + 4);
        const float4 gs0 = *reinterpret_cast<const float4*>(gs + j);
        const float4 gs1 = *reinterpret_cast<const float4*>(gs + j + 4);
        const float d[8] = {gt0.x - gs0.x, gt0.y - gs0.y, gt0.z - gs0.z, gt0.w - gs0.w,
                            gt1.x - gs1.x, gt1.y - gs1.y, gt1.z - gs1.z, gt1.w - gs1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float m = fks[e] * ex2_approx(d[e]);
          if (DELTA) accA = fmaf(fkt[e], m, accA);
          accP = fmaf(fqt[e], m, accP);
        }
      }
    } else {   // diagonal: q_t . k_t (KDA), (u (.) k_t) . r_t (RWKV6)
      t = s = p - NSPLIT;
      const __nv_bfloat16* kt = sK + t * LDK;
      const __nv_bfloat16* qt = sQ + t * LDK;
#pragma unroll 2
      for (int j = 0; j < DK; j += 8) {
        float fkt[8], fqt[8];
        bf16x8_to_f32(kt + j, fkt);
        bf16x8_to_f32(qt + j, fqt);
#pragma unroll
        for (int e = 0; e < 8; ++e) accP = fmaf(fqt[e], OP == OP_RWKV6 ? sBonus[j + e] * fkt[e] : fkt[e], accP);
      }
    }
    // every lane of the warp reaches the shuffles
#pragma unroll
    for (int o = 1; o < KS; o <<= 1) {
      const float oA = __shfl_xor_sync(0xffffffffu, accA, o), oP = __shfl_xor_sync(0xffffffffu, accP, o);
      if (split) {
        accA += oA;
        accP += oP;
      }
    }
    if (!split || p % KS == 0) {
      if (DELTA && s < t) sA[t * LDA + s] = sBeta[t] * accA;
      sP[t * LDA + s] = wm::__float_to_tf32(accP);
    }
  }
  __syncthreads();   // the last level's partial blocks are stored
  if (TWO) {
    for (int idx = tid; idx < 128; idx += NT) {   // the two 8 x 8 diagonal blocks of that product
      const int b = idx >> 6, r = (idx >> 3) & 7, c = idx & 7;
      sum_entry((8 * b + r) * 16 + 8 * b + c, 16 * b + 8 + r, 16 * b + c);
    }
  } else {
    for (int idx = tid; idx < 256; idx += NT) sum_entry(idx, 16 + (idx >> 4), idx & 15);
  }
  for (int idx = tid; idx < C * C; idx += NT) {
    const int t = idx / C, s = idx % C;
    if (s > t) sP[t * LDA + s] = 0.f;
    if (DELTA && s >= t) sA[t * LDA + s] = 0.f;
  }
}

}  // namespace dl
