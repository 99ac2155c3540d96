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

// A (KDA: beta_t-weighted, strictly lower) and P (lower; RWKV6: strictly
// lower plus the bonus diagonal) of one chunk, pair by pair with one exp2 per
// (pair, key) from Gamma in log2 units; the upper triangles zero.  P is stored
// tf32-rounded.  When twice the strict pairs plus the diagonal make exactly
// one item per thread, each strict pair is split between two adjacent lanes,
// one half of the keys each.
template <int OP, int DK, int C, int NT, int LDK, int LDG, int LDA>
__device__ __forceinline__ void key_pair_phase(const __nv_bfloat16* sK, const __nv_bfloat16* sQ, const float* sG,
                                               const float* sBeta, const float* sBonus, float* sA, float* sP) {
  constexpr bool DELTA = OP == OP_KDA;
  const int tid = threadIdx.x;
  constexpr int NSTRICT = C * (C - 1) / 2;
  constexpr bool SPLIT = 2 * NSTRICT + C == NT;
  constexpr int NITEMS = SPLIT ? NT : NSTRICT + C;
  for (int p = tid; p < NITEMS; p += NT) {
    const int nstr = SPLIT ? 2 * NSTRICT : NSTRICT;   // strict items come first
    const bool strict = p < nstr;
    int t, s;
    if (strict) {
      strict_pair(SPLIT ? p >> 1 : p, t, s);
    } else {
      t = s = p - nstr;
    }
    const int j0 = SPLIT && strict ? (p & 1) * (DK / 2) : 0;
    const int j1 = SPLIT && strict ? j0 + DK / 2 : DK;
    const __nv_bfloat16* kt = sK + t * LDK;
    const __nv_bfloat16* ks = sK + s * LDK;
    const __nv_bfloat16* qt = sQ + t * LDK;
    float accA = 0.f, accP = 0.f;
    if (strict) {
      // exponent rows: Gamma_t (KDA) or Gamma_{t-1} (RWKV6), against Gamma_s
      const float* gt = sG + (OP == OP_RWKV6 ? t - 1 : t) * LDG;
      const float* gs = sG + s * LDG;
#pragma unroll 2
      for (int j = j0; j < j1; j += 8) {
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
    } else {
      // diagonal: q_t . k_t (KDA), (u (.) k_t) . r_t (RWKV6)
#pragma unroll 2
      for (int j = 0; j < DK; j += 8) {
        float fkt[8], fqt[8];
        bf16x8_to_f32(kt + j, fkt);
        bf16x8_to_f32(qt + j, fqt);
#pragma unroll
        for (int e = 0; e < 8; ++e) accP = fmaf(fqt[e], OP == OP_RWKV6 ? sBonus[j + e] * fkt[e] : fkt[e], accP);
      }
    }
    if (SPLIT) {   // one item per thread: every lane of the warp reaches the shuffles
      const float oA = __shfl_xor_sync(0xffffffffu, accA, 1), oP = __shfl_xor_sync(0xffffffffu, accP, 1);
      if (strict) {
        accA += oA;
        accP += oP;
      }
    }
    if (!SPLIT || !strict || (p & 1) == 0) {
      if (DELTA && strict) sA[t * LDA + s] = sBeta[t] * accA;
      sP[t * LDA + s] = wm::__float_to_tf32(accP);
    }
  }
  for (int idx = tid; idx < C * C; idx += NT) {
    const int t = idx / C, s = idx % C;
    if (s > t) sP[t * LDA + s] = 0.f;
    if (DELTA && s >= t) sA[t * LDA + s] = 0.f;
  }
}

}  // namespace dl
