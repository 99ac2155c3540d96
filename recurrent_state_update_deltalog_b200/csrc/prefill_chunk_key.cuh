// Chunked KDA and RWKV6 prefill on tensor cores: the hand-off of
// prefill_kernel (each prompt's final state written as its slot's base, log
// entries cleared) for bf16-input handles whose decay is per key.
//
// With Gamma_t in R^{d_k} the cumulative log-decay inside a chunk, S the state
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
//
// One CTA per (row, head, value tile) keeps its d_k x VT state slice in shared
// memory for the whole prompt, with K, Q, V and the gates of the next chunk
// streaming in (cp.async, double-buffered).  Two geometries:
//   VT = 128: a whole 128 x 128 head per 512-thread CTA, 32-token chunks, one
//     CTA per SM (the key-side work is done once per head);
//   VT = 64: 256-thread CTAs, two per SM; 32-token chunks at d_k = 64, 16 at
//     d_k = 128 (to fit two CTAs).  Where a C x 64 product has fewer 16 x 16
//     output tiles than the CTA has warps, its contraction is split between
//     two warps per tile.
#pragma once

#include <type_traits>

#include "prefill_chunk.cuh"

namespace dl {

template <int DK, int VT_>
struct KeyChunkGeom {
  // value columns per CTA: 128 (a whole d_v = 128 head, 512 threads, one CTA
  // per SM) or 64 (256 threads, two CTAs per SM)
  static constexpr int VT = VT_;
  static constexpr int C = DK == 128 && VT == 64 ? 16 : 32;   // tokens per chunk
  static constexpr int NT = VT == 128 ? 512 : 256, NW = NT / 32;   // threads, warps
  static constexpr int MINB = NT == 512 ? 1 : 2;                    // resident CTAs per SM
  static constexpr int LDK = DK + 8;    // bf16 row stride of K and Q (16-byte multiple)
  static constexpr int LDV = VT + 8;    // bf16 row stride of the V tile
  static constexpr int LDS = VT + 8;    // fp32 row stride of the state tile, U and B
  static constexpr int LDG = DK + 4;    // fp32 row stride of the gates / Gamma
  static constexpr int LDA = C + 4;     // fp32 row stride of A and P
  static constexpr int LDW = DK + 4;    // fp32 row stride of W and the scaled queries
  static constexpr int LDT = C + 4;     // fp32 row stride of the scaled keys, stored transposed
  static constexpr size_t al(size_t x) { return (x + 127) & ~size_t(127); }
  static constexpr size_t K_BYTES = al(size_t(C) * LDK * 2);
  static constexpr size_t V_BYTES = al(size_t(C) * LDV * 2);
  static constexpr size_t G_BYTES = al(size_t(C) * LDG * 4);
  // K, Q, V and the gates are double-buffered: buffer (chunk index & 1)
  static constexpr size_t S_OFF = 0;
  static constexpr size_t K_OFF = al(size_t(DK) * LDS * 4);
  static constexpr size_t Q_OFF = K_OFF + 2 * K_BYTES;
  static constexpr size_t V_OFF = Q_OFF + 2 * K_BYTES;
  static constexpr size_t G_OFF = V_OFF + 2 * V_BYTES;
  static constexpr size_t A_OFF = G_OFF + 2 * G_BYTES;
  static constexpr size_t P_OFF = al(A_OFF + size_t(C) * LDA * 4);
  static constexpr size_t W_FLOATS = size_t(C) * LDW > size_t(DK) * LDT ? size_t(C) * LDW : size_t(DK) * LDT;
  static constexpr size_t W_OFF = al(P_OFF + size_t(C) * LDA * 4);
  static constexpr size_t U_OFF = al(W_OFF + W_FLOATS * 4);
  static constexpr size_t E_OFF = al(U_OFF + size_t(C) * LDS * 4);   // e^{Gamma_end} [DK], u [DK], beta [C]
  static constexpr size_t BYTES = al(E_OFF + (2 * DK + C) * 4);
  static constexpr int TILES = (C / 16) * (VT / 16);   // 16 x 16 tiles of a C x VT product
  static constexpr int KSPLIT = NW / TILES;            // warps per such tile
  static_assert(TILES * KSPLIT == NW, "a C x VT product must cover the warps exactly");
};

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

template <int OP, int DK, int DV, int VT_>
__global__ void __launch_bounds__(KeyChunkGeom<DK, VT_>::NT, KeyChunkGeom<DK, VT_>::MINB)
    key_chunk_prefill_kernel(const PrefillArgs a) {
  using G = KeyChunkGeom<DK, VT_>;
  constexpr int C = G::C, VT = G::VT, NSPLIT = DV / VT;
  constexpr bool DELTA = OP == OP_KDA;
  constexpr float LOG2E = 1.4426950408889634f;
  static_assert(OP == OP_KDA || OP == OP_RWKV6, "per-key decay operators");
  static_assert(DV % VT == 0 && DK % 16 == 0, "chunk tile shape");
  extern __shared__ __align__(128) unsigned char smem[];
  float* sS = reinterpret_cast<float*>(smem + G::S_OFF);   // [DK][LDS] state slice
  auto kbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::K_OFF + b * G::K_BYTES); };
  auto qbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::Q_OFF + b * G::K_BYTES); };
  auto vbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::V_OFF + b * G::V_BYTES); };
  auto gbuf = [&](int b) { return reinterpret_cast<float*>(smem + G::G_OFF + b * G::G_BYTES); };
  float* sA = reinterpret_cast<float*>(smem + G::A_OFF);   // [C][LDA] A (KDA)
  float* sP = reinterpret_cast<float*>(smem + G::P_OFF);   // [C][LDA] P
  float* sW = reinterpret_cast<float*>(smem + G::W_OFF);   // [C][LDW] W, then scaled Q; [DK][LDT] scaled K^T
  float* sU = reinterpret_cast<float*>(smem + G::U_OFF);   // [C][LDS] U, then B
  float* sE = reinterpret_cast<float*>(smem + G::E_OFF);   // [DK] e^{Gamma_end}
  float* sBonus = sE + DK;                                 // [DK] u (RWKV6)
  float* sBeta = sE + 2 * DK;                              // [C] beta (KDA)
  __shared__ __align__(32) float s_patch[G::NW][16 * 16];  // per-warp tile

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = static_cast<int>(blockIdx.x) / NSPLIT;
  const int col0 = (static_cast<int>(blockIdx.x) % NSPLIT) * VT;
  const int r = blockIdx.y;

  const int slot = a.slot_idx ? __ldg(a.slot_idx + r) : r;
  if (slot < 0) return;
  if (slot >= a.slots) {
    if (tid == 0) atomicOr(a.err, kErrSlotIndex);
    return;
  }
  const long t0 = __ldg(a.cu_seqlens + r), t1 = __ldg(a.cu_seqlens + r + 1);
  if (t0 < 0 || t1 < t0 || t1 > a.total) {
    if (tid == 0) atomicOr(a.err, kErrSeqlen);
    return;
  }
  const long sh = static_cast<long>(slot) * a.H + h;
  float* Sg = a.Sbar + sh * (DK * DV) + col0;

  for (int idx = tid; idx < DK * VT / 4; idx += G::NT) {
    const int row = idx / (VT / 4), c4 = idx % (VT / 4);
    const float4 x = a.zero_state ? make_float4(0.f, 0.f, 0.f, 0.f) : ld_state(Sg + row * DV + 4 * c4);
    *reinterpret_cast<float4*>(&sS[row * G::LDS + 4 * c4]) = x;
  }
  if (OP == OP_RWKV6)
    for (int j = tid; j < DK; j += G::NT) sBonus[j] = a.u[h * DK + j];

  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* Og = static_cast<__nv_bfloat16*>(a.o);

  // Stage rows [c, c + C) of a [total][H][stride] input (columns off..off +
  // width) into dst; rows past the prompt are zeros.  16-byte async copies
  // when every input allows them.
  const bool async_ok = aligned_to(a.q, 16) && aligned_to(a.k, 16) && aligned_to(a.v, 16) &&
                        aligned_to(a.log_decay, 16);
  auto stage_rows = [&](auto* dst, const auto* src, long c, int width, int ld, int stride, int off) {
    using T = typename std::remove_const<typename std::remove_pointer<decltype(src)>::type>::type;
    constexpr int PER_SEG = 16 / static_cast<int>(sizeof(T));
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
    if (async_ok) {
      const int seg_per_row = width / PER_SEG;
      for (int idx = tid; idx < C * seg_per_row; idx += G::NT) {
        const int t = idx / seg_per_row, seg = idx % seg_per_row;
        const long row = ((c + (t < nv ? t : nv - 1)) * a.H + h) * stride + off + PER_SEG * seg;
        cp_async16(dst + t * ld + PER_SEG * seg, src + row, t < nv ? 16u : 0u);
      }
    } else {
      for (int idx = tid; idx < C * width; idx += G::NT) {
        const int t = idx / width, j = idx % width;
        dst[t * ld + j] = t < nv ? src[((c + t) * a.H + h) * stride + off + j] : T(0.f);
      }
    }
  };
  auto stage = [&](int b, long c) {
    stage_rows(kbuf(b), Kg, c, DK, G::LDK, DK, 0);
    stage_rows(qbuf(b), Qg, c, DK, G::LDK, DK, 0);
    stage_rows(vbuf(b), Vg, c, VT, G::LDV, DV, col0);
    stage_rows(gbuf(b), a.log_decay, c, DK, G::LDG, DK, 0);
  };
  float bnext = 0.f;   // beta of row tid of the next chunk (KDA)
  if (t0 < t1) {
    stage(0, t0);
    if (DELTA && tid < C && t0 + tid < t1) bnext = a.beta[(t0 + tid) * a.H + h];
  }
  cp_async_commit();

  // One copy group per chunk: chunk c + 1's inputs are committed at the start
  // of chunk c, into the buffers chunk c - 1 used.
  int buf = 0;
  for (long c0 = t0; c0 < t1; c0 += C, buf ^= 1) {
    const int n = static_cast<int>(t1 - c0 < C ? t1 - c0 : C);   // valid rows of this chunk
    const bool has_next = c0 + C < t1;
    __syncthreads();   // the previous chunk is done with buffer buf ^ 1 and every work buffer
    if (has_next) stage(buf ^ 1, c0 + C);
    cp_async_commit();
    if (DELTA && tid < C) {
      sBeta[tid] = bnext;
      bnext = has_next && c0 + C + tid < t1 ? a.beta[(c0 + C + tid) * a.H + h] : 0.f;
    }
    cp_async_wait<1>();   // this chunk's group has landed
    __syncthreads();
    const __nv_bfloat16 *sK = kbuf(buf), *sQ = qbuf(buf), *sV = vbuf(buf);
    float* sG = gbuf(buf);

    // 1. Gamma, in log2 units: per key, the inclusive prefix sum of the
    // chunk's log-gates (rows past the prompt hold zero gates), in place
    for (int j = tid; j < DK; j += G::NT) {
      float run = 0.f;
#pragma unroll 4
      for (int t = 0; t < C; ++t) {
        run = fmaf(sG[t * G::LDG + j], LOG2E, run);
        sG[t * G::LDG + j] = run;
      }
      sE[j] = ex2_approx(run);
    }
    __syncthreads();

    // 2. A and P pair by pair; the upper triangles zero; right-hand sides
    key_pair_phase<OP, DK, C, G::NT, G::LDK, G::LDG, G::LDA>(sK, sQ, sG, sBeta, sBonus, sA, sP);
    // four consecutive columns per thread in the element-wise passes below
    if (DELTA) {
      // beta (e^{Gamma} (.) K) into W, beta V into U
      for (int idx = tid; idx < C * DK / 4; idx += G::NT) {
        const int t = idx / (DK / 4), j = 4 * (idx % (DK / 4));
        const float4 g = *reinterpret_cast<const float4*>(sG + t * G::LDG + j);
        float k4[4];
        bf16x4_to_f32(sK + t * G::LDK + j, k4);
        const float bt = sBeta[t];
        *reinterpret_cast<float4*>(sW + t * G::LDW + j) =
            make_float4(bt * ex2_approx(g.x) * k4[0], bt * ex2_approx(g.y) * k4[1], bt * ex2_approx(g.z) * k4[2],
                        bt * ex2_approx(g.w) * k4[3]);
      }
      for (int idx = tid; idx < C * VT / 4; idx += G::NT) {
        const int t = idx / (VT / 4), c = 4 * (idx % (VT / 4));
        float v4[4];
        bf16x4_to_f32(sV + t * G::LDV + c, v4);
        const float bt = sBeta[t];
        *reinterpret_cast<float4*>(sU + t * G::LDS + c) = make_float4(bt * v4[0], bt * v4[1], bt * v4[2], bt * v4[3]);
      }
    } else {
      for (int idx = tid; idx < C * VT / 4; idx += G::NT) {   // B = V, a tf32 operand (bf16 is tf32-exact)
        const int t = idx / (VT / 4), c = 4 * (idx % (VT / 4));
        float v4[4];
        bf16x4_to_f32(sV + t * G::LDV + c, v4);
        *reinterpret_cast<float4*>(sU + t * G::LDS + c) = make_float4(v4[0], v4[1], v4[2], v4[3]);
      }
    }
    __syncthreads();

    // warp -> (output tile, contraction part) of a C x VT product
    constexpr int TJ = VT / 16;
    const int tile = warp % G::TILES, part = warp / G::TILES;
    const int ti = tile / TJ, tj = tile % TJ;
    constexpr int KR = DK / G::KSPLIT;   // contraction range of a part

    if (DELTA) {
      // 3. (I + A) X = R, one right-hand-side column per thread (W is a tf32
      // operand later and is stored tf32-rounded; U stays fp32)
      if (tid < DK + VT) {
        const bool isw = tid < DK;
        float* col = isw ? sW + tid : sU + (tid - DK);
        const int ld = isw ? G::LDW : G::LDS;
        float x[C];
#pragma unroll
        for (int t = 0; t < C; ++t) {
          float acc0 = col[t * ld], acc1 = 0.f;
          const float* arow = sA + t * G::LDA;
#pragma unroll
          for (int s = 0; s + 3 < t; s += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(arow + s);
            acc0 = fmaf(-a4.x, x[s], acc0);
            acc1 = fmaf(-a4.y, x[s + 1], acc1);
            acc0 = fmaf(-a4.z, x[s + 2], acc0);
            acc1 = fmaf(-a4.w, x[s + 3], acc1);
          }
#pragma unroll
          for (int s = t & ~3; s < t; ++s) acc0 = fmaf(-arow[s], x[s], acc0);
          x[t] = acc0 + acc1;
          col[t * ld] = isw ? wm::__float_to_tf32(x[t]) : x[t];
        }
      }
      __syncthreads();

      // 4. B = U - W S
      AccTf acc;
      wm::fill_fragment(acc, 0.f);
#pragma unroll 4
      for (int kk = part * KR; kk < (part + 1) * KR; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * ti) * G::LDW + kk, G::LDW);
        wm::load_matrix_sync(fb, sS + kk * G::LDS + 16 * tj, G::LDS);
        to_tf32(fb);
        wm::mma_sync(acc, fa, fb, acc);
      }
      if (part > 0) wm::store_matrix_sync(s_patch[warp], acc, 16, wm::mem_row_major);
      __syncthreads();
      if (part == 0) {
#pragma unroll
        for (int q = 1; q < G::KSPLIT; ++q) {
          AccTf other;
          wm::load_matrix_sync(other, s_patch[warp + q * G::TILES], 16, wm::mem_row_major);
#pragma unroll
          for (int e = 0; e < acc.num_elements; ++e) acc.x[e] += other.x[e];
        }
        AccTf u;
        float* p = sU + (16 * ti) * G::LDS + 16 * tj;
        wm::load_matrix_sync(u, p, G::LDS, wm::mem_row_major);
#pragma unroll
        for (int e = 0; e < u.num_elements; ++e) u.x[e] = wm::__float_to_tf32(u.x[e] - acc.x[e]);
        wm::store_matrix_sync(p, u, G::LDS, wm::mem_row_major);
      }
      __syncthreads();
    }

    // 5. the scaled queries e^{Gamma_t} (.) q_t (KDA), e^{Gamma_{t-1}} (.) r_t (RWKV6) into W
    for (int idx = tid; idx < C * DK / 4; idx += G::NT) {
      const int t = idx / (DK / 4), j = 4 * (idx % (DK / 4));
      const int tg = OP == OP_KDA ? t : t - 1;
      const float4 g = tg >= 0 ? *reinterpret_cast<const float4*>(sG + tg * G::LDG + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      float q4[4];
      bf16x4_to_f32(sQ + t * G::LDK + j, q4);
      *reinterpret_cast<float4*>(sW + t * G::LDW + j) =
          make_float4(wm::__float_to_tf32(ex2_approx(g.x) * q4[0]), wm::__float_to_tf32(ex2_approx(g.y) * q4[1]),
                      wm::__float_to_tf32(ex2_approx(g.z) * q4[2]), wm::__float_to_tf32(ex2_approx(g.w) * q4[3]));
    }
    __syncthreads();

    // 6. O = (scaled Q) S + P B, rows < n to global through the warp's patch
    {
      AccTf acc;
      wm::fill_fragment(acc, 0.f);
#pragma unroll 4
      for (int kk = part * KR; kk < (part + 1) * KR; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * ti) * G::LDW + kk, G::LDW);
        wm::load_matrix_sync(fb, sS + kk * G::LDS + 16 * tj, G::LDS);
        to_tf32(fb);
        wm::mma_sync(acc, fa, fb, acc);
      }
      if (part == 0) {
        for (int kk = 0; kk < 16 * (ti + 1); kk += 8) {   // P is lower triangular
          TfA fa;
          TfB fb;
          wm::load_matrix_sync(fa, sP + (16 * ti) * G::LDA + kk, G::LDA);
          wm::load_matrix_sync(fb, sU + kk * G::LDS + 16 * tj, G::LDS);
          wm::mma_sync(acc, fa, fb, acc);
        }
      } else {
        wm::store_matrix_sync(s_patch[warp], acc, 16, wm::mem_row_major);
      }
      __syncthreads();
      if (part == 0) {
#pragma unroll
        for (int q = 1; q < G::KSPLIT; ++q) {
          AccTf other;
          wm::load_matrix_sync(other, s_patch[warp + q * G::TILES], 16, wm::mem_row_major);
#pragma unroll
          for (int e = 0; e < acc.num_elements; ++e) acc.x[e] += other.x[e];
        }
        float* patch = s_patch[warp];
        wm::store_matrix_sync(patch, acc, 16, wm::mem_row_major);
        __syncwarp();
        for (int e = lane; e < 256; e += 32) {
          const int t = 16 * ti + e / 16;
          if (t < n) Og[((c0 + t) * a.H + h) * DV + col0 + 16 * tj + e % 16] = __float2bfloat16_rn(patch[e]);
        }
      }
    }
    __syncthreads();

    // 7. (e^{Gamma_end - Gamma} (.) K)^T into W, transposed; S rows scaled by e^{Gamma_end}
    for (int idx = tid; idx < C * DK / 4; idx += G::NT) {   // four rows t of one key j
      const int j = idx / (C / 4), t = 4 * (idx % (C / 4));
      const float gend = sG[(C - 1) * G::LDG + j];
      float w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = wm::__float_to_tf32(ex2_approx(gend - sG[(t + e) * G::LDG + j]) *
                                   __bfloat162float(sK[(t + e) * G::LDK + j]));
      *reinterpret_cast<float4*>(sW + j * G::LDT + t) = make_float4(w[0], w[1], w[2], w[3]);
    }
    for (int idx = tid; idx < DK * VT / 4; idx += G::NT) {
      const int row = idx / (VT / 4), c4 = idx % (VT / 4);
      float4* p = reinterpret_cast<float4*>(&sS[row * G::LDS + 4 * c4]);
      const float e = sE[row];
      float4 x = *p;
      x.x *= e;
      x.y *= e;
      x.z *= e;
      x.w *= e;
      *p = x;
    }
    __syncthreads();

    // 8. S += (scaled K)^T B
    for_tiles<DK, VT>([&](int i, int j) {
      AccTf acc;
      float* p = sS + (16 * i) * G::LDS + 16 * j;
      wm::load_matrix_sync(acc, p, G::LDS, wm::mem_row_major);
#pragma unroll
      for (int kk = 0; kk < C; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * i) * G::LDT + kk, G::LDT);
        wm::load_matrix_sync(fb, sU + kk * G::LDS + 16 * j, G::LDS);
        wm::mma_sync(acc, fa, fb, acc);
      }
      wm::store_matrix_sync(p, acc, G::LDS, wm::mem_row_major);
    });
  }
  __syncthreads();

  for (int idx = tid; idx < DK * VT / 4; idx += G::NT) {
    const int row = idx / (VT / 4), c4 = idx % (VT / 4);
    st_state(Sg + row * DV + 4 * c4, *reinterpret_cast<const float4*>(&sS[row * G::LDS + 4 * c4]));
  }
  clear_log_tile<OP, DK, DV, __nv_bfloat16>(a, sh, col0, VT);
}

}  // namespace dl
