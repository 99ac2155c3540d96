// Chunked GDN prefill on tensor cores: the same hand-off as prefill_kernel
// (each prompt's final state written as its slot's base, log entries
// cleared), for bf16-input GDN handles.
//
// Within a chunk of C tokens the delta rule unrolls into dense products (the
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
// One CTA per (row, head, 64-column value tile) keeps its d_k x 64 state
// slice in shared memory for the whole prompt.  K K^T and Q K^T run as bf16
// tensor-core products (the inputs are bf16-exact); the products with the
// state, W and B use tf32 operands with fp32 accumulation.  The two
// triangular solves share one forward substitution per right-hand-side
// column.  tf32 rounding (2^-11 relative) fits the bf16-input tolerance, so
// the path serves bf16 handles only.
#pragma once

#include <mma.h>

#include "prefill.cuh"

namespace dl {

template <int DK, int VT_>
struct ChunkGeom {
  static constexpr int C = 32;           // tokens per chunk
  static constexpr int VT = VT_;         // value columns per CTA (64 or 128)
  static constexpr int NT = 4 * VT;      // threads (8 or 16 warps)
  static constexpr int NW = NT / 32;
  static constexpr int MINB = VT == 128 ? 1 : 2;   // resident CTAs per SM
  static constexpr int LDK = DK + 8;     // bf16 row stride of K and Q (16-byte multiple)
  static constexpr int LDV = VT + 8;     // bf16 row stride of the V tile
  static constexpr int LDS = VT + 8;     // fp32 row stride of the state tile, B and U (8 banks:
                                         // conflict-free tf32 B-operand reads)
  static constexpr int LDA = C + 4;      // fp32 row stride of A and P
  static constexpr int LDW = DK + 4;     // fp32 row stride of W and e^Gamma Q
  static constexpr int LDT = C + 4;      // fp32 row stride of (e^{..} K)^T, stored transposed
  // shared-memory carve-up (bytes; every region 128-byte aligned)
  static constexpr size_t al(size_t x) { return (x + 127) & ~size_t(127); }
  // K and the V tile are double-buffered (chunk c + 1 streams in while chunk
  // c computes); Q streams in during the chunk's first steps
  static constexpr size_t KQ_BYTES = al(size_t(C) * LDK * 2), V_BYTES = al(size_t(C) * LDV * 2);
  static constexpr size_t S_OFF = 0;
  static constexpr size_t K_OFF = al(S_OFF + size_t(DK) * LDS * 4);
  static constexpr size_t Q_OFF = K_OFF + 2 * KQ_BYTES;
  static constexpr size_t V_OFF = Q_OFF + KQ_BYTES;
  static constexpr size_t A_OFF = V_OFF + 2 * V_BYTES;
  static constexpr size_t W_OFF = al(A_OFF + size_t(C) * LDA * 4);
  static constexpr size_t W_FLOATS = size_t(C) * LDW > size_t(DK) * LDT ? size_t(C) * LDW : size_t(DK) * LDT;
  static constexpr size_t U_OFF = al(W_OFF + W_FLOATS * 4);
  static constexpr size_t G_OFF = al(U_OFF + size_t(C) * LDS * 4);
  static constexpr size_t BYTES = al(G_OFF + 5 * C * 4);   // Gamma, beta and three per-row factors
};

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
using AccTf = wm::fragment<wm::accumulator, 16, 16, 8, float>;    // of tf32 products
using TfA = wm::fragment<wm::matrix_a, 16, 16, 8, wm::precision::tf32, wm::row_major>;
using TfAc = wm::fragment<wm::matrix_a, 16, 16, 8, wm::precision::tf32, wm::col_major>;
using TfB = wm::fragment<wm::matrix_b, 16, 16, 8, wm::precision::tf32, wm::row_major>;
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

template <typename Frag>
__device__ __forceinline__ void to_tf32(Frag& f) {
#pragma unroll
  for (int e = 0; e < f.num_elements; ++e) f.x[e] = wm::__float_to_tf32(f.x[e]);
}

template <int DK, int DV, int VT_>
__global__ void __launch_bounds__(ChunkGeom<DK, VT_>::NT, ChunkGeom<DK, VT_>::MINB)
    gdn_chunk_prefill_kernel(const PrefillArgs a) {
  using G = ChunkGeom<DK, VT_>;
  constexpr int C = G::C, VT = G::VT, NSPLIT = DV / VT;
  static_assert(DV % VT == 0 && DK % 16 == 0, "chunk tile shape");
  extern __shared__ __align__(128) unsigned char smem[];
  float* sS = reinterpret_cast<float*>(smem + G::S_OFF);                  // [DK][LDS] state slice
  // [2][C][LDK] K and Q, [2][C][LDV] V tile: buffer (chunk index & 1)
  auto kbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::K_OFF + b * G::KQ_BYTES); };
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + G::Q_OFF);
  auto vbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::V_OFF + b * G::V_BYTES); };
  float* sA = reinterpret_cast<float*>(smem + G::A_OFF);                  // [C][LDA] A, then P
  float* sW = reinterpret_cast<float*>(smem + G::W_OFF);                  // [C][LDW] W, then e^G Q; [DK][LDT] (e^{..} K)^T
  float* sU = reinterpret_cast<float*>(smem + G::U_OFF);                  // [C][LDS] U, then B
  float* sG = reinterpret_cast<float*>(smem + G::G_OFF);                  // [C] Gamma
  float* sBeta = sG + C;                                                  // [C] beta
  float* sEG = sG + 2 * C;    // [C] e^{Gamma_t}
  float* sBEG = sG + 3 * C;   // [C] beta_t e^{Gamma_t}
  float* sEnd = sG + 4 * C;   // [C] e^{Gamma_end - Gamma_t} (0 past the prompt)
  __shared__ __align__(32) float s_patch[G::NW][16 * 16];                 // per-warp output tile

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

  // state slice into shared memory
  for (int idx = tid; idx < DK * VT / 4; idx += G::NT) {
    const int row = idx / (VT / 4), c4 = idx % (VT / 4);
    const float4 x = a.zero_state ? make_float4(0.f, 0.f, 0.f, 0.f) : ld_state(Sg + row * DV + 4 * c4);
    *reinterpret_cast<float4*>(&sS[row * G::LDS + 4 * c4]) = x;
  }

  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* Og = static_cast<__nv_bfloat16*>(a.o);
  const __nv_bfloat16 zero_bf = __float2bfloat16_rn(0.f);

  // Stage chunk [c, c + C) of K and the V tile into buffer b, or of Q; rows
  // past the prompt are zeros.  16-byte async copies when the inputs allow.
  const bool async_ok = aligned_to(a.q, 16) && aligned_to(a.k, 16) && aligned_to(a.v, 16);
  auto stage_rows = [&](__nv_bfloat16* dst, const __nv_bfloat16* src, long c, int width, int ld, int stride,
                        int off) {
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
    if (async_ok) {
      const int seg_per_row = width / 8;   // 16-byte segments
      for (int idx = tid; idx < C * seg_per_row; idx += G::NT) {
        const int t = idx / seg_per_row, seg = idx % seg_per_row;
        const long row = ((c + (t < nv ? t : nv - 1)) * a.H + h) * stride + off + 8 * seg;
        cp_async16(dst + t * ld + 8 * seg, src + row, t < nv ? 16u : 0u);
      }
    } else {
      for (int idx = tid; idx < C * width; idx += G::NT) {
        const int t = idx / width, j = idx % width;
        dst[t * ld + j] = t < nv ? src[((c + t) * a.H + h) * stride + off + j] : zero_bf;
      }
    }
  };
  auto stage_kv = [&](int b, long c) {
    stage_rows(kbuf(b), Kg, c, DK, G::LDK, DK, 0);
    stage_rows(vbuf(b), Vg, c, VT, G::LDV, DV, col0);
  };
  constexpr int EPL = C / 32;   // chunk rows per lane of warp 0
  float gn[EPL], bnv[EPL];
  auto fetch_gates = [&](long c) {
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int t = EPL * lane + e;
      gn[e] = t < nv ? a.log_decay[(c + t) * a.H + h] : 0.f;
      bnv[e] = t < nv ? a.beta[(c + t) * a.H + h] : 0.f;
    }
  };
  if (t0 < t1) {
    stage_kv(0, t0);
    if (warp == 0) fetch_gates(t0);
  }
  cp_async_commit();

  // Copy groups, in commit order: K/V of chunk c (committed one chunk ahead),
  // then at chunk c: Q of chunk c, K/V of chunk c + 1 (possibly empty).
  int buf = 0;
  for (long c0 = t0; c0 < t1; c0 += C, buf ^= 1) {
    const int n = static_cast<int>(t1 - c0 < C ? t1 - c0 : C);   // valid rows of this chunk
    const bool has_next = c0 + C < t1;
    __syncthreads();   // the previous chunk is done with every buffer
    stage_rows(sQ, Qg, c0, DK, G::LDK, DK, 0);
    cp_async_commit();
    if (has_next) stage_kv(buf ^ 1, c0 + C);
    cp_async_commit();
    cp_async_wait<2>();   // K/V of this chunk have landed (Q and the next K/V may be in flight)
    __nv_bfloat16 *sK = kbuf(buf), *sV = vbuf(buf);

    // 1. Gamma = inclusive prefix sum of the chunk's log-gates (rows past the
    // prompt: 0), and beta; then the next chunk's gates
    if (warp == 0) {
      float loc[EPL], run = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) loc[e] = (run += gn[e]);
      float incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float excl = incl - run;
      float sel = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        loc[e] += excl;
        if (e == (n - 1) % EPL) sel = loc[e];
      }
      const float gend = __shfl_sync(0xffffffffu, sel, (n - 1) / EPL);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int t = EPL * lane + e;
        const float eg = expf(loc[e]);
        sG[t] = loc[e];
        sBeta[t] = bnv[e];
        sEG[t] = eg;
        sBEG[t] = bnv[e] * eg;
        sEnd[t] = t < n ? expf(gend - loc[e]) : 0.f;
      }
      if (has_next) fetch_gates(c0 + C);
    }
    __syncthreads();

    // 2. A = strictly lower (beta_t e^{G_t - G_s} k_t . k_s)
    lower_xyt<C, DK, G::LDK, G::LDA>(sK, sK, sA);
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += G::NT) {
      const int t = idx / C, s = idx % C;
      float& x = sA[t * G::LDA + s];
      x = s < t ? sBeta[t] * expf(sG[t] - sG[s]) * x : 0.f;
    }
    // right-hand sides: beta e^{G} K into W, beta V into U
    for (int idx = tid; idx < C * DK; idx += G::NT) {
      const int t = idx / DK, j = idx % DK;
      sW[t * G::LDW + j] = sBEG[t] * __bfloat162float(sK[t * G::LDK + j]);
    }
    for (int idx = tid; idx < C * VT; idx += G::NT) {
      const int t = idx / VT, c = idx % VT;
      sU[t * G::LDS + c] = sBeta[t] * __bfloat162float(sV[t * G::LDV + c]);
    }
    __syncthreads();

    // 3. (I + A) X = R, one right-hand-side column per thread
    // (W is a tf32 operand later and is stored tf32-rounded; U stays fp32.)
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
    for_tiles<C, VT>([&](int i, int j) {
      AccTf acc;
      wm::fill_fragment(acc, 0.f);
#pragma unroll 4
      for (int kk = 0; kk < DK; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * i) * G::LDW + kk, G::LDW);   // tf32-rounded already
        wm::load_matrix_sync(fb, sS + kk * G::LDS + 16 * j, G::LDS);
        to_tf32(fb);
        wm::mma_sync(acc, fa, fb, acc);
      }
      AccTf u;
      float* p = sU + (16 * i) * G::LDS + 16 * j;
      wm::load_matrix_sync(u, p, G::LDS, wm::mem_row_major);
#pragma unroll
      for (int e = 0; e < u.num_elements; ++e) u.x[e] = wm::__float_to_tf32(u.x[e] - acc.x[e]);   // B, a tf32 operand
      wm::store_matrix_sync(p, u, G::LDS, wm::mem_row_major);
    });
    __syncthreads();

    // 5. P = Q K^T (.) [e^{G_t - G_s}]_{s <= t} into A;  e^{G} Q into W
    cp_async_wait<1>();   // Q of this chunk has landed
    __syncthreads();
    lower_xyt<C, DK, G::LDK, G::LDA>(sQ, sK, sA);
    for (int idx = tid; idx < C * DK; idx += G::NT) {
      const int t = idx / DK, j = idx % DK;
      sW[t * G::LDW + j] = wm::__float_to_tf32(sEG[t] * __bfloat162float(sQ[t * G::LDK + j]));
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += G::NT) {
      const int t = idx / C, s = idx % C;
      float& x = sA[t * G::LDA + s];
      x = s <= t ? wm::__float_to_tf32(expf(sG[t] - sG[s]) * x) : 0.f;
    }
    __syncthreads();

    // 6. O = (e^{G} Q) S + P B, rows < n to global (through a per-warp patch)
    for_tiles<C, VT>([&](int i, int j) {
      AccTf acc;
      wm::fill_fragment(acc, 0.f);
#pragma unroll 4
      for (int kk = 0; kk < DK; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * i) * G::LDW + kk, G::LDW);   // e^G Q, tf32-rounded
        wm::load_matrix_sync(fb, sS + kk * G::LDS + 16 * j, G::LDS);
        to_tf32(fb);
        wm::mma_sync(acc, fa, fb, acc);
      }
      for (int kk = 0; kk < 16 * (i + 1); kk += 8) {   // P is lower triangular
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sA + (16 * i) * G::LDA + kk, G::LDA);   // P, tf32-rounded
        wm::load_matrix_sync(fb, sU + kk * G::LDS + 16 * j, G::LDS);     // B, tf32-rounded
        wm::mma_sync(acc, fa, fb, acc);
      }
      float* patch = s_patch[warp];
      wm::store_matrix_sync(patch, acc, 16, wm::mem_row_major);
      __syncwarp();
      for (int e = lane; e < 256; e += 32) {
        const int t = 16 * i + e / 16;
        if (t < n) Og[((c0 + t) * a.H + h) * DV + col0 + 16 * j + e % 16] = __float2bfloat16_rn(patch[e]);
      }
      __syncwarp();
    });
    __syncthreads();

    // 7. S <- e^{G_end} S + (e^{G_end - G} K)^T B
    for (int idx = tid; idx < C * DK; idx += G::NT) {   // transposed, rows of keys
      const int j = idx / C, t = idx % C;
      sW[j * G::LDT + t] = wm::__float_to_tf32(sEnd[t] * __bfloat162float(sK[t * G::LDK + j]));
    }
    __syncthreads();
    const float dend = sEG[n - 1];
    for_tiles<DK, VT>([&](int i, int j) {
      AccTf acc;
      float* p = sS + (16 * i) * G::LDS + 16 * j;
      wm::load_matrix_sync(acc, p, G::LDS, wm::mem_row_major);
#pragma unroll
      for (int e = 0; e < acc.num_elements; ++e) acc.x[e] *= dend;
#pragma unroll 4
      for (int kk = 0; kk < C; kk += 8) {
        TfA fa;
        TfB fb;
        wm::load_matrix_sync(fa, sW + (16 * i) * G::LDT + kk, G::LDT);  // (e^{..} K)^T, tf32
        wm::load_matrix_sync(fb, sU + kk * G::LDS + 16 * j, G::LDS);     // B, tf32
        wm::mma_sync(acc, fa, fb, acc);
      }
      wm::store_matrix_sync(p, acc, G::LDS, wm::mem_row_major);
    });
  }
  __syncthreads();

  // final state slice to Sbar; clear the slot's log entries
  for (int idx = tid; idx < DK * VT / 4; idx += G::NT) {
    const int row = idx / (VT / 4), c4 = idx % (VT / 4);
    st_state(Sg + row * DV + 4 * c4, *reinterpret_cast<const float4*>(&sS[row * G::LDS + 4 * c4]));
  }
  clear_log_tile<OP_GDN, DK, DV, __nv_bfloat16>(a, sh, col0, VT);
}

// Grid (H * d_v/VT, rows), 4 VT threads, ChunkGeom<DK, VT>::BYTES of dynamic
// shared memory.  Instantiated in prefill.cu.
template <int DK, int DV, int VT>
cudaError_t launch_gdn_chunk_prefill(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);

}  // namespace dl
