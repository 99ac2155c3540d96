// Chunked prefill with the state in tensor memory: the chunk forms of
// prefill_chunk.cuh with their three products with the state issued as
// 5th-generation tensor-core MMAs (tcgen05, tf32 operands, fp32 accumulation)
// on a whole head per CTA, for every head shape (d_k, d_v in {64, 128}).
//
// The state is kept transposed, S^T (value column c on TMEM lane c, key j on
// column j), so that it serves directly as the A operand of
//   B^T = U^T - S^T W^T                  (M = 128 lanes, N = C tokens)
//   O^T = S^T (e^{Gamma} Q)^T + B^T P^T
//   S^T <- e^{Gamma_end} S^T + B^T (e^{Gamma_end - Gamma} K)
// and receives the last as its accumulator; it never leaves tensor memory
// between the prompt's first and last chunk.  A d_v = 64 head uses lanes
// 0 .. 63 of the M = 128 products and keeps lanes 64 .. 127 zero: each row of
// an MMA result depends only on the same row of its tensor-memory operand,
// and every element-wise pass stays on its own lane.  B^T, O^T and U^T live
// in tensor memory too.  The triangular solve forms T = (I + A)^{-1} in
// 16 x 16 blocks on the SIMT lanes and W^T, U^T as two tcgen05 products with
// T^T, into tensor memory.  W, the scaled queries, P, T, the solve's
// right-hand sides and the scaled keys are written by the SIMT lanes into
// shared memory in K-major no-swizzle operand layouts.  One thread issues the MMAs; their
// completion is tracked by mbarriers (bounded waits: a wait that runs out
// raises DL_DEVERR_WAIT_TIMEOUT and the CTA stops).  The state update of
// chunk i runs while chunk i + 1 computes its gates, A and the solve.
//
// Two CTAs of 256 threads share an SM (and its 512 TMEM columns) when the
// launch has more CTAs than SMs; one CTA of 512 threads otherwise.
#pragma once

#include "prefill_chunk.cuh"

namespace dl {

// ---- tcgen05 / tensor-memory wrappers --------------------------------------

// K-major tf32 operands with no swizzle are made of 8-row x 4-element core
// matrices of 128 contiguous bytes.  In the dense form used for P and the
// scaled keys, the core matrices of one 8-row group are adjacent along k and
// the groups KT/4 x 128 bytes apart: element (r, k) of an R x KT operand sits
// at byte (r/8)(KT/4)128 + (k/4)128 + (r%8)16 + (k%4)4.
//
// Shared-memory matrix descriptor of such an operand: start address, leading
// byte offset 128 (next core matrix along k), stride byte offset `sbo` (next
// 8-row group), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fff) | (static_cast<uint64_t>(128 >> 4) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32) | (static_cast<uint64_t>(1) << 46);
}

// Instruction descriptor: kind::tf32, fp32 accumulator, both operands K-major.
template <int M, int N>
__host__ __device__ constexpr uint32_t umma_idesc_tf32() {
  static_assert(M == 128 && N % 16 == 0 && N >= 16 && N <= 256, "tcgen05 tf32 tile shape");
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] B[smem desc]; one thread issues.
__device__ __forceinline__ void umma_tf32_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

// D[tmem] (+)= A[smem desc] B[smem desc]; one thread issues.
__device__ __forceinline__ void umma_tf32_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make this thread's shared-memory writes visible to the tensor cores' reads.
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Warp-collective 32 lanes x 8 / x 32 columns of 32 bits (lane i of the warp
// gets TMEM lane (address lane + i)).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- geometry ----------------------------------------------------------------

constexpr size_t tc_align128(size_t x) { return (x + 127) & ~size_t(127); }

// K-major operand of R rows whose 8-row groups are adjacent (stride byte
// offset 128) and whose 16-byte k-chunks are R/8 x 128 + 16 bytes apart
// (leading byte offset): the 16-byte pad puts the 32 consecutive k of one
// row on 32 different banks, so a warp writes a row (one k a lane, as the
// copy of W^T out of tensor memory does) without bank conflicts.
template <int R>
__host__ __device__ constexpr uint32_t kmajor_pad_lbo() { return (R / 8) * 128 + 16; }
template <int R>
__device__ __forceinline__ uint32_t kmajor_pad_off(int r, int k) {
  return static_cast<uint32_t>((r >> 3) * 128 + (k >> 2) * kmajor_pad_lbo<R>() + (r & 7) * 16 + (k & 3) * 4);
}
__device__ __forceinline__ uint64_t umma_desc_lbo(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fff) | (static_cast<uint64_t>((lbo >> 4) & 0x3fff) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32) | (static_cast<uint64_t>(1) << 46);
}

template <int NT_, int DK_ = 128, int DV_ = 128>
struct TcChunkGeom {
  // a whole head per CTA; value columns sit on tensor-memory lanes 0 .. DV-1
  // of the 128 an M = 128 MMA covers (a d_v = 64 head leaves the upper 64
  // lanes zero: every MMA row and every element-wise pass stays within its own
  // lane, so padding never reaches a value column)
  static constexpr int DK = DK_, DV = DV_;
  static_assert((DK == 64 || DK == 128) && (DV == 64 || DV == 128), "head shape");
  static constexpr int C = 32;               // tokens per chunk
  // 256 threads (two CTAs per SM) or 512 (one CTA per SM, for launches with
  // fewer CTAs than SMs)
  static constexpr int NT = NT_, NW = NT / 32;
  static constexpr int NG = NW / 4;          // column groups of the TMEM epilogues
  static constexpr int MINB = NT == 256 ? 2 : 1;
  static constexpr int LDK = DK + 8;         // bf16 row stride of K and Q
  static constexpr int LDV = DV + 8;         // bf16 row stride of V
  static constexpr int LDA = C + 4;          // fp32 row stride of A and P (WMMA outputs)
  static constexpr uint32_t WQ_LBO = kmajor_pad_lbo<C>();             // W and e^G Q operand layout
  // the W and e^G Q buffers also hold the solve's right-hand sides R_W^T and
  // R_U^T, dense K-major 128 x C operands
  static constexpr size_t WQ_BYTES = size_t(DK / 4) * WQ_LBO > size_t(128) * C * 4 ? size_t(DK / 4) * WQ_LBO
                                                                                    : size_t(128) * C * 4;
  static constexpr size_t KQ_BYTES = tc_align128(size_t(C) * LDK * 2), V_BYTES = tc_align128(size_t(C) * LDV * 2);
  static constexpr size_t K_OFF = 0;                                  // [2][C][LDK] bf16
  static constexpr size_t Q_OFF = K_OFF + 2 * KQ_BYTES;               // [C][LDK] bf16
  static constexpr size_t V_OFF = Q_OFF + KQ_BYTES;                   // [C][LDV] bf16
  static constexpr size_t A_OFF = V_OFF + V_BYTES;                    // [C][LDA] fp32
  static constexpr size_t WC_OFF = tc_align128(A_OFF + size_t(C) * LDA * 4);   // W, padded K-major C x DK
  static constexpr size_t QC_OFF = tc_align128(WC_OFF + WQ_BYTES);    // e^G Q, padded K-major C x DK
  static constexpr size_t PC_OFF = tc_align128(QC_OFF + WQ_BYTES);    // P, K-major C x C
  static constexpr size_t KC_OFF = PC_OFF + size_t(C) * C * 4;        // (e^{..} K)^T, K-major DK x C
  static constexpr size_t G_OFF = tc_align128(KC_OFF + size_t(DK) * C * 4);    // 5 x [C] per-row factors
  static constexpr size_t T_OFF = tc_align128(G_OFF + 5 * C * 4);              // [C][LDA] T = (I + A)^-1
  static constexpr size_t X_OFF = T_OFF + size_t(C) * LDA * 4;                 // [16][17] A21 T11
  static constexpr size_t BAR_OFF = tc_align128(X_OFF + 16 * 17 * 4);          // 4 mbarriers, TMEM base, abort flag, drain
  static constexpr size_t BYTES = BAR_OFF + 64;
  // tensor-memory columns
  static constexpr uint32_t TM_COLS = 256;   // allocation (power of two)
  static constexpr uint32_t TM_S = 0;        // S^T: DK columns (keys)
  static constexpr uint32_t TM_B = DK;       // W S, then B^T: C columns (tokens)
  static constexpr uint32_t TM_O = DK + 32;  // O^T: C columns
  static constexpr uint32_t TM_U = DK + 64;  // U^T: C columns (the solve's product writes it)
  static constexpr uint32_t TM_W = DK + 96;  // W^T: C columns (the solve's product, then W's operand)
};

template <int NT_, int DK_, int DV_>
__global__ void __launch_bounds__(NT_, TcChunkGeom<NT_, DK_, DV_>::MINB) gdn_chunk_prefill_tc_kernel(const PrefillArgs a) {
  using G = TcChunkGeom<NT_, DK_, DV_>;
  constexpr int C = G::C, DK = G::DK, DV = G::DV;
  extern __shared__ __align__(128) unsigned char smem[];
  auto kbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + G::K_OFF + b * G::KQ_BYTES); };
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + G::Q_OFF);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + G::V_OFF);
  float* sA = reinterpret_cast<float*>(smem + G::A_OFF);
  unsigned char* sWc = smem + G::WC_OFF;
  unsigned char* sQc = smem + G::QC_OFF;
  unsigned char* sPc = smem + G::PC_OFF;
  unsigned char* sKc = smem + G::KC_OFF;
  float* sG = reinterpret_cast<float*>(smem + G::G_OFF);
  float* sBeta = sG + C;
  float* sEG = sG + 2 * C;
  float* sBEG = sG + 3 * C;
  float* sEnd = sG + 4 * C;
  float* sT = reinterpret_cast<float*>(smem + G::T_OFF);
  float* sX = reinterpret_cast<float*>(smem + G::X_OFF);
  uint64_t* barB = reinterpret_cast<uint64_t*>(smem + G::BAR_OFF);   // W S done
  uint64_t* barO = barB + 1;                                          // O^T done
  uint64_t* barS = barB + 2;                                          // state update done
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(barB + 3);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
  uint64_t* barF = barB + 4;                                          // drain after an abort
  uint64_t* barT = barB + 5;                                          // the solve's products done
  auto fp = [](unsigned char* base, uint32_t off) { return reinterpret_cast<float*>(base + off); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quarter = warp & 3, group = warp >> 2;   // TMEM lanes 32 quarter .., column group
  constexpr int NG = G::NG;
  const int h = blockIdx.x;
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
  float* Sg = a.Sbar + sh * (DK * DV);

  if (tid == 0) {
    mbar_init(barB, 1);
    mbar_init(barO, 1);
    mbar_init(barS, 1);
    mbar_init(barF, 1);
    mbar_init(barT, 1);
    fence_mbar_init();
    *sAbort = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sTmem)),
                 "r"(G::TM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
  const int c_own = 32 * quarter + lane;   // this thread's value column in TMEM epilogues
  const bool own_col = c_own < DV;         // false on the padding lanes of a d_v = 64 head

  // S^T into tensor memory: this warp's 32 lanes (value columns), key blocks 32 cb ..
  for (int cb = group; cb < DK / 32; cb += NG) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = a.zero_state || !own_col ? 0.f : __ldcs(Sg + (32 * cb + i) * DV + c_own);
    tmem_st32(tmem + lane_base + G::TM_S + 32 * cb, v);
  }
  tmem_wait_st();

  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* Og = static_cast<__nv_bfloat16*>(a.o);
  const __nv_bfloat16 zero_bf = __float2bfloat16_rn(0.f);

  // Stage rows [c, c + C) of a [total][H][width] bf16 input into dst (row
  // stride ld); rows past the prompt are zeros.
  const bool async_ok = aligned_to(a.q, 16) && aligned_to(a.k, 16) && aligned_to(a.v, 16);
  auto stage_rows = [&](__nv_bfloat16* dst, const __nv_bfloat16* src, long c, int width, int ld) {
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
    if (async_ok) {
      const int seg_per_row = width / 8;
      for (int idx = tid; idx < C * seg_per_row; idx += G::NT) {
        const int t = idx / seg_per_row, seg = idx % seg_per_row;
        const long row = ((c + (t < nv ? t : nv - 1)) * a.H + h) * width + 8 * seg;
        cp_async16(dst + t * ld + 8 * seg, src + row, t < nv ? 16u : 0u);
      }
    } else {
      for (int idx = tid; idx < C * width; idx += G::NT) {
        const int t = idx / width, j = idx % width;
        dst[t * ld + j] = t < nv ? src[((c + t) * a.H + h) * width + j] : zero_bf;
      }
    }
  };

  float gn = 0.f, bnv = 0.f;   // warp 0, lane t: gate and beta of row t of the next chunk
  auto fetch_gates = [&](long c) {
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
    gn = lane < nv ? a.log_decay[(c + lane) * a.H + h] : 0.f;
    bnv = lane < nv ? a.beta[(c + lane) * a.H + h] : 0.f;
  };
  // Copy groups, in commit order: K and V of chunk 0; then per chunk c: Q of c
  // and K of c + 1 at its start, V of c + 1 once V of c has been consumed
  // (V is single-buffered).  Groups may be empty.
  if (t0 < t1) {
    stage_rows(kbuf(0), Kg, t0, DK, G::LDK);
    if (warp == 0) fetch_gates(t0);
  }
  cp_async_commit();
  if (t0 < t1) stage_rows(sV, Vg, t0, DV, G::LDV);
  cp_async_commit();

  // (r, k) of element e of a K-major operand with kt columns, enumerated in
  // storage order (e * 4 is its byte offset)
  auto kmajor_rk = [](int e, int kt, int& rr, int& kk) {
    const int core = e >> 5, within = e & 31;
    rr = (core / (kt >> 2)) * 8 + (within >> 2);
    kk = (core % (kt >> 2)) * 4 + (within & 3);
  };

  int buf = 0, ci = 0;
  for (long c0 = t0; c0 < t1; c0 += C, buf ^= 1, ++ci) {
    const int n = static_cast<int>(t1 - c0 < C ? t1 - c0 : C);
    const bool has_next = c0 + C < t1;
    const uint32_t par = static_cast<uint32_t>(ci & 1);
    __syncthreads();   // the previous chunk is done with every buffer
    stage_rows(sQ, Qg, c0, DK, G::LDK);
    cp_async_commit();
    if (has_next) stage_rows(kbuf(buf ^ 1), Kg, c0 + C, DK, G::LDK);
    cp_async_commit();
    cp_async_wait<2>();   // K and V of this chunk have landed
    __nv_bfloat16* sK = kbuf(buf);

    // 1. Gamma (inclusive prefix of the log-gates), beta and per-row factors
    if (warp == 0) {
      float incl = gn;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float gend = __shfl_sync(0xffffffffu, incl, n - 1);
      const float eg = expf(incl);
      sG[lane] = incl;
      sBeta[lane] = bnv;
      sEG[lane] = eg;
      sBEG[lane] = bnv * eg;
      sEnd[lane] = lane < n ? expf(gend - incl) : 0.f;
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
    __syncthreads();

    // 3. (I + A) W = diag(beta e^G) K and (I + A) U = diag(beta) V as
    // W^T = R_W^T T^T and U^T = R_U^T T^T with T = (I + A)^{-1}: T on the SIMT
    // lanes in 16 x 16 blocks (T11, T22 column by column on warp 0, then
    // T21 = -T22 (A21 T11)), the two products on the tensor cores.  Meanwhile
    // the other warps write the right-hand sides as dense K-major 128 x C
    // operands, R_W^T into the e^G Q buffer and R_U^T into the W buffer
    // (rows past d_k or d_v are zero).
    if (warp == 0) {
      const int c = lane, r0 = c & ~15;   // column c of the diagonal block at rows r0 ..
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = r0 + i;
        const float* arow = sA + t * G::LDA + r0;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int k = 0; k + 1 < i; k += 2) {
          acc0 = fmaf(-arow[k], x[k], acc0);
          acc1 = fmaf(-arow[k + 1], x[k + 1], acc1);
        }
        if (i & 1) acc0 = fmaf(-arow[i - 1], x[i - 1], acc0);
        x[i] = t == c ? 1.f : t < c ? 0.f : acc0 + acc1;
        sT[t * G::LDA + c] = x[i];
        sT[(t ^ 16) * G::LDA + c] = 0.f;   // the other block row of column c: T12 = 0, T21 filled below
      }
    } else {   // four tokens of one key (one 16-byte run of the layout) a thread
      for (int e = 4 * (tid - 32); e < 128 * C; e += 4 * (G::NT - 32)) {
        int rr, s;
        kmajor_rk(e, C, rr, s);
        float4 w = make_float4(0.f, 0.f, 0.f, 0.f), u = w;
        if (rr < DK) {
          const __nv_bfloat16* kc = sK + s * G::LDK + rr;
          w = make_float4(wm::__float_to_tf32(sBEG[s] * __bfloat162float(kc[0])),
                          wm::__float_to_tf32(sBEG[s + 1] * __bfloat162float(kc[G::LDK])),
                          wm::__float_to_tf32(sBEG[s + 2] * __bfloat162float(kc[2 * G::LDK])),
                          wm::__float_to_tf32(sBEG[s + 3] * __bfloat162float(kc[3 * G::LDK])));
        }
        if (rr < DV) {
          const __nv_bfloat16* vc = sV + s * G::LDV + rr;
          u = make_float4(wm::__float_to_tf32(sBeta[s] * __bfloat162float(vc[0])),
                          wm::__float_to_tf32(sBeta[s + 1] * __bfloat162float(vc[G::LDV])),
                          wm::__float_to_tf32(sBeta[s + 2] * __bfloat162float(vc[2 * G::LDV])),
                          wm::__float_to_tf32(sBeta[s + 3] * __bfloat162float(vc[3 * G::LDV])));
        }
        *reinterpret_cast<float4*>(sQc + 4 * e) = w;
        *reinterpret_cast<float4*>(sWc + 4 * e) = u;
      }
    }
    __syncthreads();
    // The blocks hold explicit zeros above their diagonals, so both products
    // run over all 16 terms.
    if (tid < 256) {   // X = A21 T11
      const int i = 16 + (tid >> 4), j = tid & 15;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int l = 0; l < 16; l += 2) {
        acc0 = fmaf(sA[i * G::LDA + l], sT[l * G::LDA + j], acc0);
        acc1 = fmaf(sA[i * G::LDA + l + 1], sT[(l + 1) * G::LDA + j], acc1);
      }
      sX[(i - 16) * 17 + j] = acc0 + acc1;
    }
    __syncthreads();
    if (tid < 256) {   // T21 = -T22 X
      const int i = 16 + (tid >> 4), j = tid & 15;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        acc0 = fmaf(sT[i * G::LDA + 16 + k], sX[k * 17 + j], acc0);
        acc1 = fmaf(sT[i * G::LDA + 17 + k], sX[(k + 1) * 17 + j], acc1);
      }
      sT[i * G::LDA + j] = -(acc0 + acc1);
    }
    __syncthreads();
    for (int e = 4 * tid; e < C * C; e += 4 * G::NT) {   // T as the B operand (N = t, K = s), tf32
      int t, s;
      kmajor_rk(e, C, t, s);
      const float* tr = sT + t * G::LDA + s;
      *reinterpret_cast<float4*>(sPc + 4 * e) = make_float4(wm::__float_to_tf32(tr[0]), wm::__float_to_tf32(tr[1]),
                                                            wm::__float_to_tf32(tr[2]), wm::__float_to_tf32(tr[3]));
    }
    fence_smem_to_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, C>();
      const uint32_t t0 = smem_u32(sPc), rw = smem_u32(sQc), ru = smem_u32(sWc);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        umma_tf32_ss(tmem + G::TM_W, umma_desc(rw + 256 * s, (C / 4) * 128), umma_desc(t0 + 256 * s, (C / 4) * 128),
                     ID, s > 0);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        umma_tf32_ss(tmem + G::TM_U, umma_desc(ru + 256 * s, (C / 4) * 128), umma_desc(t0 + 256 * s, (C / 4) * 128),
                     ID, s > 0);
      umma_commit(barT);
    }
    if (!mbar_wait_abortable(barT, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_after();
    if (!*sAbort && c_own < DK) {   // W^T (key j on lane j) into W's padded operand layout, tf32
      for (int b8 = group; b8 < C / 8; b8 += NG) {
        float v[8];
        tmem_ld8(tmem + lane_base + G::TM_W + 8 * b8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) fp(sWc, kmajor_pad_off<C>(8 * b8 + i, c_own))[0] = wm::__float_to_tf32(v[i]);
      }
    }
    fence_smem_to_async();
    tc_fence_before();
    __syncthreads();
    if (has_next) stage_rows(sV, Vg, c0 + C, DV, G::LDV);   // V of this chunk is consumed
    cp_async_commit();

    // 4. the previous chunk's state update must be complete before S^T is read
    if (ci > 0 && !mbar_wait_abortable(barS, par ^ 1u, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_before();
    __syncthreads();
    if (*sAbort) break;
    tc_fence_after();
    if (tid == 0) {   // W S  (M = 128 value columns, N = C tokens, K = DK)
      constexpr uint32_t ID = umma_idesc_tf32<128, C>();
      const uint32_t w0 = smem_u32(sWc);
#pragma unroll
      for (int s = 0; s < DK / 8; ++s)
        umma_tf32_ts(tmem + G::TM_B, tmem + G::TM_S + 8 * s, umma_desc_lbo(w0 + 2 * G::WQ_LBO * s, G::WQ_LBO, 128),
                     ID, s > 0);
      umma_commit(barB);
    }

    // 5. P = Q K^T (.) [e^{G_t - G_s}]_{s <= t}, e^G Q and (e^{G_end - G} K)^T as operands
    cp_async_wait<2>();   // Q of this chunk has landed (K and V of the next may be in flight)
    __syncthreads();
    lower_xyt<C, DK, G::LDK, G::LDA>(sQ, sK, sA);
    __syncthreads();
    for (int e = 4 * tid; e < C * C; e += 4 * G::NT) {   // four columns s of one row t a thread
      int t, s;
      kmajor_rk(e, C, t, s);
      float p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        p[i] = s + i <= t ? wm::__float_to_tf32(expf(sG[t] - sG[s + i]) * sA[t * G::LDA + s + i]) : 0.f;
      *reinterpret_cast<float4*>(sPc + 4 * e) = make_float4(p[0], p[1], p[2], p[3]);
    }
    for (int idx = tid; idx < C * DK / 4; idx += G::NT) {   // e^G Q, four keys a thread
      const int t = idx / (DK / 4), j = 4 * (idx % (DK / 4));
      float q4[4];
      bf16x4_to_f32(sQ + t * G::LDK + j, q4);
      const float f = sEG[t];
      *reinterpret_cast<float4*>(sQc + kmajor_pad_off<C>(t, j)) =
          make_float4(wm::__float_to_tf32(f * q4[0]), wm::__float_to_tf32(f * q4[1]), wm::__float_to_tf32(f * q4[2]),
                      wm::__float_to_tf32(f * q4[3]));
    }
    for (int e = 4 * tid; e < DK * C; e += 4 * G::NT) {   // four tokens t of one key j a thread
      int j, t;
      kmajor_rk(e, C, j, t);
      const __nv_bfloat16* kc = sK + t * G::LDK + j;
      *reinterpret_cast<float4*>(sKc + 4 * e) =
          make_float4(wm::__float_to_tf32(sEnd[t] * __bfloat162float(kc[0])),
                      wm::__float_to_tf32(sEnd[t + 1] * __bfloat162float(kc[G::LDK])),
                      wm::__float_to_tf32(sEnd[t + 2] * __bfloat162float(kc[2 * G::LDK])),
                      wm::__float_to_tf32(sEnd[t + 3] * __bfloat162float(kc[3 * G::LDK])));
    }
    fence_smem_to_async();
    __syncthreads();
    if (tid == 0) {   // O^T = S^T (e^G Q)^T, first term
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, C>();
      const uint32_t q0 = smem_u32(sQc);
#pragma unroll
      for (int s = 0; s < DK / 8; ++s)
        umma_tf32_ts(tmem + G::TM_O, tmem + G::TM_S + 8 * s, umma_desc_lbo(q0 + 2 * G::WQ_LBO * s, G::WQ_LBO, 128),
                     ID, s > 0);
    }

    // 6. B^T = U^T - (W S)^T in tensor memory, tf32-rounded (columns 8 group ..)
    if (!mbar_wait_abortable(barB, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_after();
    if (!*sAbort) {
      for (int b8 = group; b8 < C / 8; b8 += NG) {
        float v[8], u[8];
        const uint32_t ta = tmem + lane_base + G::TM_B + 8 * b8;
        tmem_ld8(ta, v);
        tmem_ld8(tmem + lane_base + G::TM_U + 8 * b8, u);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = wm::__float_to_tf32(u[i] - v[i]);
        tmem_st8(ta, v);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (*sAbort) break;
    if (tid == 0) {   // O^T += B^T P^T
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, C>();
      const uint32_t p0 = smem_u32(sPc);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        umma_tf32_ts(tmem + G::TM_O, tmem + G::TM_B + 8 * s, umma_desc(p0 + 256 * s, (C / 4) * 128), ID, 1u);
      umma_commit(barO);
    }

    // 7. O rows < n to global; S^T scaled by e^{G_end} (every MMA reading it is done)
    if (!mbar_wait_abortable(barO, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_after();
    if (!*sAbort) {
      for (int b8 = group; b8 < C / 8; b8 += NG) {
        float v[8];
        tmem_ld8(tmem + lane_base + G::TM_O + 8 * b8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int t = 8 * b8 + i;
          if (t < n && own_col) Og[((c0 + t) * a.H + h) * DV + c_own] = __float2bfloat16_rn(v[i]);
        }
      }
      const float dend = sEG[n - 1];
      for (int cb = group; cb < DK / 32; cb += NG) {
        float sv[32];
        const uint32_t ts = tmem + lane_base + G::TM_S + 32 * cb;
        tmem_ld32(ts, sv);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] *= dend;
        tmem_st32(ts, sv);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (*sAbort) break;
    if (tid == 0) {   // S^T += B^T (e^{G_end - G} K)   (N = DK keys, K = C tokens)
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, DK>();
      const uint32_t k0 = smem_u32(sKc);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        umma_tf32_ts(tmem + G::TM_S, tmem + G::TM_B + 8 * s, umma_desc(k0 + 256 * s, (C / 4) * 128), ID, 1u);
      umma_commit(barS);
    }
  }

  // the last state update, then S^T back to Sbar
  if (ci > 0 && !*sAbort && !mbar_wait_abortable(barS, static_cast<uint32_t>((ci - 1) & 1), sAbort) && tid == 0)
    atomicOr(a.err, kErrWaitTimeout);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool ok = !*sAbort;
  if (ok) {
    for (int cb = group; cb < DK / 32; cb += NG) {
      float v[32];
      tmem_ld32(tmem + lane_base + G::TM_S + 32 * cb, v);
      if (own_col) {
#pragma unroll
        for (int i = 0; i < 32; ++i) __stcs(Sg + (32 * cb + i) * DV + c_own, v[i]);
      }
    }
  }
  if (!ok && tid == 0) {
    // After a timed-out wait, MMAs this thread issued (and their arrivals on
    // the barriers above) may still be pending: one more commit tracks all of
    // them, and the tensor memory is freed only once it arrives (or its own
    // bounded wait gives up).
    umma_commit(barF);
    mbar_wait_bounded(barF, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TM_COLS) : "memory");
  }
  if (ok) clear_log_tile<OP_GDN, DK, DV, __nv_bfloat16>(a, sh, 0, DV);
}

// Grid (H, rows), 256 threads (two CTAs per SM) once the launch has more CTAs
// than SMs, else 512; TcChunkGeom<NT, DK, DV>::BYTES of dynamic shared memory;
// bf16 inputs.  Instantiated in prefill.cu.
template <int DK, int DV>
cudaError_t launch_gdn_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);

// ---- KDA and RWKV6 (per-key decay) ---------------------------------------------
//
// The per-key chunk form (prefill_chunk.cuh) with the same tensor-memory
// state: A and P on the SIMT lanes (pairs across the chunk's halves as
// products of rows scaled once each), the blocked solve of the GDN kernel,
// its two products and the three products with the state on tcgen05.  RWKV6 has no W S product: its B^T is
// V^T, written straight into tensor memory.  The per-key decay of the state
// update scales the columns of S^T.

template <int NT_, int DK_ = 128, int DV_ = 128>
struct KeyTcChunkGeom {
  // 256 threads (two CTAs per SM) or 512 (one per SM, for launches with
  // fewer CTAs than SMs); value columns on lanes 0 .. DV-1 as in TcChunkGeom
  static constexpr int DK = DK_, DV = DV_, C = 32, NT = NT_, NW = NT / 32;
  static_assert((DK == 64 || DK == 128) && (DV == 64 || DV == 128), "head shape");
  static constexpr int NG = NW / 4;                 // column groups of the TMEM epilogues
  static constexpr int MINB = NT == 256 ? 2 : 1;
  static constexpr int LDK = DK + 8, LDV = DV + 8, LDG = DK + 4, LDA = C + 4;
  static constexpr int LDX = DK + 4;                                   // fp32 rows scaled through token 15
  static constexpr uint32_t WQ_LBO = kmajor_pad_lbo<C>();             // W and scaled-query operand layout
  // the W and scaled-query buffers also hold the solve's right-hand sides
  // R_W^T and R_U^T (dense K-major 128 x C) and, before them, the scaled rows
  // of the pair phase (two [16][LDX] arrays in the scaled-query buffer)
  static constexpr size_t WQ_MIN = size_t(128) * C * 4 > size_t(32) * LDX * 4 ? size_t(128) * C * 4 : size_t(32) * LDX * 4;
  static constexpr size_t WQ_BYTES = size_t(DK / 4) * WQ_LBO > WQ_MIN ? size_t(DK / 4) * WQ_LBO : WQ_MIN;
  static constexpr size_t KQ_BYTES = tc_align128(size_t(C) * LDK * 2), V_BYTES = tc_align128(size_t(C) * LDV * 2);
  static constexpr size_t G_BYTES = tc_align128(size_t(C) * LDG * 4);
  // single-buffered inputs: the next chunk's V streams in once the solve has
  // consumed V, its K, Q and gates once the operands have been built
  static constexpr size_t K_OFF = 0;                                   // [C][LDK] bf16
  static constexpr size_t Q_OFF = K_OFF + KQ_BYTES;                    // [C][LDK] bf16
  static constexpr size_t V_OFF = Q_OFF + KQ_BYTES;                    // [C][LDV] bf16
  static constexpr size_t G_OFF = V_OFF + V_BYTES;                     // [C][LDG] gates, then Gamma
  static constexpr size_t A_OFF = G_OFF + G_BYTES;                     // [C][LDA] A (KDA)
  static constexpr size_t P_OFF = tc_align128(A_OFF + size_t(C) * LDA * 4);   // [C][LDA] P
  static constexpr size_t WC_OFF = tc_align128(P_OFF + size_t(C) * LDA * 4);  // W, padded K-major C x DK
  static constexpr size_t QC_OFF = tc_align128(WC_OFF + WQ_BYTES);     // scaled queries, padded K-major C x DK
  static constexpr size_t PC_OFF = tc_align128(QC_OFF + WQ_BYTES);     // P, K-major C x C
  static constexpr size_t KC_OFF = PC_OFF + size_t(C) * C * 4;         // scaled keys^T, K-major DK x C
  static constexpr size_t E_OFF = tc_align128(KC_OFF + size_t(DK) * C * 4);  // e^{G_end} [DK], u [DK], beta [C]
  static constexpr size_t T_OFF = tc_align128(E_OFF + (2 * DK + C) * 4);     // [C][LDA] T = (I + A)^-1 (KDA)
  static constexpr size_t X_OFF = T_OFF + size_t(C) * LDA * 4;               // [16][17] A21 T11
  static constexpr size_t BAR_OFF = tc_align128(X_OFF + 16 * 17 * 4);
  static constexpr size_t BYTES = BAR_OFF + 64;
  // tensor-memory columns: S^T, W S then B^T, O^T, and the solve's products
  // U^T and W^T (KDA)
  static constexpr uint32_t TM_COLS = 256, TM_S = 0, TM_B = DK, TM_O = DK + 32, TM_U = DK + 64, TM_W = DK + 96;
};

template <int OP, int NT_, int DK_, int DV_>
__global__ void __launch_bounds__(NT_, KeyTcChunkGeom<NT_, DK_, DV_>::MINB)
key_chunk_prefill_tc_kernel(const PrefillArgs a) {
  using G = KeyTcChunkGeom<NT_, DK_, DV_>;
  constexpr int NG = G::NG;
  constexpr int C = G::C, DK = G::DK, DV = G::DV;
  constexpr bool DELTA = OP == OP_KDA;
  constexpr float LOG2E = 1.4426950408889634f;
  static_assert(OP == OP_KDA || OP == OP_RWKV6, "per-key decay operators");
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + G::K_OFF);
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + G::Q_OFF);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + G::V_OFF);
  float* sG = reinterpret_cast<float*>(smem + G::G_OFF);
  float* sA = reinterpret_cast<float*>(smem + G::A_OFF);
  float* sP = reinterpret_cast<float*>(smem + G::P_OFF);
  unsigned char* sWc = smem + G::WC_OFF;
  unsigned char* sQc = smem + G::QC_OFF;
  unsigned char* sPc = smem + G::PC_OFF;
  unsigned char* sKc = smem + G::KC_OFF;
  float* sE = reinterpret_cast<float*>(smem + G::E_OFF);
  float* sBonus = sE + DK;
  float* sBeta = sE + 2 * DK;
  float* sT = reinterpret_cast<float*>(smem + G::T_OFF);
  float* sX = reinterpret_cast<float*>(smem + G::X_OFF);
  uint64_t* barB = reinterpret_cast<uint64_t*>(smem + G::BAR_OFF);
  uint64_t* barO = barB + 1;
  uint64_t* barS = barB + 2;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(barB + 3);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
  uint64_t* barF = barB + 4;                                          // drain after an abort
  uint64_t* barT = barB + 5;                                          // the solve's products (KDA)
  auto fp = [](unsigned char* base, uint32_t off) { return reinterpret_cast<float*>(base + off); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quarter = warp & 3, group = warp >> 2;
  const int h = blockIdx.x;
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
  float* Sg = a.Sbar + sh * (DK * DV);

  if (tid == 0) {
    mbar_init(barB, 1);
    mbar_init(barO, 1);
    mbar_init(barS, 1);
    mbar_init(barF, 1);
    mbar_init(barT, 1);
    fence_mbar_init();
    *sAbort = 0;
  }
  if (OP == OP_RWKV6)
    for (int j = tid; j < DK; j += G::NT) sBonus[j] = a.u[h * DK + j];
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sTmem)),
                 "r"(G::TM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
  const int c_own = 32 * quarter + lane;
  const bool own_col = c_own < DV;
  for (int cb = group; cb < DK / 32; cb += NG) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = a.zero_state || !own_col ? 0.f : __ldcs(Sg + (32 * cb + i) * DV + c_own);
    tmem_st32(tmem + lane_base + G::TM_S + 32 * cb, v);
  }
  tmem_wait_st();

  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* Og = static_cast<__nv_bfloat16*>(a.o);
  const bool async_ok = aligned_to(a.q, 16) && aligned_to(a.k, 16) && aligned_to(a.v, 16) &&
                        aligned_to(a.log_decay, 16);
  auto stage_rows = [&](auto* dst, const auto* src, long c, int width, int ld) {
    using T = typename std::remove_const<typename std::remove_pointer<decltype(src)>::type>::type;
    constexpr int PER_SEG = 16 / static_cast<int>(sizeof(T));
    const int nv = static_cast<int>(t1 - c < C ? t1 - c : C);
    if (async_ok) {
      const int seg_per_row = width / PER_SEG;
      for (int idx = tid; idx < C * seg_per_row; idx += G::NT) {
        const int t = idx / seg_per_row, seg = idx % seg_per_row;
        const long row = ((c + (t < nv ? t : nv - 1)) * a.H + h) * width + PER_SEG * seg;
        cp_async16(dst + t * ld + PER_SEG * seg, src + row, t < nv ? 16u : 0u);
      }
    } else {
      for (int idx = tid; idx < C * width; idx += G::NT) {
        const int t = idx / width, j = idx % width;
        dst[t * ld + j] = t < nv ? src[((c + t) * a.H + h) * width + j] : T(0.f);
      }
    }
  };
  auto stage_kqg = [&](long c) {
    stage_rows(sK, Kg, c, DK, G::LDK);
    stage_rows(sQ, Qg, c, DK, G::LDK);
    stage_rows(sG, a.log_decay, c, DK, G::LDG);
  };
  float bnext = 0.f;
  if (t0 < t1) {
    stage_kqg(t0);
    stage_rows(sV, Vg, t0, DV, G::LDV);
    if (DELTA && tid < C && t0 + tid < t1) bnext = a.beta[(t0 + tid) * a.H + h];
  }
  cp_async_commit();
  auto kmajor_rk = [](int e, int kt, int& rr, int& kk) {
    const int core = e >> 5, within = e & 31;
    rr = (core / (kt >> 2)) * 8 + (within >> 2);
    kk = (core % (kt >> 2)) * 4 + (within & 3);
  };

  int ci = 0;
  for (long c0 = t0; c0 < t1; c0 += C, ++ci) {
    const int n = static_cast<int>(t1 - c0 < C ? t1 - c0 : C);
    const bool has_next = c0 + C < t1;
    const uint32_t par = static_cast<uint32_t>(ci & 1);
    __syncthreads();   // the previous chunk is done with every work buffer
    if (DELTA && tid < C) {
      sBeta[tid] = bnext;
      bnext = has_next && c0 + C + tid < t1 ? a.beta[(c0 + C + tid) * a.H + h] : 0.f;
    }
    cp_async_wait<0>();   // this chunk's inputs have landed
    __syncthreads();

    // 1. Gamma in log2 units, per key, in place; e^{Gamma_end}
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

    // 2. A and P; the rows scaled through token 15 sit in the scaled-query and
    // W buffers, free until the solve, the partial products in the T and P
    // operand buffers, free until then too
    key_pair_phase<OP, DK, C, G::NT, G::LDK, G::LDG, G::LDA, G::LDX>(
        sK, sQ, sG, sBeta, sBonus, fp(sQc, 0), fp(sQc, 16 * G::LDX * 4), fp(sWc, 0), sT, fp(sPc, 0), sA, sP);
    __syncthreads();

    if (DELTA) {
      // 3. (I + A) W = diag(beta) (2^Gamma (.) K) and (I + A) U = diag(beta) V as
      // W^T = R_W^T T^T and U^T = R_U^T T^T with T = (I + A)^{-1}, as in the GDN
      // kernel: T11 and T22 column by column on warp 0 while the other warps
      // write R_W^T (into the scaled-query buffer) and R_U^T (into the W buffer)
      // as dense K-major 128 x C operands, then T21 = -T22 (A21 T11), then the
      // two products on the tensor cores.
      if (warp == 0) {
        const int c = lane, r0 = c & ~15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = r0 + i;
          const float* arow = sA + t * G::LDA + r0;
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int k = 0; k + 1 < i; k += 2) {
            acc0 = fmaf(-arow[k], x[k], acc0);
            acc1 = fmaf(-arow[k + 1], x[k + 1], acc1);
          }
          if (i & 1) acc0 = fmaf(-arow[i - 1], x[i - 1], acc0);
          x[i] = t == c ? 1.f : t < c ? 0.f : acc0 + acc1;
          sT[t * G::LDA + c] = x[i];
          sT[(t ^ 16) * G::LDA + c] = 0.f;
        }
      } else {   // four tokens of one key a thread
        for (int e = 4 * (tid - 32); e < 128 * C; e += 4 * (G::NT - 32)) {
          int rr, s;
          kmajor_rk(e, C, rr, s);
          float w[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
          if (rr < DK) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = wm::__float_to_tf32(sBeta[s + i] * ex2_approx(sG[(s + i) * G::LDG + rr]) *
                                         __bfloat162float(sK[(s + i) * G::LDK + rr]));
          }
          if (rr < DV) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              u[i] = wm::__float_to_tf32(sBeta[s + i] * __bfloat162float(sV[(s + i) * G::LDV + rr]));
          }
          *reinterpret_cast<float4*>(sQc + 4 * e) = make_float4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<float4*>(sWc + 4 * e) = make_float4(u[0], u[1], u[2], u[3]);
        }
      }
      __syncthreads();
      if (tid < 256) {   // X = A21 T11 (zeros above the diagonals: 16 terms)
        const int i = 16 + (tid >> 4), j = tid & 15;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int l = 0; l < 16; l += 2) {
          acc0 = fmaf(sA[i * G::LDA + l], sT[l * G::LDA + j], acc0);
          acc1 = fmaf(sA[i * G::LDA + l + 1], sT[(l + 1) * G::LDA + j], acc1);
        }
        sX[(i - 16) * 17 + j] = acc0 + acc1;
      }
      __syncthreads();
      if (tid < 256) {   // T21 = -T22 X
        const int i = 16 + (tid >> 4), j = tid & 15;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          acc0 = fmaf(sT[i * G::LDA + 16 + k], sX[k * 17 + j], acc0);
          acc1 = fmaf(sT[i * G::LDA + 17 + k], sX[(k + 1) * 17 + j], acc1);
        }
        sT[i * G::LDA + j] = -(acc0 + acc1);
      }
      __syncthreads();
      for (int e = 4 * tid; e < C * C; e += 4 * G::NT) {   // T as the B operand (N = t, K = s), tf32
        int t, s;
        kmajor_rk(e, C, t, s);
        const float* tr = sT + t * G::LDA + s;
        *reinterpret_cast<float4*>(sPc + 4 * e) = make_float4(wm::__float_to_tf32(tr[0]), wm::__float_to_tf32(tr[1]),
                                                              wm::__float_to_tf32(tr[2]), wm::__float_to_tf32(tr[3]));
      }
      fence_smem_to_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID = umma_idesc_tf32<128, C>();
        const uint32_t t0 = smem_u32(sPc), rw = smem_u32(sQc), ru = smem_u32(sWc);
#pragma unroll
        for (int s = 0; s < C / 8; ++s)
          umma_tf32_ss(tmem + G::TM_W, umma_desc(rw + 256 * s, (C / 4) * 128), umma_desc(t0 + 256 * s, (C / 4) * 128),
                       ID, s > 0);
#pragma unroll
        for (int s = 0; s < C / 8; ++s)
          umma_tf32_ss(tmem + G::TM_U, umma_desc(ru + 256 * s, (C / 4) * 128), umma_desc(t0 + 256 * s, (C / 4) * 128),
                       ID, s > 0);
        umma_commit(barT);
      }
      if (!mbar_wait_abortable(barT, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
      tc_fence_after();
      if (!*sAbort && c_own < DK) {   // W^T (key j on lane j) into W's padded operand layout, tf32
        for (int b8 = group; b8 < C / 8; b8 += NG) {
          float v[8];
          tmem_ld8(tmem + lane_base + G::TM_W + 8 * b8, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) fp(sWc, kmajor_pad_off<C>(8 * b8 + i, c_own))[0] = wm::__float_to_tf32(v[i]);
        }
      }
      fence_smem_to_async();
    }

    // 4. the previous chunk's state update must be complete (it reads B^T and
    // the scaled keys, and writes S^T)
    if (ci > 0 && !mbar_wait_abortable(barS, par ^ 1u, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_before();
    __syncthreads();
    if (*sAbort) break;
    tc_fence_after();
    if (DELTA) {
      if (tid == 0) {   // W S
        constexpr uint32_t ID = umma_idesc_tf32<128, C>();
        const uint32_t w0 = smem_u32(sWc);
#pragma unroll
        for (int s = 0; s < DK / 8; ++s)
          umma_tf32_ts(tmem + G::TM_B, tmem + G::TM_S + 8 * s,
                       umma_desc_lbo(w0 + 2 * G::WQ_LBO * s, G::WQ_LBO, 128), ID, s > 0);
        umma_commit(barB);
      }
    } else {
      // B^T = V^T (bf16 values are tf32-exact), column blocks 8 b8 ..
      for (int b8 = group; b8 < C / 8; b8 += NG) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = own_col ? __bfloat162float(sV[(8 * b8 + i) * G::LDV + c_own]) : 0.f;
        tmem_st8(tmem + lane_base + G::TM_B + 8 * b8, v);
      }
      tmem_wait_st();
    }

    // 5. P, the scaled queries and the scaled keys^T into their operand layouts
    for (int e = 4 * tid; e < C * C; e += 4 * G::NT) {   // tf32-rounded, zero above the diagonal
      int t, s;
      kmajor_rk(e, C, t, s);
      const float* pr = sP + t * G::LDA + s;
      *reinterpret_cast<float4*>(sPc + 4 * e) = make_float4(pr[0], pr[1], pr[2], pr[3]);
    }
    for (int idx = tid; idx < C * DK / 4; idx += G::NT) {   // four keys a thread
      const int t = idx / (DK / 4), j = 4 * (idx % (DK / 4));
      const int tg = DELTA ? t : t - 1;   // Gamma_t (KDA), Gamma_{t-1} (RWKV6)
      const float4 g = tg >= 0 ? *reinterpret_cast<const float4*>(sG + tg * G::LDG + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      float q4[4];
      bf16x4_to_f32(sQ + t * G::LDK + j, q4);
      *reinterpret_cast<float4*>(sQc + kmajor_pad_off<C>(t, j)) =
          make_float4(wm::__float_to_tf32(ex2_approx(g.x) * q4[0]), wm::__float_to_tf32(ex2_approx(g.y) * q4[1]),
                      wm::__float_to_tf32(ex2_approx(g.z) * q4[2]), wm::__float_to_tf32(ex2_approx(g.w) * q4[3]));
    }
    for (int e = 4 * tid; e < DK * C; e += 4 * G::NT) {   // four tokens t of one key j a thread
      int j, t;
      kmajor_rk(e, C, j, t);
      const float gend = sG[(C - 1) * G::LDG + j];
      float k4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        k4[i] = wm::__float_to_tf32(ex2_approx(gend - sG[(t + i) * G::LDG + j]) *
                                    __bfloat162float(sK[(t + i) * G::LDK + j]));
      *reinterpret_cast<float4*>(sKc + 4 * e) = make_float4(k4[0], k4[1], k4[2], k4[3]);
    }
    fence_smem_to_async();
    tc_fence_before();
    __syncthreads();
    // every read of this chunk's K, Q, V and gates is done: the next chunk's stream in
    if (has_next) {
      stage_kqg(c0 + C);
      stage_rows(sV, Vg, c0 + C, DV, G::LDV);
    }
    cp_async_commit();
    if (tid == 0) {   // O^T = S^T (scaled Q)^T  (+ B^T P^T at once for RWKV6)
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, C>();
      const uint32_t q0 = smem_u32(sQc);
#pragma unroll
      for (int s = 0; s < DK / 8; ++s)
        umma_tf32_ts(tmem + G::TM_O, tmem + G::TM_S + 8 * s, umma_desc_lbo(q0 + 2 * G::WQ_LBO * s, G::WQ_LBO, 128),
                     ID, s > 0);
      if (!DELTA) {
        const uint32_t p0 = smem_u32(sPc);
#pragma unroll
        for (int s = 0; s < C / 8; ++s)
          umma_tf32_ts(tmem + G::TM_O, tmem + G::TM_B + 8 * s, umma_desc(p0 + 256 * s, (C / 4) * 128), ID, 1u);
        umma_commit(barO);
      }
    }

    if (DELTA) {
      // 6. B^T = U^T - (W S)^T, tf32-rounded, then O^T += B^T P^T
      if (!mbar_wait_abortable(barB, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
      tc_fence_after();
      if (!*sAbort) {
        for (int b8 = group; b8 < C / 8; b8 += NG) {
          float v[8], u[8];
          const uint32_t ta = tmem + lane_base + G::TM_B + 8 * b8;
          tmem_ld8(ta, v);
          tmem_ld8(tmem + lane_base + G::TM_U + 8 * b8, u);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = wm::__float_to_tf32(u[i] - v[i]);
          tmem_st8(ta, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncthreads();
      if (*sAbort) break;
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID = umma_idesc_tf32<128, C>();
        const uint32_t p0 = smem_u32(sPc);
#pragma unroll
        for (int s = 0; s < C / 8; ++s)
          umma_tf32_ts(tmem + G::TM_O, tmem + G::TM_B + 8 * s, umma_desc(p0 + 256 * s, (C / 4) * 128), ID, 1u);
        umma_commit(barO);
      }
    }

    // 7. O rows < n to global; S^T columns scaled by e^{Gamma_end}; S^T += B^T (scaled K)
    if (!mbar_wait_abortable(barO, par, sAbort) && tid == 0) atomicOr(a.err, kErrWaitTimeout);
    tc_fence_after();
    if (!*sAbort) {
      for (int b8 = group; b8 < C / 8; b8 += NG) {
        float v[8];
        tmem_ld8(tmem + lane_base + G::TM_O + 8 * b8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int t = 8 * b8 + i;
          if (t < n && own_col) Og[((c0 + t) * a.H + h) * DV + c_own] = __float2bfloat16_rn(v[i]);
        }
      }
      for (int cb = group; cb < DK / 32; cb += NG) {
        float sv[32];
        const uint32_t ts = tmem + lane_base + G::TM_S + 32 * cb;
        tmem_ld32(ts, sv);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] *= sE[32 * cb + i];
        tmem_st32(ts, sv);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (*sAbort) break;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ID = umma_idesc_tf32<128, DK>();
      const uint32_t k0 = smem_u32(sKc);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        umma_tf32_ts(tmem + G::TM_S, tmem + G::TM_B + 8 * s, umma_desc(k0 + 256 * s, (C / 4) * 128), ID, 1u);
      umma_commit(barS);
    }
  }

  if (ci > 0 && !*sAbort && !mbar_wait_abortable(barS, static_cast<uint32_t>((ci - 1) & 1), sAbort) && tid == 0)
    atomicOr(a.err, kErrWaitTimeout);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool ok = !*sAbort;
  if (ok) {
    for (int cb = group; cb < DK / 32; cb += NG) {
      float v[32];
      tmem_ld32(tmem + lane_base + G::TM_S + 32 * cb, v);
      if (own_col) {
#pragma unroll
        for (int i = 0; i < 32; ++i) __stcs(Sg + (32 * cb + i) * DV + c_own, v[i]);
      }
    }
  }
  if (!ok && tid == 0) {
    // After a timed-out wait, MMAs this thread issued (and their arrivals on
    // the barriers above) may still be pending: one more commit tracks all of
    // them, and the tensor memory is freed only once it arrives (or its own
    // bounded wait gives up).
    umma_commit(barF);
    mbar_wait_bounded(barF, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TM_COLS) : "memory");
  }
  if (ok) clear_log_tile<OP, DK, DV, __nv_bfloat16>(a, sh, 0, DV);
}

// Grid (H, rows), 256 threads (two CTAs per SM) once the launch has more CTAs
// than SMs, else 512; KeyTcChunkGeom<NT, DK, DV>::BYTES of dynamic shared
// memory; bf16 inputs.  Instantiated in prefill.cu.
template <int OP, int DK, int DV>
cudaError_t launch_key_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);

}  // namespace dl
