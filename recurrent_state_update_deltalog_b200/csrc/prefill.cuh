// Prefill -> decode hand-off: the recurrence over a packed batch of prompts,
// ending with each prompt's state written as its slot's dense base Sbar.
//
// The pages' path starts from a dense base state that a prefill produced
// (DeltaLog technical summary, gist.science, "Method -- core mechanism:
// base + log": the base holds the accumulated history up to the last merge
// point).  A prompt's final state is such a point, so the prefill writes it
// straight into Sbar and clears the slot's log entries; decode steps then
// append to it like to any merged base.
//
// One warp per (row, head, 16-column value tile) keeps its d_k x 16 slice of
// the state in registers for the row's whole prompt; only q, k, v, gates and
// o stream through HBM (state read once, written once).  Each token runs the
// eager update of the operator (same arithmetic as the eager step kernel)
// with the next token's inputs prefetched into registers during the current
// one.  The per-row key-side values pass through double-buffered shared
// memory behind one __syncwarp, the cross-row reduction is three xor
// shuffles, and each lane finalises its own four columns: no block barrier
// on the per-token chain.
#pragma once

#include "launch.cuh"

namespace dl {

// Device error bit: a row whose cu_seqlens range is invalid (the row is skipped).
constexpr int kErrSeqlen = 4;

struct PrefillArgs {
  float* Sbar;             // [B*H][DK][DV]
  const void* q;           // [total][H][DK] (r for RWKV6), input dtype
  const void* k;           // [total][H][DK]
  const void* v;           // [total][H][DV]
  const float* log_decay;  // [total][H] (GDN) or [total][H][DK]
  const float* beta;       // [total][H] (GDN/KDA)
  void* o;                 // [total][H][DV], input dtype
  const float* u;          // [H][DK] (RWKV6)
  const int* slot_idx;     // [rows] slot of each row (< 0: skip), or null (row r = slot r)
  const int* cu_seqlens;   // [rows + 1] token offsets of the rows
  void* logA;              // log regions whose entries [0, n) are cleared
  void* logB;
  float* logLam;
  int* err;
  long total;              // tokens in the packed batch
  int H, slots, Mcap, n;
  int b_esize;             // bytes of one b_i element in the log (2 or 4)
  int lam_esize;           // bytes of one per-key Lam element in the log (4, or 2 for fp16 log-gates)
  int zero_state;          // 1: every row starts from S = 0; 0: from Sbar
};

// Clear entries [0, n) of unit `sh`'s log: the b_i columns of this value tile,
// and (first tile only) a_i and Lam_i.  Zero entries add nothing to S_t, and
// Lam_i = 0 (or zero log-gates, with fp16 per-key snapshots) restarts the
// unit's cumulative decay at the hand-off.
template <int OP, int DK, int DV, typename TI>
__device__ __forceinline__ void clear_log_tile(const PrefillArgs& a, long sh, int col0, int ncols) {
  const int n = a.n;
  if (n == 0) return;
  const int halves_per_col = a.b_esize / 2;
  unsigned short* b = static_cast<unsigned short*>(a.logB);
  for (int idx = threadIdx.x; idx < n * ncols * halves_per_col; idx += blockDim.x) {
    const int i = idx / (ncols * halves_per_col), w = idx % (ncols * halves_per_col);
    b[((sh * a.Mcap + i) * DV + col0) * halves_per_col + w] = 0;
  }
  if (col0 != 0) return;
  TI* A = static_cast<TI*>(a.logA) + sh * a.Mcap * DK;
  for (int idx = threadIdx.x; idx < n * DK; idx += blockDim.x) A[idx] = from_f<TI>(0.f);
  if (OP == OP_GDN) {
    for (int idx = threadIdx.x; idx < n; idx += blockDim.x) a.logLam[sh * gdn_lam_stride(a.Mcap) + idx] = 0.f;
  } else {
    const int halves = a.lam_esize / 2;
    unsigned short* lam = reinterpret_cast<unsigned short*>(a.logLam) + sh * a.Mcap * DK * halves;
    for (int idx = threadIdx.x; idx < n * DK * halves; idx += blockDim.x) lam[idx] = 0;
  }
}

// Geometry of the one-warp prefill tile: 16 value columns, lane = 4 x row
// group + column group; each lane holds RPT rows x 4 columns of the state.
// Rows are interleaved so that a lane's rows come in runs of four
// (row = 32 jb + 4 rg + i): its shared-memory reads of per-row values are
// 128-bit and the eight row groups hit eight different bank quads.
template <int DK>
struct PrefillTile {
  static constexpr int CW = 16;          // value columns per CTA
  static constexpr int RG = 8;           // row groups
  static constexpr int RPT = DK / RG;    // rows per lane
  static constexpr int KPL = DK / 32;    // keys per lane when loading
  // resident warps per SM the register budget is sized for (measured on
  // B200: 16 warps of <= 128 registers beat 12 warps with a two-token input
  // lookahead by 25% at d_k = 128)
  static constexpr int MINB = DK == 128 ? 16 : 24;
  __device__ static int row(int jj, int rg) { return (jj >> 2) * 32 + rg * 4 + (jj & 3); }
};

template <int OP, int DK, int DV, typename TI>
__global__ void __launch_bounds__(32, PrefillTile<DK>::MINB)
prefill_kernel(const PrefillArgs a) {
  using PT = PrefillTile<DK>;
  constexpr int CW = PT::CW, RPT = PT::RPT, KPL = PT::KPL;
  constexpr int NSPLIT = DV / CW;
  constexpr bool DELTA = OP != OP_RWKV6;
  static_assert(RPT % 4 == 0 && KPL * 32 == DK, "prefill tile shape");

  // per-row key-side values of a token, double-buffered across tokens
  __shared__ __align__(16) float s_kx[2][DK];   // contraction vector for p
  __shared__ __align__(16) float s_qx[2][DK];   // contraction vector for s
  __shared__ __align__(16) float s_dec[2][DK];  // per-row decay
  __shared__ __align__(16) float s_k[2][DK];    // k_t rows of the rank-1 update

  const int lane = threadIdx.x;
  const int c4 = lane & 3, rg = lane >> 2;
  const int h = static_cast<int>(blockIdx.x) / NSPLIT;
  const int col0 = (static_cast<int>(blockIdx.x) % NSPLIT) * CW;
  const int r = blockIdx.y;

  const int slot = a.slot_idx ? __ldg(a.slot_idx + r) : r;
  if (slot < 0) return;
  if (slot >= a.slots) {
    if (lane == 0) atomicOr(a.err, kErrSlotIndex);
    return;
  }
  const long t0 = __ldg(a.cu_seqlens + r), t1 = __ldg(a.cu_seqlens + r + 1);
  if (t0 < 0 || t1 < t0 || t1 > a.total) {
    if (lane == 0) atomicOr(a.err, kErrSeqlen);
    return;
  }
  const long sh = static_cast<long>(slot) * a.H + h;
  float* Sp = a.Sbar + sh * (DK * DV) + col0 + 4 * c4;

  float4 st[RPT];
#pragma unroll
  for (int jj = 0; jj < RPT; ++jj)
    st[jj] = a.zero_state ? make_float4(0.f, 0.f, 0.f, 0.f) : ld_state(Sp + PT::row(jj, rg) * DV);

  // The next token's inputs, in registers: keys j = lane + 32 m, and this
  // lane's four value columns (scalar accesses: inputs need only element
  // alignment).
  float kn[KPL], qn[KPL], gn[KPL], vn[4], bn = 0.f;
  auto fetch = [&](long t) {
    const long bu = t * a.H + h;
    const TI* qg = static_cast<const TI*>(a.q) + bu * DK;
    const TI* kg = static_cast<const TI*>(a.k) + bu * DK;
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      const int j = lane + 32 * m;
      kn[m] = to_f(kg[j]);
      qn[m] = to_f(qg[j]);
      gn[m] = OP == OP_GDN ? 0.f : a.log_decay[bu * DK + j];
    }
    if (OP == OP_GDN) gn[0] = a.log_decay[bu];
    const TI* vg = static_cast<const TI*>(a.v) + bu * DV + col0 + 4 * c4;
#pragma unroll
    for (int i = 0; i < 4; ++i) vn[i] = to_f(vg[i]);
    if (DELTA) bn = a.beta[bu];
  };
  if (t0 < t1) fetch(t0);
  float ur[KPL];
#pragma unroll
  for (int m = 0; m < KPL; ++m) ur[m] = OP == OP_RWKV6 ? a.u[h * DK + lane + 32 * m] : 0.f;

  for (long t = t0; t < t1; ++t) {
    const int buf = static_cast<int>(t & 1);
    const float4 vc = make_float4(vn[0], vn[1], vn[2], vn[3]);
    const float betac = bn;
    const float alpha = OP == OP_GDN ? expf(gn[0]) : 1.f;
    float kap = 0.f;
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      const int j = lane + 32 * m;
      const float dec = OP == OP_GDN ? alpha : expf(gn[m]);
      s_dec[buf][j] = dec;
      s_k[buf][j] = kn[m];
      if (OP == OP_GDN) {          // p = S^T k, s = S^T q (alpha applied after)
        s_kx[buf][j] = kn[m];
        s_qx[buf][j] = qn[m];
        kap = fmaf(kn[m], qn[m], kap);
      } else if (OP == OP_KDA) {   // p = S^T (alpha (.) k), s = S^T (alpha (.) q)
        s_kx[buf][j] = dec * kn[m];
        s_qx[buf][j] = dec * qn[m];
        kap = fmaf(kn[m], qn[m], kap);
      } else {                     // RWKV6: s = S^T r, kappa = (u (.) k) . r
        s_qx[buf][j] = qn[m];
        kap = fmaf(ur[m] * kn[m], qn[m], kap);
      }
    }
    kap = warp_sum(kap);
    if (t + 1 < t1) fetch(t + 1);  // in flight during this token's passes
    __syncwarp();

    // contraction over this lane's rows, then over the eight row groups
    float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = p4;
#pragma unroll
    for (int jb = 0; jb < RPT / 4; ++jb) {
      const int base = jb * 32 + rg * 4;
      const float4 qx = *reinterpret_cast<const float4*>(&s_qx[buf][base]);
      fma4(s4, qx.x, st[4 * jb + 0]);
      fma4(s4, qx.y, st[4 * jb + 1]);
      fma4(s4, qx.z, st[4 * jb + 2]);
      fma4(s4, qx.w, st[4 * jb + 3]);
      if (DELTA) {
        const float4 kx = *reinterpret_cast<const float4*>(&s_kx[buf][base]);
        fma4(p4, kx.x, st[4 * jb + 0]);
        fma4(p4, kx.y, st[4 * jb + 1]);
        fma4(p4, kx.z, st[4 * jb + 2]);
        fma4(p4, kx.w, st[4 * jb + 3]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      s4.x += __shfl_xor_sync(0xffffffffu, s4.x, off);
      s4.y += __shfl_xor_sync(0xffffffffu, s4.y, off);
      s4.z += __shfl_xor_sync(0xffffffffu, s4.z, off);
      s4.w += __shfl_xor_sync(0xffffffffu, s4.w, off);
      if (DELTA) {
        p4.x += __shfl_xor_sync(0xffffffffu, p4.x, off);
        p4.y += __shfl_xor_sync(0xffffffffu, p4.y, off);
        p4.z += __shfl_xor_sync(0xffffffffu, p4.z, off);
        p4.w += __shfl_xor_sync(0xffffffffu, p4.w, off);
      }
    }

    // this lane's four columns: b_t and o_t (every row group holds the same)
    float bt[4], oc[4];
    const float pv[4] = {p4.x, p4.y, p4.z, p4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
    const float vv[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (OP == OP_GDN) {
        bt[i] = betac * (vv[i] - alpha * pv[i]);
        oc[i] = fmaf(kap, bt[i], alpha * sv[i]);
      } else if (OP == OP_KDA) {
        bt[i] = betac * (vv[i] - pv[i]);
        oc[i] = fmaf(kap, bt[i], sv[i]);
      } else {
        bt[i] = vv[i];
        oc[i] = fmaf(kap, vv[i], sv[i]);
      }
    }
    if (rg == 0) {
      TI* og = static_cast<TI*>(a.o) + (t * a.H + h) * DV + col0 + 4 * c4;
#pragma unroll
      for (int i = 0; i < 4; ++i) og[i] = from_f<TI>(oc[i]);
    }

    // S_t = diag(dec) S_{t-1} + k_t b_t^T on this lane's rows and columns
    const float4 b4 = make_float4(bt[0], bt[1], bt[2], bt[3]);
#pragma unroll
    for (int jb = 0; jb < RPT / 4; ++jb) {
      const int base = jb * 32 + rg * 4;
      const float4 d4 = *reinterpret_cast<const float4*>(&s_dec[buf][base]);
      const float4 k4 = *reinterpret_cast<const float4*>(&s_k[buf][base]);
      const float dd[4] = {d4.x, d4.y, d4.z, d4.w}, kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        scale4(st[4 * jb + i], dd[i]);
        fma4(st[4 * jb + i], kk[i], b4);
      }
    }
  }

#pragma unroll
  for (int jj = 0; jj < RPT; ++jj) st_state(Sp + PT::row(jj, rg) * DV, st[jj]);
  clear_log_tile<OP, DK, DV, TI>(a, sh, col0, CW);
}

// Chunked GDN prefill with the state in tensor memory (bf16 inputs;
// prefill_chunk_tc.cuh), any supported d_k x d_v: grid (H, rows).
// cudaErrorNotSupported when its shared memory does not fit the device.
cudaError_t launch_gdn_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);

// Chunked KDA / RWKV6 prefill with the state in tensor memory (bf16 inputs;
// prefill_chunk_tc.cuh): grid (H, rows).  cudaErrorNotSupported when its
// shared memory does not fit the device.
template <int OP>
cudaError_t launch_key_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);
extern template cudaError_t launch_key_chunk_prefill_dims<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
extern template cudaError_t launch_key_chunk_prefill_dims<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

// Grid (H * d_v/16, rows), one warp per CTA.  Instantiated in prefill.cu.
template <int OP>
cudaError_t launch_prefill_op(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);
extern template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
extern template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
extern template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
