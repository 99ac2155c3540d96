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
// One CTA per (row, head, 32-column value tile) keeps its d_k x 32 slice of
// the state in registers for the row's whole prompt; only q, k, v, gates and
// o stream through HBM (state read once, written once).  Each token runs the
// eager update of the operator (same arithmetic as the eager step kernel),
// with the next token's inputs prefetched into registers during the current
// one, so the per-token chain is three block barriers and no global-memory
// latency.
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
  int zero_state;          // 1: every row starts from S = 0; 0: from Sbar
};

// Clear entries [0, n) of unit `sh`'s log: the b_i columns of this value tile,
// and (first tile only) a_i and Lam_i.  Zero entries add nothing to S_t, and
// Lam_i = 0 restarts the unit's cumulative decay at the hand-off.
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
    for (int idx = threadIdx.x; idx < n * DK; idx += blockDim.x) a.logLam[sh * a.Mcap * DK + idx] = 0.f;
  }
}

// d_k = 128 tiles hold 64 state registers per thread next to the prefetched
// inputs: six CTAs per SM leave them 170 registers without spills.
template <int DK>
constexpr int kPrefillMinBlocks = DK == 128 ? 6 : 8;

template <int OP, int DK, int DV, typename TI>
__global__ void __launch_bounds__(Tile<DK, 32>::NT, kPrefillMinBlocks<DK>)
prefill_kernel(const PrefillArgs a) {
  constexpr int DVT = 32;                 // value columns per CTA
  constexpr int NSPLIT = DV / DVT;
  using TL = Tile<DK, DVT>;
  constexpr bool DELTA = OP != OP_RWKV6;
  static_assert(TL::NT == 64 && TL::KPL * 32 == DK, "prefill tile: two warps, warp 0 owns keys and columns");

  __shared__ __align__(16) float s_kx[DK];      // contraction vector for p
  __shared__ __align__(16) float s_qx[DK];      // contraction vector for s
  __shared__ __align__(16) float s_dec[2][DK];  // per-row decay (double-buffered: read after the last barrier)
  __shared__ __align__(16) float s_k[2][DK];    // k_t rows of the rank-1 update (double-buffered)
  __shared__ __align__(16) float s_b[DVT];      // b_t columns of the rank-1 update
  __shared__ __align__(16) float s_red[2][TL::RG][DVT];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % TL::TPR, rg = tid / TL::TPR;
  const int h = static_cast<int>(blockIdx.x) / NSPLIT;
  const int col0 = (static_cast<int>(blockIdx.x) % NSPLIT) * DVT;
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
  float* Sp = a.Sbar + sh * (DK * DV);

  float4 st[TL::RPT];
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j)
    st[j] = a.zero_state ? make_float4(0.f, 0.f, 0.f, 0.f) : ld_state(Sp + (rg * TL::RPT + j) * DV + col0 + 4 * c4);

  // Warp 0 holds the next token's inputs: keys j = lane + 32 m, and value
  // column `lane` of this tile.
  float kn[TL::KPL], qn[TL::KPL], gn[TL::KPL], vn = 0.f, bn = 0.f;
  auto fetch = [&](long t) {
    const long bu = t * a.H + h;
    const TI* qg = static_cast<const TI*>(a.q) + bu * DK;
    const TI* kg = static_cast<const TI*>(a.k) + bu * DK;
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      kn[m] = to_f(kg[j]);
      qn[m] = to_f(qg[j]);
      gn[m] = OP == OP_GDN ? (m == 0 ? a.log_decay[bu] : 0.f) : a.log_decay[bu * DK + j];
    }
    vn = to_f(static_cast<const TI*>(a.v)[bu * DV + col0 + lane]);
    if (DELTA) bn = a.beta[bu];
  };
  if (warp == 0 && t0 < t1) fetch(t0);
  float ur[TL::KPL];
#pragma unroll
  for (int m = 0; m < TL::KPL; ++m) ur[m] = OP == OP_RWKV6 && warp == 0 ? a.u[h * DK + lane + 32 * m] : 0.f;

  for (long t = t0; t < t1; ++t) {
    const int buf = static_cast<int>(t & 1);
    float kap = 0.f, alpha = 1.f;
    const float vc = vn, betac = bn;
    if (warp == 0) {
      if (OP == OP_GDN) alpha = expf(__shfl_sync(0xffffffffu, gn[0], 0));
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) {
        const int j = lane + 32 * m;
        const float dec = OP == OP_GDN ? alpha : expf(gn[m]);
        s_dec[buf][j] = dec;
        s_k[buf][j] = kn[m];
        if (OP == OP_GDN) {          // p = S^T k, s = S^T q (alpha applied after)
          s_kx[j] = kn[m];
          s_qx[j] = qn[m];
          kap = fmaf(kn[m], qn[m], kap);
        } else if (OP == OP_KDA) {   // p = S^T (alpha (.) k), s = S^T (alpha (.) q)
          s_kx[j] = dec * kn[m];
          s_qx[j] = dec * qn[m];
          kap = fmaf(kn[m], qn[m], kap);
        } else {                     // RWKV6: s = S^T r, kappa = (u (.) k) . r
          s_qx[j] = qn[m];
          kap = fmaf(ur[m] * kn[m], qn[m], kap);
        }
      }
      kap = warp_sum(kap);
      if (t + 1 < t1) fetch(t + 1);  // in flight during this token's passes
    }
    __syncthreads();

    {
      float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = p4;
#pragma unroll
      for (int j = 0; j < TL::RPT; ++j) {
        const int row = rg * TL::RPT + j;
        if (DELTA) fma4(p4, s_kx[row], st[j]);
        fma4(s4, s_qx[row], st[j]);
      }
      if (DELTA) *reinterpret_cast<float4*>(&s_red[0][rg][4 * c4]) = p4;
      *reinterpret_cast<float4*>(&s_red[1][rg][4 * c4]) = s4;
    }
    __syncthreads();

    if (warp == 0) {  // value column `lane` of the tile
      float p = 0.f, s = 0.f;
#pragma unroll
      for (int g = 0; g < TL::RG; ++g) {
        if (DELTA) p += s_red[0][g][lane];
        s += s_red[1][g][lane];
      }
      float oc, bt;
      if (OP == OP_GDN) {
        bt = betac * (vc - alpha * p);
        oc = fmaf(kap, bt, alpha * s);
      } else if (OP == OP_KDA) {
        bt = betac * (vc - p);
        oc = fmaf(kap, bt, s);
      } else {
        bt = vc;
        oc = fmaf(kap, vc, s);
      }
      s_b[lane] = bt;
      static_cast<TI*>(a.o)[(t * a.H + h) * DV + col0 + lane] = from_f<TI>(oc);
    }
    __syncthreads();

    const float4 b4 = *reinterpret_cast<const float4*>(&s_b[4 * c4]);
#pragma unroll
    for (int j = 0; j < TL::RPT; ++j) {
      const int row = rg * TL::RPT + j;
      scale4(st[j], s_dec[buf][row]);
      fma4(st[j], s_k[buf][row], b4);
    }
  }

#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) st_state(Sp + (rg * TL::RPT + j) * DV + col0 + 4 * c4, st[j]);
  clear_log_tile<OP, DK, DV, TI>(a, sh, col0, DVT);
}

// Grid (H * d_v/32, rows), 64 threads.  Instantiated in prefill.cu.
template <int OP>
cudaError_t launch_prefill_op(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st);
extern template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
extern template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
extern template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
