// Persistent, TMA-pipelined DeltaLog step for sm_100a.
//
// Same arithmetic as deltalog_step_kernel (kernels.cuh), different data
// movement.  A grid of (CTAs per SM) x (SM count) persistent CTAs walks the
// (slot, head) units round-robin.  The fp32 state is cut into 16 KB chunks
// (CR rows x d_v) that one producer thread streams into a ring of NS
// shared-memory stages with TMA bulk copies (cp.async.bulk, no multicast),
// each stage completing on its own mbarrier.  A unit's log (a_i, Lam_i, b_i),
// its q/k/v, per-key gates and RWKV6 bonus row go into one of two unit slots
// (double buffered: unit iu+1's slot is issued when unit iu starts).  Consumers accumulate Sbar^T k~ and
// Sbar^T q~ chunk by chunk from shared memory and release each stage as soon
// as it is consumed (append), or after the unit's merged state has been
// written back (merge), so up to NS-1 chunks are in flight per CTA at all
// times instead of one CTA's worth of registers.
//
// Every mbarrier wait is bounded: a timeout raises kErrWaitTimeout in the
// device error word, the CTA leaves its loop at the next barrier (all threads
// agree through __syncthreads_or) and thread 0 waits, again bounded, for the
// copies it issued before the CTA exits.
#pragma once

#include "kernels.cuh"

namespace dl {

constexpr int kChunkBytes = 16384;
constexpr int kMaxStages = 12;
constexpr int kUnitSlots = 2;

__host__ __device__ constexpr size_t round_up16(size_t x) { return (x + 15) & ~size_t(15); }

template <int OP, int DK, int DV, typename TI>
struct StreamGeom {
  using TB = typename std::conditional<OP == OP_RWKV6, TI, float>::type;
  static constexpr bool PERKEY = OP != OP_GDN;
  static constexpr int CR = kChunkBytes / (DV * 4);  // state rows per chunk
  static constexpr int CPU = DK / CR;                 // chunks per (slot, head)
  static constexpr int RPC = CR / 8;                  // rows per thread per chunk
  static_assert(CR % 8 == 0 && DK % CR == 0, "chunk shape");

  // Unit slot layout (bytes, each region 16-byte aligned):
  //   A [n][DK] TI | L: [n][DK] f32 (per-key) or round4(n) f32 (GDN) | B [n][DV] TB |
  //   q [DK] TI | k [DK] TI | v [DV] TI | log_decay [DK] f32 (per-key) | u [DK] f32 (RWKV6)
  __host__ __device__ static constexpr size_t a_bytes(int n) { return size_t(n) * DK * sizeof(TI); }
  __host__ __device__ static constexpr size_t l_bytes(int n) {
    return PERKEY ? size_t(n) * DK * 4 : size_t((n + 3) & ~3) * 4;
  }
  __host__ __device__ static constexpr size_t b_bytes(int n) { return size_t(n) * DV * sizeof(TB); }
  __host__ __device__ static constexpr size_t log_bytes(int n) { return a_bytes(n) + l_bytes(n) + b_bytes(n); }
  __host__ __device__ static constexpr size_t io_bytes() {
    return size_t(2 * DK + DV) * sizeof(TI) + (PERKEY ? DK * 4 : 0) + (OP == OP_RWKV6 ? DK * 4 : 0);
  }
  __host__ __device__ static constexpr size_t slot_bytes(int n) { return round_up16(log_bytes(n) + io_bytes()); }
  __host__ __device__ static constexpr size_t merge_bytes(int n) { return size_t(n + 1) * DK * 4 + DV * 4; }
  __host__ __device__ static constexpr size_t smem(int n, bool merge, int ns) {
    return size_t(ns) * kChunkBytes + kUnitSlots * slot_bytes(n) + (merge ? merge_bytes(n) : 0);
  }
};

struct StreamCfg {
  int BH;   // units
  int ns;   // ring stages (16 KB each)
};

template <int OP, int DK, int DV, typename TI, bool MERGE>
__global__ void __launch_bounds__(Tile<DK, DV>::NT, 2)
deltalog_stream_kernel(const StepArgs a, const StreamCfg cfg) {
  using TL = Tile<DK, DV>;
  using SG = StreamGeom<OP, DK, DV, TI>;
  using TB = typename SG::TB;
  constexpr bool DELTA = OP != OP_RWKV6;
  constexpr bool PERKEY = SG::PERKEY;
  constexpr int CR = SG::CR, CPU = SG::CPU, RPC = SG::RPC;
  constexpr int CHF = kChunkBytes / 4;  // floats per chunk

  __shared__ __align__(16) float s_kt[DK];
  __shared__ __align__(16) float s_qt[DK];
  __shared__ __align__(16) float s_dec[DK];
  __shared__ __align__(16) float s_red[2][TL::RG][DV];
  __shared__ float s_ck[kMaxM], s_cq[kMaxM];
  __shared__ float s_kappa;
  __shared__ __align__(8) uint64_t s_full[kMaxStages];
  __shared__ __align__(8) uint64_t s_unit[kUnitSlots];
  extern __shared__ __align__(128) unsigned char s_dyn[];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % TL::TPR, rg = tid / TL::TPR;
  const int n = a.n;
  const int NS = cfg.ns;
  const long G = gridDim.x;
  const int nunits = static_cast<int>((cfg.BH - 1 - blockIdx.x) / G) + 1;
  const int nchunks = nunits * CPU;
  const size_t SB = SG::slot_bytes(n);
  const long LS = PERKEY ? long(a.Mcap) * DK : gdn_lam_stride(a.Mcap);  // Lam floats per unit

  float* ring = reinterpret_cast<float*>(s_dyn);
  unsigned char* slots = s_dyn + size_t(NS) * kChunkBytes;
  float* As = reinterpret_cast<float*>(slots + kUnitSlots * SB);  // merge only
  float* Bc = As + (n + 1) * DK;                            // merge only

  // ---- producer (thread 0): chunk g into ring stage g % NS; unit iu's slot.
  int issued = 0;
  auto issue = [&](int g) {
    if (g >= nchunks) return;
    const int iu = g / CPU, kc = g % CPU;
    const long u = blockIdx.x + iu * G;
    const int stage = g % NS;
    mbar_arrive_expect_tx(&s_full[stage], kChunkBytes);
    bulk_g2s(ring + stage * CHF, a.Sbar + u * (DK * DV) + kc * (CR * DV), kChunkBytes, &s_full[stage]);
    issued = g + 1;
  };
  auto issue_slot = [&](int iu) {
    if (iu >= nunits) return;
    const long u = blockIdx.x + iu * G;
    unsigned char* sl = slots + (iu % kUnitSlots) * SB;
    uint64_t* ub = &s_unit[iu % kUnitSlots];
    mbar_arrive_expect_tx(ub, static_cast<uint32_t>(SG::log_bytes(n) + SG::io_bytes()));
    if (n > 0) {
      bulk_g2s(sl, static_cast<const TI*>(a.logA) + u * a.Mcap * DK, SG::a_bytes(n), ub);
      bulk_g2s(sl + SG::a_bytes(n), a.logLam + u * LS, SG::l_bytes(n), ub);
      bulk_g2s(sl + SG::a_bytes(n) + SG::l_bytes(n), static_cast<const TB*>(a.logB) + u * a.Mcap * DV,
               SG::b_bytes(n), ub);
    }
    unsigned char* io = sl + SG::log_bytes(n);
    bulk_g2s(io, static_cast<const TI*>(a.q) + u * DK, DK * sizeof(TI), ub);
    bulk_g2s(io + DK * sizeof(TI), static_cast<const TI*>(a.k) + u * DK, DK * sizeof(TI), ub);
    bulk_g2s(io + 2 * DK * sizeof(TI), static_cast<const TI*>(a.v) + u * DV, DV * sizeof(TI), ub);
    if (PERKEY) bulk_g2s(io + (2 * DK + DV) * sizeof(TI), a.log_decay + u * DK, DK * 4, ub);
    if (OP == OP_RWKV6)
      bulk_g2s(io + (2 * DK + DV) * sizeof(TI) + DK * 4, a.u + (u % a.H) * DK, DK * 4, ub);
  };

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&s_full[s], 1);
    for (int s = 0; s < kUnitSlots; ++s) mbar_init(&s_unit[s], 1);
    fence_mbar_init();
    issue_slot(0);
    issue_slot(1);
    const int pre = NS < nchunks ? NS : nchunks;
    for (int g = 0; g < pre; ++g) issue(g);
  }
  __syncthreads();

  // Per-unit scalars that are too small for a bulk copy, prefetched one unit ahead.
  auto scalars = [&](int iu, float& ld, float& be) {
    if (iu >= nunits) return;
    const long u = blockIdx.x + iu * G;
    if (!PERKEY) ld = a.log_decay[u];
    if (DELTA) be = a.beta[u];
  };
  float nx_ld = 0.f, nx_be = 0.f;
  scalars(0, nx_ld, nx_be);

  int g = 0;        // next chunk to consume
  int g0 = 0;       // first chunk of the current unit
  int iu = 0;
  bool aborted = false;
  for (; iu < nunits; ++iu) {
    const long u = blockIdx.x + iu * G;
    g0 = g;
    const float cur_ld = nx_ld, cur_be = nx_be;
    scalars(iu + 1, nx_ld, nx_be);

    // Unit iu-1 is finished (end-of-unit barrier): its slot takes unit iu+1.
    if (tid == 0 && iu >= 1) issue_slot(iu + 1);
    const int slot = iu % kUnitSlots;
    const unsigned char* sl = slots + slot * SB;
    const TI* sA = reinterpret_cast<const TI*>(sl);
    const float* sL = reinterpret_cast<const float*>(sl + SG::a_bytes(n));
    const TB* sB = reinterpret_cast<const TB*>(sl + SG::a_bytes(n) + SG::l_bytes(n));
    const TI* sq = reinterpret_cast<const TI*>(sl + SG::log_bytes(n));
    const TI* sk = sq + DK;
    const TI* sv = sk + DK;
    const float* sld = reinterpret_cast<const float*>(sv + DV);
    const float* sub = sld + DK;

    int bad = !mbar_wait_bounded(&s_unit[slot], (iu / kUnitSlots) & 1);
    if (bad) atomicOr(a.err, kErrWaitTimeout);

    // ReplayPrep for unit u (from the staged slot).
    float kr[TL::KPL], qr[TL::KPL], lt[TL::KPL], lp[TL::KPL];
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      kr[m] = to_f(sk[j]);
      qr[m] = to_f(sq[j]);
      if (PERKEY) {
        lp[m] = n > 0 ? sL[(n - 1) * DK + j] : 0.f;
        lt[m] = lp[m] + sld[j];
      } else {
        lp[m] = n > 0 ? sL[n - 1] : 0.f;
        lt[m] = lp[m] + cur_ld;
      }
    }
    for (int i = warp; i <= n; i += TL::NW) {
      float dk = 0.f, dq = 0.f;
      if (i < n) {
#pragma unroll
        for (int m = 0; m < TL::KPL; ++m) {
          const int j = lane + 32 * m;
          const float ai = to_f(sA[i * DK + j]);
          const float lam_i = PERKEY ? sL[i * DK + j] : sL[i];
          const float r_t = expf(lt[m] - lam_i);
          if (DELTA) {
            dk = fmaf(r_t * ai, kr[m], dk);
            dq = fmaf(r_t * ai, qr[m], dq);
          } else {
            dq = fmaf(expf(lp[m] - lam_i) * ai, qr[m], dq);
          }
          if (MERGE) As[i * DK + j] = r_t * ai;
        }
      } else {
#pragma unroll
        for (int m = 0; m < TL::KPL; ++m) {
          const int j = lane + 32 * m;
          dq = DELTA ? fmaf(kr[m], qr[m], dq) : fmaf(sub[j] * kr[m], qr[m], dq);
          if (MERGE) As[n * DK + j] = kr[m];
        }
      }
      if (DELTA) dk = warp_sum(dk);
      dq = warp_sum(dq);
      if (lane == 0) {
        if (i < n) {
          s_ck[i] = dk;
          s_cq[i] = dq;
        } else {
          s_kappa = dq;
        }
      }
    }
    if (warp == 0) {
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) {
        const int j = lane + 32 * m;
        const float et = expf(lt[m]);
        if (DELTA) {
          s_kt[j] = et * kr[m];
          s_qt[j] = et * qr[m];
        } else {
          s_qt[j] = expf(lp[m]) * qr[m];
        }
        if (MERGE) s_dec[j] = et;
      }
      if (!MERGE && !bad) {  // append: a_n = k_t and its snapshot
        TI* dstA = static_cast<TI*>(a.logA) + (u * a.Mcap + n) * DK;
#pragma unroll
        for (int m = 0; m < TL::KPL; ++m) {
          const int j = lane + 32 * m;
          dstA[j] = sk[j];
          if (PERKEY) a.logLam[u * LS + n * DK + j] = lt[m];
        }
        if (!PERKEY && lane == 0) a.logLam[u * LS + n] = lt[0];
      }
    }
    if (__syncthreads_or(bad)) {
      aborted = true;
      break;
    }

    // Base contraction, chunk by chunk from the ring.
    float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = p4;
    for (int kc = 0; kc < CPU; ++kc, ++g) {
      const int stage = g % NS;
      const bool ok = mbar_wait_bounded(&s_full[stage], (g / NS) & 1);
      if (!ok) {
        bad = 1;
        atomicOr(a.err, kErrWaitTimeout);
      } else {
        const float* ch = ring + stage * CHF;
#pragma unroll
        for (int j = 0; j < RPC; ++j) {
          const int rl = rg * RPC + j;
          const int row = kc * CR + rl;
          const float4 x = *reinterpret_cast<const float4*>(ch + rl * DV + 4 * c4);
          if (DELTA) fma4(p4, s_kt[row], x);
          fma4(s4, s_qt[row], x);
        }
      }
      if (!MERGE) {
        if (__syncthreads_or(bad)) break;
        if (tid == 0) issue(g + NS);   // stage consumed by every thread: refill
      }
    }
    if (DELTA) *reinterpret_cast<float4*>(&s_red[0][rg][4 * c4]) = p4;
    *reinterpret_cast<float4*>(&s_red[1][rg][4 * c4]) = s4;
    if (__syncthreads_or(bad)) {
      aborted = true;
      break;
    }

    // Finalize for value column c: replay, delta correction, output, append.
    const int c = tid;
    if (c < DV) {
      float p = 0.f, s = 0.f;
#pragma unroll
      for (int gg = 0; gg < TL::RG; ++gg) {
        if (DELTA) p += s_red[0][gg][c];
        s += s_red[1][gg][c];
      }
      float oc = s;
      for (int i = 0; i < n; ++i) {
        const float bi = to_f(sB[i * DV + c]);
        if (DELTA) p = fmaf(s_ck[i], bi, p);
        oc = fmaf(s_cq[i], bi, oc);
      }
      const float vc = to_f(sv[c]);
      const float bt = DELTA ? cur_be * (vc - p) : vc;
      oc = fmaf(s_kappa, bt, oc);
      static_cast<TI*>(a.o)[u * DV + c] = from_f<TI>(oc);
      if (MERGE) {
        Bc[c] = bt;
      } else {
        TB* dstB = static_cast<TB*>(a.logB) + (u * a.Mcap + n) * DV;
        if constexpr (DELTA) {
          dstB[c] = bt;
        } else {
          dstB[c] = sv[c];
        }
      }
    }
    __syncthreads();

    if (MERGE) {
      // S_t = diag(e^{Lam_t}) Sbar + sum_{i<=n} (ratio_i (.) a_i) b_i^T, chunk by chunk.
      for (int kc = 0; kc < CPU; ++kc) {
        const float* ch = ring + ((g - CPU + kc) % NS) * CHF;
        float4 x[RPC];
#pragma unroll
        for (int j = 0; j < RPC; ++j) {
          const int rl = rg * RPC + j;
          const float d = s_dec[kc * CR + rl];
          x[j] = *reinterpret_cast<const float4*>(ch + rl * DV + 4 * c4);
          x[j].x *= d;
          x[j].y *= d;
          x[j].z *= d;
          x[j].w *= d;
        }
        for (int i = 0; i <= n; ++i) {
          const float4 b4 = i < n ? load4f(sB + i * DV + 4 * c4) : load4f(Bc + 4 * c4);
          const float* ai = As + i * DK + kc * CR + rg * RPC;
#pragma unroll
          for (int j4 = 0; j4 < RPC; j4 += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(ai + j4);
            fma4(x[j4 + 0], a4.x, b4);
            fma4(x[j4 + 1], a4.y, b4);
            fma4(x[j4 + 2], a4.z, b4);
            fma4(x[j4 + 3], a4.w, b4);
          }
        }
        float* dst = a.Sbar + u * (DK * DV) + (kc * CR + rg * RPC) * DV + 4 * c4;
#pragma unroll
        for (int j = 0; j < RPC; ++j) st_state(dst + j * DV, x[j]);
      }
      __syncthreads();
      if (tid == 0)
        for (int kc = 0; kc < CPU; ++kc) issue(g - CPU + kc + NS);
    }
  }

  // Abort path: every copy this CTA issued must land before it exits.
  if (aborted && tid == 0) {
    for (int gg = g0; gg < issued; ++gg) mbar_wait_bounded(&s_full[gg % NS], (gg / NS) & 1);
    for (int uu = iu; uu <= iu + 1 && uu < nunits; ++uu)
      mbar_wait_bounded(&s_unit[uu % kUnitSlots], (uu / kUnitSlots) & 1);
  }
}

}  // namespace dl
