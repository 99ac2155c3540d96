// Persistent, warp-specialised, TMA-pipelined DeltaLog step for sm_100a.
//
// Same arithmetic as deltalog_step_kernel (kernels.cuh), different schedule.
// A grid of persistent CTAs walks the (slot, head) units round-robin; each CTA
// has three roles that never wait on a CTA-wide barrier inside the loop:
//
//  * producer warp (lane 0): streams the fp32 state as 16 KB chunks (CR rows x
//    d_v) into a ring of NS shared-memory stages with TMA bulk copies
//    (cp.async.bulk, no multicast); stage s completes on full[s] and is
//    refilled once every consumer warp has arrived on empty[s];
//    the same producer also stages each unit's log (a_i, Lam_i, b_i), q/k/v,
//    per-key gates and RWKV6 bonus row into one of three slots (bulk copies)
//    one unit ahead of the unit's first chunk;
//  * consumer warps, one per row group (two for d_v = 64).  Per unit each warp
//    computes k~, q~ and e^{Lam_t} for its own rows only (warp-private), and
//    the ReplayPrep coefficients of the log entries i = warp, warp+NWC, ...
//    (decay ratios, c^k_i, c^q_i, and for a merge the ratio-scaled a_i) into a
//    double-buffered shared block, so the key-side work is done once per
//    (slot, head) and split across warps.  The warps then accumulate
//    Sbar^T k~ and Sbar^T q~ from the ring, exchange the row-group partials
//    through a double-buffered reduction block whose mbarrier also certifies
//    the shared coefficients, finalise their float4 column group (replay,
//    delta correction, output, appended b_n) and, on a merge, write S_t back
//    chunk by chunk before releasing each stage.
//
// So the state stream never stops for per-unit bookkeeping: while consumers
// finish one unit the producer keeps up to NS chunks and the next unit's slot
// in flight.  Every wait is bounded and also stops as soon as any role has
// given up (shared abort flag); the CTA then meets at one final barrier,
// thread 0 waits (bounded) for its own copies still in flight, raises
// kErrWaitTimeout and the kernel returns.
#pragma once

#include "kernels.cuh"

namespace dl {

constexpr int kChunkBytes = 16384;
constexpr int kMaxStages = 12;
constexpr int kSlots = 3;   // unit slots (log + io staging)
constexpr int kCoefs = 2;   // coefficient blocks

__host__ __device__ constexpr size_t round_up16(size_t x) { return (x + 15) & ~size_t(15); }

template <int OP, int DK, int DV, typename TI>
struct StreamGeom {
  using TB = typename std::conditional<OP == OP_RWKV6, TI, float>::type;
  static constexpr bool PERKEY = OP != OP_GDN;
  static constexpr int CR = kChunkBytes / (DV * 4);  // state rows per chunk
  static constexpr int CPU = DK / CR;                 // chunks per (slot, head)
  static constexpr int RPC = CR / 8;                  // rows per row group per chunk
  static constexpr int NTC = 2 * DV;                  // consumer threads
  static constexpr int NWC = NTC / 32;                // consumer warps
  static constexpr int NT = NTC + 32;                 // + producer warp
  static constexpr int TPR = DV / 4;                  // threads per state row
  static constexpr int RW = 4 * DK / TPR;             // rows owned by one consumer warp
  static_assert(CR % 8 == 0 && DK % CR == 0 && RPC % 4 == 0, "chunk shape");

  // Unit slot (bytes, each region 16-byte aligned):
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
  // Shared coefficient block (floats): ck[kMaxM] cq[kMaxM] kappa beta pad[2] | merge: As[(n+1)][DK]
  __host__ __device__ static constexpr size_t coef_floats(int n, bool merge) {
    return 2 * kMaxM + 4 + (merge ? size_t(n + 1) * DK : 0);
  }
  __host__ __device__ static constexpr size_t coef_bytes(int n, bool merge) {
    return round_up16(coef_floats(n, merge) * 4);
  }
  // Row-group partials: [2][8][DV] floats per block, two blocks.
  __host__ __device__ static constexpr size_t red_bytes() { return size_t(2) * 8 * DV * 4; }
  // Warp-private row values: kt, qt, dec for RW rows per consumer warp.
  __host__ __device__ static constexpr size_t rows_bytes() { return size_t(NWC) * 3 * RW * 4; }
  __host__ __device__ static constexpr size_t smem(int n, bool merge, int ns) {
    return size_t(ns) * kChunkBytes + kSlots * slot_bytes(n) + kCoefs * coef_bytes(n, merge) + 2 * red_bytes() +
           rows_bytes();
  }
};

// Register cap of the streaming kernel (d_v): two CTAs per SM put
// ceil(2 * warps / 4) warps on each of the SM's four sub-partitions, whose
// register files hold 16 K registers each.
template <int DV>
constexpr int stream_maxreg = (16384 / (((2 * (2 * DV + 32) / 32) + 3) / 4) / 32) & ~7;

struct StreamCfg {
  int BH;  // units
  int ns;  // ring stages (16 KB each)
};

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&lo);
  r.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = r;
}

template <int OP, int DK, int DV, typename TI, bool MERGE>
__global__ void __launch_bounds__(StreamGeom<OP, DK, DV, TI>::NT) __maxnreg__(stream_maxreg<DV>)
deltalog_stream_kernel(const StepArgs a, const StreamCfg cfg) {
  using SG = StreamGeom<OP, DK, DV, TI>;
  using TL = Tile<DK, DV>;
  using TB = typename SG::TB;
  constexpr bool DELTA = OP != OP_RWKV6;
  constexpr bool PERKEY = SG::PERKEY;
  constexpr int CR = SG::CR, CPU = SG::CPU, RPC = SG::RPC, NWC = SG::NWC, RW = SG::RW;
  constexpr int TPR = SG::TPR, GPW = 32 / TPR;  // row groups per consumer warp
  constexpr int CHF = kChunkBytes / 4;

  __shared__ __align__(8) uint64_t s_full[kMaxStages];
  __shared__ __align__(8) uint64_t s_empty[kMaxStages];
  __shared__ __align__(8) uint64_t s_slot[kSlots];
  __shared__ __align__(8) uint64_t s_sempty[kSlots];
  __shared__ __align__(8) uint64_t s_rfull[2];
  __shared__ int s_abort_word, s_nchunks_issued, s_nslots_issued;
  extern __shared__ __align__(128) unsigned char s_dyn[];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n = a.n;
  const int NS = cfg.ns;
  const long G = gridDim.x;
  const int nunits = static_cast<int>((cfg.BH - 1 - blockIdx.x) / G) + 1;
  const int nchunks = nunits * CPU;
  const size_t SB = SG::slot_bytes(n);
  const size_t CB = SG::coef_bytes(n, MERGE);
  const long LS = PERKEY ? long(a.Mcap) * DK : gdn_lam_stride(a.Mcap);  // Lam floats per unit
  volatile int* abort = &s_abort_word;

  float* ring = reinterpret_cast<float*>(s_dyn);
  unsigned char* slots = s_dyn + size_t(NS) * kChunkBytes;
  unsigned char* coefs = slots + kSlots * SB;
  float* red = reinterpret_cast<float*>(coefs + kCoefs * CB);
  float* rowvals = red + 2 * (2 * 8 * DV);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], NWC);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&s_slot[s], 1);
      mbar_init(&s_sempty[s], NWC);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&s_rfull[s], NWC);
    fence_mbar_init();
    s_abort_word = 0;
    s_nchunks_issued = 0;
    s_nslots_issued = 0;
  }
  __syncthreads();

  if (warp == NWC) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Unit iu's slot is issued together with chunk 0 of unit iu-1, one unit
      // ahead of its chunks; it reuses the slot of unit iu - kSlots.
      auto issue_slot = [&](int iu) -> bool {
        if (iu >= nunits) return true;
        if (iu >= kSlots && !mbar_wait_abortable(&s_sempty[iu % kSlots], ((iu / kSlots) - 1) & 1, abort))
          return false;
        const long u = blockIdx.x + iu * G;
        unsigned char* sl = slots + (iu % kSlots) * SB;
        uint64_t* ub = &s_slot[iu % kSlots];
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
        s_nslots_issued = iu + 1;
        return true;
      };
      bool live = issue_slot(0);
      for (int g = 0; live && g < nchunks; ++g) {
        const int iu = g / CPU, kc = g % CPU;
        const long u = blockIdx.x + iu * G;
        if (kc == 0 && !issue_slot(iu + 1)) break;
        const int stage = g % NS;
        if (g >= NS && !mbar_wait_abortable(&s_empty[stage], ((g / NS) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&s_full[stage], kChunkBytes);
        bulk_g2s(ring + stage * CHF, a.Sbar + u * (DK * DV) + kc * (CR * DV), kChunkBytes, &s_full[stage]);
        s_nchunks_issued = g + 1;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int c4 = tid % TPR, rg = tid / TPR;
    const int rg0 = warp * GPW;  // first row group of this warp
    float* kt_w = rowvals + warp * 3 * RW;
    float* qt_w = kt_w + RW;
    float* dec_w = qt_w + RW;

    // Scalar gates (GDN decay, GDN/KDA beta) are prefetched one unit ahead.
    float nx_ld = 0.f, nx_be = 0.f;
    auto scalars = [&](int iu) {
      if (iu >= nunits) return;
      const long u = blockIdx.x + iu * G;
      if (!PERKEY) nx_ld = a.log_decay[u];
      if (DELTA) nx_be = a.beta[u];
    };
    scalars(0);

    int g = 0;
    for (int iu = 0; iu < nunits; ++iu) {
      const long u = blockIdx.x + iu * G;
      const float cur_ld = nx_ld, cur_be = nx_be;
      scalars(iu + 1);
      if (!mbar_wait_abortable(&s_slot[iu % kSlots], (iu / kSlots) & 1, abort)) break;

      const unsigned char* sl = slots + (iu % kSlots) * SB;
      const TI* sA = reinterpret_cast<const TI*>(sl);
      const float* sL = reinterpret_cast<const float*>(sl + SG::a_bytes(n));
      const TB* sB = reinterpret_cast<const TB*>(sl + SG::a_bytes(n) + SG::l_bytes(n));
      const TI* sq = reinterpret_cast<const TI*>(sl + SG::log_bytes(n));
      const TI* sk = sq + DK;
      const TI* sv = sk + DK;
      const float* sld = reinterpret_cast<const float*>(sv + DV);
      const float* sub = sld + DK;
      float* cf = reinterpret_cast<float*>(coefs + (iu & 1) * CB);
      float* ck = cf;
      float* cq = ck + kMaxM;
      float* scal = cq + kMaxM;  // kappa, beta
      float* As = scal + 4;      // merge only

      // (a) k~, q~, e^{Lam_t} for this warp's rows (row index ri = (kc*GPW + group)*RPC + j).
      if (lane < RW) {
        const int kcl = lane / (GPW * RPC), rem = lane % (GPW * RPC);
        const int row = kcl * CR + (rg0 + rem / RPC) * RPC + rem % RPC;
        const float lp = n > 0 ? (PERKEY ? sL[(n - 1) * DK + row] : sL[n - 1]) : 0.f;
        const float lt = lp + (PERKEY ? sld[row] : cur_ld);
        const float et = expf(lt);
        if (DELTA) {
          kt_w[lane] = et * to_f(sk[row]);
          qt_w[lane] = et * to_f(sq[row]);
        } else {
          qt_w[lane] = expf(lp) * to_f(sq[row]);
        }
        if (MERGE) dec_w[lane] = et;
      }

      // (b) ReplayPrep for the log entries of this warp; entry n (the current
      // token: kappa, beta, and on an append the new a_n / Lam_n) by warp n % NWC.
      if (warp <= n) {
        float kr[TL::KPL], qr[TL::KPL], lt[TL::KPL], lp[TL::KPL];
#pragma unroll
        for (int m = 0; m < TL::KPL; ++m) {
          const int j = lane + 32 * m;
          kr[m] = to_f(sk[j]);
          qr[m] = to_f(sq[j]);
          lp[m] = n > 0 ? (PERKEY ? sL[(n - 1) * DK + j] : sL[n - 1]) : 0.f;
          lt[m] = lp[m] + (PERKEY ? sld[j] : cur_ld);
        }
        for (int i = warp; i <= n; i += NWC) {
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
            if (DELTA) dk = warp_sum(dk);
            dq = warp_sum(dq);
            if (lane == 0) {
              ck[i] = dk;
              cq[i] = dq;
            }
          } else {
#pragma unroll
            for (int m = 0; m < TL::KPL; ++m) {
              const int j = lane + 32 * m;
              dq = DELTA ? fmaf(kr[m], qr[m], dq) : fmaf(sub[j] * kr[m], qr[m], dq);
              if (MERGE) As[n * DK + j] = kr[m];
            }
            dq = warp_sum(dq);
            if (lane == 0) {
              scal[0] = dq;
              scal[1] = cur_be;
            }
            if (!MERGE) {  // append: a_n = k_t and its snapshot
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
        }
      }
      __syncwarp();

      // (c) Base contraction over this thread's rows of every chunk of the unit.
      float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = p4;
      bool ok = true;
      for (int kc = 0; kc < CPU; ++kc) {
        const int gg = g + kc, stage = gg % NS;
        if (!mbar_wait_abortable(&s_full[stage], (gg / NS) & 1, abort)) {
          ok = false;
          break;
        }
        const float* ch = ring + stage * CHF;
        const int ri0 = (kc * GPW + (rg - rg0)) * RPC;
#pragma unroll
        for (int j = 0; j < RPC; ++j) {
          const float4 x = *reinterpret_cast<const float4*>(ch + (rg * RPC + j) * DV + 4 * c4);
          if (DELTA) fma4(p4, kt_w[ri0 + j], x);
          fma4(s4, qt_w[ri0 + j], x);
        }
        if (!MERGE) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[stage]);
        }
      }
      if (!ok) break;

      // (d) Exchange the row-group partials (block iu & 1).  The same barrier
      // certifies every warp's ReplayPrep coefficients of this unit.
      float* rd = red + (iu & 1) * (2 * 8 * DV);
      if (DELTA) *reinterpret_cast<float4*>(rd + rg * DV + 4 * c4) = p4;
      *reinterpret_cast<float4*>(rd + (8 + rg) * DV + 4 * c4) = s4;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_rfull[iu & 1]);
      if (!mbar_wait_abortable(&s_rfull[iu & 1], (iu >> 1) & 1, abort)) break;

      // (e) Finalise columns 4*c4 .. 4*c4+3 (every row group does it; row group 0 writes).
      float4 P = make_float4(0.f, 0.f, 0.f, 0.f), S = P;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (DELTA) {
          const float4 x = *reinterpret_cast<const float4*>(rd + r * DV + 4 * c4);
          P.x += x.x;
          P.y += x.y;
          P.z += x.z;
          P.w += x.w;
        }
        const float4 y = *reinterpret_cast<const float4*>(rd + (8 + r) * DV + 4 * c4);
        S.x += y.x;
        S.y += y.y;
        S.z += y.z;
        S.w += y.w;
      }
      for (int i = 0; i < n; ++i) {
        const float4 b4 = load4f(sB + i * DV + 4 * c4);
        if (DELTA) fma4(P, ck[i], b4);
        fma4(S, cq[i], b4);
      }
      const float4 v4 = load4f(sv + 4 * c4);
      const float kap = scal[0], be = scal[1];
      float4 bt = v4;
      if (DELTA) {
        bt.x = be * (v4.x - P.x);
        bt.y = be * (v4.y - P.y);
        bt.z = be * (v4.z - P.z);
        bt.w = be * (v4.w - P.w);
      }
      fma4(S, kap, bt);
      if (rg == 0) {
        store4<TI>(static_cast<TI*>(a.o) + u * DV + 4 * c4, S);
        if (!MERGE) {
          TB* dstB = static_cast<TB*>(a.logB) + (u * a.Mcap + n) * DV + 4 * c4;
          if constexpr (DELTA) {
            store4<float>(dstB, bt);
          } else if constexpr (sizeof(TI) == 2) {
            *reinterpret_cast<uint2*>(dstB) = *reinterpret_cast<const uint2*>(sv + 4 * c4);  // raw v bits
          } else {
            *reinterpret_cast<uint4*>(dstB) = *reinterpret_cast<const uint4*>(sv + 4 * c4);
          }
        }
      }

      // (f) Merge: S_t = diag(e^{Lam_t}) Sbar + sum_{i<=n} (ratio_i (.) a_i) b_i^T, chunk by chunk.
      if (MERGE) {
        for (int kc = 0; kc < CPU; ++kc) {
          const int gg = g + kc, stage = gg % NS;
          const float* ch = ring + stage * CHF;
          const int r0 = kc * CR + rg * RPC;
          const int ri0 = (kc * GPW + (rg - rg0)) * RPC;
          float4 x[RPC];
#pragma unroll
          for (int j = 0; j < RPC; ++j) {
            x[j] = *reinterpret_cast<const float4*>(ch + (rg * RPC + j) * DV + 4 * c4);
            scale4(x[j], dec_w[ri0 + j]);
          }
          for (int i = 0; i <= n; ++i) {
            const float4 b4 = i < n ? load4f(sB + i * DV + 4 * c4) : bt;
            const float* ai = As + i * DK + r0;
#pragma unroll
            for (int j4 = 0; j4 < RPC; j4 += 4) {
              const float4 a4 = *reinterpret_cast<const float4*>(ai + j4);
              fma4(x[j4 + 0], a4.x, b4);
              fma4(x[j4 + 1], a4.y, b4);
              fma4(x[j4 + 2], a4.z, b4);
              fma4(x[j4 + 3], a4.w, b4);
            }
          }
          float* dst = a.Sbar + u * (DK * DV) + r0 * DV + 4 * c4;
#pragma unroll
          for (int j = 0; j < RPC; ++j) st_state(dst + j * DV, x[j]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[stage]);
        }
      }
      g += CPU;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_sempty[iu % kSlots]);
    }
  }

  __syncthreads();
  if (*abort && tid == 0) {
    // Every copy this CTA issued must land before it exits.
    const int ci = s_nchunks_issued, si = s_nslots_issued;
    for (int gg = ci > NS ? ci - NS : 0; gg < ci; ++gg) mbar_wait_bounded(&s_full[gg % NS], (gg / NS) & 1);
    for (int su = si > kSlots ? si - kSlots : 0; su < si; ++su)
      mbar_wait_bounded(&s_slot[su % kSlots], (su / kSlots) & 1);
    atomicOr(a.err, kErrWaitTimeout);
  }
}

}  // namespace dl
