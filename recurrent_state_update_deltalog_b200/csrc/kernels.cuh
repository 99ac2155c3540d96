// DeltaLog decode kernels for sm_100a: deferred step (append / merge-fused),
// eager dense baseline, and log materialisation.
//
// Method (DeltaLog technical summary, gist.science, sections "Method -- core
// mechanism: base + log" and "Kernel implementation"): the logical state of a
// (slot, head) after step t is
//     S_t = diag(e^{Lam_t}) Sbar + sum_{i in log} diag(e^{Lam_t - Lam_i}) a_i b_i^T
// with a_i = k_i and Lam the cumulative natural-log decay since the last
// merge (a scalar for GDN, a per-key vector for KDA and RWKV6).  Append steps
// read Sbar and add one log entry; every M-th step writes S_t back to Sbar.
//
// Work decomposition on B200.  One CTA owns one (slot, head): the key-side
// "ReplayPrep" coefficients (decay ratios, a_i.k_t, a_i.q_t) are computed once
// per CTA by its warps and shared through shared memory with every value tile
// of that head, so nothing key-side is recomputed per value tile.  Value tiles
// are the float4 column groups of the CTA's threads: thread (rg, c4) holds
// rows [rg*RPT, rg*RPT+RPT) x columns [4*c4, 4*c4+4) of the fp32 state in
// registers.  All state loads of a CTA are issued up front as 128-bit
// streaming loads (64 KB in flight per CTA at d = 128) while one thread stages
// the head's whole log (a_i, Lam_i, b_i) into shared memory with TMA bulk
// copies on an mbarrier, so the log costs one round trip, not one per entry.
// The two contractions
// Sbar^T k~ and Sbar^T q~ are formed in one pass over those registers, and the
// d_k reduction crosses row groups through a small shared-memory stage.  On a
// merge step the rank-(n+1) update is applied to the same registers and
// stored back with 128-bit streaming stores, so Sbar crosses HBM once each
// way.  No tensor cores: this is matrix-vector work at ~1 flop/byte.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "ptx.cuh"

namespace dl {

enum { OP_GDN = 0, OP_KDA = 1, OP_RWKV6 = 2 };

// Arguments of one deferred step (device pointers; sizes in elements).
// Units: a pool unit (slot, head) owns Sbar and log storage; a batch unit
// (row, head) owns inputs and outputs.  Without an index map, row b is slot b.
struct StepArgs {
  float* Sbar;             // [BH][DK][DV]                 pool units
  const void* q;           // [rows*H][DK] (r for RWKV6), input dtype   batch units
  const void* k;           // [rows*H][DK]
  const void* v;           // [rows*H][DV]
  const float* log_decay;  // [rows*H] (GDN) or [rows*H][DK]
  const float* beta;       // [rows*H] (GDN/KDA)
  void* o;                 // [rows*H][DV], input dtype
  const int* slot_idx;     // [rows] pool slot of each batch row (< 0: padding; kSlotHold
                           // bit: the slot sits this token out), or null
  int slots;               // pool slots B (bound of slot_idx)
  void* logA;              // [BH][Mcap][DK], input dtype (a_i = k_i)
  void* logB;              // [BH][Mcap][DV], fp32 (GDN/KDA) or input dtype (RWKV6)
  float* logLam;           // [BH][gdn_lam_stride(Mcap)] (GDN) or [BH][Mcap][DK]
  const float* u;          // [H][DK] (RWKV6)
  int* err;               // device error word (kErr* bits)
  int H;
  int M;                   // merge interval
  int Mcap;                // log capacity per (slot, head), >= 1
  int n;                   // entries in the log before this step (lockstep launches)
  int stall_log;           // test only: arm the log barrier but issue no copy (see stage_log)
};

// Bound of the log wait when a test stalls the log on purpose: long enough
// for nothing, short enough that the timeout path is quick.
constexpr uint64_t kStallWaitNs = 20000;

// Step kernel modes: every slot appends, or every slot merges.
enum { MODE_APPEND = 0, MODE_MERGE = 1 };

// Device error bit: a slot index at or past the pool size (the row is skipped).
constexpr int kErrSlotIndex = 2;

// Slot-map bit of a held slot: the row names slot (index & ~kSlotHold), which
// takes no input and writes no output this token but keeps its state exact
// (an append gives it a null log entry; a merge folds its log).
constexpr int kSlotHold = 0x40000000;

// Which unit a CTA of a step kernel serves.  `bu` (row * H + head) indexes
// inputs and outputs, `sh` (slot * H + head) the state and the log, `col0` is
// the tile's first value column.  Unmapped launches: a 1-D grid of
// B * H * NSPLIT CTAs and sh == bu.  Mapped launches (template switch, so the
// unmapped kernels carry none of it): grid (H * NSPLIT, rows), row r on slot
// slot_idx[r]; ok is false for a padding row (negative index) and for an
// index past the pool, which also raises kErrSlotIndex; hold is set for a
// held slot.
struct UnitIx {
  long bu, sh;
  int h, col0;
  bool ok, hold;
};

template <int NSPLIT, int DVT, bool MAP>
__device__ __forceinline__ UnitIx unit_of(const StepArgs& a) {
  UnitIx u;
  if constexpr (MAP) {
    u.h = static_cast<int>(blockIdx.x) / NSPLIT;
    u.col0 = (static_cast<int>(blockIdx.x) % NSPLIT) * DVT;
    u.bu = static_cast<long>(blockIdx.y) * a.H + u.h;
    const int raw = __ldg(a.slot_idx + blockIdx.y);
    u.hold = raw >= 0 && (raw & kSlotHold);
    const int slot = raw & ~kSlotHold;
    u.ok = raw >= 0 && slot < a.slots;
    if (raw >= 0 && slot >= a.slots && threadIdx.x == 0) atomicOr(a.err, kErrSlotIndex);
    u.sh = static_cast<long>(slot) * a.H + u.h;
  } else {
    u.bu = blockIdx.x / NSPLIT;
    u.col0 = (blockIdx.x % NSPLIT) * DVT;
    u.h = static_cast<int>(u.bu % a.H);  // only RWKV6 reads it
    u.sh = u.bu;
    u.ok = true;
    u.hold = false;
  }
  return u;
}

// Arguments of log materialisation: Sout = Sbar + replayed log, for the
// units [unit0, unit0 + gridDim.x); Sout points at the first of them.
struct MaterializeArgs {
  const float* Sin;
  float* Sout;
  const void* logA;
  const void* logB;
  const float* logLam;
  int* err;
  long unit0;
  const int* slot_idx;  // null: units [unit0, unit0 + gridDim.x) into Sout;
                        // else grid (H, rows): slot slot_idx[r]'s heads, in place
                        // (Sout == Sin), rows with a negative index skipped
  int slots;            // pool slots (bound of slot_idx)
  int H;
  int Mcap;
  int n;
};

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// 128-bit loads/stores of the state: streaming (evict-first) so the state,
// which is far larger than L2, does not push the log and inputs out of L2.
__device__ __forceinline__ float4 ld_state(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void st_state(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }

// e^x as 2^(x log2 e) on the SFU (ex2.approx): relative error about 2^-22,
// plus the rounding of x log2 e (2^-24 |x| in the exponent); results below
// the normal range flush to zero.  The ratios exp(Lam_t - Lam_i) <= 1 of the
// replay take it: a few instructions each on every CTA's serial path.
__device__ __forceinline__ float exp_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
  return y;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// acc += a * b on a float4, as two packed fp32x2 FMAs (sm_100 FFMA2; each
// lane rounds exactly like fmaf).
__device__ __forceinline__ void fma4(float4& acc, float a, float4 b) {
  const float2 aa = make_float2(a, a);
  const float2 lo = __ffma2_rn(aa, make_float2(b.x, b.y), make_float2(acc.x, acc.y));
  const float2 hi = __ffma2_rn(aa, make_float2(b.z, b.w), make_float2(acc.z, acc.w));
  acc = make_float4(lo.x, lo.y, hi.x, hi.y);
}

// v *= d on a float4 (two packed fp32x2 multiplies).
__device__ __forceinline__ void scale4(float4& v, float d) {
  const float2 dd = make_float2(d, d);
  const float2 lo = __fmul2_rn(dd, make_float2(v.x, v.y));
  const float2 hi = __fmul2_rn(dd, make_float2(v.z, v.w));
  v = make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Largest supported merge interval M (log capacity M-1).
constexpr int kMaxM = 64;

template <int DK, int DV>
struct Tile {
  // The whole 64 x 64 tile (a d = 64 head, one value tile) runs on 64 threads
  // with 16 rows each ("slim"); every other tile on 2 DV threads with DK / 8
  // rows each.
  static constexpr bool SLIM = DK == 64 && DV == 64;
  static constexpr int NT = SLIM ? 64 : 2 * DV;   // threads per CTA
  static constexpr int TPR = DV / 4;     // threads that cover one state row with float4s
  static constexpr int RG = NT / TPR;    // row groups (8; 4 for the slim tile)
  static constexpr int RPT = DK / RG;    // rows held by each thread
  static constexpr int NW = NT / 32;     // warps
  static constexpr int KPL = DK / 32;    // keys per lane in warp-wide key loops
  // CTAs per SM the register budget is sized for.  128-thread tiles at d_k =
  // 64 keep 32 state registers per thread, so eight CTAs (64 registers each)
  // fit; the slim tile keeps 64 and fits eight at 128 registers.
  static constexpr int MINB = NT >= 256 ? 2 : (NT >= 128 ? (DK == 64 ? 8 : 4) : 8);
  // Append launches keep more state loads in flight per SM: 128-thread tiles
  // at d_k = 128 fit five CTAs (96 registers, no spills), 160 KB instead of
  // 128 KB; measured on B200, GDN B=256 appends 86.9 -> 83.8 us.  Six (80
  // registers) spill and lose; merge launches need their 128.  The slim tile
  // fits ten (102 registers), also 160 KB.
  static constexpr int MINB_APPEND = (NT == 128 && DK == 128) ? 5 : (SLIM ? 10 : MINB);
  static_assert(DV % 32 == 0 && DK % 32 == 0 && (RG == 8 || (SLIM && RG == 4)) && RPT % 4 == 0, "tile shape");
  static_assert(NT >= kMaxM - 1 && DV <= NT, "one thread per log entry / value column in setup phases");
};


// GDN keeps one scalar snapshot per entry; each head's row of snapshots is
// padded to a multiple of 4 floats so that it can be staged by a bulk copy.
__host__ __device__ constexpr int gdn_lam_stride(int Mcap) { return (Mcap + 3) & ~3; }

// Shared-memory image of a (slot, head)'s log, staged by TMA bulk copies.
// Byte layout (every region starts 16-byte aligned):
//   A   n x DK input dtype     a_i = k_i
//   L   n x DK fp32 | fp16     Lam_i (KDA / RWKV6 only; GDN keeps n scalars
//                              apart); LAMC: the step's log-gates g_i in fp16
//   B   n x DV (fp32 | input)  b_i (RWKV6: raw v_i in the input dtype; BLOW:
//                              GDN/KDA b_i rounded to bf16)
// then, with LAMC, the fp32 snapshots rebuilt from the gates
//   Lf  n x DK fp32            Lam_i = g_0 + ... + g_i, summed in entry order
// followed, for merge-type launches, by the fp32 work arrays
//   As  (n+1) x DK             ratio-scaled a_i, current entry last (ratio 1)
//   Bc  DV                     the current entry's b_t
// LAMC (compact per-key snapshots) stores each entry's own log-gate rather
// than its cumulative snapshot.  A rounded gate errs by at most 2^-11 of
// itself, so a rebuilt Lam_i errs by at most 2^-11 |Lam_i| and the decay
// factor e^{Lam_i} by at most e^{Lam} |Lam| 2^-11 <= 2^-11 / e of the state:
// rounding the snapshot itself would err by 2^-11 |Lam_i| in every ratio,
// however close the two snapshots of the ratio are.
template <int OP, int DK, int DV, typename TI, bool BLOW = false, bool LAMC = false>
struct LogLayout {
  static_assert(!BLOW || (OP != OP_RWKV6 && std::is_same<TI, __nv_bfloat16>::value),
                "a bf16 b-log is an option of bf16-input GDN/KDA handles");
  static_assert(!LAMC || (OP != OP_GDN && std::is_same<TI, __nv_bfloat16>::value),
                "compact snapshots are an option of bf16-input KDA/RWKV6 handles");
  using TB = typename std::conditional<OP == OP_RWKV6 || BLOW, TI, float>::type;
  using TL = typename std::conditional<LAMC, __half, float>::type;   // L elements in the log
  static constexpr bool PERKEY = OP != OP_GDN;
  __host__ __device__ static constexpr size_t a_bytes(int n) { return size_t(n) * DK * sizeof(TI); }
  __host__ __device__ static constexpr size_t l_bytes(int n) { return PERKEY ? size_t(n) * DK * sizeof(TL) : 0; }
  __host__ __device__ static constexpr size_t b_bytes(int n) { return size_t(n) * DV * sizeof(TB); }
  __host__ __device__ static constexpr size_t staged(int n) { return a_bytes(n) + l_bytes(n) + b_bytes(n); }
  __host__ __device__ static constexpr size_t table(int n) { return LAMC ? size_t(n) * DK * 4 : 0; }
  __host__ __device__ static constexpr size_t step_smem(int n, bool merge) {
    return staged(n) + table(n) + (merge ? size_t(n + 1) * DK * 4 + size_t(DV) * 4 : 0);
  }
  __host__ __device__ static constexpr size_t materialize_smem(int n) {
    return staged(n) + table(n) + size_t(n) * DK * 4;
  }
};

// LAMC: rebuild the fp32 snapshots Lam_i = g_0 + ... + g_i (i < n) from the
// staged fp16 gates, one key per thread, always in entry order (so every
// launch that reads a log sees the same values).  The caller synchronises.
template <int DK>
__device__ __forceinline__ void rebuild_snapshots(const __half* g, float* lam, int n) {
  for (int j = threadIdx.x; j < DK; j += blockDim.x) {
    float s = 0.f;
    for (int i0 = 0; i0 < n; i0 += 8) {
      // eight gates in flight at once; the sums stay in entry order
      float gi[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) gi[u] = i0 + u < n ? __half2float(g[(i0 + u) * DK + j]) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (i0 + u < n) {
          s += gi[u];
          lam[(i0 + u) * DK + j] = s;
        }
      }
    }
  }
}

// Four consecutive log values as floats (fp32 or bf16 storage).
__device__ __forceinline__ float4 load4f(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4f(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&r.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&r.y);
  const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

// Thread 0 starts the bulk copies of entries [0, n) of this (slot, head)'s log
// into shared memory; completion arrives on `bar` (phase 0).  With `stall`
// (a test of the timeout path) the barrier expects the bytes but no copy is
// issued: the wait runs out with nothing in flight.
template <int OP, int DK, int DV, typename TI, bool BLOW, bool LAMC>
__device__ __forceinline__ void stage_log(unsigned char* smem, uint64_t* bar, const void* logA,
                                          const float* logLam, const void* logB, long sh, int Mcap,
                                          int n, bool stall = false) {
  using LL = LogLayout<OP, DK, DV, TI, BLOW, LAMC>;
  using TB = typename LL::TB;
  using TLE = typename LL::TL;
  mbar_init(bar, 1);
  fence_mbar_init();
  if (n == 0) return;
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(LL::staged(n)));
  if (stall) return;
  bulk_g2s(smem, static_cast<const TI*>(logA) + sh * Mcap * DK, static_cast<uint32_t>(LL::a_bytes(n)), bar);
  if (LL::PERKEY)
    bulk_g2s(smem + LL::a_bytes(n), reinterpret_cast<const TLE*>(logLam) + sh * Mcap * DK,
             static_cast<uint32_t>(LL::l_bytes(n)), bar);
  bulk_g2s(smem + LL::a_bytes(n) + LL::l_bytes(n), static_cast<const TB*>(logB) + sh * Mcap * DV,
           static_cast<uint32_t>(LL::b_bytes(n)), bar);
}

// Every thread waits for the staged log.  On a timeout the whole CTA agrees to
// stop: the error word is raised, copies still in flight get one more bounded
// wait (the CTA must not exit while they target its shared memory), and the
// caller returns.
__device__ __forceinline__ bool wait_log(uint64_t* bar, int n, int* err, uint64_t limit_ns = kWaitNs) {
  int ok = n == 0 ? 1 : static_cast<int>(mbar_wait_bounded(bar, 0, limit_ns));
  if (__syncthreads_and(ok)) return true;
  if (threadIdx.x == 0) {
    atomicOr(err, kErrWaitTimeout);
    mbar_wait_bounded(bar, 0, limit_ns);
  }
  __syncthreads();
  return false;
}

// A held slot's append: the null entry a_n = 0, b_n = 0, Lam_n = Lam_{n-1}
// adds nothing to its state and does not advance its decay, so its logical
// state stays exact without reading Sbar.  Each value tile writes its b_n
// columns; the first tile writes a_n and the snapshot.
template <int OP, int DK, int DV, typename TI, bool BLOW, bool LAMC>
__device__ __forceinline__ void hold_entry(const StepArgs& a, long sh, int col0, int dvt, int n) {
  using TB = typename LogLayout<OP, DK, DV, TI, BLOW, LAMC>::TB;
  const int tid = threadIdx.x, nt = blockDim.x;
  TB* dstB = static_cast<TB*>(a.logB) + (sh * a.Mcap + n) * DV + col0;
  for (int c = tid; c < dvt; c += nt) dstB[c] = from_f<TB>(0.f);
  if (col0 != 0) return;
  TI* dstA = static_cast<TI*>(a.logA) + (sh * a.Mcap + n) * DK;
  for (int j = tid; j < DK; j += nt) dstA[j] = from_f<TI>(0.f);
  if constexpr (LAMC) {   // a zero gate
    __half* g = reinterpret_cast<__half*>(a.logLam) + (sh * a.Mcap + n) * DK;
    for (int j = tid; j < DK; j += nt) g[j] = __float2half_rn(0.f);
  } else if constexpr (OP != OP_GDN) {
    float* lam = a.logLam + sh * a.Mcap * DK;
    for (int j = tid; j < DK; j += nt) lam[n * DK + j] = n > 0 ? lam[(n - 1) * DK + j] : 0.f;
  } else if (tid == 0) {
    float* lam = a.logLam + sh * gdn_lam_stride(a.Mcap);
    lam[n] = n > 0 ? lam[n - 1] : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Deferred step.  MODE_APPEND: every slot appends (Sbar read only).
// MODE_MERGE: every slot is at n+1 == M; it also writes S_t over Sbar.  NSPLIT > 1 splits each head's
// d_v columns into NSPLIT value tiles, one CTA each (grid B*H*NSPLIT); every
// tile recomputes the head's ReplayPrep coefficients and the first tile
// appends the key-side entry.
// ---------------------------------------------------------------------------
template <int OP, int DK, int DV, typename TI, int MODE, int NSPLIT, bool MAP, bool BLOW, bool LAMC>
__global__ void __launch_bounds__(Tile<DK, DV / NSPLIT>::NT,
                                  MODE == MODE_APPEND ? Tile<DK, DV / NSPLIT>::MINB_APPEND : Tile<DK, DV / NSPLIT>::MINB)
deltalog_step_kernel(const StepArgs a) {
  constexpr int DVT = DV / NSPLIT;  // value-tile width owned by this CTA
  using TL = Tile<DK, DVT>;
  using LL = LogLayout<OP, DK, DV, TI, BLOW, LAMC>;
  using TB = typename LL::TB;
  constexpr bool DELTA = OP != OP_RWKV6;
  constexpr bool PERKEY = OP != OP_GDN;

  __shared__ __align__(16) float s_kt[DK];       // k~ = e^{Lam_t} (.) k   (GDN/KDA)
  __shared__ __align__(16) float s_qt[DK];       // q~ (GDN/KDA: e^{Lam_t}; RWKV6: e^{Lam_{t-1}})
  __shared__ __align__(16) float s_dec[DK];      // e^{Lam_t} per row (merge)
  __shared__ __align__(16) float s_red[2][TL::RG][DVT];
  __shared__ float s_ck[kMaxM], s_cq[kMaxM];
  __shared__ float s_lam[kMaxM];                 // GDN: scalar Lam_i of the log entries
  __shared__ float s_kappa;
  __shared__ __align__(8) uint64_t s_bar;
  extern __shared__ __align__(128) unsigned char s_dyn[];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % TL::TPR, rg = tid / TL::TPR;
  // Launch order.  When the host launches this step as a programmatic
  // dependent (only after an append of the same handle), the kernel just
  // before it in the stream may still be running, and its writes become
  // visible only after griddep_wait.  That kernel need not be this handle's
  // append: a caller's kernel that writes this token's inputs or slot map can
  // sit in between.  So nothing but Sbar, which only this handle's own
  // launches write (and appends never do), is read before the wait.  Mapped
  // launches need the slot map to find their Sbar, and the per-key operators
  // load their inputs ahead of the state tile (measured on B200: KDA and
  // RWKV6 appends 5-6% faster than behind 32 KB of state loads), so both wait
  // first; GDN streams its tile before the wait and loads its few input
  // words after it.
  constexpr bool WAIT_FIRST = MAP || OP != OP_GDN;
  if constexpr (WAIT_FIRST) griddep_wait();
  const UnitIx ux = unit_of<NSPLIT, DVT, MAP>(a);
  if (!ux.ok) return;
  const long bu = ux.bu;      // batch unit: inputs and output
  const long sh = ux.sh;      // pool unit: Sbar and the log
  const int col0 = ux.col0;   // first value column of this tile
  const int h = ux.h;
  const int n = a.n;
  constexpr bool MERGE = MODE == MODE_MERGE;
  // A held slot: an append writes its null entry and stops; a merge runs with
  // zero inputs (a null current entry) and writes no output, which folds the
  // slot's log into its base at its unchanged logical state.
  const bool hold = MAP && ux.hold;
  if (!MERGE && hold) {
    hold_entry<OP, DK, DV, TI, BLOW, LAMC>(a, sh, col0, DVT, n);
    return;
  }

  const TI* sA = reinterpret_cast<const TI*>(s_dyn);
  float* sLf = reinterpret_cast<float*>(s_dyn + LL::staged(n));       // LAMC: rebuilt snapshots
  const float* sL = LAMC ? sLf : reinterpret_cast<const float*>(s_dyn + LL::a_bytes(n));
  const TB* sB = reinterpret_cast<const TB*>(s_dyn + LL::a_bytes(n) + LL::l_bytes(n));
  float* As = reinterpret_cast<float*>(s_dyn + LL::staged(n) + LL::table(n));   // merge only
  float* Bc = As + (n + 1) * DK;                                      // merge only

  // 1. The token's inputs and this head's Sbar tile into registers (all
  // state loads in flight; order as above), then the log once the preceding
  // kernel has completed.  An append lets the next step launch early; a
  // merge, which writes Sbar, does not.
  const TI* qg = static_cast<const TI*>(a.q) + bu * DK;
  const TI* kg = static_cast<const TI*>(a.k) + bu * DK;
  float kr[TL::KPL], qr[TL::KPL], gt[TL::KPL], lt[TL::KPL], lp[TL::KPL];
  float g_head = 0.f, vc = 0.f, betac = 0.f;
  const int c = tid;
  auto load_inputs = [&]() {
    if (hold) {   // k = q = v = 0, gate 0, beta 0: a null current entry
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) kr[m] = qr[m] = gt[m] = 0.f;
      return;
    }
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      kr[m] = to_f(kg[j]);
      qr[m] = to_f(qg[j]);
      gt[m] = PERKEY ? a.log_decay[bu * DK + j] : 0.f;
    }
    if (!PERKEY) g_head = a.log_decay[bu];   // GDN: scalar log-gate
    if (c < DVT) {
      vc = to_f(static_cast<const TI*>(a.v)[bu * DV + col0 + c]);
      if (DELTA) betac = a.beta[bu];
    }
  };
  if constexpr (PERKEY) load_inputs();
  // This thread's rows of the tile, addressed from one register with
  // immediate row offsets (rows are DV floats apart).
  float* Sp = a.Sbar + sh * (DK * DV) + (rg * TL::RPT) * DV + col0 + 4 * c4;
  float4 st[TL::RPT];
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) st[j] = ld_state(Sp + j * DV);
  if (MODE == MODE_APPEND) griddep_launch_dependents();
  if constexpr (!WAIT_FIRST) griddep_wait();
  if (tid == 0)
    stage_log<OP, DK, DV, TI, BLOW, LAMC>(s_dyn, &s_bar, a.logA, a.logLam, a.logB, sh, a.Mcap, n,
                                          a.stall_log != 0);
  if constexpr (!PERKEY) load_inputs();

  // 2. Decay snapshots: Lam_{t-1} from the newest entry, Lam_t = Lam_{t-1} +
  // log-gate; GDN's scalar snapshots of every entry.  (LAMC rebuilds the
  // snapshots from the staged gates below, once the log has arrived.)
  if (PERKEY && !LAMC) {
    const float* lamp = a.logLam + (sh * a.Mcap + (n > 0 ? n - 1 : 0)) * DK;
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      lp[m] = n > 0 ? lamp[lane + 32 * m] : 0.f;
      lt[m] = lp[m] + gt[m];
    }
  } else if (!PERKEY) {
    if (tid < n) s_lam[tid] = a.logLam[sh * gdn_lam_stride(a.Mcap) + tid];
    const float lprev = n > 0 ? a.logLam[sh * gdn_lam_stride(a.Mcap) + (n - 1)] : 0.f;
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      lp[m] = lprev;
      lt[m] = lprev + g_head;
    }
  }
  __syncthreads();                              // barrier init and s_lam visible
  if (!wait_log(&s_bar, n, a.err, a.stall_log ? kStallWaitNs : kWaitNs)) return;
  if constexpr (LAMC) {
    rebuild_snapshots<DK>(reinterpret_cast<const __half*>(s_dyn + LL::a_bytes(n)), sLf, n);
    __syncthreads();
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      lp[m] = n > 0 ? sLf[(n - 1) * DK + lane + 32 * m] : 0.f;
      lt[m] = lp[m] + gt[m];
    }
  }

  // 3. ReplayPrep: per-entry coefficients once per (slot, head).  Warp w takes
  // entries i = w, w+NW, ...; i == n is the current token (kappa).
  for (int i = warp; i <= n; i += TL::NW) {
    float dk = 0.f, dq = 0.f;
    if (i < n) {
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) {
        const int j = lane + 32 * m;
        const float ai = to_f(sA[i * DK + j]);
        const float lam_i = PERKEY ? sL[i * DK + j] : s_lam[i];
        const float r_t = exp_sfu(lt[m] - lam_i);              // ratio to Lam_t
        if (DELTA) {
          dk = fmaf(r_t * ai, kr[m], dk);
          dq = fmaf(r_t * ai, qr[m], dq);
        } else {
          const float r_p = exp_sfu(lp[m] - lam_i);            // RWKV6 reads S_{t-1}
          dq = fmaf(r_p * ai, qr[m], dq);
        }
        if (MERGE) As[i * DK + j] = r_t * ai;
      }
    } else {
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) {
        const int j = lane + 32 * m;
        if (DELTA) {
          dq = fmaf(kr[m], qr[m], dq);                           // kappa = k . q
        } else {
          dq = fmaf(a.u[h * DK + j] * kr[m], qr[m], dq);         // kappa = (u (.) k) . r
        }
        if (MERGE) As[n * DK + j] = kr[m];                       // current entry, ratio 1
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
      const float et = exp_sfu(lt[m]);
      if (DELTA) {
        s_kt[j] = et * kr[m];
        s_qt[j] = et * qr[m];
      } else {
        s_qt[j] = exp_sfu(lp[m]) * qr[m];
      }
      if (MERGE) s_dec[j] = et;
    }
    if (!MERGE && col0 == 0) {  // append (first value tile): a_n = k_t and its snapshot
      TI* dstA = static_cast<TI*>(a.logA) + (sh * a.Mcap + n) * DK;
#pragma unroll
      for (int m = 0; m < TL::KPL; ++m) {
        const int j = lane + 32 * m;
        dstA[j] = kg[j];
        if (LAMC) {
          reinterpret_cast<__half*>(a.logLam)[(sh * a.Mcap + n) * DK + j] = __float2half_rn(gt[m]);
        } else if (PERKEY) {
          a.logLam[(sh * a.Mcap + n) * DK + j] = lt[m];
        }
      }
      if (!PERKEY && lane == 0) a.logLam[sh * gdn_lam_stride(a.Mcap) + n] = lt[0];
    }
  }
  __syncthreads();

  // 4. One pass over the register tile: partial Sbar^T k~ and Sbar^T q~.
  {
    float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = p4;
#pragma unroll
    for (int j = 0; j < TL::RPT; ++j) {
      const int row = rg * TL::RPT + j;
      if (DELTA) fma4(p4, s_kt[row], st[j]);
      fma4(s4, s_qt[row], st[j]);
    }
    if (DELTA) *reinterpret_cast<float4*>(&s_red[0][rg][4 * c4]) = p4;
    *reinterpret_cast<float4*>(&s_red[1][rg][4 * c4]) = s4;
  }
  __syncthreads();

  // 5. AppendDecode finalize for value column c: replay, delta correction, output.
  if (c < DVT) {
    float p = 0.f, s = 0.f;
#pragma unroll
    for (int g = 0; g < TL::RG; ++g) {
      if (DELTA) p += s_red[0][g][c];
      s += s_red[1][g][c];
    }
    float oc = s, bt;
    for (int i = 0; i < n; ++i) {
      const float bi = to_f(sB[i * DV + col0 + c]);
      if (DELTA) p = fmaf(s_ck[i], bi, p);
      oc = fmaf(s_cq[i], bi, oc);
    }
    if (DELTA) {
      bt = betac * (vc - p);
    } else {
      bt = vc;
    }
    oc = fmaf(s_kappa, bt, oc);
    if (!hold) static_cast<TI*>(a.o)[bu * DV + col0 + c] = from_f<TI>(oc);
    if (MERGE) {
      Bc[c] = bt;
    } else {
      TB* dstB = static_cast<TB*>(a.logB) + (sh * a.Mcap + n) * DV + col0;
      if constexpr (DELTA) {
        dstB[c] = from_f<TB>(bt);
      } else {
        dstB[c] = static_cast<const TI*>(a.v)[bu * DV + col0 + c];   // raw v, bit copy
      }
    }
  }

  // 6. Merge: S_t = diag(e^{Lam_t}) Sbar + sum_{i<=n} (ratio_i (.) a_i) b_i^T.
  if (MERGE) {
    __syncthreads();
#pragma unroll
    for (int j = 0; j < TL::RPT; ++j) {
      scale4(st[j], s_dec[rg * TL::RPT + j]);
    }
    for (int i = 0; i <= n; ++i) {
      const float4 b4 = i < n ? load4f(sB + i * DV + col0 + 4 * c4) : load4f(Bc + 4 * c4);
      const float* ai = &As[i * DK + rg * TL::RPT];
#pragma unroll
      for (int j4 = 0; j4 < TL::RPT; j4 += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(ai + j4);
        fma4(st[j4 + 0], a4.x, b4);
        fma4(st[j4 + 1], a4.y, b4);
        fma4(st[j4 + 2], a4.z, b4);
        fma4(st[j4 + 3], a4.w, b4);
      }
    }
    // Re-derive the store addresses from the one base register rather than
    // keep the load addresses live across the kernel (measured with ptxas:
    // the merge variants drop from 128 registers with 32 bytes of spills to
    // 114-118 registers and none).
    float* Sw = Sp;
    asm volatile("" : "+l"(Sw));
#pragma unroll
    for (int j = 0; j < TL::RPT; ++j) st_state(Sw + j * DV, st[j]);
  }
}

// ---------------------------------------------------------------------------
// Eager dense baseline: S_{t-1} -> S_t read and written every token.  Same
// tile mapping (and value-tile split) as the deferred step.
// ---------------------------------------------------------------------------
template <int OP, int DK, int DV, typename TI, int NSPLIT, bool MAP>
__global__ void __launch_bounds__(Tile<DK, DV / NSPLIT>::NT, Tile<DK, DV / NSPLIT>::MINB)
eager_step_kernel(const StepArgs a) {
  constexpr int DVT = DV / NSPLIT;  // value-tile width owned by this CTA
  using TL = Tile<DK, DVT>;
  constexpr bool DELTA = OP != OP_RWKV6;

  __shared__ __align__(16) float s_kx[DK];   // contraction vector for p
  __shared__ __align__(16) float s_qx[DK];   // contraction vector for s
  __shared__ __align__(16) float s_dec[DK];  // per-row decay of S_{t-1}
  __shared__ __align__(16) float s_k[DK];    // k_t (rank-1 update rows)
  __shared__ __align__(16) float s_b[DVT];   // b_t (rank-1 update columns)
  __shared__ __align__(16) float s_red[2][TL::RG][DVT];
  __shared__ float s_kappa;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % TL::TPR, rg = tid / TL::TPR;
  const UnitIx ux = unit_of<NSPLIT, DVT, MAP>(a);
  if (!ux.ok || ux.hold) return;   // the dense state of a held slot needs nothing
  const long bu = ux.bu;      // batch unit: inputs and output
  const long sh = ux.sh;      // pool unit: the state
  const int col0 = ux.col0;
  const int h = ux.h;

  float* Sp = a.Sbar + sh * (DK * DV) + (rg * TL::RPT) * DV + col0 + 4 * c4;   // this thread's rows
  float4 st[TL::RPT];
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) st[j] = ld_state(Sp + j * DV);

  const int c = tid;
  float vc = 0.f, betac = 0.f;
  if (c < DVT) {
    vc = to_f(static_cast<const TI*>(a.v)[bu * DV + col0 + c]);
    if (DELTA) betac = a.beta[bu];
  }

  if (warp == 0) {
    const TI* qg = static_cast<const TI*>(a.q) + bu * DK;
    const TI* kg = static_cast<const TI*>(a.k) + bu * DK;
    float kap = 0.f;
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      const float kj = to_f(kg[j]), qj = to_f(qg[j]);
      const float dec = expf(OP == OP_GDN ? a.log_decay[bu] : a.log_decay[bu * DK + j]);
      s_dec[j] = dec;
      s_k[j] = kj;
      if (OP == OP_GDN) {          // p = S^T k, s = S^T q (alpha applied after)
        s_kx[j] = kj;
        s_qx[j] = qj;
        kap = fmaf(kj, qj, kap);
      } else if (OP == OP_KDA) {   // p = S^T (alpha (.) k), s = S^T (alpha (.) q)
        s_kx[j] = dec * kj;
        s_qx[j] = dec * qj;
        kap = fmaf(kj, qj, kap);
      } else {                     // RWKV6: s = S^T r, kappa = (u (.) k) . r
        s_qx[j] = qj;
        kap = fmaf(a.u[h * DK + j] * kj, qj, kap);
      }
    }
    kap = warp_sum(kap);
    if (lane == 0) s_kappa = kap;
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

  if (c < DVT) {
    float p = 0.f, s = 0.f;
#pragma unroll
    for (int g = 0; g < TL::RG; ++g) {
      if (DELTA) p += s_red[0][g][c];
      s += s_red[1][g][c];
    }
    float oc, bt;
    if (OP == OP_GDN) {
      const float alpha = s_dec[0];
      bt = betac * (vc - alpha * p);
      oc = fmaf(s_kappa, bt, alpha * s);
    } else if (OP == OP_KDA) {
      bt = betac * (vc - p);
      oc = fmaf(s_kappa, bt, s);
    } else {
      bt = vc;
      oc = fmaf(s_kappa, vc, s);
    }
    s_b[c] = bt;
    static_cast<TI*>(a.o)[bu * DV + col0 + c] = from_f<TI>(oc);
  }
  __syncthreads();

  const float4 b4 = *reinterpret_cast<const float4*>(&s_b[4 * c4]);
  float* Sw = Sp;
  asm volatile("" : "+l"(Sw));   // store addresses from one register (see the step kernel)
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) {
    const int row = rg * TL::RPT + j;
    float4 x = st[j];
    scale4(x, s_dec[row]);
    fma4(x, s_k[row], b4);
    st_state(Sw + j * DV, x);
  }
}

// ---------------------------------------------------------------------------
// Materialise base + log into Sout (dl_merge with Sout == Sin, dl_read_state
// otherwise).  Lam_last = Lam_{n-1}, the newest snapshot; a unit with an
// empty log is copied through.
// ---------------------------------------------------------------------------
template <int OP, int DK, int DV, typename TI, bool BLOW, bool LAMC>
__global__ void __launch_bounds__(Tile<DK, DV>::NT, Tile<DK, DV>::MINB)
materialize_kernel(const MaterializeArgs a) {
  using TL = Tile<DK, DV>;
  using LL = LogLayout<OP, DK, DV, TI, BLOW, LAMC>;
  using TB = typename LL::TB;
  constexpr bool PERKEY = OP != OP_GDN;
  __shared__ __align__(16) float s_dec[DK];
  __shared__ float s_lam[kMaxM];
  __shared__ __align__(8) uint64_t s_bar;
  extern __shared__ __align__(128) unsigned char s_dyn[];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % TL::TPR, rg = tid / TL::TPR;
  long sh = a.unit0 + blockIdx.x;
  float* Sq = a.Sout + blockIdx.x * (DK * DV);
  if (a.slot_idx) {
    const int slot = __ldg(a.slot_idx + blockIdx.y);
    if (slot < 0) return;
    if (slot >= a.slots) {
      if (tid == 0) atomicOr(a.err, kErrSlotIndex);
      return;
    }
    sh = static_cast<long>(slot) * a.H + blockIdx.x;
    Sq = a.Sout + sh * (DK * DV);
  }
  const int n = a.n;

  const TI* sA = reinterpret_cast<const TI*>(s_dyn);
  float* sLf = reinterpret_cast<float*>(s_dyn + LL::staged(n));       // LAMC: rebuilt snapshots
  const float* sL = LAMC ? sLf : reinterpret_cast<const float*>(s_dyn + LL::a_bytes(n));
  const TB* sB = reinterpret_cast<const TB*>(s_dyn + LL::a_bytes(n) + LL::l_bytes(n));
  float* As = reinterpret_cast<float*>(s_dyn + LL::staged(n) + LL::table(n));

  const float* Sp = a.Sin + sh * (DK * DV) + (rg * TL::RPT) * DV + 4 * c4;   // this thread's rows
  float4 st[TL::RPT];
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) st[j] = ld_state(Sp + j * DV);
  if (tid == 0) stage_log<OP, DK, DV, TI, BLOW, LAMC>(s_dyn, &s_bar, a.logA, a.logLam, a.logB, sh, a.Mcap, n);

  float ll[TL::KPL];
  if constexpr (!LAMC) {
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      ll[m] = n == 0 ? 0.f
              : PERKEY ? a.logLam[(sh * a.Mcap + (n - 1)) * DK + j]
                       : a.logLam[sh * gdn_lam_stride(a.Mcap) + (n - 1)];
    }
  }
  if (!PERKEY && tid < n) s_lam[tid] = a.logLam[sh * gdn_lam_stride(a.Mcap) + tid];
  __syncthreads();
  if (!wait_log(&s_bar, n, a.err)) return;
  if constexpr (LAMC) {
    rebuild_snapshots<DK>(reinterpret_cast<const __half*>(s_dyn + LL::a_bytes(n)), sLf, n);
    __syncthreads();
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) ll[m] = n == 0 ? 0.f : sLf[(n - 1) * DK + lane + 32 * m];
  }

  for (int i = warp; i < n; i += TL::NW) {
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) {
      const int j = lane + 32 * m;
      const float lam_i = PERKEY ? sL[i * DK + j] : s_lam[i];
      As[i * DK + j] = expf(ll[m] - lam_i) * to_f(sA[i * DK + j]);
    }
  }
  if (warp == 0) {
#pragma unroll
    for (int m = 0; m < TL::KPL; ++m) s_dec[lane + 32 * m] = expf(ll[m]);
  }
  __syncthreads();

#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) {
    scale4(st[j], s_dec[rg * TL::RPT + j]);
  }
  for (int i = 0; i < n; ++i) {
    const float4 b4 = load4f(sB + i * DV + 4 * c4);
    const float* ai = &As[i * DK + rg * TL::RPT];
#pragma unroll
    for (int j4 = 0; j4 < TL::RPT; j4 += 4) {
      const float4 a4 = *reinterpret_cast<const float4*>(ai + j4);
      fma4(st[j4 + 0], a4.x, b4);
      fma4(st[j4 + 1], a4.y, b4);
      fma4(st[j4 + 2], a4.z, b4);
      fma4(st[j4 + 3], a4.w, b4);
    }
  }
  float* Sw = Sq + (rg * TL::RPT) * DV + 4 * c4;
  asm volatile("" : "+l"(Sw));   // store addresses from one register (see the step kernel)
#pragma unroll
  for (int j = 0; j < TL::RPT; ++j) st_state(Sw + j * DV, st[j]);
}

}  // namespace dl
