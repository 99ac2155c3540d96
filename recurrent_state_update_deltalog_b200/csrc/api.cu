// C ABI of libdeltalog: handle lifetime, argument validation and launches.
// The contract of every entry point is documented in include/deltalog.h.
#include "deltalog.h"
#include "launch.cuh"
#include "prefill.cuh"

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <new>
#include <string>

static_assert(DL_DEVERR_WAIT_TIMEOUT == dl::kErrWaitTimeout, "device error bits");
static_assert(DL_DEVERR_SLOT_INDEX == dl::kErrSlotIndex, "device error bits");
static_assert(DL_DEVERR_SEQLEN == dl::kErrSeqlen, "device error bits");
static_assert(DL_SLOT_HOLD == dl::kSlotHold, "held-slot bit of the slot map");

struct dl_handle {
  int B, H, dk, dv, M, op, dtype, device;
  int sms, smem_block_optin, smem_sm, smem_reserved;  // device limits
  int step_kernel;                                    // DL_STEP_* requested
  int last_kernel;                                    // DL_STEP_* used by the last dl_step
  // Entries in every slot's log, tracked on the host in stream order.  All
  // slots share it: a slot loaded or merged mid-cycle keeps its n positions,
  // zeroed, so every step is one lockstep launch.
  int n;
  bool wrote_state;    // the last launch on this handle may have written Sbar
  int Mcap;    // log capacity per (slot, head): max(M - 1, 1)
  size_t esize;
  float* Sbar;
  void* logA;
  void* logB;
  float* logLam;
  float* u;
  int* err;
  // device staging for dl_step_host: two sets, so that with host prefetch the
  // inputs of call t+1 upload (on copy_stream) while call t computes
  struct Staging {
    void* q;
    void* k;
    void* v;
    void* o;
    float* ld;
    float* beta;
  } st[2];
  cudaStream_t copy_stream;
  cudaEvent_t in_ready[2];  // recorded on copy_stream after a set's uploads
  cudaEvent_t set_free[2];  // recorded on the caller's stream after a set's download
  bool set_used[2];
  int host_calls;
  int host_prefetch;        // DL_OPT_HOST_PREFETCH
  int pdl;                  // DL_OPT_PDL
  int value_tiles;          // DL_OPT_VALUE_TILES (0 = automatic)
  int log_b_bf16;           // DL_OPT_LOG_B_BF16
  int prefill_kernel;       // DL_OPT_PREFILL_KERNEL (DL_PREFILL_*)
  int last_prefill;         // DL_PREFILL_* used by the last dl_prefill
  int stall_log;            // DL_OPT_TEST_STALL_LOG
  int log_lam_f16;          // DL_OPT_LOG_LAM_F16
};

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Makes the handle's device current for the scope of a call and restores the
// caller's device afterwards.
class DeviceScope {
 public:
  explicit DeviceScope(int dev) {
    ok_ = cudaGetDevice(&prev_) == cudaSuccess;
    if (ok_ && prev_ != dev) {
      ok_ = cudaSetDevice(dev) == cudaSuccess;
      changed_ = ok_;
    }
  }
  ~DeviceScope() {
    if (changed_) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = 0;
  bool ok_ = false;
  bool changed_ = false;
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t lam_per_entry(const dl_handle* h) { return h->op == DL_GDN ? 1 : static_cast<size_t>(h->dk); }
size_t lam_unit_floats(const dl_handle* h) {
  return h->op == DL_GDN ? static_cast<size_t>(dl::gdn_lam_stride(h->Mcap)) : static_cast<size_t>(h->Mcap) * h->dk;
}
// Bytes of one Lam element in the log: per-key snapshots are fp16 log-gates
// with DL_OPT_LOG_LAM_F16 (the buffer is sized for fp32, so the option needs
// no reallocation); GDN keeps fp32 scalars.
size_t lam_esize(const dl_handle* h) { return h->op != DL_GDN && h->log_lam_f16 ? 2 : 4; }
// Element size of b_i in the log: RWKV6 keeps raw v_i in the input dtype;
// GDN/KDA keep fp32, or bf16 with DL_OPT_LOG_B_BF16.  The buffer is sized
// for fp32 (logb_alloc_esize) so that the option needs no reallocation.
size_t logb_esize(const dl_handle* h) { return h->op == DL_RWKV6 || h->log_b_bf16 ? h->esize : sizeof(float); }
size_t logb_alloc_esize(const dl_handle* h) { return h->op == DL_RWKV6 ? h->esize : sizeof(float); }
size_t bh(const dl_handle* h) { return static_cast<size_t>(h->B) * h->H; }
size_t state_bytes(const dl_handle* h) { return bh(h) * h->dk * h->dv * sizeof(float); }
size_t decay_elems(const dl_handle* h) { return bh(h) * lam_per_entry(h); }

void free_all(dl_handle* h) {
  void* ptrs[] = {h->Sbar, h->logA, h->logB, h->logLam, h->u, h->err};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (auto& st : h->st) {
    void* sp[] = {st.q, st.k, st.v, st.o, st.ld, st.beta};
    for (void* p : sp)
      if (p) cudaFree(p);
  }
  for (int j = 0; j < 2; ++j) {
    if (h->in_ready[j]) cudaEventDestroy(h->in_ready[j]);
    if (h->set_free[j]) cudaEventDestroy(h->set_free[j]);
  }
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
}

// Launch geometry and policies for the handle's current log length and
// `units` launched (slot, head) units (0: every slot).
dl::LaunchShape shape_of(const dl_handle* h, long units = 0) {
  dl::LaunchShape s;
  s.BH = static_cast<int>(units > 0 ? units : bh(h));
  s.H = h->H;
  s.dk = h->dk;
  s.dv = h->dv;
  s.dtype = h->dtype;
  s.sms = h->sms;
  s.smem_block_optin = h->smem_block_optin;
  s.smem_sm = h->smem_sm;
  s.smem_reserved = h->smem_reserved;
  s.variant = h->step_kernel;
  // Programmatic launch only when the previous launch of this handle did not
  // write Sbar (an append): the step may then read Sbar before it completes.
  s.pdl = h->pdl && !h->wrote_state;
  if (h->value_tiles == 0) {
    // measured on B200: two 64-column tiles per head win for d_v = 128 while
    // the log is short (each tile recomputes the key-side coefficients) and
    // the launch has at least two units per SM; below that (GDN B=4, H=32:
    // 128 units) one tile is 7.7% faster
    s.split = h->dv == 128 && h->n < 16 && s.BH >= 2 * h->sms ? 2 : 1;
  } else {
    s.split = h->dv / h->value_tiles >= 32 ? h->value_tiles : 1;
  }
  s.max_n = h->n;
  s.units = s.BH;
  s.blow = h->log_b_bf16 && h->op != DL_RWKV6;
  s.lamc = h->log_lam_f16 && h->op != DL_GDN;
  return s;
}

int check_step_args(const dl_handle* h, const void* q, const void* k, const void* v,
                    const float* log_decay, const float* beta, const void* o) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (!q || !k || !v || !log_decay || !o) return fail(DL_ERR_ARG, "null input/output pointer");
  if (h->op == DL_RWKV6 && beta) return fail(DL_ERR_ARG, "beta must be NULL for RWKV6");
  if (h->op != DL_RWKV6 && !beta) return fail(DL_ERR_ARG, "beta is required for GDN/KDA");
  const void* tp[] = {q, k, v, o};
  for (const void* p : tp)
    if (!aligned(p, h->esize)) return fail(DL_ERR_ARG, "input/output pointer not aligned to its element size");
  if (!aligned(log_decay, 4) || (beta && !aligned(beta, 4))) return fail(DL_ERR_ARG, "gate pointer not 4-byte aligned");
  return DL_OK;
}

// A slot index map of `rows` rows; rows == 0 needs no pointer at all.
int check_slot_map(const dl_handle* h, const int* slot_idx, int rows) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (rows < 0 || rows > h->B) return fail(DL_ERR_ARG, "rows=%d outside [0, %d]", rows, h->B);
  if (rows > 65535) return fail(DL_ERR_UNSUPPORTED, "slot index maps take at most 65535 rows (grid y)");
  if (rows > 0 && (!slot_idx || !aligned(slot_idx, 4)))
    return fail(DL_ERR_ARG, "slot index pointer null or not 4-byte aligned");
  return DL_OK;
}

dl::StepArgs step_args(dl_handle* h, const void* q, const void* k, const void* v,
                       const float* log_decay, const float* beta, void* o) {
  dl::StepArgs a;
  a.Sbar = h->Sbar;
  a.q = q;
  a.k = k;
  a.v = v;
  a.log_decay = log_decay;
  a.beta = beta;
  a.o = o;
  a.slot_idx = nullptr;
  a.slots = h->B;
  a.logA = h->logA;
  a.logB = h->logB;
  a.logLam = h->logLam;
  a.u = h->u;
  a.err = h->err;
  a.H = h->H;
  a.M = h->M;
  a.Mcap = h->Mcap;
  a.n = h->n;
  a.stall_log = h->stall_log;
  return a;
}

// Empty slot `b`'s log without changing its logical state: zero factors
// contribute nothing, and Lam_i = 0 restarts its cumulative decay at the
// present token.  Only positions [0, n) are ever read; the whole slot is
// cleared.
cudaError_t zero_slot_log(const dl_handle* h, int b, cudaStream_t s) {
  const size_t units = static_cast<size_t>(h->H), first = static_cast<size_t>(b) * units;
  const size_t a_unit = static_cast<size_t>(h->Mcap) * h->dk * h->esize;
  const size_t b_unit = static_cast<size_t>(h->Mcap) * h->dv * logb_esize(h);
  const size_t l_unit = lam_unit_floats(h) * lam_esize(h);
  cudaError_t e = cudaMemsetAsync(static_cast<char*>(h->logA) + first * a_unit, 0, units * a_unit, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(static_cast<char*>(h->logB) + first * b_unit, 0, units * b_unit, s);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(reinterpret_cast<char*>(h->logLam) + first * l_unit, 0, units * l_unit, s);
  return e;
}

// `rows` batch rows of H units each are launched (B without an index map).
cudaError_t launch_step(dl_handle* h, int mode, const dl::StepArgs& a, int rows, cudaStream_t s) {
  const dl::LaunchShape sh = shape_of(h, static_cast<long>(rows) * h->H);
  int* used = &h->last_kernel;
  switch (h->op) {
    case DL_GDN: return dl::launch_step_op<dl::OP_GDN>(sh, mode, a, s, used);
    case DL_KDA: return dl::launch_step_op<dl::OP_KDA>(sh, mode, a, s, used);
    default: return dl::launch_step_op<dl::OP_RWKV6>(sh, mode, a, s, used);
  }
}

cudaError_t launch_eager(const dl_handle* h, const dl::StepArgs& a, int rows, cudaStream_t s) {
  dl::LaunchShape sh = shape_of(h, static_cast<long>(rows) * h->H);
  // the eager kernel has no per-tile ReplayPrep to repeat: two tiles for
  // d_v = 128 at every batch size measured (B = 1..1024)
  if (h->value_tiles == 0) sh.split = h->dv == 128 ? 2 : 1;
  switch (h->op) {
    case DL_GDN: return dl::launch_eager_op<dl::OP_GDN>(sh, a, s);
    case DL_KDA: return dl::launch_eager_op<dl::OP_KDA>(sh, a, s);
    default: return dl::launch_eager_op<dl::OP_RWKV6>(sh, a, s);
  }
}

// Base + log of units [unit0, unit0 + units) into `out` (which points at the
// first of them).
cudaError_t launch_materialize(const dl_handle* h, float* out, cudaStream_t s, long unit0, int units) {
  dl::MaterializeArgs a;
  a.Sin = h->Sbar;
  a.Sout = out;
  a.logA = h->logA;
  a.logB = h->logB;
  a.logLam = h->logLam;
  a.err = h->err;
  a.unit0 = unit0;
  a.slot_idx = nullptr;
  a.slots = h->B;
  a.H = h->H;
  a.Mcap = h->Mcap;
  a.n = h->n;
  dl::LaunchShape sh = shape_of(h);
  sh.units = units;
  switch (h->op) {
    case DL_GDN: return dl::launch_materialize_op<dl::OP_GDN>(sh, a, s);
    case DL_KDA: return dl::launch_materialize_op<dl::OP_KDA>(sh, a, s);
    default: return dl::launch_materialize_op<dl::OP_RWKV6>(sh, a, s);
  }
}

// Fold the logs of slots slot_idx[0..rows) into their bases, in place.
cudaError_t materialize_slots(const dl_handle* h, const int* slot_idx, int rows, cudaStream_t s) {
  dl::MaterializeArgs a;
  a.Sin = h->Sbar;
  a.Sout = h->Sbar;
  a.logA = h->logA;
  a.logB = h->logB;
  a.logLam = h->logLam;
  a.err = h->err;
  a.unit0 = 0;
  a.slot_idx = slot_idx;
  a.slots = h->B;
  a.H = h->H;
  a.Mcap = h->Mcap;
  a.n = h->n;
  dl::LaunchShape sh = shape_of(h);
  sh.units = slot_idx ? rows : rows * h->H;
  switch (h->op) {
    case DL_GDN: return dl::launch_materialize_op<dl::OP_GDN>(sh, a, s);
    case DL_KDA: return dl::launch_materialize_op<dl::OP_KDA>(sh, a, s);
    default: return dl::launch_materialize_op<dl::OP_RWKV6>(sh, a, s);
  }
}

// The chunked prefills (state in tensor memory) serve bf16-input handles.
// AUTO picks them once the prompts average enough tokens to fill their
// 32-token chunks.  Measured on B200 against the recurrent kernel (bf16):
//   d = 128, H = 32: GDN L=8 0.90, L=16 1.32, L=24 1.86, B=64 L=512 4.2;
//               KDA L=16 1.05, B=64 L=512 2.4; RWKV6 L=8 0.69;
//   d = 64:     GDN (H=32) L=16 0.73, L=32 1.15; KDA (H=32) L=32 1.10;
//               RWKV6 (H=64) L=16 0.65, L=32 1.05, B=64 L=512 1.6.
// Thresholds: 16 tokens at d_k = d_v = 128, 32 at the other shapes.
bool chunked_prefill(const dl_handle* h, int rows, long long total) {
  if (h->prefill_kernel != DL_PREFILL_AUTO) return h->prefill_kernel == DL_PREFILL_CHUNKED;
  const bool big = h->dk == 128 && h->dv == 128;
  const long long min_avg = big ? 16 : 32;
  return h->dtype == DL_BF16 && total >= min_avg * rows;
}

cudaError_t launch_prefill(dl_handle* h, const dl::PrefillArgs& a, int rows, cudaStream_t s) {
  dl::LaunchShape sh = shape_of(h);
  sh.units = rows;
  if (chunked_prefill(h, rows, a.total)) {
    if (h->dtype != DL_BF16) return cudaErrorNotSupported;
    h->last_prefill = DL_PREFILL_CHUNKED;
    switch (h->op) {
      case DL_GDN: return dl::launch_gdn_chunk_prefill_dims(sh, a, s);
      case DL_KDA: return dl::launch_key_chunk_prefill_dims<dl::OP_KDA>(sh, a, s);
      default: return dl::launch_key_chunk_prefill_dims<dl::OP_RWKV6>(sh, a, s);
    }
  }
  h->last_prefill = DL_PREFILL_RECURRENT;
  switch (h->op) {
    case DL_GDN: return dl::launch_prefill_op<dl::OP_GDN>(sh, a, s);
    case DL_KDA: return dl::launch_prefill_op<dl::OP_KDA>(sh, a, s);
    default: return dl::launch_prefill_op<dl::OP_RWKV6>(sh, a, s);
  }
}

// One token: `rows` batch rows, row r on slot idx[r] (row r itself when idx
// is null).
int do_step(dl_handle* h, const int* idx, int rows, const void* q, const void* k, const void* v,
            const float* log_decay, const float* beta, void* o, cudaStream_t s) {
  const bool merge = h->n + 1 == h->M;
  dl::StepArgs a = step_args(h, q, k, v, log_decay, beta, o);
  a.slot_idx = idx;
  cudaError_t e = launch_step(h, merge ? dl::MODE_MERGE : dl::MODE_APPEND, a, rows, s);
  if (e != cudaSuccess) return cuda_fail(e, "deltalog step launch");
  h->n = merge ? 0 : h->n + 1;
  h->wrote_state = merge;
  return DL_OK;
}

// Replay cost of one log entry over its bytes, c(op, d_k, d_v), measured on
// B200 for the square shapes: two fine M sweeps (4..16) per shape, averaged
// and fitted with the cost model of dl_suggest_m (residuals under 1%).  It
// exceeds 1 where the replay's arithmetic, repeated per value tile, outweighs
// its bytes.  RWKV6 at d = 64 fits 1.12, whose optimum (7) measured 1.25%
// below the best; it takes 1.10, the nearest ratio whose optimum (8) lies
// within 1% of it.  Mixed shapes take the pure traffic model (1).
double replay_cost_ratio(int op, int dk, int dv) {
  if (dk != dv) return 1.0;
  const bool big = dk == 128;
  switch (op) {
    case DL_GDN: return big ? 1.33 : 0.98;
    case DL_KDA: return big ? 1.53 : 1.26;
    default: return big ? 1.47 : 1.10;
  }
}

// Bytes of one log entry: a_i (input dtype), b_i (fp32, raw v for RWKV6), Lam_i.
double entry_bytes(int op, int dk, int dv, int esize) {
  const double a = static_cast<double>(dk) * esize;
  const double b = static_cast<double>(dv) * (op == DL_RWKV6 ? esize : 4);
  const double lam = op == DL_GDN ? 4.0 : 4.0 * dk;
  return a + b + lam;
}

int suggest_m(int op, int dk, int dv, int esize) {
  const double S = 4.0 * dk * dv;
  const double e = entry_bytes(op, dk, dv, esize);
  const double rho = e * replay_cost_ratio(op, dk, dv);
  int best = 2;
  double fbest = 0.0;
  for (int M = 2; M <= DL_MAX_M; ++M) {
    const double f = S / M + e * (M - 1) / M + rho * (M - 1) / 2.0;
    if (M == 2 || f < fbest) {
      best = M;
      fbest = f;
    }
  }
  return best;
}

// Read and clear the device error word in one atomic step (err[0]) into its
// snapshot (err[1]): bits that work on other streams raises meanwhile stay in
// the word for the next check instead of being cleared unseen.
__global__ void take_error_word(int* err) { err[1] = atomicExch(err, 0); }

}  // namespace

namespace dl {
// The last-error message of this thread, for entry points defined in other
// translation units.
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace dl

extern "C" {

int dl_suggest_m(int op, int d_k, int d_v, int in_dtype, int* M) {
  if (!M) return fail(DL_ERR_ARG, "null output pointer");
  if (op < DL_GDN || op > DL_RWKV6) return fail(DL_ERR_ARG, "unknown op %d", op);
  if (in_dtype != DL_F32 && in_dtype != DL_BF16) return fail(DL_ERR_ARG, "unknown dtype %d", in_dtype);
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128))
    return fail(DL_ERR_ARG, "d_k=%d d_v=%d not in {64,128}", d_k, d_v);
  *M = suggest_m(op, d_k, d_v, in_dtype == DL_BF16 ? 2 : 4);
  return DL_OK;
}

int dl_merge_interval(dl_t h, int* M) {
  if (!h || !M) return fail(DL_ERR_ARG, "null argument");
  *M = h->M;
  return DL_OK;
}


int dl_create(dl_t* out, int B, int H, int d_k, int d_v, int M, int op, int in_dtype) {
  if (!out) return fail(DL_ERR_ARG, "null output handle pointer");
  *out = nullptr;
  if (B <= 0 || H <= 0) return fail(DL_ERR_ARG, "B and H must be positive (B=%d H=%d)", B, H);
  if (M != DL_M_AUTO && (M < 1 || M > DL_MAX_M))
    return fail(DL_ERR_UNSUPPORTED, "M=%d outside [1, %d] and not DL_M_AUTO", M, DL_MAX_M);
  if (op < DL_GDN || op > DL_RWKV6) return fail(DL_ERR_ARG, "unknown op %d", op);
  if (in_dtype != DL_F32 && in_dtype != DL_BF16) return fail(DL_ERR_ARG, "unknown dtype %d", in_dtype);
  const bool dk_ok = d_k == 64 || d_k == 128, dv_ok = d_v == 64 || d_v == 128;
  if (!dk_ok || !dv_ok) return fail(DL_ERR_UNSUPPORTED, "d_k=%d d_v=%d not in {64,128}", d_k, d_v);
  if (M == DL_M_AUTO) M = suggest_m(op, d_k, d_v, in_dtype == DL_BF16 ? 2 : 4);
  if (static_cast<long long>(B) * H > (1ll << 30)) return fail(DL_ERR_ARG, "B*H too large");

  dl_handle* h = new (std::nothrow) dl_handle();
  if (!h) return fail(DL_ERR_OOM, "host allocation failed");
  h->B = B;
  h->H = H;
  h->dk = d_k;
  h->dv = d_v;
  h->M = M;
  h->op = op;
  h->dtype = in_dtype;
  h->n = 0;
  h->wrote_state = true;
  h->Mcap = M > 1 ? M - 1 : 1;
  h->esize = in_dtype == DL_BF16 ? 2 : 4;
  h->step_kernel = DL_STEP_AUTO;
  h->last_kernel = DL_STEP_AUTO;
  h->pdl = 1;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return fail(DL_ERR_CUDA, "no current CUDA device");
  }
  {
    const struct {
      int* dst;
      cudaDeviceAttr attr;
    } q[] = {{&h->sms, cudaDevAttrMultiProcessorCount},
             {&h->smem_block_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin},
             {&h->smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor},
             {&h->smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock}};
    for (auto& x : q) {
      cudaError_t e = cudaDeviceGetAttribute(x.dst, x.attr, h->device);
      if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "device attribute query");
      }
    }
  }
  const size_t nbh = bh(h);
  struct {
    void** p;
    size_t bytes;
  } allocs[] = {
      {reinterpret_cast<void**>(&h->Sbar), state_bytes(h)},
      {&h->logA, nbh * h->Mcap * d_k * h->esize},
      {&h->logB, nbh * h->Mcap * d_v * logb_alloc_esize(h)},
      {reinterpret_cast<void**>(&h->logLam), nbh * lam_unit_floats(h) * sizeof(float)},
      {reinterpret_cast<void**>(&h->u), static_cast<size_t>(H) * d_k * sizeof(float)},
      {reinterpret_cast<void**>(&h->err), 2 * sizeof(int)},   // the word and a snapshot of it
      {&h->st[0].q, nbh * d_k * h->esize},
      {&h->st[0].k, nbh * d_k * h->esize},
      {&h->st[0].v, nbh * d_v * h->esize},
      {&h->st[0].o, nbh * d_v * h->esize},
      {reinterpret_cast<void**>(&h->st[0].ld), decay_elems(h) * sizeof(float)},
      {reinterpret_cast<void**>(&h->st[0].beta), nbh * sizeof(float)},
      {&h->st[1].q, nbh * d_k * h->esize},
      {&h->st[1].k, nbh * d_k * h->esize},
      {&h->st[1].v, nbh * d_v * h->esize},
      {&h->st[1].o, nbh * d_v * h->esize},
      {reinterpret_cast<void**>(&h->st[1].ld), decay_elems(h) * sizeof(float)},
      {reinterpret_cast<void**>(&h->st[1].beta), nbh * sizeof(float)},
  };
  for (auto& a : allocs) {
    cudaError_t e = cudaMalloc(a.p, a.bytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      free_all(h);
      delete h;
      return fail(e == cudaErrorMemoryAllocation ? DL_ERR_OOM : DL_ERR_CUDA,
                  "cudaMalloc of %zu bytes failed: %s", a.bytes, cudaGetErrorString(e));
    }
  }
  cudaError_t e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking);
  for (int j = 0; j < 2 && e == cudaSuccess; ++j) {
    e = cudaEventCreateWithFlags(&h->in_ready[j], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->set_free[j], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaMemset(h->Sbar, 0, state_bytes(h));
  if (e == cudaSuccess) e = cudaMemset(h->u, 0, static_cast<size_t>(H) * d_k * sizeof(float));
  if (e == cudaSuccess) e = cudaMemset(h->err, 0, 2 * sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    free_all(h);
    delete h;
    return cuda_fail(e, "dl_create initialisation");
  }
  *out = h;
  return DL_OK;
}

int dl_destroy(dl_t h) {
  if (!h) return DL_OK;
  DeviceScope ds(h->device);
  free_all(h);
  delete h;
  return ds.ok() ? DL_OK : fail(DL_ERR_CUDA, "could not select the handle's device");
}

int dl_load_state(dl_t h, const float* S, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (!S || !aligned(S, 16)) return fail(DL_ERR_ARG, "state pointer null or not 16-byte aligned");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaError_t e = cudaMemcpyAsync(h->Sbar, S, state_bytes(h), cudaMemcpyDeviceToDevice,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dl_load_state copy");
  h->n = 0;
  h->wrote_state = true;
  return DL_OK;
}

int dl_set_bonus(dl_t h, const float* u, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (h->op != DL_RWKV6) return fail(DL_ERR_STATE, "dl_set_bonus is for RWKV6 handles only");
  if (!u || !aligned(u, 4)) return fail(DL_ERR_ARG, "bonus pointer null or misaligned");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaError_t e = cudaMemcpyAsync(h->u, u, static_cast<size_t>(h->H) * h->dk * sizeof(float),
                                  cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DL_OK : cuda_fail(e, "dl_set_bonus copy");
}

int dl_step(dl_t h, const void* q, const void* k, const void* v, const float* log_decay,
            const float* beta, void* o, void* stream) {
  int rc = check_step_args(h, q, k, v, log_decay, beta, o);
  if (rc != DL_OK) return rc;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  return do_step(h, nullptr, h->B, q, k, v, log_decay, beta, o, static_cast<cudaStream_t>(stream));
}

int dl_step_indexed(dl_t h, const int* slot_idx, int rows, const void* q, const void* k, const void* v,
                    const float* log_decay, const float* beta, void* o, void* stream) {
  int rc = check_slot_map(h, slot_idx, rows);
  if (rc != DL_OK || rows == 0) return rc;
  rc = check_step_args(h, q, k, v, log_decay, beta, o);
  if (rc != DL_OK) return rc;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  return do_step(h, slot_idx, rows, q, k, v, log_decay, beta, o, static_cast<cudaStream_t>(stream));
}

int dl_prefill(dl_t h, const int* slot_idx, int rows, const int* cu_seqlens, long long total, int flags,
               const void* q, const void* k, const void* v, const float* log_decay, const float* beta, void* o,
               void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (rows < 0 || rows > h->B) return fail(DL_ERR_ARG, "rows=%d outside [0, %d]", rows, h->B);
  if (rows > 65535) return fail(DL_ERR_UNSUPPORTED, "a prefill takes at most 65535 rows (grid y)");
  if (flags & ~DL_PREFILL_ZERO_STATE) return fail(DL_ERR_ARG, "unknown prefill flags 0x%x", flags);
  if (total < 0) return fail(DL_ERR_ARG, "negative token count");
  if (rows == 0) return DL_OK;
  if (!cu_seqlens || !aligned(cu_seqlens, 4)) return fail(DL_ERR_ARG, "cu_seqlens null or not 4-byte aligned");
  if (slot_idx && !aligned(slot_idx, 4)) return fail(DL_ERR_ARG, "slot index pointer not 4-byte aligned");
  if (total > 0) {
    int rc = check_step_args(h, q, k, v, log_decay, beta, o);
    if (rc != DL_OK) return rc;
  }
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool zero = flags & DL_PREFILL_ZERO_STATE;
  if (!zero && h->n > 0) {  // start from the logical state: fold the rows' logs first
    cudaError_t e = materialize_slots(h, slot_idx, rows, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill: log fold");
  }
  dl::PrefillArgs a;
  a.Sbar = h->Sbar;
  a.q = q;
  a.k = k;
  a.v = v;
  a.log_decay = log_decay;
  a.beta = beta;
  a.o = o;
  a.u = h->u;
  a.slot_idx = slot_idx;
  a.cu_seqlens = cu_seqlens;
  a.logA = h->logA;
  a.logB = h->logB;
  a.logLam = h->logLam;
  a.err = h->err;
  a.total = static_cast<long>(total);
  a.H = h->H;
  a.slots = h->B;
  a.Mcap = h->Mcap;
  a.n = h->n;
  a.b_esize = static_cast<int>(logb_esize(h));
  a.lam_esize = static_cast<int>(lam_esize(h));
  a.zero_state = zero ? 1 : 0;
  cudaError_t e = launch_prefill(h, a, rows, s);
  if (e == cudaErrorNotSupported)
    return fail(DL_ERR_UNSUPPORTED, "the chunked prefill serves bf16-input handles that fit its shared memory");
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  h->wrote_state = true;
  return DL_OK;
}

int dl_step_host(dl_t h, const void* q, const void* k, const void* v, const float* log_decay,
                 const float* beta, void* o, void* stream) {
  int rc = check_step_args(h, q, k, v, log_decay, beta, o);
  if (rc != DL_OK) return rc;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t nbh = bh(h);
  // Without prefetch the uploads are ordered on the caller's stream like any
  // other work there; with it they run on the handle's copy stream, gated
  // only by the reuse of their staging set, and the caller's stream waits for
  // them before the step.
  const int j = h->host_prefetch ? (h->host_calls & 1) : 0;
  dl_handle::Staging& st = h->st[j];
  cudaStream_t cs = h->host_prefetch ? h->copy_stream : s;
  cudaError_t e = cudaSuccess;
  if (h->host_prefetch && h->set_used[j]) e = cudaStreamWaitEvent(cs, h->set_free[j], 0);
  struct {
    void* dst;
    const void* src;
    size_t bytes;
  } in[] = {
      {st.q, q, nbh * h->dk * h->esize},
      {st.k, k, nbh * h->dk * h->esize},
      {st.v, v, nbh * h->dv * h->esize},
      {st.ld, log_decay, decay_elems(h) * sizeof(float)},
      {st.beta, beta, beta ? nbh * sizeof(float) : 0},
  };
  for (auto& c : in) {
    if (e != cudaSuccess) break;
    if (c.bytes) e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, cs);
  }
  if (e == cudaSuccess && h->host_prefetch) {
    e = cudaEventRecord(h->in_ready[j], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->in_ready[j], 0);
  }
  if (e != cudaSuccess) return cuda_fail(e, "dl_step_host input upload");
  // A pinned, device-mapped output buffer is written by the kernel itself
  // (its stores cross PCIe while the step streams the state); anything else
  // goes through the staging set and one download.
  void* o_dev = nullptr;
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, o) == cudaSuccess && pa.type == cudaMemoryTypeHost && pa.devicePointer &&
      aligned(pa.devicePointer, 16))
    o_dev = pa.devicePointer;
  else
    cudaGetLastError();  // pageable memory reports an error on some drivers
  rc = do_step(h, nullptr, h->B, st.q, st.k, st.v, st.ld, beta ? st.beta : nullptr, o_dev ? o_dev : st.o, s);
  if (rc != DL_OK) return rc;
  if (!o_dev) e = cudaMemcpyAsync(o, st.o, nbh * h->dv * h->esize, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && h->host_prefetch) e = cudaEventRecord(h->set_free[j], s);
  if (e != cudaSuccess) return cuda_fail(e, "dl_step_host output download");
  h->set_used[j] = true;
  ++h->host_calls;
  return DL_OK;
}

int dl_eager_step(dl_t h, const void* q, const void* k, const void* v, const float* log_decay,
                  const float* beta, void* o, void* stream) {
  int rc = check_step_args(h, q, k, v, log_decay, beta, o);
  if (rc != DL_OK) return rc;
  if (h->n != 0) return fail(DL_ERR_STATE, "eager step needs every slot's log empty; call dl_merge");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaError_t e =
      launch_eager(h, step_args(h, q, k, v, log_decay, beta, o), h->B, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "eager step launch");
  h->wrote_state = true;
  return DL_OK;
}

int dl_eager_step_indexed(dl_t h, const int* slot_idx, int rows, const void* q, const void* k, const void* v,
                          const float* log_decay, const float* beta, void* o, void* stream) {
  int rc = check_slot_map(h, slot_idx, rows);
  if (rc != DL_OK) return rc;
  if (h->n != 0) return fail(DL_ERR_STATE, "eager step needs every slot's log empty; call dl_merge");
  if (rows == 0) return DL_OK;
  rc = check_step_args(h, q, k, v, log_decay, beta, o);
  if (rc != DL_OK) return rc;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  dl::StepArgs a = step_args(h, q, k, v, log_decay, beta, o);
  a.slot_idx = slot_idx;
  cudaError_t e = launch_eager(h, a, rows, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "eager step launch");
  h->wrote_state = true;
  return DL_OK;
}

int dl_merge(dl_t h, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (h->n == 0) return DL_OK;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaError_t e = launch_materialize(h, h->Sbar, static_cast<cudaStream_t>(stream), 0, static_cast<int>(bh(h)));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  h->n = 0;
  h->wrote_state = true;
  return DL_OK;
}

int dl_read_state(dl_t h, float* S_out, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (!S_out || !aligned(S_out, 16)) return fail(DL_ERR_ARG, "output pointer null or not 16-byte aligned");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = h->n == 0 ? cudaMemcpyAsync(S_out, h->Sbar, state_bytes(h), cudaMemcpyDeviceToDevice, s)
                            : launch_materialize(h, S_out, s, 0, static_cast<int>(bh(h)));
  return e == cudaSuccess ? DL_OK : cuda_fail(e, "dl_read_state");
}

int dl_slot_load(dl_t h, int slot, const float* S, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (slot < 0 || slot >= h->B) return fail(DL_ERR_ARG, "slot %d outside [0, %d)", slot, h->B);
  if (S && !aligned(S, 16)) return fail(DL_ERR_ARG, "state pointer not 16-byte aligned");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(h->H) * h->dk * h->dv * sizeof(float);
  float* dst = h->Sbar + static_cast<size_t>(slot) * h->H * h->dk * h->dv;
  cudaError_t e = S ? cudaMemcpyAsync(dst, S, bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(dst, 0, bytes, s);
  if (e == cudaSuccess && h->n > 0) e = zero_slot_log(h, slot, s);
  if (e != cudaSuccess) return cuda_fail(e, "dl_slot_load");
  h->wrote_state = true;
  return DL_OK;
}

int dl_slot_merge(dl_t h, int slot, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (slot < 0 || slot >= h->B) return fail(DL_ERR_ARG, "slot %d outside [0, %d)", slot, h->B);
  if (h->n == 0) return DL_OK;
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long unit0 = static_cast<long>(slot) * h->H;
  cudaError_t e = launch_materialize(h, h->Sbar + unit0 * h->dk * h->dv, s, unit0, h->H);
  if (e == cudaSuccess) e = zero_slot_log(h, slot, s);
  if (e != cudaSuccess) return cuda_fail(e, "dl_slot_merge");
  h->wrote_state = true;
  return DL_OK;
}

int dl_slot_read(dl_t h, int slot, float* S_out, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  if (slot < 0 || slot >= h->B) return fail(DL_ERR_ARG, "slot %d outside [0, %d)", slot, h->B);
  if (!S_out || !aligned(S_out, 16)) return fail(DL_ERR_ARG, "output pointer null or not 16-byte aligned");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long unit0 = static_cast<long>(slot) * h->H;
  cudaError_t e = h->n == 0 ? cudaMemcpyAsync(S_out, h->Sbar + unit0 * h->dk * h->dv,
                                           static_cast<size_t>(h->H) * h->dk * h->dv * sizeof(float),
                                           cudaMemcpyDeviceToDevice, s)
                            : launch_materialize(h, S_out, s, unit0, h->H);
  return e == cudaSuccess ? DL_OK : cuda_fail(e, "dl_slot_read");
}

int dl_set_option(dl_t h, int option, int value) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  switch (option) {
    case DL_OPT_STEP_KERNEL:
      if (value != DL_STEP_AUTO && value != DL_STEP_REGISTER) return fail(DL_ERR_ARG, "bad step-kernel value %d", value);
      h->step_kernel = value;
      return DL_OK;
    case DL_OPT_HOST_PREFETCH:
      if (value != 0 && value != 1) return fail(DL_ERR_ARG, "bad host-prefetch value %d", value);
      h->host_prefetch = value;
      return DL_OK;
    case DL_OPT_PDL:
      if (value != 0 && value != 1) return fail(DL_ERR_ARG, "bad PDL value %d", value);
      h->pdl = value;
      return DL_OK;
    case DL_OPT_PREFILL_KERNEL:
      if (value < DL_PREFILL_AUTO || value > DL_PREFILL_CHUNKED)
        return fail(DL_ERR_ARG, "bad prefill-kernel value %d", value);
      h->prefill_kernel = value;
      return DL_OK;
    case DL_OPT_LOG_B_BF16:
      if (value != 0 && value != 1) return fail(DL_ERR_ARG, "bad log-b-bf16 value %d", value);
      if (value && h->dtype != DL_BF16) return fail(DL_ERR_UNSUPPORTED, "a bf16 b-log needs bf16 inputs");
      if (value != h->log_b_bf16 && h->n != 0)
        return fail(DL_ERR_STATE, "change the b-log precision only with an empty log (call dl_merge)");
      h->log_b_bf16 = value;
      return DL_OK;
    case DL_OPT_LOG_LAM_F16:
      if (value != 0 && value != 1) return fail(DL_ERR_ARG, "bad log-lam-f16 value %d", value);
      if (value && h->dtype != DL_BF16) return fail(DL_ERR_UNSUPPORTED, "fp16 log-gates need bf16 inputs");
      if (value != h->log_lam_f16 && h->n != 0)
        return fail(DL_ERR_STATE, "change the snapshot precision only with an empty log (call dl_merge)");
      h->log_lam_f16 = value;
      return DL_OK;
    case DL_OPT_TEST_STALL_LOG:
      if (value != 0 && value != 1) return fail(DL_ERR_ARG, "bad stall-log value %d", value);
      h->stall_log = value;
      return DL_OK;
    case DL_OPT_VALUE_TILES:
      if (value != 0 && value != 1 && value != 2 && value != 4)
        return fail(DL_ERR_ARG, "bad value-tile count %d", value);
      h->value_tiles = value;
      return DL_OK;
    default:
      return fail(DL_ERR_ARG, "unknown option %d", option);
  }
}

int dl_last_step_kernel(dl_t h, int* kind) {
  if (!h || !kind) return fail(DL_ERR_ARG, "null argument");
  *kind = h->last_kernel;
  return DL_OK;
}

int dl_last_prefill_kernel(dl_t h, int* kind) {
  if (!h || !kind) return fail(DL_ERR_ARG, "null argument");
  *kind = h->last_prefill;
  return DL_OK;
}

int dl_log_len(dl_t h, int* n) {
  if (!h || !n) return fail(DL_ERR_ARG, "null argument");
  *n = h->n;
  return DL_OK;
}

int dl_check_device(dl_t h, void* stream) {
  if (!h) return fail(DL_ERR_ARG, "null handle");
  DeviceScope ds(h->device);
  if (!ds.ok()) return fail(DL_ERR_CUDA, "could not select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int flag = 0;
  take_error_word<<<1, 1, 0, s>>>(h->err);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, h->err + 1, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "dl_check_device");
  return flag ? fail(DL_ERR_DEVICE, "device error word 0x%x", flag) : DL_OK;
}

const char* dl_strerror(int status) {
  switch (status) {
    case DL_OK: return "ok";
    case DL_ERR_ARG: return "invalid argument";
    case DL_ERR_UNSUPPORTED: return "unsupported configuration";
    case DL_ERR_CUDA: return "CUDA error";
    case DL_ERR_OOM: return "out of memory";
    case DL_ERR_DEVICE: return "device-side error flag raised";
    case DL_ERR_STATE: return "call not valid in the current handle state";
    default: return "unknown status";
  }
}

const char* dl_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
