// dl_decode_static: DeltaLog decode over a caller's dense state with the log
// in a fixed device array of this library, for callers that cannot allocate
// device memory.  The contract is documented in include/deltalog.h.
//
// The step and materialisation kernels are the library's own; only where
// their log lives differs.  A handle (dl_create) allocates its log with
// cudaMalloc; here the log and the error word sit in `dl_static_scratch`, a
// file-scope __device__ array that every device which loads the library holds
// until the process exits.  Host code never names the array as an address:
// its symbol on the host is only a stand-in, so each device's address is
// looked up once with cudaGetSymbolAddress (with that device current) and
// passed to the kernels.
#include "deltalog.h"
#include "launch.cuh"

#include <atomic>
#include <cstdio>
#include <mutex>

namespace dl {
int record_error(int code, const char* msg);   // api.cu: dl_last_error's message
}  // namespace dl

namespace {

static_assert(DL_STATIC_SCRATCH_BYTES % 256 == 0, "scratch regions are 256-byte aligned");

static __device__ __align__(256) unsigned char dl_static_scratch[DL_STATIC_SCRATCH_BYTES];

constexpr size_t kErrRegion = 256;   // the error word, then padding to the first log region
constexpr int kMaxDevices = 64;

struct DeviceSetup {
  unsigned char* scratch;   // device address of dl_static_scratch on this device
  int sms, smem_block_optin, smem_sm, smem_reserved;
};

std::atomic<bool> g_ready[kMaxDevices];
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mutex;

int fail(int code, const char* msg) { return dl::record_error(code, msg); }

// Once per device, with that device current: the array's device address and
// the limits the launchers size their grids and shared memory by.
int device_setup(int dev, DeviceSetup* out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(DL_ERR_UNSUPPORTED, "device ordinal beyond 63");
  if (!g_ready[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_ready[dev].load(std::memory_order_relaxed)) {
      DeviceSetup s{};
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, dl_static_scratch);
      if (e != cudaSuccess || !p) {
        cudaGetLastError();
        return fail(DL_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
      }
      s.scratch = static_cast<unsigned char*>(p);
      const struct {
        int* dst;
        cudaDeviceAttr attr;
      } q[] = {{&s.sms, cudaDevAttrMultiProcessorCount},
               {&s.smem_block_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin},
               {&s.smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor},
               {&s.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock}};
      for (auto& x : q)
        if (cudaDeviceGetAttribute(x.dst, x.attr, dev) != cudaSuccess) {
          cudaGetLastError();
          return fail(DL_ERR_CUDA, "device attribute query failed");
        }
      g_setup[dev] = s;
      g_ready[dev].store(true, std::memory_order_release);
    }
  }
  *out = g_setup[dev];
  return DL_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" int dl_decode_static(int op, int B, int H, int d_k, int d_v, int M, int in_dtype, float* S,
                                const float* u, int T, const void* q, const void* k, const void* v,
                                const float* log_decay, const float* beta, void* o, int* dev_err,
                                void* stream) {
  if (op < DL_GDN || op > DL_RWKV6) return fail(DL_ERR_ARG, "unknown op");
  if (in_dtype != DL_F32 && in_dtype != DL_BF16) return fail(DL_ERR_ARG, "unknown dtype");
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128))
    return fail(DL_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128");
  if (M < 1 || M > DL_MAX_M) return fail(DL_ERR_UNSUPPORTED, "M outside [1, DL_MAX_M]");
  if (B <= 0 || H <= 0 || T < 0) return fail(DL_ERR_ARG, "B and H must be positive and T not negative");
  if (!S || !aligned(S, 16)) return fail(DL_ERR_ARG, "state pointer null or not 16-byte aligned");
  if (op == DL_RWKV6 && (!u || !aligned(u, 4))) return fail(DL_ERR_ARG, "RWKV6 needs the bonus u");
  if (dev_err && !aligned(dev_err, 4)) return fail(DL_ERR_ARG, "error word not 4-byte aligned");

  // Scratch plan: the error word, then the log regions of every (slot, head).
  const size_t units = static_cast<size_t>(B) * H;
  if (units > (size_t(1) << 30)) return fail(DL_ERR_ARG, "B*H too large");
  const size_t es = in_dtype == DL_BF16 ? 2 : 4;
  const int Mcap = M > 1 ? M - 1 : 1;
  const size_t b_es = op == DL_RWKV6 ? es : 4;
  const size_t lam_unit = op == DL_GDN ? static_cast<size_t>(dl::gdn_lam_stride(Mcap)) : static_cast<size_t>(Mcap) * d_k;
  const size_t a_bytes = round256(units * Mcap * d_k * es);
  const size_t b_bytes = round256(units * Mcap * d_v * b_es);
  const size_t l_bytes = round256(units * lam_unit * sizeof(float));
  const size_t need = kErrRegion + a_bytes + b_bytes + l_bytes;
  if (need > DL_STATIC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "the log of B*H = %zu units at M = %d needs %zu bytes; the static scratch holds %u "
             "(split the batch over calls, take a smaller M, or use a handle)",
             units, M, need, static_cast<unsigned>(DL_STATIC_SCRATCH_BYTES));
    return fail(DL_ERR_ARG, buf);
  }
  if (T == 0) return DL_OK;
  if (!q || !k || !v || !log_decay || !o) return fail(DL_ERR_ARG, "null input/output pointer");
  if (op == DL_RWKV6 && beta) return fail(DL_ERR_ARG, "beta must be NULL for RWKV6");
  if (op != DL_RWKV6 && !beta) return fail(DL_ERR_ARG, "beta is required for GDN/KDA");
  const void* tp[] = {q, k, v, o};
  for (const void* p : tp)
    if (!aligned(p, es)) return fail(DL_ERR_ARG, "input/output pointer not aligned to its element size");
  if (!aligned(log_decay, 4) || (beta && !aligned(beta, 4))) return fail(DL_ERR_ARG, "gate pointer not 4-byte aligned");

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(DL_ERR_CUDA, "no current CUDA device");
  }
  DeviceSetup ds;
  int rc = device_setup(dev, &ds);
  if (rc != DL_OK) return rc;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* base = ds.scratch;
  int* err = dev_err ? dev_err : reinterpret_cast<int*>(base);
  // Only the error word must start at zero: every log entry is written by an
  // append of this call before any later step of the call reads it.
  if (!dev_err) {
    cudaError_t e = cudaMemsetAsync(base, 0, sizeof(int), st);
    if (e != cudaSuccess) return fail(DL_ERR_CUDA, "clearing the scratch error word failed");
  }

  dl::LaunchShape sh{};
  sh.BH = static_cast<int>(units);
  sh.H = H;
  sh.dk = d_k;
  sh.dv = d_v;
  sh.dtype = in_dtype == DL_BF16 ? 1 : 0;
  sh.sms = ds.sms;
  sh.smem_block_optin = ds.smem_block_optin;
  sh.smem_sm = ds.smem_sm;
  sh.smem_reserved = ds.smem_reserved;
  sh.variant = dl::STEP_REGISTER;
  sh.units = sh.BH;
  sh.blow = false;

  dl::StepArgs a{};
  a.Sbar = S;
  a.slot_idx = nullptr;
  a.slots = B;
  a.logA = base + kErrRegion;
  a.logB = base + kErrRegion + a_bytes;
  a.logLam = reinterpret_cast<float*>(base + kErrRegion + a_bytes + b_bytes);
  a.u = u;
  a.err = err;
  a.H = H;
  a.M = M;
  a.Mcap = Mcap;

  const size_t qk_tok = units * d_k * es, v_tok = units * d_v * es;
  const size_t ld_tok = (op == DL_GDN ? units : units * d_k) * sizeof(float);
  int n = 0;
  for (int t = 0; t < T; ++t) {
    const bool merge = n + 1 == M;
    a.q = static_cast<const char*>(q) + t * qk_tok;
    a.k = static_cast<const char*>(k) + t * qk_tok;
    a.v = static_cast<const char*>(v) + t * v_tok;
    a.log_decay = reinterpret_cast<const float*>(reinterpret_cast<const char*>(log_decay) + t * ld_tok);
    a.beta = beta ? beta + t * units : nullptr;
    a.o = static_cast<char*>(o) + t * v_tok;
    a.n = n;
    // The first step of a call may follow a caller's kernel that wrote S, so
    // only steps after an append of this call are programmatic dependents.
    sh.pdl = n > 0;
    sh.split = d_v == 128 && n < 16 && sh.BH >= 2 * ds.sms ? 2 : 1;
    sh.max_n = n;
    int used = 0;
    cudaError_t e;
    switch (op) {
      case DL_GDN: e = dl::launch_step_op<dl::OP_GDN>(sh, merge ? dl::MODE_MERGE : dl::MODE_APPEND, a, st, &used); break;
      case DL_KDA: e = dl::launch_step_op<dl::OP_KDA>(sh, merge ? dl::MODE_MERGE : dl::MODE_APPEND, a, st, &used); break;
      default: e = dl::launch_step_op<dl::OP_RWKV6>(sh, merge ? dl::MODE_MERGE : dl::MODE_APPEND, a, st, &used); break;
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(DL_ERR_CUDA, "step launch failed");
    }
    n = merge ? 0 : n + 1;
  }
  if (n > 0) {   // fold the remaining entries into S in place
    dl::MaterializeArgs ma{};
    ma.Sin = S;
    ma.Sout = S;
    ma.logA = a.logA;
    ma.logB = a.logB;
    ma.logLam = a.logLam;
    ma.err = err;
    ma.unit0 = 0;
    ma.slot_idx = nullptr;
    ma.slots = B;
    ma.H = H;
    ma.Mcap = Mcap;
    ma.n = n;
    sh.max_n = n;
    cudaError_t e;
    switch (op) {
      case DL_GDN: e = dl::launch_materialize_op<dl::OP_GDN>(sh, ma, st); break;
      case DL_KDA: e = dl::launch_materialize_op<dl::OP_KDA>(sh, ma, st); break;
      default: e = dl::launch_materialize_op<dl::OP_RWKV6>(sh, ma, st); break;
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(DL_ERR_CUDA, "log fold launch failed");
    }
  }
  return DL_OK;
}
