// Host-side launchers: shape/dtype dispatch onto the kernel templates.
// Each operator's instantiations live in their own translation unit
// (step_gdn.cu, step_kda.cu, step_rwkv6.cu) so they compile in parallel.
#pragma once

#include "kernels.cuh"

namespace dl {

// Step-kernel variants (dl_set_option DL_OPT_STEP_KERNEL).
enum { STEP_AUTO = 0, STEP_REGISTER = 1 };

struct LaunchShape {
  int BH;     // launched (slot or batch row) x heads
  int H;      // heads
  int dk;
  int dv;
  int dtype;  // 0 = fp32, 1 = bf16 inputs
  // device limits, queried once per handle
  int sms;
  int smem_block_optin;
  int smem_sm;
  int smem_reserved;
  int variant;     // STEP_*
  bool pdl;        // launch the step as a programmatic dependent of the previous kernel
  int split;       // value tiles per head for the register-tile step kernel (1, 2 or 4)
  int max_n;       // log length of the launched units (shared-memory sizing)
  int units;       // materialisation: units in the launch
  bool blow;       // GDN/KDA b_i stored in bf16 (bf16-input handles only)
  bool lamc;       // KDA/RWKV6 snapshots stored as fp16 log-gates (bf16-input handles only)
};

// Launch with the programmatic-stream-serialisation attribute when `pdl`.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(void (*kern)(KArgs...), dim3 grid, int block, size_t smem, cudaStream_t st, bool pdl,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Opt a kernel into more than the default 48 KB of shared memory (static +
// dynamic) when a launch needs it; `worst` is the largest dynamic size any
// launch of this kernel can ask for.
template <typename K>
cudaError_t allow_smem(K kern, size_t smem, size_t worst) {
  if (smem <= 16 * 1024) return cudaSuccess;  // every kernel's static part is < 32 KB
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.sharedSizeBytes + smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(worst));
}

// Grid of a step kernel: unmapped B * H * NSPLIT CTAs; mapped (H * NSPLIT, rows).
template <int NSPLIT, bool MAP>
dim3 step_grid(const LaunchShape& s) {
  if (MAP) return dim3(s.H * NSPLIT, s.BH / s.H);
  return dim3(s.BH * NSPLIT);
}

template <int OP, int DK, int DV, typename TI, int MODE, int NSPLIT, bool MAP, bool BLOW, bool LAMC>
cudaError_t register_step_mode(const LaunchShape& s, const StepArgs& a, cudaStream_t st) {
  using TL = Tile<DK, DV / NSPLIT>;
  using LL = LogLayout<OP, DK, DV, TI, BLOW, LAMC>;
  const size_t smem = LL::step_smem(a.n, MODE == MODE_MERGE);
  auto kern = deltalog_step_kernel<OP, DK, DV, TI, MODE, NSPLIT, MAP, BLOW, LAMC>;
  cudaError_t e = allow_smem(kern, smem, LL::step_smem(kMaxM - 1, MODE != MODE_APPEND));
  if (e != cudaSuccess) return e;
  return launch_maybe_pdl(kern, step_grid<NSPLIT, MAP>(s), TL::NT, smem, st, s.pdl, a);
}

template <int OP, int DK, int DV, typename TI, int NSPLIT, bool BLOW, bool LAMC>
cudaError_t register_step_log(const LaunchShape& s, int mode, const StepArgs& a, cudaStream_t st) {
  if (a.slot_idx) {
    if (mode == MODE_MERGE) return register_step_mode<OP, DK, DV, TI, MODE_MERGE, NSPLIT, true, BLOW, LAMC>(s, a, st);
    return register_step_mode<OP, DK, DV, TI, MODE_APPEND, NSPLIT, true, BLOW, LAMC>(s, a, st);
  }
  if (mode == MODE_MERGE) return register_step_mode<OP, DK, DV, TI, MODE_MERGE, NSPLIT, false, BLOW, LAMC>(s, a, st);
  return register_step_mode<OP, DK, DV, TI, MODE_APPEND, NSPLIT, false, BLOW, LAMC>(s, a, st);
}

// A bf16 b-log exists for bf16-input GDN/KDA handles, compact fp16
// snapshots for bf16-input KDA/RWKV6 handles; other instantiations are never
// built.
template <int OP, typename TI>
constexpr bool kHasBlow = OP != OP_RWKV6 && std::is_same<TI, __nv_bfloat16>::value;
template <int OP, typename TI>
constexpr bool kHasLamc = OP != OP_GDN && std::is_same<TI, __nv_bfloat16>::value;

// Calls FN<BLOW, LAMC>() for the handle's log storage.
template <int OP, typename TI, typename FN>
cudaError_t with_log_kind(const LaunchShape& s, FN fn) {
  if constexpr (kHasLamc<OP, TI>) {
    if (s.lamc) {
      if constexpr (kHasBlow<OP, TI>) {
        if (s.blow) return fn(std::true_type{}, std::true_type{});
      }
      return fn(std::false_type{}, std::true_type{});
    }
  }
  if constexpr (kHasBlow<OP, TI>) {
    if (s.blow) return fn(std::true_type{}, std::false_type{});
  }
  return fn(std::false_type{}, std::false_type{});
}

template <int OP, int DK, int DV, typename TI, int NSPLIT>
cudaError_t register_step(const LaunchShape& s, int mode, const StepArgs& a, cudaStream_t st) {
  return with_log_kind<OP, TI>(s, [&](auto blow, auto lamc) {
    return register_step_log<OP, DK, DV, TI, NSPLIT, decltype(blow)::value, decltype(lamc)::value>(s, mode, a, st);
  });
}

template <int OP, int DK, int DV, typename TI>
cudaError_t step_dims(const LaunchShape& s, int mode, const StepArgs& a, cudaStream_t st, int* used) {
  *used = STEP_REGISTER;
  if constexpr (DV >= 128) {
    if (s.split == 4) return register_step<OP, DK, DV, TI, 4>(s, mode, a, st);
  }
  if constexpr (DV >= 64) {
    if (s.split == 2) return register_step<OP, DK, DV, TI, 2>(s, mode, a, st);
  }
  return register_step<OP, DK, DV, TI, 1>(s, mode, a, st);
}

template <int OP, int DK, int DV, typename TI, bool MAP>
cudaError_t eager_map(const LaunchShape& s, const StepArgs& a, cudaStream_t st) {
  if constexpr (DV >= 64) {
    if (s.split == 2) {
      eager_step_kernel<OP, DK, DV, TI, 2, MAP><<<step_grid<2, MAP>(s), Tile<DK, DV / 2>::NT, 0, st>>>(a);
      return cudaGetLastError();
    }
  }
  eager_step_kernel<OP, DK, DV, TI, 1, MAP><<<step_grid<1, MAP>(s), Tile<DK, DV>::NT, 0, st>>>(a);
  return cudaGetLastError();
}

template <int OP, int DK, int DV, typename TI>
cudaError_t eager_dims(const LaunchShape& s, const StepArgs& a, cudaStream_t st) {
  return a.slot_idx ? eager_map<OP, DK, DV, TI, true>(s, a, st) : eager_map<OP, DK, DV, TI, false>(s, a, st);
}

template <int OP, int DK, int DV, typename TI, bool BLOW, bool LAMC>
cudaError_t materialize_log(const LaunchShape& s, const MaterializeArgs& a, cudaStream_t st) {
  using LL = LogLayout<OP, DK, DV, TI, BLOW, LAMC>;
  auto kern = materialize_kernel<OP, DK, DV, TI, BLOW, LAMC>;
  const size_t smem = LL::materialize_smem(s.max_n);
  cudaError_t e = allow_smem(kern, smem, LL::materialize_smem(kMaxM - 1));
  if (e != cudaSuccess) return e;
  const dim3 grid = a.slot_idx ? dim3(s.H, s.units) : dim3(s.units);  // mapped: (heads, rows)
  kern<<<grid, Tile<DK, DV>::NT, smem, st>>>(a);
  return cudaGetLastError();
}

template <int OP, int DK, int DV, typename TI>
cudaError_t materialize_dims(const LaunchShape& s, const MaterializeArgs& a, cudaStream_t st) {
  return with_log_kind<OP, TI>(s, [&](auto blow, auto lamc) {
    return materialize_log<OP, DK, DV, TI, decltype(blow)::value, decltype(lamc)::value>(s, a, st);
  });
}

#define DL_DISPATCH_DIMS(FN, ...)                                                          \
  do {                                                                                     \
    if (s.dk == 64 && s.dv == 64)                                                          \
      return s.dtype ? FN<OP, 64, 64, __nv_bfloat16>(__VA_ARGS__) : FN<OP, 64, 64, float>(__VA_ARGS__);     \
    if (s.dk == 128 && s.dv == 128)                                                        \
      return s.dtype ? FN<OP, 128, 128, __nv_bfloat16>(__VA_ARGS__) : FN<OP, 128, 128, float>(__VA_ARGS__); \
    if (s.dk == 64 && s.dv == 128)                                                         \
      return s.dtype ? FN<OP, 64, 128, __nv_bfloat16>(__VA_ARGS__) : FN<OP, 64, 128, float>(__VA_ARGS__);   \
    if (s.dk == 128 && s.dv == 64)                                                         \
      return s.dtype ? FN<OP, 128, 64, __nv_bfloat16>(__VA_ARGS__) : FN<OP, 128, 64, float>(__VA_ARGS__);   \
    return cudaErrorInvalidValue;                                                          \
  } while (0)

template <int OP>
cudaError_t launch_step_op(const LaunchShape& s, int mode, const StepArgs& a, cudaStream_t st, int* used) {
  DL_DISPATCH_DIMS(step_dims, s, mode, a, st, used);
}

template <int OP>
cudaError_t launch_eager_op(const LaunchShape& s, const StepArgs& a, cudaStream_t st) {
  DL_DISPATCH_DIMS(eager_dims, s, a, st);
}

template <int OP>
cudaError_t launch_materialize_op(const LaunchShape& s, const MaterializeArgs& a, cudaStream_t st) {
  DL_DISPATCH_DIMS(materialize_dims, s, a, st);
}

#define DL_DECLARE_OP(OPV)                                                                      \
  extern template cudaError_t launch_step_op<OPV>(const LaunchShape&, int, const StepArgs&, cudaStream_t, int*); \
  extern template cudaError_t launch_eager_op<OPV>(const LaunchShape&, const StepArgs&, cudaStream_t);      \
  extern template cudaError_t launch_materialize_op<OPV>(const LaunchShape&, const MaterializeArgs&, cudaStream_t);

#define DL_INSTANTIATE_OP(OPV)                                                                  \
  template cudaError_t launch_step_op<OPV>(const LaunchShape&, int, const StepArgs&, cudaStream_t, int*); \
  template cudaError_t launch_eager_op<OPV>(const LaunchShape&, const StepArgs&, cudaStream_t);      \
  template cudaError_t launch_materialize_op<OPV>(const LaunchShape&, const MaterializeArgs&, cudaStream_t);

DL_DECLARE_OP(OP_GDN)
DL_DECLARE_OP(OP_KDA)
DL_DECLARE_OP(OP_RWKV6)

}  // namespace dl
