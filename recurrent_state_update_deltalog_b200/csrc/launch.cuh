// Host-side launchers: shape/dtype dispatch onto the kernel templates.
// Each operator's instantiations live in their own translation unit
// (step_gdn.cu, step_kda.cu, step_rwkv6.cu) so they compile in parallel.
#pragma once

#include "kernels.cuh"

namespace dl {

struct LaunchShape {
  int BH;     // slots x heads = grid size
  int dk;
  int dv;
  int dtype;  // 0 = fp32, 1 = bf16 inputs
};

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

template <int OP, int DK, int DV, typename TI>
cudaError_t step_dims(const LaunchShape& s, bool merge, const StepArgs& a, cudaStream_t st) {
  using TL = Tile<DK, DV>;
  using LL = LogLayout<OP, DK, DV, TI>;
  const size_t smem = LL::step_smem(a.n, merge);
  if (merge) {
    auto kern = deltalog_step_kernel<OP, DK, DV, TI, true>;
    cudaError_t e = allow_smem(kern, smem, LL::step_smem(kMaxM - 1, true));
    if (e != cudaSuccess) return e;
    kern<<<s.BH, TL::NT, smem, st>>>(a);
  } else {
    auto kern = deltalog_step_kernel<OP, DK, DV, TI, false>;
    cudaError_t e = allow_smem(kern, smem, LL::step_smem(kMaxM - 1, false));
    if (e != cudaSuccess) return e;
    kern<<<s.BH, TL::NT, smem, st>>>(a);
  }
  return cudaGetLastError();
}

template <int OP, int DK, int DV, typename TI>
cudaError_t eager_dims(const LaunchShape& s, const StepArgs& a, cudaStream_t st) {
  eager_step_kernel<OP, DK, DV, TI><<<s.BH, Tile<DK, DV>::NT, 0, st>>>(a);
  return cudaGetLastError();
}

template <int OP, int DK, int DV, typename TI>
cudaError_t materialize_dims(const LaunchShape& s, const MaterializeArgs& a, cudaStream_t st) {
  using LL = LogLayout<OP, DK, DV, TI>;
  auto kern = materialize_kernel<OP, DK, DV, TI>;
  const size_t smem = LL::materialize_smem(a.n);
  cudaError_t e = allow_smem(kern, smem, LL::materialize_smem(kMaxM - 1));
  if (e != cudaSuccess) return e;
  kern<<<s.BH, Tile<DK, DV>::NT, smem, st>>>(a);
  return cudaGetLastError();
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
cudaError_t launch_step_op(const LaunchShape& s, bool merge, const StepArgs& a, cudaStream_t st) {
  DL_DISPATCH_DIMS(step_dims, s, merge, a, st);
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
  extern template cudaError_t launch_step_op<OPV>(const LaunchShape&, bool, const StepArgs&, cudaStream_t); \
  extern template cudaError_t launch_eager_op<OPV>(const LaunchShape&, const StepArgs&, cudaStream_t);      \
  extern template cudaError_t launch_materialize_op<OPV>(const LaunchShape&, const MaterializeArgs&, cudaStream_t);

#define DL_INSTANTIATE_OP(OPV)                                                                  \
  template cudaError_t launch_step_op<OPV>(const LaunchShape&, bool, const StepArgs&, cudaStream_t); \
  template cudaError_t launch_eager_op<OPV>(const LaunchShape&, const StepArgs&, cudaStream_t);      \
  template cudaError_t launch_materialize_op<OPV>(const LaunchShape&, const MaterializeArgs&, cudaStream_t);

DL_DECLARE_OP(OP_GDN)
DL_DECLARE_OP(OP_KDA)
DL_DECLARE_OP(OP_RWKV6)

}  // namespace dl
