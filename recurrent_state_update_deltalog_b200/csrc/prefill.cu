// Instantiations of the prefill hand-off kernel (every operator, shape and
// input dtype) in a translation unit of their own.
#include "prefill.cuh"

namespace dl {

template <int OP, int DK, int DV, typename TI>
cudaError_t prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  prefill_kernel<OP, DK, DV, TI><<<dim3(s.H * (DV / PrefillTile<DK>::CW), s.units), 32, 0, st>>>(a);
  return cudaGetLastError();
}

template <int OP>
cudaError_t launch_prefill_op(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  DL_DISPATCH_DIMS(prefill_dims, s, a, st);
}

template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
