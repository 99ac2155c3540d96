// Instantiations of the prefill hand-off kernel (every operator, shape and
// input dtype) in a translation unit of their own.
#include "prefill.cuh"
#include "prefill_chunk.cuh"
#include "prefill_chunk_key.cuh"

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

template <int DK, int DV>
cudaError_t launch_gdn_chunk_prefill(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = ChunkGeom<DK>;
  auto kern = gdn_chunk_prefill_kernel<DK, DV>;
  if (G::BYTES + 8 * 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H * (DV / G::VT), s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gdn_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_gdn_chunk_prefill<64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128) return launch_gdn_chunk_prefill<128, 128>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_gdn_chunk_prefill<64, 128>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_gdn_chunk_prefill<128, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template <int OP, int DK, int DV>
cudaError_t launch_key_chunk_prefill(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = KeyChunkGeom<DK>;
  auto kern = key_chunk_prefill_kernel<OP, DK, DV>;
  if (G::BYTES + 8 * 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H * (DV / G::VT), s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

template <int OP>
cudaError_t launch_key_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_key_chunk_prefill<OP, 64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128) return launch_key_chunk_prefill<OP, 128, 128>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_key_chunk_prefill<OP, 64, 128>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_key_chunk_prefill<OP, 128, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template cudaError_t launch_key_chunk_prefill_dims<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_key_chunk_prefill_dims<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
