// Instantiations of the prefill hand-off kernel (every operator, shape and
// input dtype) in a translation unit of their own.
#include "prefill.cuh"
#include "prefill_chunk.cuh"
#include "prefill_chunk_key.cuh"
#include "prefill_chunk_tc.cuh"

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

// Whole-head CTAs (VT = 128) for d_k = d_v = 128 once they cover at least
// half the SMs (rows x heads), 64-column tiles below that.  Measured on B200
// for the KDA kernel (H=32): whole-head CTAs 1.18x at B=64 L=512, 1.21x at
// B=4 L=4096, but 0.83x at B=1 L=8192 (32 CTAs).
inline bool whole_head_tiles(const LaunchShape& s) { return 2LL * s.units * s.H > s.sms; }

template <int DK, int DV, int VT>
cudaError_t launch_gdn_chunk_prefill(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = ChunkGeom<DK, VT>;
  auto kern = gdn_chunk_prefill_kernel<DK, DV, VT>;
  if (G::BYTES + G::NW * 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H * (DV / G::VT), s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gdn_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = TcChunkGeom;
  auto kern = gdn_chunk_prefill_tc_kernel<0>;
  if (G::BYTES + 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H, s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gdn_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_gdn_chunk_prefill<64, 64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128)
    return whole_head_tiles(s) ? launch_gdn_chunk_prefill_tc(s, a, st)
                               : launch_gdn_chunk_prefill<128, 128, 64>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_gdn_chunk_prefill<64, 128, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_gdn_chunk_prefill<128, 64, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template <int OP, int DK, int DV, int VT>
cudaError_t launch_key_chunk_prefill(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = KeyChunkGeom<DK, VT>;
  auto kern = key_chunk_prefill_kernel<OP, DK, DV, VT>;
  if (G::BYTES + G::NW * 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H * (DV / VT), s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

template <int OP>
cudaError_t launch_key_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = KeyTcChunkGeom;
  auto kern = key_chunk_prefill_tc_kernel<OP>;
  if (G::BYTES + 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H, s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

template <int OP>
cudaError_t launch_key_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_key_chunk_prefill<OP, 64, 64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128)
    return whole_head_tiles(s) ? launch_key_chunk_prefill_tc<OP>(s, a, st)
                               : launch_key_chunk_prefill<OP, 128, 128, 64>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_key_chunk_prefill<OP, 64, 128, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_key_chunk_prefill<OP, 128, 64, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template cudaError_t launch_key_chunk_prefill_dims<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_key_chunk_prefill_dims<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
