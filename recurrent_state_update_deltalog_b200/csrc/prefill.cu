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

template <int NT>
cudaError_t launch_gdn_chunk_prefill_tc_nt(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = TcChunkGeom<NT>;
  auto kern = gdn_chunk_prefill_tc_kernel<NT>;
  if (G::BYTES + 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H, s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

// Two 256-thread CTAs per SM once the launch has more CTAs (rows x heads) than
// SMs; one 512-thread CTA per SM below that.  Measured on B200, GDN H=32:
// 256 threads 1.33x at B=64 L=512 and 1.41x at B=512 L=32, but 0.84x at
// B=4 L=4096 (128 CTAs) and 0.85x at B=1.
cudaError_t launch_gdn_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  return static_cast<long long>(s.units) * s.H > s.sms ? launch_gdn_chunk_prefill_tc_nt<256>(s, a, st)
                                                        : launch_gdn_chunk_prefill_tc_nt<512>(s, a, st);
}

cudaError_t launch_gdn_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_gdn_chunk_prefill<64, 64, 64>(s, a, st);
  // d_k = d_v = 128: whole heads with the state in tensor memory.  Measured on
  // B200 against the warp-MMA kernel (64-column tiles, or 512-thread whole-head
  // tiles), H = 32: 2.06x at B=64 L=512 and B=4 L=4096, and 1.55x at B=1 where
  // it launches half the CTAs.
  if (s.dk == 128 && s.dv == 128) return launch_gdn_chunk_prefill_tc(s, a, st);
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

template <int OP, int NT>
cudaError_t launch_key_chunk_prefill_tc_nt(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = KeyTcChunkGeom<NT>;
  auto kern = key_chunk_prefill_tc_kernel<OP, NT>;
  if (G::BYTES + 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H, s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

// Two 256-thread CTAs per SM once the launch has more CTAs than SMs, as for GDN.
template <int OP>
cudaError_t launch_key_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  return static_cast<long long>(s.units) * s.H > s.sms ? launch_key_chunk_prefill_tc_nt<OP, 256>(s, a, st)
                                                        : launch_key_chunk_prefill_tc_nt<OP, 512>(s, a, st);
}

template <int OP>
cudaError_t launch_key_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_key_chunk_prefill<OP, 64, 64, 64>(s, a, st);
  // d_k = d_v = 128: whole heads with the state in tensor memory (KDA, H = 32:
  // 1.68x the warp-MMA kernel at B=64 L=512, 1.40x at B=1 L=8192)
  if (s.dk == 128 && s.dv == 128) return launch_key_chunk_prefill_tc<OP>(s, a, st);
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
