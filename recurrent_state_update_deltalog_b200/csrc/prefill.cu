// Instantiations of the prefill hand-off kernel (every operator, shape and
// input dtype) in a translation unit of their own.
#include "prefill.cuh"
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

template <int NT, int DK, int DV>
cudaError_t launch_gdn_chunk_prefill_tc_nt(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = TcChunkGeom<NT, DK, DV>;
  auto kern = gdn_chunk_prefill_tc_kernel<NT, DK, DV>;
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
template <int DK, int DV>
cudaError_t launch_gdn_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  return static_cast<long long>(s.units) * s.H > s.sms ? launch_gdn_chunk_prefill_tc_nt<256, DK, DV>(s, a, st)
                                                        : launch_gdn_chunk_prefill_tc_nt<512, DK, DV>(s, a, st);
}

// Every head shape runs with its state in tensor memory (a d_v = 64 head on
// the lower 64 of the 128 lanes).  Measured on B200 against the warp-MMA
// kernel (64-column tiles, or 512-thread whole-head tiles), d_k = d_v = 128,
// H = 32: 2.06x at B=64 L=512 and B=4 L=4096, and 1.55x at B=1 where it
// launches half the CTAs.
cudaError_t launch_gdn_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_gdn_chunk_prefill_tc<64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128) return launch_gdn_chunk_prefill_tc<128, 128>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_gdn_chunk_prefill_tc<64, 128>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_gdn_chunk_prefill_tc<128, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template <int OP, int NT, int DK, int DV>
cudaError_t launch_key_chunk_prefill_tc_nt(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  using G = KeyTcChunkGeom<NT, DK, DV>;
  auto kern = key_chunk_prefill_tc_kernel<OP, NT, DK, DV>;
  if (G::BYTES + 1024 > static_cast<size_t>(s.smem_block_optin)) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::BYTES));
  if (e != cudaSuccess) return e;
  kern<<<dim3(s.H, s.units), G::NT, G::BYTES, st>>>(a);
  return cudaGetLastError();
}

// Two 256-thread CTAs per SM once the launch has more CTAs than SMs, as for GDN.
template <int OP, int DK, int DV>
cudaError_t launch_key_chunk_prefill_tc(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  return static_cast<long long>(s.units) * s.H > s.sms ? launch_key_chunk_prefill_tc_nt<OP, 256, DK, DV>(s, a, st)
                                                        : launch_key_chunk_prefill_tc_nt<OP, 512, DK, DV>(s, a, st);
}

// Every head shape with the state in tensor memory, as for GDN (KDA, H = 32,
// d = 128: 1.68x the warp-MMA kernel at B=64 L=512, 1.40x at B=1 L=8192).
template <int OP>
cudaError_t launch_key_chunk_prefill_dims(const LaunchShape& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.dk == 64 && s.dv == 64) return launch_key_chunk_prefill_tc<OP, 64, 64>(s, a, st);
  if (s.dk == 128 && s.dv == 128) return launch_key_chunk_prefill_tc<OP, 128, 128>(s, a, st);
  if (s.dk == 64 && s.dv == 128) return launch_key_chunk_prefill_tc<OP, 64, 128>(s, a, st);
  if (s.dk == 128 && s.dv == 64) return launch_key_chunk_prefill_tc<OP, 128, 64>(s, a, st);
  return cudaErrorInvalidValue;
}

template cudaError_t launch_key_chunk_prefill_dims<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_key_chunk_prefill_dims<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

template cudaError_t launch_prefill_op<OP_GDN>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_KDA>(const LaunchShape&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill_op<OP_RWKV6>(const LaunchShape&, const PrefillArgs&, cudaStream_t);

}  // namespace dl
