// CUDA-core tree verification: any dk, dv in {16, ..., 128}, fp32 or bf16 inputs, scalar
// decay or gated delta rule, up to 256 nodes per tree.  One CTA of 128 threads per
// (sequence, head); the per-item algorithm is in simt_item.cuh.
#include "simt_item.cuh"

namespace tv {
namespace {

constexpr int kThreads = 128;

template <typename Tin, typename Tout, bool kGdn>
__global__ void __launch_bounds__(kThreads) verify_simt_kernel(VerifyArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  simt_item<Tin, Tout, kGdn, kThreads>(a, blockIdx.x / a.H, blockIdx.x % a.H, smem_raw);
}

template <typename Tin, typename Tout, bool kGdn>
cudaError_t launch_simt_t(const VerifyArgs &a, cudaStream_t st) {
  const size_t smem = simt_smem_bytes(a.dk, a.dv);
  auto kern = verify_simt_kernel<Tin, Tout, kGdn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.B * a.H, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_verify_simt(const VerifyArgs &a, int mode, int in_dtype, int out_dtype,
                               cudaStream_t st) {
  const bool gdn = mode == TV_MODE_GDN;
  if (in_dtype == TV_F32)
    return gdn ? launch_simt_t<float, float, true>(a, st) : launch_simt_t<float, float, false>(a, st);
  if (out_dtype == TV_BF16)
    return gdn ? launch_simt_t<__nv_bfloat16, __nv_bfloat16, true>(a, st)
               : launch_simt_t<__nv_bfloat16, __nv_bfloat16, false>(a, st);
  return gdn ? launch_simt_t<__nv_bfloat16, float, true>(a, st)
             : launch_simt_t<__nv_bfloat16, float, false>(a, st);
}

}  // namespace tv
