// tv_tree_verify_noalloc: tree verification for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they verify a tree: code running
// inside a custom allocator or memory pool callback (allocating there would re-enter it),
// serving loops that forbid allocation after start-up so that memory use stays fixed, and
// hosts that hand this library only pointers to buffers they own.  This entry point runs
// the same verification as tv_tree_verify but takes its device scratch (the status word
// that tv_tree_verify keeps in the caller's workspace) from a fixed array that lives in
// this library's device image, so the caller passes only inputs, outputs and a stream.
#include <mutex>

#include "tv_internal.cuh"

namespace {

// Device scratch shared by every call on a device; every GPU that loads the library holds
// it until the process exits.
constexpr size_t kStaticScratchBytes = 4096;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up (and zeroed) once
// per device.  In host code `g_static_scratch` names a host-side stand-in, not device
// memory, so the address must come from cudaGetSymbolAddress with the device current.
cudaError_t scratch_for_current_device(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemset(p, 0, kStaticScratchBytes);   // status word starts clear
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" tv_status tv_tree_verify_noalloc(const tv_problem *p, const void *q, const void *k,
                                            const void *v, const float *log_a, const float *b,
                                            const int32_t *parent, const int32_t *node_offsets,
                                            const float *S_root, void *out, float *U,
                                            void **scratch_out, tv_stream_t stream) {
  const size_t need = tv_workspace_size(p);
  if (need == 0)   // invalid or unsupported problem: tv_tree_verify names the reason
    return tv_tree_verify(p, q, k, v, log_a, b, parent, node_offsets, S_root, out, U, nullptr,
                          0, stream);
  if (need > kStaticScratchBytes) return TV_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return tv::record_cuda_error(e);   // readable via tv_last_cuda_error
  if (scratch_out) *scratch_out = scratch;
  return tv_tree_verify(p, q, k, v, log_a, b, parent, node_offsets, S_root, out, U, scratch,
                        kStaticScratchBytes, stream);
}
