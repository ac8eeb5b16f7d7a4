// Diagnostic for the time-out path that every kernel of the library relies on, exercised
// without a fault and without a hang.  One thread initialises an mbarrier that expects one
// arrival and waits on its first phase with the library's bounded poll loop.  Nothing ever
// arrives, so the loop runs out and the kernel records TV_ERR_TIMEOUT on the workspace status
// word -- what a verify or commit CTA does after a wait that does not complete -- and
// returns, leaving the context usable.
#include "tc_ptx.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

__global__ void timeout_probe(int *ws, uint32_t polls) {
  __shared__ unsigned long long bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = ptx::smem_addr(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  if (!ptx::mbar_wait_bounded(b, 0, polls)) set_status(ws, TV_ERR_TIMEOUT, -1);
}

}  // namespace

cudaError_t launch_timeout_probe(int *ws, uint32_t polls, cudaStream_t st) {
  timeout_probe<<<1, 32, 0, st>>>(ws, polls);
  return cudaGetLastError();
}

}  // namespace tv
