// Tree metadata: parent array -> depth, strict-ancestor bitmask, cumulative path log-decay.
//
// The Bole summary's worked example weights a node's path terms by powers of lambda set
// by depth (lambda^2 S_root for the depth-2 node a2); with per-token gates the power
// becomes the cumulative log-decay cl_n = sum of log_a over the root->n path.  The
// verify and commit kernels recompute these in shared memory; this kernel exports them
// (one CTA per sequence) so that they can be checked bit for bit and cached by callers.
// cl is accumulated in fp32 from the root down, cl_n = cl_parent + log_a_n, which is the
// exact rounding sequence the other kernels use.
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) meta_kernel(MetaArgs a) {
  __shared__ int par[kMaxNodes];
  __shared__ int dep[kMaxNodes];
  __shared__ int flag, maxdep;
  const int tid = threadIdx.x, s = blockIdx.x, H = a.H;
  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n_nodes = hi - lo;
  if (tid == 0) { flag = 0; maxdep = 0; }
  __syncthreads();
  for (int i = tid; i < n_nodes; i += kThreads) {
    const int p = a.parent[lo + i];
    if (p < -1 || p >= i) flag = 1;
    par[i] = p;
  }
  __syncthreads();
  if (flag) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  for (int i = tid; i < n_nodes; i += kThreads) {
    unsigned long long words[kAncWords] = {0ull, 0ull, 0ull, 0ull};
    int d = 1;
    for (int x = par[i]; x >= 0; x = par[x]) {
#pragma unroll
      for (int w = 0; w < kAncWords; ++w)
        if ((x >> 6) == w) words[w] |= 1ull << (x & 63);
      ++d;
    }
    dep[i] = d;
    a.depth[lo + i] = d;
    atomicMax(&maxdep, d);
#pragma unroll
    for (int w = 0; w < kAncWords; ++w)
      if (w < a.anc_words) a.anc[(size_t)(lo + i) * a.anc_words + w] = words[w];
  }
  __syncthreads();
  // cl for every (node, head), level by level from the root (parents are final first)
  for (int lvl = 1; lvl <= maxdep; ++lvl) {
    for (int e = tid; e < n_nodes * H; e += kThreads) {
      const int i = e / H, h = e % H;
      if (dep[i] == lvl) {
        const float up = par[i] < 0 ? 0.f : a.cumlog[(size_t)(lo + par[i]) * H + h];
        a.cumlog[(size_t)(lo + i) * H + h] = up + a.log_a[(size_t)(lo + i) * H + h];
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_meta(const MetaArgs &a, cudaStream_t st) {
  meta_kernel<<<a.B, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace tv
