// Commit of the accepted path: rebuild one state per (sequence, head) from pseudo-values.
//
// Along the accepted root-first path p_1..p_m the state is the closed form
//     S_new = exp(c_m) S_root + sum_j exp(c_m - c_j) u_{p_j} k_{p_j}^T,  c_j = sum_{l<=j} log_a_{p_l}
// (the Bole summary's worked example rebuilds S_c3 this way for scalar decay; with the
// pseudo-values of the tree solve the same form holds for the gated delta rule).  The
// kernel streams S_root once with 128-bit loads, applies the m rank-one terms held in
// shared memory, and streams S_new out; it is HBM bound (two state passes per head).
// Paths are processed in chunks of kChunk entries so any path length fits.
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 16;
constexpr int kMaxVec = 128 * 128 / 4 / kThreads;  // float4 slots per thread at dk=dv=128

struct CommitSmem {
  float cu[kChunk][128];   // exp(c_m - c_j) u_{p_j}
  float kk[kChunk][128];   // k_{p_j}
  int path[kMaxNodes];
  float c[kMaxNodes];      // cumulative log-decay along the path (root first, fp32)
  int m;
  int flag;
};

template <typename Tk>
__global__ void __launch_bounds__(kThreads) commit_kernel(CommitArgs a) {
  __shared__ __align__(16) CommitSmem sm;
  const int tid = threadIdx.x;
  const int s = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int H = a.H, dk = a.dk, dv = a.dv;
  const Tk *k = static_cast<const Tk *>(a.k);

  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n_nodes = hi - lo;
  if (tid == 0) {
    // root-first entries, then only -1 padding; each entry a node of this tree; with the
    // parent array, each entry the child of the previous one (the first a root child)
    const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
    int m = 0, bad = 0;
    while (m < a.max_path && row[m] >= 0) {
      const int p = row[m];
      if (p >= n_nodes || m >= kMaxNodes) { bad = 1; break; }
      if (a.parent && a.parent[lo + p] != (m == 0 ? -1 : row[m - 1])) { bad = 1; break; }
      sm.path[m] = p;
      ++m;
    }
    for (int j = m; !bad && j < a.max_path; ++j)
      if (row[j] != -1) bad = 1;
    float c = 0.f;
    for (int j = 0; !bad && j < m; ++j) {
      c += a.log_a[(size_t)(lo + sm.path[j]) * H + h];
      sm.c[j] = c;
    }
    sm.m = m;
    sm.flag = bad;
    if (bad) set_status(a.ws, TV_ERR_BAD_PATH, s);
  }
  __syncthreads();
  if (sm.flag) return;
  const int m = sm.m;
  const float cm = m ? sm.c[m - 1] : 0.f;
  const float gam = m ? expf(cm) : 1.f;

  const size_t base = ((size_t)s * H + h) * dv * dk;
  const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + base);
  float4 *Sn = reinterpret_cast<float4 *>(a.S_new + base);
  const int nvec = dv * dk / 4;
  float4 acc[kMaxVec];
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) {
      const float4 x = Sg[e];
      acc[r] = make_float4(gam * x.x, gam * x.y, gam * x.z, gam * x.w);
    }
  }
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    const int cnt = min(kChunk, m - j0);
    __syncthreads();
    for (int e = tid; e < cnt * 128; e += kThreads) {
      const int j = e / 128, x = e % 128;
      const size_t node = (size_t)(lo + sm.path[j0 + j]) * H + h;
      if (x < dv) sm.cu[j][x] = expf(cm - sm.c[j0 + j]) * a.U[node * dv + x];
      if (x < dk) sm.kk[j][x] = to_f32(k[node * dk + x]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaxVec; ++r) {
      const int e = tid + r * kThreads;
      if (e < nvec) {
        const int row = (e * 4) / dk, col = (e * 4) % dk;
        for (int j = 0; j < cnt; ++j) {
          const float cu = sm.cu[j][row];
          const float4 kv = *reinterpret_cast<const float4 *>(&sm.kk[j][col]);
          acc[r].x = fmaf(cu, kv.x, acc[r].x);
          acc[r].y = fmaf(cu, kv.y, acc[r].y);
          acc[r].z = fmaf(cu, kv.z, acc[r].z);
          acc[r].w = fmaf(cu, kv.w, acc[r].w);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) Sn[e] = acc[r];
  }
}

}  // namespace

cudaError_t launch_commit(const CommitArgs &a, int in_dtype, cudaStream_t st) {
  if (in_dtype == TV_F32)
    commit_kernel<float><<<a.B * a.H, kThreads, 0, st>>>(a);
  else
    commit_kernel<__nv_bfloat16><<<a.B * a.H, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace tv
