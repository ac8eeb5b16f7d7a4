// Commit of the accepted path: rebuild one state per (sequence, head) from pseudo-values.
//
// Along the accepted root-first path p_1..p_m the state is the closed form
//     S_new = exp(c_m) S_root + sum_j exp(c_m - c_j) u_{p_j} k_{p_j}^T,  c_j = sum_{l<=j} log_a_{p_l}
// (the Bole summary's worked example rebuilds S_c3 this way for scalar decay; with the
// pseudo-values of the tree solve the same form holds for the gated delta rule).
//
// One CTA per (sequence, head, slice of kRows state rows).  The kernel is HBM bound (one
// read and one write of the state), so the S_root loads are issued first, before anything
// that depends on the path; the path is then checked by all threads at once, its rank-one
// factors are staged in shared memory in chunks of kChunk entries, and S_new is streamed
// out with 128-bit stores.  Small CTAs keep many slices in flight per SM, which hides the
// chain of dependent loads (offsets -> path -> parent, log_a -> u, k rows) of each slice.
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = 32;                          // state rows (v) per CTA
constexpr int kChunk = 16;
constexpr int kMaxVec = kRows * 128 / 4 / kThreads;  // float4 slots per thread at dk=128
constexpr int kMaxPathWidth = 1024;

struct CommitSmem {
  float cu[kChunk][kRows]; // exp(c_m - c_j) u_{p_j}, this CTA's rows
  float kk[kChunk][128];   // k_{p_j}
  int prow[kMaxPathWidth]; // the accepted_path row
  float la[kMaxNodes];     // log_a of the path nodes
  float c[kMaxNodes];      // cumulative log-decay along the path (root first, fp32)
  int m;
  int flag;
};

template <typename Tk>
__global__ void __launch_bounds__(kThreads) commit_kernel(CommitArgs a) {
  __shared__ __align__(16) CommitSmem sm;
  const int tid = threadIdx.x;
  const int H = a.H, dk = a.dk, dv = a.dv;
  const int slices = (dv + kRows - 1) / kRows;
  const int s = blockIdx.x / (H * slices), h = (blockIdx.x / slices) % H;
  const int r0 = (blockIdx.x % slices) * kRows;           // first state row of the slice
  const int rows = min(kRows, dv - r0);
  const Tk *k = static_cast<const Tk *>(a.k);

  // 1. stream the state slice in (independent of everything else)
  const size_t base = (((size_t)s * H + h) * dv + r0) * dk;
  const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + base);
  const int nvec = rows * dk / 4;
  float4 acc[kMaxVec];
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) acc[r] = __ldcs(Sg + e);
  }

  // 2. the path row and its checks, all threads at once
  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0 && r0 == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n_nodes = hi - lo;
  const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
  if (tid == 0) { sm.flag = 0; sm.m = a.max_path; }
  for (int t = tid; t < a.max_path; t += kThreads) sm.prow[t] = row[t];
  __syncthreads();
  for (int t = tid; t < a.max_path; t += kThreads)
    if (sm.prow[t] < 0 && (t == 0 || sm.prow[t - 1] >= 0)) atomicMin(&sm.m, t);
  __syncthreads();
  const int m = sm.m;
  for (int t = tid; t < a.max_path; t += kThreads) {
    const int p = sm.prow[t];
    bool ok;
    if (t < m) {
      ok = p < n_nodes && t < kMaxNodes;
      if (ok && a.parent) ok = a.parent[lo + p] == (t == 0 ? -1 : sm.prow[t - 1]);
      if (ok) sm.la[t] = a.log_a[(size_t)(lo + p) * H + h];
    } else {
      ok = p == -1;
    }
    if (!ok) sm.flag = 1;
  }
  __syncthreads();
  if (sm.flag) {
    if (tid == 0 && r0 == 0) set_status(a.ws, TV_ERR_BAD_PATH, s);
    return;
  }
  if (tid == 0) {
    float c = 0.f;
    for (int j = 0; j < m; ++j) {
      c += sm.la[j];
      sm.c[j] = c;
    }
  }
  __syncthreads();
  const float cm = m ? sm.c[m - 1] : 0.f;
  const float gam = m ? expf(cm) : 1.f;
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    acc[r].x *= gam; acc[r].y *= gam; acc[r].z *= gam; acc[r].w *= gam;
  }

  // 3. rank-one terms of the path, kChunk at a time
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    const int cnt = min(kChunk, m - j0);
    if (j0) __syncthreads();
    for (int e = tid; e < cnt * 128; e += kThreads) {
      const int j = e / 128, x = e % 128;
      const size_t node = (size_t)(lo + sm.prow[j0 + j]) * H + h;
      if (x < rows) sm.cu[j][x] = expf(cm - sm.c[j0 + j]) * a.U[node * dv + r0 + x];
      if (x < dk) sm.kk[j][x] = to_f32(k[node * dk + x]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaxVec; ++r) {
      const int e = tid + r * kThreads;
      if (e < nvec) {
        const int rr = (e * 4) / dk, col = (e * 4) % dk;
        for (int j = 0; j < cnt; ++j) {
          const float cu = sm.cu[j][rr];
          const float4 kv = *reinterpret_cast<const float4 *>(&sm.kk[j][col]);
          acc[r].x = fmaf(cu, kv.x, acc[r].x);
          acc[r].y = fmaf(cu, kv.y, acc[r].y);
          acc[r].z = fmaf(cu, kv.z, acc[r].z);
          acc[r].w = fmaf(cu, kv.w, acc[r].w);
        }
      }
    }
  }

  // 4. stream the state out
  float4 *Sn = reinterpret_cast<float4 *>(a.S_new + base);
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) __stcs(Sn + e, acc[r]);
  }
}

}  // namespace

int commit_max_path_width() { return kMaxPathWidth; }

cudaError_t launch_commit(const CommitArgs &a, int in_dtype, cudaStream_t st) {
  const int grid = a.B * a.H * ((a.dv + kRows - 1) / kRows);
  if (in_dtype == TV_F32)
    commit_kernel<float><<<grid, kThreads, 0, st>>>(a);
  else
    commit_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace tv
