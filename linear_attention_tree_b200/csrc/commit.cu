// Commit of the accepted path: rebuild one state per (sequence, head) from pseudo-values.
//
// Along the accepted root-first path p_1..p_m the state is the closed form
//     S_new = exp(c_m) S_root + sum_j exp(c_m - c_j) u_{p_j} k_{p_j}^T,  c_j = sum_{l<=j} log_a_{p_l}
// (the Bole summary's worked example rebuilds S_c3 this way for scalar decay; with the
// pseudo-values of the tree solve the same form holds for the gated delta rule).
//
// One CTA per (sequence, head, slice of kRows state rows).  The kernel is HBM bound (one
// read and one write of the state), so everything that depends on the path is kept to
// two rounds of dependent global loads, overlapped with the state loads:
//   round 0: the state slice (registers), node_offsets, the accepted_path row (warp 0,
//            checked with one ballot per 32 entries);
//   round 1: parent and log_a of the path nodes and their u and k rows, all at once.
// Then one thread forms the fp32 prefix sums c_j (root first, the order the verify
// kernels use for cl), the u rows are scaled, and S_new streams out with 128-bit stores.
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = 32;                            // state rows (v) per CTA
constexpr int kChunk = 16;                           // path entries staged at a time
constexpr int kMaxVec = kRows * 128 / 4 / kThreads;  // float4 slots per thread at dk=128
constexpr int kMaxPathWidth = 1024;

struct CommitSmem {
  float cu[kChunk][kRows]; // exp(c_m - c_j) u_{p_j}, this CTA's rows
  float kk[kChunk][128];   // k_{p_j}
  int prow[kMaxNodes];     // root-first path nodes
  float la[kMaxNodes];     // log_a of the path nodes
  float e[kMaxNodes];      // exp(c_m - c_j)
  int m;
  int lo;
  int bad;
};

// kD128: dk == 128, so thread t always owns column block 4*(t%32) and rows t/32 + 4r.
template <typename Tk, bool kD128>
__global__ void __launch_bounds__(kThreads) commit_kernel(CommitArgs a) {
  __shared__ __align__(16) CommitSmem sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, dk = a.dk, dv = a.dv;
  const int slices = (dv + kRows - 1) / kRows;
  const int s = blockIdx.x / (H * slices), h = (blockIdx.x / slices) % H;
  const int r0 = (blockIdx.x % slices) * kRows;           // first state row of the slice
  const int rows = min(kRows, dv - r0);
  const Tk *k = static_cast<const Tk *>(a.k);

  // ---- round 0 ---------------------------------------------------------------------
  const size_t base = (((size_t)s * H + h) * dv + r0) * dk;
  const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + base);
  const int nvec = rows * dk / 4;
  float4 acc[kMaxVec];
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) acc[r] = __ldcs(Sg + e);
  }
  if (warp == 0) {
    const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
    const bool tree_ok = !(lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
                           (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T));
    const int n_nodes = hi - lo;
    const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
    // m = number of leading non-negative entries; after them only -1 may follow
    int m = -1;
    bool bad = false;
    for (int t0 = 0; t0 < a.max_path; t0 += 32) {
      const int t = t0 + lane;
      const int p = t < a.max_path ? row[t] : -1;
      const unsigned neg = __ballot_sync(0xffffffffu, t < a.max_path && p < 0);
      if (m < 0 && neg) m = t0 + __ffs(neg) - 1;
      const bool in_path = m < 0 || t < m;
      if (t < a.max_path) {
        if (in_path) {
          if (p < 0 || p >= n_nodes || t >= kMaxNodes) bad = true;
          else sm.prow[t] = p;
        } else if (p != -1) {
          bad = true;
        }
      }
    }
    if (m < 0) m = a.max_path;
    bad = __any_sync(0xffffffffu, bad) || !tree_ok;
    if (lane == 0) {
      sm.m = bad ? 0 : m;
      sm.lo = lo;
      sm.bad = bad ? (tree_ok ? TV_ERR_BAD_PATH : TV_ERR_BAD_TREE) : 0;
    }
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0 && r0 == 0) set_status(a.ws, sm.bad, s);
    return;
  }
  const int m = sm.m, lo = sm.lo;

  // ---- round 1: parent / log_a of the path, the first chunk of u and k rows ----------
  int chain_bad = 0;
  for (int t = tid; t < m; t += kThreads) {
    const int p = sm.prow[t];
    sm.la[t] = a.log_a[(size_t)(lo + p) * H + h];
    if (a.parent && a.parent[lo + p] != (t == 0 ? -1 : sm.prow[t - 1])) chain_bad = 1;
  }
  const int cnt0 = min(kChunk, m);
  for (int e = tid; e < cnt0 * 128; e += kThreads) {
    const int j = e >> 7, x = e & 127;
    const size_t node = (size_t)(lo + sm.prow[j]) * H + h;
    if (x < rows) sm.cu[j][x] = a.U[node * dv + r0 + x];
    if (x < dk) sm.kk[j][x] = to_f32(k[node * dk + x]);
  }
  if (__syncthreads_or(chain_bad)) {
    if (tid == 0 && r0 == 0) set_status(a.ws, TV_ERR_BAD_PATH, s);
    return;
  }
  if (tid == 0) {
    float c = 0.f;
    for (int j = 0; j < m; ++j) {
      c += sm.la[j];
      sm.la[j] = c;                    // now c_j
    }
    for (int j = 0; j < m; ++j) sm.e[j] = expf(c - sm.la[j]);
  }
  __syncthreads();
  for (int e = tid; e < cnt0 * kRows; e += kThreads) sm.cu[e / kRows][e % kRows] *= sm.e[e / kRows];
  __syncthreads();
  const float gam = m ? expf(sm.la[m - 1]) : 1.f;
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    acc[r].x *= gam; acc[r].y *= gam; acc[r].z *= gam; acc[r].w *= gam;
  }

  // ---- rank-one terms of the path, kChunk entries at a time --------------------------
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    const int cnt = min(kChunk, m - j0);
    if (j0) {
      __syncthreads();
      for (int e = tid; e < cnt * 128; e += kThreads) {
        const int j = e >> 7, x = e & 127;
        const size_t node = (size_t)(lo + sm.prow[j0 + j]) * H + h;
        if (x < rows) sm.cu[j][x] = sm.e[j0 + j] * a.U[node * dv + r0 + x];
        if (x < dk) sm.kk[j][x] = to_f32(k[node * dk + x]);
      }
      __syncthreads();
    }
    if (kD128) {
      // fixed column block per thread: one k chunk per path entry serves all its rows
      const int col = (tid & 31) * 4, rb = tid >> 5;
      for (int j = 0; j < cnt; ++j) {
        const float4 kv = *reinterpret_cast<const float4 *>(&sm.kk[j][col]);
#pragma unroll
        for (int r = 0; r < kMaxVec; ++r) {
          const float cu = sm.cu[j][rb + 4 * r];
          acc[r].x = fmaf(cu, kv.x, acc[r].x);
          acc[r].y = fmaf(cu, kv.y, acc[r].y);
          acc[r].z = fmaf(cu, kv.z, acc[r].z);
          acc[r].w = fmaf(cu, kv.w, acc[r].w);
        }
      }
    } else {
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
  }

  // ---- stream the state slice out ------------------------------------------------------
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
  const bool d128 = a.dk == 128 && a.dv % kRows == 0;
  if (in_dtype == TV_F32) {
    if (d128) commit_kernel<float, true><<<grid, kThreads, 0, st>>>(a);
    else commit_kernel<float, false><<<grid, kThreads, 0, st>>>(a);
  } else {
    if (d128) commit_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, st>>>(a);
    else commit_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace tv
