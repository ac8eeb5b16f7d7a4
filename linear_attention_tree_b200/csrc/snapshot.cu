// The per-node-snapshot baseline: the draft tree verified the way the pages' baseline does it
// (Twig / Bole abstracts: trees verified sequentially, with the full recurrent state
// snapshotted for every node), on the same inputs and with the same outputs as
// tv_tree_verify, so that speed and transient memory can be compared on one GPU.
//
// One CTA of 128 threads per (sequence, head); thread v owns row v of every state.  Nodes go
// in index order (topological): node n starts from its parent's snapshot (S_root for a
// first-level node), takes one step of the recurrence,
//     gated delta rule:  u = b (v_n - a S_par k_n),  S_n = a S_par + u k_n^T   (= a S_par (I - b k k^T) + b v k^T)
//     scalar decay:      u = v_n,                    S_n = lambda S_par + v_n k_n^T
// writes S_n into the snapshot buffer ([T][H][dv][dk] fp32, dv x dk floats per node and
// head), and reads out o_n = S_n q_n.  Row v of S_n only depends on row v of S_par, so each
// thread reads back what it wrote itself and no synchronisation is needed for the states.
// The commit then copies the snapshot of the accepted path's last node.
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 128;

template <typename Tin, typename Tout, bool kGdn>
__global__ void __launch_bounds__(kThreads) snapshot_verify_kernel(VerifyArgs a, float *snap) {
  __shared__ float qn[128], kn[128], vn[128];
  __shared__ float la, bb;
  __shared__ int par, bad;
  const int t = threadIdx.x;
  const int s = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int H = a.H, dk = a.dk, dv = a.dv, kh = qk_head(h, H, a.Hk);
  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes || (s == 0 && lo != 0) ||
      (s == a.B - 1 && hi != a.T)) {
    if (t == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const Tin *q = static_cast<const Tin *>(a.q);
  const Tin *k = static_cast<const Tin *>(a.k);
  const Tin *v = static_cast<const Tin *>(a.v);
  const size_t state = (size_t)dv * dk;
  for (int n = 0; n < hi - lo; ++n) {
    const size_t node = (size_t)(lo + n) * H + h;
    const size_t qk_row = ((size_t)(lo + n) * a.Hk + kh) * dk;
    for (int j = t; j < dk; j += kThreads) {
      qn[j] = to_f32(q[qk_row + j]);
      kn[j] = to_f32(k[qk_row + j]);
    }
    for (int j = t; j < dv; j += kThreads) vn[j] = to_f32(v[node * dv + j]);
    if (t == 0) {
      const int p = a.parent[lo + n];
      par = p;
      bad = p < -1 || p >= n;
      la = a.log_a[node];
      bb = kGdn ? a.b[node] : 0.f;
    }
    __syncthreads();
    if (bad) {
      if (t == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
      return;
    }
    if (t < dv) {
      const float *src = par < 0 ? a.S_root + ((size_t)s * H + h) * state
                                 : snap + ((size_t)(lo + par) * H + h) * state;
      float *dst = snap + node * state;
      const float4 *row = reinterpret_cast<const float4 *>(src + (size_t)t * dk);
      float4 *out_row = reinterpret_cast<float4 *>(dst + (size_t)t * dk);
      float dot = 0.f;
      for (int j = 0; j < dk / 4; ++j) {
        const float4 r = row[j];
        dot = fmaf(r.x, kn[4 * j], dot);
        dot = fmaf(r.y, kn[4 * j + 1], dot);
        dot = fmaf(r.z, kn[4 * j + 2], dot);
        dot = fmaf(r.w, kn[4 * j + 3], dot);
      }
      const float dec = expf(la);
      const float u = kGdn ? bb * (vn[t] - dec * dot) : vn[t];
      float o = 0.f;
      for (int j = 0; j < dk / 4; ++j) {
        const float4 r = row[j];
        float4 x;
        x.x = fmaf(u, kn[4 * j], dec * r.x);
        x.y = fmaf(u, kn[4 * j + 1], dec * r.y);
        x.z = fmaf(u, kn[4 * j + 2], dec * r.z);
        x.w = fmaf(u, kn[4 * j + 3], dec * r.w);
        out_row[j] = x;
        o = fmaf(x.x, qn[4 * j], o);
        o = fmaf(x.y, qn[4 * j + 1], o);
        o = fmaf(x.z, qn[4 * j + 2], o);
        o = fmaf(x.w, qn[4 * j + 3], o);
      }
      static_cast<Tout *>(a.out)[node * dv + t] = from_f32<Tout>(o);
      store_u(a.U, node * dv + t, u, a.u_bf16);
    }
    __syncthreads();   // qn / kn / vn are rewritten for the next node
  }
}

// S_new = the snapshot of the accepted path's last node (S_root for an empty path), after
// the same checks of the path as tv_tree_commit makes.
__global__ void __launch_bounds__(kThreads) snapshot_commit_kernel(CommitArgs a, const float *snap) {
  __shared__ int src_node, status;
  const int t = threadIdx.x;
  const int s = blockIdx.x / a.H, h = blockIdx.x % a.H;
  if (t == 0) {
    const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
    int st = (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes || (s == 0 && lo != 0) ||
              (s == a.B - 1 && hi != a.T)) ? TV_ERR_BAD_TREE : 0;
    const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
    int last = -1, prev = -1;
    for (int j = 0; j < a.max_path && !st; ++j) {
      const int p = row[j];
      if (p < 0) {
        for (int r = j; r < a.max_path; ++r)
          if (row[r] != -1) st = TV_ERR_BAD_PATH;
        break;
      }
      if (p >= hi - lo || (a.parent && a.parent[lo + p] != prev)) st = TV_ERR_BAD_PATH;
      prev = p;
      last = lo + p;
    }
    src_node = last;
    status = st;
    if (st) set_status(a.ws, st, s);
  }
  __syncthreads();
  if (status) return;
  const size_t state = (size_t)a.dv * a.dk;
  const float *src = src_node < 0 ? a.S_root + ((size_t)s * a.H + h) * state
                                   : snap + ((size_t)src_node * a.H + h) * state;
  float *dst = a.S_new + ((size_t)s * a.H + h) * state;
  const float4 *s4 = reinterpret_cast<const float4 *>(src);
  float4 *d4 = reinterpret_cast<float4 *>(dst);
  for (size_t e = t; e < state / 4; e += kThreads) d4[e] = s4[e];
}

template <typename Tin, typename Tout, bool kGdn>
cudaError_t launch_snap_t(const VerifyArgs &a, float *snap, cudaStream_t st) {
  snapshot_verify_kernel<Tin, Tout, kGdn><<<a.B * a.H, kThreads, 0, st>>>(a, snap);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_snapshot_verify(const VerifyArgs &a, float *snap, int mode, int in_dtype,
                                   int out_dtype, cudaStream_t st) {
  const bool gdn = mode == TV_MODE_GDN;
  if (in_dtype == TV_F32)
    return gdn ? launch_snap_t<float, float, true>(a, snap, st)
               : launch_snap_t<float, float, false>(a, snap, st);
  if (out_dtype == TV_BF16)
    return gdn ? launch_snap_t<__nv_bfloat16, __nv_bfloat16, true>(a, snap, st)
               : launch_snap_t<__nv_bfloat16, __nv_bfloat16, false>(a, snap, st);
  return gdn ? launch_snap_t<__nv_bfloat16, float, true>(a, snap, st)
             : launch_snap_t<__nv_bfloat16, float, false>(a, snap, st);
}

cudaError_t launch_snapshot_commit(const CommitArgs &a, const float *snap, cudaStream_t st) {
  snapshot_commit_kernel<<<a.B * a.H, kThreads, 0, st>>>(a, snap);
  return cudaGetLastError();
}

}  // namespace tv
