// C ABI entry points: argument validation, kernel choice, launches.  No allocation, no
// synchronisation except in tv_get_status.
#include <cstdio>
#include <cstring>

#include "tv_internal.cuh"

namespace {

using namespace tv;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape / enum checks shared by all entry points.
tv_status check_problem(const tv_problem *p) {
  if (!p) return TV_ERR_INVALID_ARG;
  if (p->B < 0 || p->H < 1 || p->total_nodes < 0) return TV_ERR_INVALID_ARG;
  if (p->max_nodes < 1) return TV_ERR_INVALID_ARG;
  if (p->mode != TV_MODE_GDN && p->mode != TV_MODE_SCALAR_DECAY) return TV_ERR_INVALID_ARG;
  if (p->in_dtype != TV_F32 && p->in_dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (p->out_dtype != TV_F32 && p->out_dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (p->kernel < TV_KERNEL_AUTO || p->kernel > TV_KERNEL_SIMT) return TV_ERR_INVALID_ARG;
  if (p->dk < 1 || p->dv < 1) return TV_ERR_INVALID_ARG;
  if (p->u_dtype != TV_F32 && p->u_dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (p->qk_heads < 0 || p->qk_heads > p->H || (p->qk_heads && p->H % p->qk_heads))
    return TV_ERR_INVALID_ARG;
  if (p->max_nodes > kMaxNodes) return TV_ERR_UNSUPPORTED;
  if (p->dk % 16 || p->dv % 16 || p->dk > 128 || p->dv > 128) return TV_ERR_UNSUPPORTED;
  if (p->in_dtype == TV_F32 && p->out_dtype == TV_BF16) return TV_ERR_UNSUPPORTED;
  // int32 indexing of every array stays in range
  const long long T = p->total_nodes, H = p->H;
  if (T * H * 128 > 0x7fffffffLL || (long long)p->B * H > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  if (T > (long long)p->B * p->max_nodes) return TV_ERR_INVALID_ARG;
  return TV_OK;
}

bool ptr_ok(const void *ptr) { return ptr && aligned16(ptr); }

int qk_heads_of(const tv_problem *p) { return p->qk_heads ? p->qk_heads : p->H; }

bool tc_supports(const tv_problem *p) {
  return p->in_dtype == TV_BF16 && p->dk == 128 && p->dv == 128 &&
         p->max_nodes <= verify_tcw_max_nodes();
}

thread_local cudaError_t g_last_cuda = cudaSuccess;

tv_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return TV_OK;
  g_last_cuda = e;
  return TV_ERR_CUDA;
}

}  // namespace

namespace tv {
tv_status record_cuda_error(cudaError_t e) { return from_cuda(e); }
}  // namespace tv

extern "C" {

int32_t tv_version(void) { return (2 << 16) | 0; }   // 2: tv_problem gained u_dtype and qk_heads

const char *tv_last_cuda_error(void) {
  if (g_last_cuda == cudaSuccess) return "";
  static thread_local char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", cudaGetErrorName(g_last_cuda),
           cudaGetErrorString(g_last_cuda));
  return buf;
}

const char *tv_status_string(tv_status s) {
  switch (s) {
    case TV_OK: return "ok";
    case TV_ERR_INVALID_ARG: return "invalid argument";
    case TV_ERR_UNSUPPORTED: return "unsupported problem";
    case TV_ERR_BAD_TREE: return "bad tree (parent not topological or node_offsets invalid)";
    case TV_ERR_BAD_PATH: return "bad accepted path";
    case TV_ERR_CUDA: return "CUDA runtime error";
    case TV_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t tv_workspace_size(const tv_problem *p) {
  return check_problem(p) == TV_OK ? kWorkspaceBytes : 0;
}

tv_status tv_tree_verify(const tv_problem *p, const void *q, const void *k, const void *v,
                         const float *log_a, const float *b, const int32_t *parent,
                         const int32_t *node_offsets, const float *S_root, void *out,
                         float *U, void *workspace, size_t workspace_bytes,
                         tv_stream_t stream) {
  tv_status st = check_problem(p);
  if (st != TV_OK) return st;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(log_a) || !ptr_ok(parent) ||
      !ptr_ok(node_offsets) || !ptr_ok(S_root) || !ptr_ok(out) || !ptr_ok(U) ||
      !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (p->mode == TV_MODE_GDN ? !ptr_ok(b) : (b && !aligned16(b))) return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  bool use_tc;
  if (p->kernel == TV_KERNEL_TC) {
    if (!tc_supports(p)) return TV_ERR_UNSUPPORTED;
    use_tc = true;
  } else {
    use_tc = p->kernel == TV_KERNEL_AUTO && tc_supports(p);
  }
  // the CUDA-core kernel reads U back as it goes: it keeps it in fp32
  if (!use_tc && p->u_dtype == TV_BF16) return TV_ERR_UNSUPPORTED;
  if (p->B == 0) return TV_OK;
  VerifyArgs a;
  a.q = q; a.k = k; a.v = v; a.log_a = log_a; a.b = b; a.parent = parent;
  a.node_offsets = node_offsets; a.S_root = S_root; a.out = out; a.U = U;
  a.ws = static_cast<int *>(workspace);
  a.B = p->B; a.H = p->H; a.dk = p->dk; a.dv = p->dv; a.T = p->total_nodes;
  a.max_nodes = p->max_nodes; a.Hk = qk_heads_of(p); a.u_bf16 = p->u_dtype == TV_BF16;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_tc)   // trees of up to 64 nodes, and wider trees, have one tensor-core kernel each
    return from_cuda(p->max_nodes <= verify_tc_max_nodes()
                         ? launch_verify_tc(a, p->mode, p->out_dtype, s)
                         : launch_verify_tcw(a, p->mode, p->out_dtype, s));
  return from_cuda(launch_verify_simt(a, p->mode, p->in_dtype, p->out_dtype, s));
}

tv_status tv_tree_commit(const tv_problem *p, const float *U, const void *k,
                         const float *log_a, const float *S_root,
                         const int32_t *node_offsets, const int32_t *accepted_path,
                         const int32_t *parent, float *S_new, void *workspace,
                         size_t workspace_bytes, tv_stream_t stream) {
  tv_status st = check_problem(p);
  if (st != TV_OK) return st;
  if (p->max_path < 1) return TV_ERR_INVALID_ARG;
  if (p->max_path > commit_max_path_width()) return TV_ERR_UNSUPPORTED;
  if (!ptr_ok(U) || !ptr_ok(k) || !ptr_ok(log_a) || !ptr_ok(S_root) || !ptr_ok(node_offsets) ||
      !ptr_ok(accepted_path) || !ptr_ok(S_new) || !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (parent && !aligned16(parent)) return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  // S_new either is S_root or does not overlap it
  const size_t state_bytes = (size_t)p->B * p->H * p->dv * p->dk * sizeof(float);
  const char *a0 = reinterpret_cast<const char *>(S_root), *b0 = reinterpret_cast<const char *>(S_new);
  if (a0 != b0 && a0 < b0 + state_bytes && b0 < a0 + state_bytes) return TV_ERR_INVALID_ARG;
  if (p->B == 0) return TV_OK;
  CommitArgs a;
  a.U = U; a.k = k; a.log_a = log_a; a.S_root = S_root; a.node_offsets = node_offsets;
  a.accepted_path = accepted_path; a.parent = parent; a.S_new = S_new;
  a.ws = static_cast<int *>(workspace);
  a.B = p->B; a.H = p->H; a.dk = p->dk; a.dv = p->dv; a.T = p->total_nodes;
  a.max_nodes = p->max_nodes; a.max_path = p->max_path;
  a.Hk = qk_heads_of(p); a.u_bf16 = p->u_dtype == TV_BF16;
  return from_cuda(launch_commit(a, p->in_dtype, reinterpret_cast<cudaStream_t>(stream)));
}

tv_status tv_tree_commit_verify(const tv_problem *prev, const float *U_prev, const void *k_prev,
                                const float *log_a_prev, const int32_t *node_offsets_prev,
                                const int32_t *accepted_path, const int32_t *parent_prev,
                                const float *S_root, float *S_new, const tv_problem *next,
                                const void *q, const void *k, const void *v, const float *log_a,
                                const float *b, const int32_t *parent,
                                const int32_t *node_offsets, void *out, float *U, void *workspace,
                                size_t workspace_bytes, tv_stream_t stream) {
  tv_status st = check_problem(prev);
  if (st == TV_OK) st = check_problem(next);
  if (st != TV_OK) return st;
  if (prev->B != next->B || prev->H != next->H || prev->dk != next->dk || prev->dv != next->dv ||
      qk_heads_of(prev) != qk_heads_of(next))
    return TV_ERR_INVALID_ARG;
  if (prev->max_path < 1) return TV_ERR_INVALID_ARG;
  if (prev->max_path > commit_max_path_width()) return TV_ERR_UNSUPPORTED;
  if (!ptr_ok(U_prev) || !ptr_ok(k_prev) || !ptr_ok(log_a_prev) || !ptr_ok(node_offsets_prev) ||
      !ptr_ok(accepted_path) || !ptr_ok(S_root) || !ptr_ok(S_new) || !ptr_ok(q) || !ptr_ok(k) ||
      !ptr_ok(v) || !ptr_ok(log_a) || !ptr_ok(parent) || !ptr_ok(node_offsets) || !ptr_ok(out) ||
      !ptr_ok(U) || !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (parent_prev && !aligned16(parent_prev)) return TV_ERR_INVALID_ARG;
  if (next->mode == TV_MODE_GDN ? !ptr_ok(b) : (b && !aligned16(b))) return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  const size_t state_bytes = (size_t)next->B * next->H * next->dv * next->dk * sizeof(float);
  const char *a0 = reinterpret_cast<const char *>(S_root), *b0 = reinterpret_cast<const char *>(S_new);
  if (a0 != b0 && a0 < b0 + state_bytes && b0 < a0 + state_bytes) return TV_ERR_INVALID_ARG;
  // the new pseudo-values must not overwrite the previous ones while they are read
  const size_t u_prev_bytes = (size_t)prev->total_nodes * prev->H * prev->dv *
                              (prev->u_dtype == TV_BF16 ? 2 : 4);
  const size_t u_bytes = (size_t)next->total_nodes * next->H * next->dv *
                         (next->u_dtype == TV_BF16 ? 2 : 4);
  const char *c0 = reinterpret_cast<const char *>(U_prev), *d0 = reinterpret_cast<const char *>(U);
  if (u_prev_bytes && u_bytes && c0 < d0 + u_bytes && d0 < c0 + u_prev_bytes) return TV_ERR_INVALID_ARG;
  if (next->kernel == TV_KERNEL_TC && !tc_supports(next)) return TV_ERR_UNSUPPORTED;
  const bool next_tc = next->kernel != TV_KERNEL_SIMT && tc_supports(next);
  if (!next_tc && next->u_dtype == TV_BF16) return TV_ERR_UNSUPPORTED;
  if (next->B == 0) return TV_OK;
  VerifyArgs a;
  a.q = q; a.k = k; a.v = v; a.log_a = log_a; a.b = b; a.parent = parent;
  a.node_offsets = node_offsets; a.S_root = S_root; a.out = out; a.U = U;
  a.ws = static_cast<int *>(workspace);
  a.B = next->B; a.H = next->H; a.dk = next->dk; a.dv = next->dv; a.T = next->total_nodes;
  a.max_nodes = next->max_nodes; a.Hk = qk_heads_of(next); a.u_bf16 = next->u_dtype == TV_BF16;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool fused = next_tc &&
                     next->max_nodes <= verify_tc_max_nodes() && prev->in_dtype == TV_BF16 &&
                     prev->max_path <= fused_max_path();
  if (fused) {
    FuseArgs f;
    f.U = U_prev; f.k = k_prev; f.log_a = log_a_prev; f.node_offsets = node_offsets_prev;
    f.accepted_path = accepted_path; f.parent = parent_prev; f.S_new = S_new;
    f.T = prev->total_nodes; f.max_nodes = prev->max_nodes; f.max_path = prev->max_path;
    f.u_bf16 = prev->u_dtype == TV_BF16;
    return from_cuda(launch_commit_verify_tc(a, f, next->mode, next->out_dtype, s));
  }
  // otherwise the commit, then the verify on its result: two launches, same results
  CommitArgs c;
  c.U = U_prev; c.k = k_prev; c.log_a = log_a_prev; c.S_root = S_root;
  c.node_offsets = node_offsets_prev; c.accepted_path = accepted_path; c.parent = parent_prev;
  c.S_new = S_new; c.ws = a.ws;
  c.B = prev->B; c.H = prev->H; c.dk = prev->dk; c.dv = prev->dv; c.T = prev->total_nodes;
  c.max_nodes = prev->max_nodes; c.max_path = prev->max_path;
  c.Hk = qk_heads_of(prev); c.u_bf16 = prev->u_dtype == TV_BF16;
  st = from_cuda(launch_commit(c, prev->in_dtype, s));
  if (st != TV_OK) return st;
  a.S_root = S_new;
  if (next_tc)
    return from_cuda(next->max_nodes <= verify_tc_max_nodes()
                         ? launch_verify_tc(a, next->mode, next->out_dtype, s)
                         : launch_verify_tcw(a, next->mode, next->out_dtype, s));
  return from_cuda(launch_verify_simt(a, next->mode, next->in_dtype, next->out_dtype, s));
}

tv_status tv_tree_meta(const tv_problem *p, const int32_t *parent,
                       const int32_t *node_offsets, const float *log_a, int32_t *depth,
                       uint64_t *anc, float *cumlog, void *workspace,
                       size_t workspace_bytes, tv_stream_t stream) {
  tv_status st = check_problem(p);
  if (st != TV_OK) return st;
  if (!ptr_ok(parent) || !ptr_ok(node_offsets) || !ptr_ok(log_a) || !ptr_ok(depth) ||
      !ptr_ok(anc) || !ptr_ok(cumlog) || !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  if (p->B == 0) return TV_OK;
  MetaArgs a;
  a.parent = parent; a.node_offsets = node_offsets; a.log_a = log_a; a.depth = depth;
  a.anc = anc; a.cumlog = cumlog; a.ws = static_cast<int *>(workspace);
  a.B = p->B; a.H = p->H; a.T = p->total_nodes; a.max_nodes = p->max_nodes;
  a.anc_words = (p->max_nodes + 63) / 64;
  return from_cuda(launch_meta(a, reinterpret_cast<cudaStream_t>(stream)));
}

tv_status tv_snapshot_verify(const tv_problem *p, const void *q, const void *k, const void *v,
                             const float *log_a, const float *b, const int32_t *parent,
                             const int32_t *node_offsets, const float *S_root, void *out,
                             float *U, float *snapshots, void *workspace, size_t workspace_bytes,
                             tv_stream_t stream) {
  tv_status st = check_problem(p);
  if (st != TV_OK) return st;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(log_a) || !ptr_ok(parent) ||
      !ptr_ok(node_offsets) || !ptr_ok(S_root) || !ptr_ok(out) || !ptr_ok(U) ||
      !ptr_ok(snapshots) || !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (p->mode == TV_MODE_GDN ? !ptr_ok(b) : (b && !aligned16(b))) return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  if (p->B == 0) return TV_OK;
  VerifyArgs a;
  a.q = q; a.k = k; a.v = v; a.log_a = log_a; a.b = b; a.parent = parent;
  a.node_offsets = node_offsets; a.S_root = S_root; a.out = out; a.U = U;
  a.ws = static_cast<int *>(workspace);
  a.B = p->B; a.H = p->H; a.dk = p->dk; a.dv = p->dv; a.T = p->total_nodes;
  a.max_nodes = p->max_nodes; a.Hk = qk_heads_of(p); a.u_bf16 = p->u_dtype == TV_BF16;
  return from_cuda(launch_snapshot_verify(a, snapshots, p->mode, p->in_dtype, p->out_dtype,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

tv_status tv_snapshot_commit(const tv_problem *p, const float *snapshots, const float *S_root,
                             const int32_t *node_offsets, const int32_t *accepted_path,
                             const int32_t *parent, float *S_new, void *workspace,
                             size_t workspace_bytes, tv_stream_t stream) {
  tv_status st = check_problem(p);
  if (st != TV_OK) return st;
  if (p->max_path < 1) return TV_ERR_INVALID_ARG;
  if (!ptr_ok(snapshots) || !ptr_ok(S_root) || !ptr_ok(node_offsets) ||
      !ptr_ok(accepted_path) || !ptr_ok(S_new) || !ptr_ok(workspace))
    return TV_ERR_INVALID_ARG;
  if (parent && !aligned16(parent)) return TV_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  if (S_new == S_root) return TV_ERR_INVALID_ARG;   // other sequences may still read S_root
  if (p->B == 0) return TV_OK;
  CommitArgs a = {};
  a.S_root = S_root; a.node_offsets = node_offsets; a.accepted_path = accepted_path;
  a.parent = parent; a.S_new = S_new; a.ws = static_cast<int *>(workspace);
  a.B = p->B; a.H = p->H; a.dk = p->dk; a.dv = p->dv; a.T = p->total_nodes;
  a.max_nodes = p->max_nodes; a.max_path = p->max_path;
  return from_cuda(launch_snapshot_commit(a, snapshots, reinterpret_cast<cudaStream_t>(stream)));
}

tv_status tv_selftest_timeout(void *workspace, size_t workspace_bytes, tv_stream_t stream) {
  if (!ptr_ok(workspace) || workspace_bytes < kWorkspaceBytes) return TV_ERR_INVALID_ARG;
  // a short poll budget: the point is the path taken when a wait runs out, not its length
  return from_cuda(launch_timeout_probe(static_cast<int *>(workspace), 4096,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

tv_status tv_get_status(void *workspace, tv_stream_t stream) {
  if (!ptr_ok(workspace)) return TV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int host[2] = {0, 0};
  tv_status st = from_cuda(cudaMemcpyAsync(host, workspace, sizeof(host),
                                           cudaMemcpyDeviceToHost, s));
  if (st == TV_OK) st = from_cuda(cudaStreamSynchronize(s));
  if (st == TV_OK && host[0] != TV_OK) {
    st = from_cuda(cudaMemsetAsync(workspace, 0, sizeof(host), s));
    if (st == TV_OK) st = from_cuda(cudaStreamSynchronize(s));
  }
  if (st != TV_OK) return st;
  return static_cast<tv_status>(host[0]);
}

}  // extern "C"
