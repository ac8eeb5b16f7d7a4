// Internal declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tree_verify.h"

namespace tv {

constexpr int kMaxNodes = 256;          // largest tree one sequence may hold
constexpr int kAncWords = kMaxNodes / 64;
constexpr size_t kWorkspaceBytes = 256; // status word + reserved

// Workspace layout (int32 words).
enum : int { kWsStatus = 0, kWsDetail = 1 };

// Device status: the first error recorded wins; later ones are dropped.
__device__ __forceinline__ void set_status(int *ws, int code, int detail) {
  if (atomicCAS(ws + kWsStatus, 0, code) == 0) ws[kWsDetail] = detail;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Everything a verify kernel needs, by value.  Hk = number of q / k heads (value head h
// reads q / k head h / (H / Hk)); u_bf16: U is stored as bf16.
struct VerifyArgs {
  const void *q, *k, *v;
  const float *log_a, *b;
  const int32_t *parent, *node_offsets;
  const float *S_root;
  void *out;
  void *U;
  int *ws;
  int B, H, dk, dv, T, max_nodes;
  int Hk, u_bf16;
};

struct CommitArgs {
  const void *U;
  const void *k;
  const float *log_a, *S_root;
  const int32_t *node_offsets, *accepted_path, *parent;
  float *S_new;
  int *ws;
  int B, H, dk, dv, T, max_nodes, max_path;
  int Hk, u_bf16;
};

// q / k head of value head h.
__host__ __device__ __forceinline__ int qk_head(int h, int H, int Hk) { return h / (H / Hk); }

// Element i of U in its storage type.
__device__ __forceinline__ void store_u(void *U, size_t i, float x, int u_bf16) {
  if (u_bf16) static_cast<__nv_bfloat16 *>(U)[i] = __float2bfloat16_rn(x);
  else __stcs(static_cast<float *>(U) + i, x);
}
__device__ __forceinline__ float load_u(const void *U, size_t i, int u_bf16) {
  return u_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(U)[i])
                : static_cast<const float *>(U)[i];
}

// The commit that a fused commit + verify launch applies to S_root before verifying: the
// previous step's tree, its pseudo-values and its accepted paths (one row per sequence).
struct FuseArgs {
  const void *U;                     // previous step's U (u_bf16: bf16)
  const void *k;                     // previous step's k (bf16)
  const float *log_a;
  const int32_t *node_offsets, *accepted_path, *parent;   // parent may be NULL
  float *S_new;                      // may be S_root
  int T, max_nodes, max_path, u_bf16;
};

struct MetaArgs {
  const int32_t *parent, *node_offsets;
  const float *log_a;
  int32_t *depth;
  uint64_t *anc;
  float *cumlog;
  int *ws;
  int B, H, T, max_nodes, anc_words;
};

// Record a failed CUDA call for tv_last_cuda_error on the calling host thread and return
// TV_ERR_CUDA (TV_OK for cudaSuccess).  Every entry point reports CUDA failures this way.
tv_status record_cuda_error(cudaError_t e);

// Launchers (host side); each returns cudaSuccess or the launch error.
cudaError_t launch_timeout_probe(int *ws, uint32_t polls, cudaStream_t st);
cudaError_t launch_verify_simt(const VerifyArgs &a, int mode, int in_dtype, int out_dtype,
                               cudaStream_t st);
int verify_tc_max_nodes();
cudaError_t launch_verify_tc(const VerifyArgs &a, int mode, int out_dtype, cudaStream_t st);
int fused_max_path();
cudaError_t launch_commit_verify_tc(const VerifyArgs &a, const FuseArgs &f, int mode, int out_dtype,
                                    cudaStream_t st);
int verify_tcw_max_nodes();
cudaError_t launch_verify_tcw(const VerifyArgs &a, int mode, int out_dtype, cudaStream_t st);
int commit_max_path_width();
cudaError_t launch_commit(const CommitArgs &a, int in_dtype, cudaStream_t st);
cudaError_t launch_meta(const MetaArgs &a, cudaStream_t st);
cudaError_t launch_snapshot_verify(const VerifyArgs &a, float *snap, int mode, int in_dtype,
                                   int out_dtype, cudaStream_t st);
cudaError_t launch_snapshot_commit(const CommitArgs &a, const float *snap, cudaStream_t st);

}  // namespace tv
