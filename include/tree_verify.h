/*
 * tree_verify.h -- C ABI of the B200 (sm_100a) draft-tree verification library for
 * recurrent linear-attention layers.
 *
 * What the library computes.  A speculative draft tree hangs off the layer's current
 * recurrent state S_root (one [dv][dk] fp32 matrix per sequence and head).  Every tree
 * node is a token whose state is the one the sequential recurrence reaches after the
 * tokens on its root-to-node path (Twig / Bole abstracts: recurrent layers carry
 * parent-dependent states, and all proposal nodes are verified in parallel).  Two
 * recurrences are supported:
 *
 *   gated delta rule (Gated DeltaNet, TreeWY abstract):
 *       S_n = a_n S_par(n) (I - b_n k_n k_n^T) + b_n v_n k_n^T,   a_n = exp(log_a_n)
 *   scalar decay (Bole machine summary, section "核心公式", first formula, stored
 *   transposed):
 *       S_n = lambda_n S_par(n) + v_n k_n^T,                        lambda_n = exp(log_a_n)
 *
 * with output o_n = S_n q_n (post-update state; no 1/sqrt(dk) scale -- pre-scale q).
 *
 * No per-node state is ever materialised.  With cl_n the sum of log_a over the root->n
 * path, every node state is  S_n = exp(cl_n) S_root + sum_{i on path(n)} exp(cl_n-cl_i) u_i k_i^T
 * (the tree-structured closed form of the Bole summary's worked example, "具体技术细节示例",
 * generalised to the delta rule), where the pseudo-values u_i (the TreeWY abstract's
 * pseudo-value matrix, which stands in for per-node snapshots) solve one
 * unit-lower-triangular system over the tree (TreeWY abstract, tree-structured WY form):
 *       u_n + sum_{i in anc(n)} b_n exp(cl_n-cl_i) (k_n.k_i) u_i = b_n (v_n - exp(cl_n) S_root k_n)
 * (scalar decay: u_n = v_n).  tv_tree_verify writes o and U; tv_tree_commit rebuilds the
 * state of the accepted path alone from U (Twig abstract: after sampling, one state is
 * rebuilt from the token-level factors).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every array is contiguous, row-major, in DEVICE memory of the current CUDA device,
 *   owned by the caller.  The library allocates nothing, never synchronises on the hot
 *   path, and enqueues all work on `stream` (NULL = legacy default stream).
 * - Every array pointer must be 16-byte aligned (TV_ERR_INVALID_ARG otherwise).
 * - Node indices are local to their sequence: sequence s owns global node rows
 *   node_offsets[s] .. node_offsets[s+1]-1, and parent[] holds local indices in
 *   topological order (parent[i] < i), -1 meaning "child of S_root".  A first-level node
 *   has depth 1.
 * - Layouts:  q, k [T][Hk][dk] (Hk = qk_heads, H by default);  v, U, out [T][H][dv];
 *   log_a, b [T][H];  parent [T];
 *   node_offsets [B+1];  S_root, S_new [B][H][dv][dk] (row v, column k);
 *   accepted_path [B][max_path] (root-first local indices, -1 padded at the tail).
 * - Errors in the arguments (NULL pointers, misalignment, bad sizes, unsupported shapes)
 *   are returned synchronously and nothing is enqueued.  Errors found in device data
 *   (a parent index outside [-1, i), inconsistent node_offsets, an accepted path that is
 *   not a root-first chain of the tree) are recorded on the device in the workspace's
 *   status word (first error wins, sticky until read); the offending sequence's outputs
 *   are then left unwritten, other sequences are unaffected.  Nothing traps or hangs.
 * - workspace: device scratch of at least tv_workspace_size() bytes, 16-byte aligned,
 *   zero-filled by the caller before its first use; it holds the device status word.
 *   One workspace may serve many calls in stream order.
 * - Stream order is kept.  The tensor-core verify kernel (dk = dv = 128) and the
 *   streaming commit kernel are launched with programmatic stream serialisation.  Their
 *   CTAs may become resident while the previous kernel on the stream drains, and may ask
 *   L2 to prefetch their first inputs then, but they load and store nothing before that
 *   kernel has completed; any sequence of library calls on one stream (commit after
 *   commit on chained or in-place states included) therefore sees plain stream order.
 *   Both kernels signal programmatic completion early.  A later kernel that the caller
 *   launches with programmatic serialisation must therefore wait for its grid dependency
 *   (griddepcontrol.wait / cudaGridDependencySynchronize) before it reads o, U or S_new.
 *   Ordinary launches and copies see the usual stream order.
 */
#ifndef TREE_VERIFY_H
#define TREE_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TV_API __attribute__((visibility("default")))
#else
#define TV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t; declared opaquely so that this header needs no CUDA include. */
typedef struct CUstream_st *tv_stream_t;

typedef enum {
  TV_OK = 0,
  TV_ERR_INVALID_ARG = 1, /* NULL / misaligned pointer, bad size or enum value          */
  TV_ERR_UNSUPPORTED = 2, /* valid but not implemented (dims, dtype, kernel choice)     */
  TV_ERR_BAD_TREE = 3,    /* device: parent[] not topological or node_offsets invalid   */
  TV_ERR_BAD_PATH = 4,    /* device: accepted_path not a root-first chain of the tree   */
  TV_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, copy, attribute)       */
  TV_ERR_TIMEOUT = 6      /* device: a bounded wait in a kernel ran out; outputs invalid */
} tv_status;

typedef enum { TV_MODE_GDN = 0, TV_MODE_SCALAR_DECAY = 1 } tv_mode;
typedef enum { TV_F32 = 0, TV_BF16 = 1 } tv_dtype;

/* Which verify kernel runs.  AUTO picks the tensor-core kernel whenever it supports the
 * problem and the CUDA-core kernel otherwise.  TC on an unsupported problem returns
 * TV_ERR_UNSUPPORTED. */
typedef enum { TV_KERNEL_AUTO = 0, TV_KERNEL_TC = 1, TV_KERNEL_SIMT = 2 } tv_kernel;

/* Problem description (all fields int32 so that the layout is fixed: 13 x 4 bytes; a
 * zero-filled struct leaves the last two fields at their defaults).
 *   B, H         sequences and (value) heads (B >= 0, H >= 1)
 *   dk, dv       key and value width: multiples of 16 in [16, 128]
 *   total_nodes  T = node_offsets[B]
 *   max_nodes    upper bound on any sequence's node count, 1..256
 *   max_path     row width of accepted_path (>= 1; commit only)
 *   mode         tv_mode
 *   in_dtype     storage type of q, k, v (TV_F32 or TV_BF16)
 *   out_dtype    storage type of out (TV_F32, or TV_BF16 when in_dtype is TV_BF16)
 *   kernel       tv_kernel (verify only)
 *   u_dtype      storage type of U (TV_F32, the default, or TV_BF16: half the bytes for the
 *                pseudo-values written by verify and read by commit; U is rounded to nearest
 *                even once it is final, so o is unaffected; not on the CUDA-core kernel, which
 *                reads its own U back)
 *   qk_heads     number of q / k heads Hk (0 = H): value head h reads q / k head
 *                h / (H / Hk), as when several value heads share one q / k head; H must be a
 *                multiple of Hk.  q and k are then [T][Hk][dk]
 * The tensor-core kernels need in_dtype = TV_BF16 and dk = dv = 128 (any max_nodes: one
 * kernel takes trees of up to 64 nodes, another wider ones; trees deeper than 16 nodes
 * in the wider kernel are verified on CUDA cores inside the same launch). */
typedef struct {
  int32_t B, H, dk, dv;
  int32_t total_nodes, max_nodes, max_path;
  int32_t mode, in_dtype, out_dtype, kernel;
  int32_t u_dtype, qk_heads;
} tv_problem;

/* Bytes of device workspace the entry points need for problem p (0 if p is invalid).
 * It is independent of the state size: O(1) today, never O(T*H*dk*dv). */
TV_API size_t tv_workspace_size(const tv_problem *p);

/* Verify every node of every tree in one call.
 *   q, k      [T][Hk][dk] in_dtype         (device, read)
 *   v         [T][H][dv] in_dtype          (device, read)
 *   log_a     [T][H] fp32, log of the decay (device, read)
 *   b         [T][H] fp32 write strength   (device, read; may be NULL in scalar mode)
 *   parent    [T] int32, local parent index (device, read)
 *   node_offsets [B+1] int32               (device, read)
 *   S_root    [B][H][dv][dk] fp32          (device, read only: verify has no side effect
 *                                            on the state)
 *   out       [T][H][dv] out_dtype, o_n = S_n q_n                (device, written)
 *   U         [T][H][dv] u_dtype pseudo-values u_n (scalar: v_n) (device, written)
 * out and U must not overlap any input.  Bit-for-bit deterministic run to run. */
TV_API tv_status tv_tree_verify(const tv_problem *p, const void *q, const void *k, const void *v,
                         const float *log_a, const float *b, const int32_t *parent,
                         const int32_t *node_offsets, const float *S_root, void *out,
                         float *U, void *workspace, size_t workspace_bytes,
                         tv_stream_t stream);

/* Rebuild the accepted state of every sequence from the pseudo-values:
 *   S_new = exp(c_m) S_root + sum_{j<=m} exp(c_m - c_j) u_{p_j} k_{p_j}^T,
 *   c_j = sum_{l<=j} log_a_{p_l}, along accepted_path p_1..p_m (root first).
 *   U          [T][H][dv] u_dtype from tv_tree_verify on the same S_root (device, read)
 *   k          [T][Hk][dk] in_dtype         (device, read)
 *   log_a      [T][H] fp32                  (device, read)
 *   S_root     [B][H][dv][dk] fp32          (device, read)
 *   node_offsets [B+1] int32                (device, read)
 *   accepted_path [B][max_path] int32, root-first local indices, -1 padded; a row of -1
 *              commits nothing (S_new = S_root)                (device, read)
 *   parent     [T] int32 or NULL.  When given, every path is checked to be a root-first
 *              chain of its tree (TV_ERR_BAD_PATH on the status word otherwise); indices
 *              are range-checked in any case.                   (device, read)
 *   S_new      [B][H][dv][dk] fp32; may be the same pointer as S_root (in place), must
 *              not partially overlap it.                          (device, written) */
TV_API tv_status tv_tree_commit(const tv_problem *p, const float *U, const void *k,
                         const float *log_a, const float *S_root,
                         const int32_t *node_offsets, const int32_t *accepted_path,
                         const int32_t *parent, float *S_new, void *workspace,
                         size_t workspace_bytes, tv_stream_t stream);

/* One decode step's commit followed by the next step's verify, against the committed state:
 *   S_new = tv_tree_commit(prev, U_prev, k_prev, log_a_prev, S_root, node_offsets_prev,
 *                          accepted_path, parent_prev)
 *   (out, U) = tv_tree_verify(next, q, k, v, log_a, b, parent, node_offsets, S_root = S_new)
 * with the results of those two calls, in one pass over the state where the shapes allow it
 * (the committed state is rebuilt in registers and verified against without being read back
 * from memory; Twig abstract: only the accepted state is rebuilt; Bole summary, worked
 * example "具体技术细节示例": only S_c3 is rebuilt, and decoding goes on from it).  That
 * single pass is taken for bf16 inputs with dk = dv = 128, next->max_nodes <= 64,
 * prev->max_path <= 32 and next->kernel AUTO or TC; otherwise the two kernels run in turn.
 *   prev       the previous step's problem (its max_path = row width of accepted_path); B, H,
 *              dk and dv must equal next's
 *   U_prev, k_prev, log_a_prev, node_offsets_prev, parent_prev (may be NULL), accepted_path:
 *              as in tv_tree_commit, for the previous step's tree          (device, read)
 *   S_root     [B][H][dv][dk] fp32, the state before the commit            (device, read)
 *   S_new      [B][H][dv][dk] fp32; may be S_root itself, must not partially overlap it
 *                                                                           (device, written)
 *   next, q, k, v, log_a, b, parent, node_offsets: as in tv_tree_verify, for the next tree
 *   out, U     as in tv_tree_verify; U must not overlap U_prev              (device, written)
 * A sequence whose next tree is empty or malformed is still committed. */
TV_API tv_status tv_tree_commit_verify(const tv_problem *prev, const float *U_prev,
                                       const void *k_prev, const float *log_a_prev,
                                       const int32_t *node_offsets_prev,
                                       const int32_t *accepted_path, const int32_t *parent_prev,
                                       const float *S_root, float *S_new, const tv_problem *next,
                                       const void *q, const void *k, const void *v,
                                       const float *log_a, const float *b, const int32_t *parent,
                                       const int32_t *node_offsets, void *out, float *U,
                                       void *workspace, size_t workspace_bytes,
                                       tv_stream_t stream);

/* Tree metadata of every node (exported for tests and for callers that cache it):
 *   depth  [T] int32: tokens on the root->n path (first-level node = 1)
 *   anc    [T][W] uint64, W = ceil(max_nodes/64): bit (i%64) of word i/64 is set iff local
 *          node i is a strict ancestor of n
 *   cumlog [T][H] fp32: cl_n = sum of log_a over the root->n path, accumulated in fp32
 *          from the root down (cl_n = cl_par(n) + log_a_n), the value the verify and
 *          commit kernels use.  All outputs are device memory, written. */
TV_API tv_status tv_tree_meta(const tv_problem *p, const int32_t *parent,
                       const int32_t *node_offsets, const float *log_a, int32_t *depth,
                       uint64_t *anc, float *cumlog, void *workspace,
                       size_t workspace_bytes, tv_stream_t stream);

/* tv_tree_verify for callers that cannot allocate device memory when they verify: code
 * running inside an allocator or memory-pool callback, serving loops that forbid
 * allocation after start-up, hosts that hand over only buffers they own.  (The pages
 * describe no such interface; this is a deployment convenience with no counterpart there.)
 * Same arguments, layouts and results as tv_tree_verify, minus the workspace: the device
 * scratch (the status word) is a fixed 4096-byte array inside this library's device image,
 * held by every GPU that loads the library until the process exits.  Nothing is
 * allocated and no allocating routine is called.
 *   scratch_out  (host, may be NULL) receives the device address of that array, which can
 *                be passed to tv_get_status to read and clear device-side errors.
 * Problems whose tv_workspace_size exceeds 4096 bytes return TV_ERR_UNSUPPORTED.
 * The first call on each device (with that device current) looks up the array's device
 * address and zeroes it; make that first call before any stream capture.  All calls on a
 * device share the one array, which keeps the last call's contents (a recorded error stays
 * until tv_get_status clears it), so calls that overlap on the GPU, from different streams
 * or threads, race on it. */
TV_API tv_status tv_tree_verify_noalloc(const tv_problem *p, const void *q, const void *k,
                                        const void *v, const float *log_a, const float *b,
                                        const int32_t *parent, const int32_t *node_offsets,
                                        const float *S_root, void *out, float *U,
                                        void **scratch_out, tv_stream_t stream);

/* The baseline the pages compare against (Twig / Bole abstracts: draft trees verified
 * sequentially, with the full recurrent state snapshotted for every node), for measuring
 * speed and transient memory against tv_tree_verify on the same GPU.  Same inputs and
 * outputs as tv_tree_verify (o and the pseudo-values U, whose meaning is identical), plus
 *   snapshots  [T][H][dv][dk] fp32: the state of every node, written  (device, written)
 * Nodes are visited in index order, each starting from its parent's snapshot.  One CTA of
 * 128 threads per (sequence, head), fp32 arithmetic on CUDA cores. */
TV_API tv_status tv_snapshot_verify(const tv_problem *p, const void *q, const void *k,
                                    const void *v, const float *log_a, const float *b,
                                    const int32_t *parent, const int32_t *node_offsets,
                                    const float *S_root, void *out, float *U, float *snapshots,
                                    void *workspace, size_t workspace_bytes, tv_stream_t stream);

/* The baseline's commit: S_new = the snapshot of each sequence's accepted path's last node
 * (S_root for an empty path), with the path checks of tv_tree_commit.  S_new must not be
 * S_root.  snapshots as written by tv_snapshot_verify on the same tree. */
TV_API tv_status tv_snapshot_commit(const tv_problem *p, const float *snapshots,
                                    const float *S_root, const int32_t *node_offsets,
                                    const int32_t *accepted_path, const int32_t *parent,
                                    float *S_new, void *workspace, size_t workspace_bytes,
                                    tv_stream_t stream);

/* Diagnostic, with no counterpart on the pages: enqueue one small kernel whose bounded
 * wait on an mbarrier phase that never completes runs out.  It then records
 * TV_ERR_TIMEOUT in `workspace`, as a verify or commit CTA does after a wait that does not
 * complete.  This is for testing the time-out path: nothing faults or hangs, and the
 * context stays usable.  A NULL, misaligned or too small workspace returns
 * TV_ERR_INVALID_ARG. */
TV_API tv_status tv_selftest_timeout(void *workspace, size_t workspace_bytes,
                                     tv_stream_t stream);

/* Synchronise `stream`, return the first device-side error recorded in `workspace` since
 * the last call (TV_OK if none) and clear it.  Not for the hot path. */
TV_API tv_status tv_get_status(void *workspace, tv_stream_t stream);

/* Name and description of the CUDA error behind the last TV_ERR_CUDA returned on the
 * calling host thread ("" if there was none).  Static storage; do not free. */
TV_API const char *tv_last_cuda_error(void);

/* Static English name of a status code. */
TV_API const char *tv_status_string(tv_status s);

/* Library ABI version, (major << 16) | minor. */
TV_API int32_t tv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TREE_VERIFY_H */
