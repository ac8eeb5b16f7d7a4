// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// Notation for one (sequence, head) item: N <= 64 nodes in topological order, path(n) =
// strict ancestors anc(n) plus n (root first, indices increase along it), cl_n = fp32 sum
// of log_a over path(n) (root first), gamma_n = exp(cl_n), D[n][i] = exp(cl_n - cl_i).
//
// The tree system (tree-structured WY form of the TreeWY abstract) is
//      (I + L) U = R,  L[n][i] = b_n D[n][i] k_n.k_i (i in anc(n)),  R_n = b_n (v_n - gamma_n S_root k_n)
// and the outputs (closed form of the Bole summary's worked example, "具体技术细节示例",
// extended to the delta rule) are  o_n = gamma_n S_root q_n + sum_i P[n][i] u_i  with
// P[n][i] = D[n][i] q_n.k_i on path(n).  With T = (I + L)^-1 and W = P T:
//      U = T R,      O = diag(gamma) S_root Q^T + W R .
// The decays factor out of both rows: T[n][i] = D[n][i] tau_i, W[n][i] = D[n][i] omega_i,
// where along path(n) = p_0 .. p_{d-1} = n (right-looking, deepest first)
//      tau_{d-1} = 1,             tau_a   = - sum_{c > a} tau_c   b_{p_c} k_{p_c}.k_{p_a}
//      omega_a = q_n.k_{p_a}                - sum_{c > a} omega_c b_{p_c} k_{p_c}.k_{p_a}
// one thread per row, in registers.  Scalar decay: T = I (U = V), W = P.
//
// The accumulator is kept transposed -- tensor-memory lane = value index, column = node --
// so that R^T can be formed in place and fed back to the tensor core from tensor memory,
// and so that every lane holds one value index of a node's output row.
// Order of work in one CTA (one item; two CTAs per SM):
//   0. before the previous kernel on the stream has completed (first resident wave): an L2
//      prefetch of the item's S_root block and node range only.
//   1. the S_root loads (64 KiB) go out first, into registers; TMA brings q, k, v in the
//      128-byte swizzled layout the MMA reads.
//   2. Gram MMA (tcgen05 kind::f16, 128 x 64 x 128): [Q ; K] . K^T into columns 128..191,
//      as soon as q and k have landed; meanwhile the tree is walked.
//   3. Gram entries by path position (they need no S_root); S_root -> bf16.
//   4-5. state MMA (kind::f16, 128 x 128 x 128): S_root . [Q ; K]^T into columns 0..127,
//      while warps 0-3 run the T and W row recursions.
//   6. per value lane: columns 0..63 scaled by gamma_n; R^T[v][j] = b_j v_j[v] -
//      b_j gamma_j (S_root k_j)[v] into columns 192..255 (tf32); [W ; T] written as the
//      shared-memory operand.
//   7. path-sum MMA (kind::tf32, A = R^T from tensor memory): columns 0..127 (o part
//      rescaled, U part zeroed in step 6) += R^T . [W ; T]^T, i.e. o^T and U^T, as two
//      N = 64 chains (W -> o, T -> U) issued by two threads.
//   8. tensor memory -> registers -> o and U node rows in shared memory -> TMA tensor
//      stores of 64, 32, ..., 1 rows, one per set bit of the tree's size.
// Trees deeper than kRegDepth take dense Gram matrices and an in-shared-memory recursion
// in step 6 instead of steps 3-4.
//
// Every wait on an mbarrier is bounded; a wait that runs out records TV_ERR_TIMEOUT on
// the status word, the CTA drains what it issued, frees its tensor memory and returns.
#include "tc_ptx.cuh"
#include "tmaps.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;                  // nodes per tree handled by this kernel
constexpr int kRegDepth = 8;               // deeper trees take the shared-memory recursion
constexpr uint32_t kTmemCols = 256;        // two CTAs per SM
constexpr uint32_t kColGram = 128;         // [Q ; K] . K^T  (lanes = q / k rows)
constexpr uint32_t kColR = 192;            // R^T            (lanes = value index)
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out
constexpr int kFuseMax = 32;               // longest accepted path of a fused commit

// Dynamic shared memory, offsets from a 1024-byte aligned base.
//   [0, 32K)    [Q ; K]: 128 rows x 128 bf16 as two 64-wide K halves of 16 KiB (TMA swizzled)
//               then [W ; T]: path-sum B operand, 128 rows x 64 fp32, two 32-wide K atoms
//   [32K, 64K)  S_root in bf16: 128 value rows x 128, two K halves
//               then (deep trees) dense q_n.k_i [32K, 48K) and b_j k_j.k_i [48K, 64K)
//   [64K, 80K)  v tile (bf16, TMA swizzled, two 64-wide value halves)
//   [80K, 84K)  root-first paths, position-major bytes: node m's a-th entry at a*64 + m
constexpr int kHalf = 128 * 128;           // one 64-wide K half of a 128-row bf16 operand
constexpr int kOffQK = 0;
constexpr int kOffA2 = 0;
constexpr int kAtom2 = 16384;              // one 32-wide K atom of the 128-row fp32 operand
constexpr int kOffS = 32768;
constexpr int kOffGQ = 32768;
constexpr int kOffLK = 49152;
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 65536;
constexpr int kOffPath = 81920;
constexpr int kOffMisc = kOffPath + kTile * kTile;

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_gram;
  unsigned long long bar_state;
  unsigned long long bar_sum;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int flag;                        // 0, or TV_ERR_TIMEOUT
  int maxdep;
  // trees no deeper than kRegDepth, position-major ([a][node]: a row-per-thread access
  // touches 32 consecutive words):
  float lpos[kRegDepth][kTile];    // b_j k_j.k_{a-th ancestor of j}
  float gpos[kRegDepth][kTile];    // q_n.k_{a-th node of path(n)}, then W[n][p_a]
  float tpos[kRegDepth][kTile];    // T[n][p_a]
  int par[kTile];
  int dep[kTile];
  float la[kTile];
  float bb[kTile];                 // b_n
  float cl[kTile];
  __align__(16) float gam[kTile];  // gamma_n
  __align__(16) float bg[kTile];   // b_n gamma_n
  __align__(16) float bq[kTile];   // b_n (copy read as float4)
  // fused commit of the previous step (kFused): its accepted path for this sequence
  int f_m, f_lo, f_stat;
  float f_gam;                     // exp(c_m)
  int f_prow[kFuseMax];            // root-first path nodes (local to the previous tree)
  float f_la[kFuseMax];            // log_a of the path nodes, then the prefix sums c_j
  float f_e[kFuseMax];             // exp(c_m - c_j)
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;

// fp32 element (row, k) of the K-major path-sum operand (128 rows, K = 64, 128-byte swizzle).
__device__ __forceinline__ int op2_off(int row, int k) {
  return ((k >> 5) * kAtom2) + (row << 7) + ((((k >> 2) & 7) ^ (row & 7)) << 4) + ((k & 3) << 2);
}
// [64][64] fp32 matrix, column XOR-swizzled by row.
__device__ __forceinline__ int coef_off(int n, int i) { return ((n << 6) + (i ^ (n & 31))) << 2; }

__device__ __forceinline__ float lds(const unsigned char *p, int off) {
  return *reinterpret_cast<const float *>(p + off);
}
__device__ __forceinline__ void sts(unsigned char *p, int off, float x) {
  *reinterpret_cast<float *>(p + off) = x;
}
// fp32 -> nearest tf32 (ties away from zero), kept in an fp32 container with the low 13
// bits clear: half a unit of the 10-bit significand is added to the magnitude bits and the
// 13 dropped bits are cleared (two integer operations; the tensor core ignores those bits).
__device__ __forceinline__ float tf32_rn(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
// Streaming 16-byte load that stays where it is written: ahead of the tree-range check.
__device__ __forceinline__ float4 ldg_first(const float4 *p) {
  float4 r;
  asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
// Tensor maps over the output rows [T][H][128] with boxes of 64, 32, 16, 8, 4, 2 and 1 node
// rows: a tree of n nodes leaves by one tensor store per set bit of n.
constexpr int kRowMaps = 7;
struct RowMaps {
  CUtensorMap m[kRowMaps];
};

// One K = 128 chain of bf16 MMAs: D = A . B^T with A and B 128-row K-major operands.
__device__ __forceinline__ void mma_chain_bf16(uint32_t a_base, uint32_t b_base, uint32_t d_tmem,
                                               uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
    ptx::mma_bf16(d_tmem, ptx::smem_desc_sw128(a_base + off, 1024),
                  ptx::smem_desc_sw128(b_base + off, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// Row m, by path position a < d:  x_a = x0_a - sum_{c > a} x_c lpos[p_c][a]
// (x0 = e_{d-1}: T row; x0 = gpos row: W row; no recursion for scalar decay), times
// D[m][p_a], rounded to tf32, stored by position (tpos, or over gpos for W).
template <bool kW, bool kGdn>
__device__ __forceinline__ void row_coefficients(Misc &ms, const uint8_t *paths, int m, int d) {
  const float clm = ms.cl[m];
  int p[kRegDepth];
  float x[kRegDepth];
#pragma unroll
  for (int a = 0; a < kRegDepth; ++a) {
    p[a] = a < d ? paths[a * kTile + m] : m;
    x[a] = kW ? (a < d ? ms.gpos[a][m] : 0.f) : (a == d - 1 ? 1.f : 0.f);
  }
#pragma unroll
  for (int c = kRegDepth - 1; c >= 1; --c) {
    if (kGdn && c < d) {
      const float xc = x[c];
#pragma unroll
      for (int a = 0; a < c; ++a) x[a] = fmaf(-xc, ms.lpos[a][p[c]], x[a]);
    }
  }
  float(*dst)[kTile] = kW ? ms.gpos : ms.tpos;
#pragma unroll
  for (int a = 0; a < kRegDepth; ++a)
    if (a < d) dst[a][m] = tf32_rn(x[a] * __expf(clm - ms.cl[p[a]]));
}

// The same for trees deeper than kRegDepth, on dense Gram matrices, in the operand row
// itself (node-indexed columns); out of line so that the register version stays small in
// the instruction cache.
template <bool kW, bool kGdn>
__device__ __noinline__ void row_coefficients_deep(unsigned char *sm, const uint8_t *paths,
                                                   const Misc &ms, int m, int d, int r2) {
  const float clm = ms.cl[m];
  for (int a = 0; a < d; ++a) {
    const int i = paths[a * kTile + m];
    sts(sm, kOffA2 + op2_off(r2, i), kW ? lds(sm, kOffGQ + coef_off(m, i)) : (a == d - 1 ? 1.f : 0.f));
  }
  if (kGdn)
    for (int c = d - 1; c >= 1; --c) {
      const int pc = paths[c * kTile + m];
      const float xc = lds(sm, kOffA2 + op2_off(r2, pc));
      for (int a = 0; a < c; ++a) {
        const int i = paths[a * kTile + m];
        const int o = kOffA2 + op2_off(r2, i);
        sts(sm, o, fmaf(-xc, lds(sm, kOffLK + coef_off(pc, i)), lds(sm, o)));
      }
    }
  for (int a = 0; a < d; ++a) {
    const int i = paths[a * kTile + m];
    const int o = kOffA2 + op2_off(r2, i);
    sts(sm, o, tf32_rn(lds(sm, o) * __expf(clm - ms.cl[i])));
  }
}

// ---- fused commit of the previous step ---------------------------------------------------
// S_new = exp(c_m) S_root + sum_j exp(c_m - c_j) u_{p_j} k_{p_j}^T along the accepted path
// p_1..p_m of the previous tree (the Bole summary's worked example rebuilds S_c3 this way;
// with the tree solve's pseudo-values the same form holds for the gated delta rule), applied
// to the S_root values this CTA holds in registers before it verifies the next tree against
// S_new.  The u and k rows of the path sit in the bf16 S_root operand region until the
// operand is written.

// One warp: the previous tree's node range and the accepted-path row of sequence s, checked.
__device__ __forceinline__ void fuse_gather_path(Misc &ms, const FuseArgs &f, int s, int B,
                                                 int lane) {
  const int lo = f.node_offsets[s], hi = f.node_offsets[s + 1];
  const bool tree_ok = !(lo < 0 || hi < lo || hi > f.T || hi - lo > f.max_nodes ||
                         (s == 0 && lo != 0) || (s == B - 1 && hi != f.T));
  const int32_t *row = f.accepted_path + (size_t)s * f.max_path;
  const int p = lane < f.max_path ? row[lane] : -1;
  // m = number of leading non-negative entries; after them only -1 may follow
  const unsigned neg = __ballot_sync(0xffffffffu, lane < f.max_path && p < 0);
  const int m = neg ? __ffs(neg) - 1 : f.max_path;
  bool bad = lane < f.max_path && (lane < m ? p >= hi - lo : p != -1);
  if (lane < m && !bad) ms.f_prow[lane] = p;
  bad = __any_sync(0xffffffffu, bad) || !tree_ok;
  if (lane == 0) {
    ms.f_m = bad ? 0 : m;
    ms.f_lo = lo;
    ms.f_stat = bad ? (tree_ok ? TV_ERR_BAD_PATH : TV_ERR_BAD_TREE) : 0;
  }
}

// All threads: the u and k rows, log_a and the parent chain of the path entries.
__device__ __forceinline__ void fuse_load_rows(unsigned char *sm, Misc &ms, const FuseArgs &f,
                                               int h, int H, int kh, int Hk, int tid) {
  const int m = ms.f_m, lo = ms.f_lo;
  float *cu = reinterpret_cast<float *>(sm + kOffS);
  float *kk = cu + kFuseMax * 128;
  const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(f.k);
  for (int idx = tid; idx < m * 128; idx += kThreads) {
    const int row = lo + ms.f_prow[idx >> 7];
    cu[idx] = load_u(f.U, ((size_t)row * H + h) * 128 + (idx & 127), f.u_bf16);
    kk[idx] = __bfloat162float(k[((size_t)row * Hk + kh) * 128 + (idx & 127)]);
  }
  if (tid < m) {
    const int p = ms.f_prow[tid];
    ms.f_la[tid] = f.log_a[(size_t)(lo + p) * H + h];
    if (f.parent && f.parent[lo + p] != (tid == 0 ? -1 : ms.f_prow[tid - 1]))
      ms.f_stat = TV_ERR_BAD_PATH;
  }
}

// One thread: fp32 prefix sums c_j root first (the order the verify kernels use for cl), the
// decay weights, and the status.
__device__ __forceinline__ void fuse_prefix(Misc &ms, int *ws, int s) {
  if (ms.f_stat) {
    set_status(ws, ms.f_stat, s);
    ms.f_m = 0;
  }
  const int m = ms.f_m;
  float c = 0.f;
  for (int j = 0; j < m; ++j) {
    c += ms.f_la[j];
    ms.f_la[j] = c;
  }
  for (int j = 0; j < m; ++j) ms.f_e[j] = expf(c - ms.f_la[j]);
  ms.f_gam = m ? expf(c) : 1.f;
}

// All threads: the update on this thread's rows v = tid/16 + 16 j, columns 8 (tid % 16) ..,
// then S_new streamed out (a malformed path leaves S_root as it is).
__device__ __forceinline__ void fuse_apply(float4 (&sr)[16], const unsigned char *sm,
                                           const Misc &ms, float *S_new, int tid) {
  const int m = ms.f_m, kc = tid & 15;
  const float g = ms.f_gam;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    sr[i].x *= g; sr[i].y *= g; sr[i].z *= g; sr[i].w *= g;
  }
  const float *cu = reinterpret_cast<const float *>(sm + kOffS);
  const float *kk = cu + kFuseMax * 128;
  for (int e = 0; e < m; ++e) {
    const float ee = ms.f_e[e];
    const float4 ka = *reinterpret_cast<const float4 *>(kk + e * 128 + kc * 8);
    const float4 kb = *reinterpret_cast<const float4 *>(kk + e * 128 + kc * 8 + 4);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float c = ee * cu[e * 128 + (tid >> 4) + 16 * j];
      sr[2 * j].x = fmaf(c, ka.x, sr[2 * j].x);
      sr[2 * j].y = fmaf(c, ka.y, sr[2 * j].y);
      sr[2 * j].z = fmaf(c, ka.z, sr[2 * j].z);
      sr[2 * j].w = fmaf(c, ka.w, sr[2 * j].w);
      sr[2 * j + 1].x = fmaf(c, kb.x, sr[2 * j + 1].x);
      sr[2 * j + 1].y = fmaf(c, kb.y, sr[2 * j + 1].y);
      sr[2 * j + 1].z = fmaf(c, kb.z, sr[2 * j + 1].z);
      sr[2 * j + 1].w = fmaf(c, kb.w, sr[2 * j + 1].w);
    }
  }
  float4 *dst = reinterpret_cast<float4 *>(S_new);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int v = (tid >> 4) + 16 * j;
    __stcs(dst + v * 32 + kc * 2, sr[2 * j]);
    __stcs(dst + v * 32 + kc * 2 + 1, sr[2 * j + 1]);
  }
}

__device__ __forceinline__ void release_tmem(int warp, uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// One thread waits on `bar`; every thread learns whether it completed.  On a time-out the
// status is recorded, the wait is retried once (bounded) and the CTA must leave.
__device__ __forceinline__ bool wait_all(Misc &ms, uint32_t bar, int tid, int *ws, int s) {
  if (tid == 0 && !ptx::mbar_wait_bounded(bar, 0, kSpinLimit)) {
    ms.flag = TV_ERR_TIMEOUT;
    set_status(ws, TV_ERR_TIMEOUT, s);
    ptx::mbar_wait_bounded(bar, 0, kSpinLimit);
  }
  __syncthreads();
  return ms.flag == 0;
}

template <bool kGdn, typename Tout, bool kFused>
__global__ void __launch_bounds__(kThreads, 2)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ RowMaps tm_o,
                     const __grid_constant__ RowMaps tm_u, VerifyArgs a, FuseArgs f,
                     int prefetch_stride) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Misc &ms = *reinterpret_cast<Misc *>(sm + kOffMisc);
  uint8_t *paths = reinterpret_cast<uint8_t *>(sm + kOffPath);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int s = blockIdx.x / H, h = blockIdx.x % H, kh = qk_head(h, H, a.Hk);
  // Launched with programmatic stream serialisation: the kernel before this one on the
  // stream may still be finishing.  Until it has (griddepcontrol.wait), a CTA of the first
  // resident wave only asks L2 for its S_root block and node range: a prefetch moves
  // nothing into the CTA, and a write by that kernel to the same lines lands in L2 after
  // it, so this is correct whatever it writes (later waves start after that kernel is done
  // and have their blocks prefetched by the wave before).  Then the kernel after this one
  // may get its CTAs resident early.
  if (threadIdx.x == 0 && (int)blockIdx.x < prefetch_stride) {
    ptx::prefetch_l2(a.S_root + (size_t)blockIdx.x * 128 * 128, 128 * 128 * 4);
    ptx::prefetch_line_l2(a.node_offsets + blockIdx.x / a.H);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- 1. S_root loads, the tree's node range, q / k / v by TMA, tree inputs ----------
  // S_root as 16 float4 per thread: thread t owns 8-element k chunk (t & 15) of value rows
  // t/16 + 16 j.  Issued before anything else; consumed in step 4.
  const int kc = tid & 15;
  float4 sr[16];
  {
    const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + ((size_t)s * H + h) * 128 * 128);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = (tid >> 4) + 16 * j;
      sr[2 * j] = ldg_first(Sg + v * 32 + kc * 2);
      sr[2 * j + 1] = ldg_first(Sg + v * 32 + kc * 2 + 1);
    }
  }
  float *const S_new_item = kFused ? f.S_new + ((size_t)s * H + h) * 128 * 128 : nullptr;
  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  const bool range_ok = !(lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
                          hi - lo > kTile || (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T));
  if (!range_ok && tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
  if (!range_ok || hi == lo) {
    if (kFused) {
      // nothing to verify in this sequence: the commit alone
      if (warp == kThreads / 32 - 1) fuse_gather_path(ms, f, s, a.B, lane);
      __syncthreads();
      fuse_load_rows(sm, ms, f, h, H, kh, a.Hk, tid);
      __syncthreads();
      if (tid == 0) fuse_prefix(ms, a.ws, s);
      __syncthreads();
      fuse_apply(sr, sm, ms, S_new_item, tid);
    }
    return;
  }
  const int n_nodes = hi - lo;

  const uint32_t sbase = ptx::smem_addr(sm);
  const uint32_t bar_tma = ptx::smem_addr(&ms.bar_tma);
  const uint32_t bar_gram = ptx::smem_addr(&ms.bar_gram);
  const uint32_t bar_state = ptx::smem_addr(&ms.bar_state);
  const uint32_t bar_sum = ptx::smem_addr(&ms.bar_sum);
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_gram, 1);
    ptx::mbar_init(bar_state, 1);
    ptx::mbar_init(bar_sum, 2);
    ptx::fence_mbar_init();
    ms.flag = 0;
    ms.maxdep = 0;
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::mbar_arrive_expect_tx(bar_tma, 6 * kTile * 128);
    for (int half = 0; half < 2; ++half) {
      const uint32_t hb = sbase + kOffQK + half * kHalf;
      ptx::tma_load_3d(hb, &tm_q, bar_tma, half * 64, kh, lo);
      ptx::tma_load_3d(hb + kTile * 128, &tm_k, bar_tma, half * 64, kh, lo);
      ptx::tma_load_3d(sbase + kOffV + half * kVHalf, &tm_v, bar_tma, half * 64, h, lo);
    }
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&ms.tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  bool bad = false;
  if (tid < kTile) {
    int p = -1;
    float la = 0.f, bb = 0.f;
    if (tid < n_nodes) {
      p = a.parent[lo + tid];
      bad = p < -1 || p >= tid;
      la = a.log_a[(size_t)(lo + tid) * H + h];
      bb = kGdn ? a.b[(size_t)(lo + tid) * H + h] : 0.f;
    }
    ms.par[tid] = p;
    ms.la[tid] = la;
    ms.bb[tid] = bb;
  }
  if (kFused && warp == kThreads / 32 - 1) fuse_gather_path(ms, f, s, a.B, lane);
  ptx::tc_fence_before();
  const bool bad_tree = __syncthreads_or(bad) != 0;
  ptx::tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  if (kFused) fuse_load_rows(sm, ms, f, h, H, kh, a.Hk, tid);   // landed by the update before step 3's conversion

  // ---- 2. Gram MMA once q / k have landed; tree walk ------------------------------------
  if (tid == kThreads - 1) {
    if (!ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit)) {
      ms.flag = TV_ERR_TIMEOUT;
    } else if (!bad_tree) {
      ptx::tc_fence_after();
      mma_chain_bf16(sbase + kOffQK, sbase + kOffQK + kTile * 128, tmem + kColGram,
                     ptx::idesc_bf16_f32(128, 64));
      ptx::mma_commit(bar_gram);
    }
  }
  if (tid < kTile) {
    // ancestors in ascending index order are the root-first path; cl summed in that order
    unsigned long long bits = 0ull;
    int d = 0;
    float cl = 0.f;
    if (!bad_tree && tid < n_nodes) {
      for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) bits |= 1ull << x;
      for (unsigned long long b = bits; b; b &= b - 1) {
        const int x = __ffsll((long long)b) - 1;
        paths[d * kTile + tid] = (uint8_t)x;
        cl += ms.la[x];
        ++d;
      }
      paths[d * kTile + tid] = (uint8_t)tid;
      cl += ms.la[tid];
      ++d;
    }
    const float gam = __expf(cl);
    ms.anc[tid] = bits;
    ms.dep[tid] = d;
    ms.cl[tid] = cl;
    ms.gam[tid] = gam;
    ms.bg[tid] = ms.bb[tid] * gam;
    ms.bq[tid] = ms.bb[tid];
    atomicMax(&ms.maxdep, d);
  }
  __syncthreads();
  if (kFused && tid == 0) fuse_prefix(ms, a.ws, s);
  if (bad_tree || ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, bad_tree ? TV_ERR_BAD_TREE : ms.flag, s);
      if (ms.flag == TV_ERR_TIMEOUT) ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit);
    }
    if (kFused) {
      __syncthreads();
      fuse_apply(sr, sm, ms, S_new_item, tid);   // the commit does not depend on the next tree
    }
    release_tmem(warp, tmem);
    return;
  }
  if (!wait_all(ms, bar_gram, tid, a.ws, s)) {
    release_tmem(warp, tmem);
    return;
  }
  ptx::tc_fence_after();
  const bool fast = ms.maxdep <= kRegDepth;

  // warp w reads tensor-memory lanes 32*(w%4)..; `set` = w/4 splits the columns in two.
  const int quarter = warp & 3, set = warp >> 2;
  const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
  // in the Gram columns, lane r is row r of [Q ; K]
  const int grow = quarter * 32 + lane;
  const bool g_is_q = grow < kTile;
  const int gn = grow & (kTile - 1);
  const bool g_live = gn < n_nodes;

  // ---- 3. Gram entries by path position: k rows b_n k_n.k_i on anc(n), q rows q_n.k_i on
  // path(n) (a node's position on a path = the number of path nodes with a smaller index)
  if (fast && (g_is_q || kGdn)) {
    const unsigned long long ancn = ms.anc[gn];
    const unsigned long long sel = !g_live ? 0ull : (g_is_q ? (ancn | (1ull << gn)) : ancn);
    const float scale = g_is_q ? 1.f : ms.bb[gn];
    float(*pos_major)[kTile] = g_is_q ? ms.gpos : ms.lpos;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float g[16];
      const int i0 = set * 32 + c * 16;
      ptx::tmem_ld16(tlane + kColGram + i0, g);
      const unsigned bits = (unsigned)(sel >> i0) & 0xFFFFu;
      int pos = __popcll(sel & ((1ull << i0) - 1ull));
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if ((bits >> j) & 1u) pos_major[pos++][gn] = scale * g[j];
    }
  }
  if (kFused) {
    // the previous step's commit, on the values in registers; S_new goes out, and the
    // verify goes on with it
    fuse_apply(sr, sm, ms, S_new_item, tid);
    __syncthreads();   // the path rows are read before the operand overwrites them
  }
  // S_root -> bf16 operand rows (all threads; the loads have long arrived by now)
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int v = (tid >> 4) + 16 * j;
    __nv_bfloat162 b0 = __floats2bfloat162_rn(sr[2 * j].x, sr[2 * j].y);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(sr[2 * j].z, sr[2 * j].w);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(sr[2 * j + 1].x, sr[2 * j + 1].y);
    __nv_bfloat162 b3 = __floats2bfloat162_rn(sr[2 * j + 1].z, sr[2 * j + 1].w);
    uint4 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&b0);
    pk.y = *reinterpret_cast<uint32_t *>(&b1);
    pk.z = *reinterpret_cast<uint32_t *>(&b2);
    pk.w = *reinterpret_cast<uint32_t *>(&b3);
    const int off = (kc >> 3) * kHalf + v * 128 + (((kc & 7) ^ (v & 7)) << 4);
    *reinterpret_cast<uint4 *>(sm + kOffS + off) = pk;
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 4. state MMA: columns 0..127 = S_root . [Q ; K]^T; meanwhile warps 0-3 run the T
  // and W row recursions of shallow trees -------------------------------------------------
  if (tid == kThreads - 1) {
    ptx::tc_fence_after();
    mma_chain_bf16(sbase + kOffS, sbase + kOffQK, tmem, ptx::idesc_bf16_f32(128, 128));
    ptx::mma_commit(bar_state);
  }
  if (fast && tid < 2 * kTile) {
    const int m = tid & (kTile - 1);
    if (m < n_nodes) {
      const int d = ms.dep[m];
      if (tid < kTile) row_coefficients<true, kGdn>(ms, paths, m, d);
      else row_coefficients<false, kGdn>(ms, paths, m, d);
    }
  }

  // ---- 5. the state product has landed (the barrier also publishes the T and W rows) -----
  if (!wait_all(ms, bar_state, tid, a.ws, s)) {
    release_tmem(warp, tmem);
    return;
  }
  ptx::tc_fence_after();
  if (tid == kThreads - 32) {
    // L2 prefetch for the CTA one resident wave ahead: its S_root block and q / k / v
    // tiles.  Issued once this CTA's own operands are consumed: earlier it competes with
    // this CTA's loads, later it arrives too late for the next CTA.
    const int nxt = blockIdx.x + prefetch_stride;
    if (nxt < a.B * H) {
      const int s2 = nxt / H, h2 = nxt % H;
      ptx::prefetch_l2(a.S_root + (size_t)nxt * 128 * 128, 128 * 128 * 4);
      const int lo2 = a.node_offsets[s2];
      if (lo2 >= 0 && lo2 < a.T)
        for (int half = 0; half < 2; ++half) {
          ptx::prefetch_tile_l2(&tm_q, half * 64, qk_head(h2, H, a.Hk), lo2);
          ptx::prefetch_tile_l2(&tm_k, half * 64, qk_head(h2, H, a.Hk), lo2);
          ptx::prefetch_tile_l2(&tm_v, half * 64, h2, lo2);
        }
    }
  }

  // ---- 6. [W ; T] operand over the dead [Q ; K] tile; gamma o^T and R^T in tensor memory --
  {
    // thread t writes K atom t/128 of operand row t%128: zeros, then its path coefficients
    const int r2 = tid & 127, atom = tid >> 7;
    const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<float4 *>(sm + kOffA2 + op2_off(r2, atom * 32 + c * 4)) = zf;
    const int n2 = r2 & (kTile - 1);
    if (fast && n2 < n_nodes) {
      const int d = ms.dep[n2];
      const float(*cf)[kTile] = r2 < kTile ? ms.gpos : ms.tpos;
#pragma unroll
      for (int a2 = 0; a2 < kRegDepth; ++a2) {
        const int i = paths[a2 * kTile + n2];
        if (a2 < d && (i >> 5) == atom) sts(sm, kOffA2 + op2_off(r2, i), cf[a2][n2]);
      }
    }
  }
  if (!fast) {
    // deep trees: dense q_n.k_i and b_n k_n.k_i over the dead S_root tile, then the row
    // recursion in the operand rows (zero-filled above)
    if (g_is_q || kGdn) {
      const unsigned long long ancn = ms.anc[gn];
      const unsigned long long sel = !g_live ? 0ull : (g_is_q ? (ancn | (1ull << gn)) : ancn);
      const float scale = g_is_q ? 1.f : ms.bb[gn];
      const int base = g_is_q ? kOffGQ : kOffLK;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float g[16];
        const int i0 = set * 32 + c * 16;
        ptx::tmem_ld16(tlane + kColGram + i0, g);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if ((sel >> (i0 + j)) & 1ull) sts(sm, base + coef_off(gn, i0 + j), scale * g[j]);
      }
    }
    __syncthreads();
    if (set == 0 && g_live) {
      const int d = ms.dep[gn];
      if (g_is_q) row_coefficients_deep<true, kGdn>(sm, paths, ms, gn, d, gn);
      else row_coefficients_deep<false, kGdn>(sm, paths, ms, gn, d, kTile + gn);
    }
  }
  {
    // lane v of columns [32 set, 32 set + 32) (o) and [64 + 32 set, ...) (S_root k_j)
    const int v = quarter * 32 + lane, j0 = set * 32;
    float o0[16], o1[16], k0[16], k1[16];
    ptx::tmem_ld16(tlane + j0, o0);
    ptx::tmem_ld16(tlane + j0 + 16, o1);
    ptx::tmem_ld16(tlane + kTile + j0, k0);
    ptx::tmem_ld16(tlane + kTile + j0 + 16, k1);
    const float4 *gam4 = reinterpret_cast<const float4 *>(&ms.gam[j0]);
    const float4 *bg4 = reinterpret_cast<const float4 *>(&ms.bg[j0]);
    const float4 *bq4 = reinterpret_cast<const float4 *>(&ms.bq[j0]);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 ga = gam4[j4], gb = gam4[4 + j4];
      o0[4 * j4] *= ga.x; o0[4 * j4 + 1] *= ga.y; o0[4 * j4 + 2] *= ga.z; o0[4 * j4 + 3] *= ga.w;
      o1[4 * j4] *= gb.x; o1[4 * j4 + 1] *= gb.y; o1[4 * j4 + 2] *= gb.z; o1[4 * j4 + 3] *= gb.w;
    }
    ptx::tmem_st16(tlane + j0, o0);
    ptx::tmem_st16(tlane + j0 + 16, o1);
    // v_j[v]: value half v/64 of node j's row in the v tile
    const unsigned char *vt = sm + kOffV + (v >> 6) * kVHalf + (v & 7) * 2;
    const int vc = (v & 63) >> 3;
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 ba = bq4[j4], bb = bq4[4 + j4], ca = bg4[j4], cb = bg4[4 + j4];
      const float bja[4] = {ba.x, ba.y, ba.z, ba.w}, bjb[4] = {bb.x, bb.y, bb.z, bb.w};
      const float cja[4] = {ca.x, ca.y, ca.z, ca.w}, cjb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * j4 + e, ja = j0 + j, jb = j0 + 16 + j;
        const float va = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(vt + ja * 128 + ((vc ^ (ja & 7)) << 4)));
        const float vb = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(vt + jb * 128 + ((vc ^ (jb & 7)) << 4)));
        k0[j] = ja < n_nodes ? tf32_rn(kGdn ? fmaf(-cja[e], k0[j], bja[e] * va) : va) : 0.f;
        k1[j] = jb < n_nodes ? tf32_rn(kGdn ? fmaf(-cjb[e], k1[j], bjb[e] * vb) : vb) : 0.f;
      }
    }
    ptx::tmem_st16(tlane + kColR + j0, k0);
    ptx::tmem_st16(tlane + kColR + j0 + 16, k1);
    // the U columns start from zero
#pragma unroll
    for (int j = 0; j < 16; ++j) k0[j] = 0.f;
    ptx::tmem_st16(tlane + kTile + j0, k0);
    ptx::tmem_st16(tlane + kTile + j0 + 16, k0);
  }
  ptx::tmem_wait_st();
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 7. path-sum MMA: columns 0..127 += R^T . [W ; T]^T (tf32), i.e. o^T and U^T ------
  // two chains of N = 64 issued by two threads: W rows into the o columns, T rows into the
  // U columns (rows 64.. of each K atom start 8 KiB into it)
  if (tid == kThreads - 1 || tid == kThreads - 33) {
    ptx::tc_fence_after();
    const uint32_t half = tid == kThreads - 1 ? 0u : 1u;
    constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 64);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      ptx::mma_tf32_tmem_a(tmem + half * kTile, tmem + kColR + kk * 8,
                           ptx::smem_desc_sw128(sbase + kOffA2 + half * (kTile * 128) + (kk >> 2) * kAtom2 + (kk & 3) * 32, 1024),
                           idesc, 1u);
    ptx::mma_commit(bar_sum);
  }
  if (!wait_all(ms, bar_sum, tid, a.ws, s)) {
    release_tmem(warp, tmem);
    return;
  }
  ptx::tc_fence_after();

  // ---- 8. o^T and U^T -> node rows in shared memory (a warp's 32 lanes are 32 adjacent v) --
  {
    const int v = quarter * 32 + lane, j0 = set * 32;
    float o0[16], o1[16], u0[16], u1[16];
    ptx::tmem_ld16(tlane + j0, o0);
    ptx::tmem_ld16(tlane + j0 + 16, o1);
    ptx::tmem_ld16(tlane + kTile + j0, u0);
    ptx::tmem_ld16(tlane + kTile + j0 + 16, u1);
    ptx::tmem_wait_ld();
    release_tmem(warp, tmem);
    // node rows into shared memory (o over the dead [W ; T] operand, U over the dead S_root
    // operand), then tensor stores of 64, 32, ..., 1 rows, one per set bit of n_nodes; the
    // CTA leaves once they have been read out of shared memory
    Tout *ost = reinterpret_cast<Tout *>(sm + kOffA2);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ost[(j0 + j) * 128 + v] = from_f32<Tout>(o0[j]);
      ost[(j0 + 16 + j) * 128 + v] = from_f32<Tout>(o1[j]);
    }
    if (a.u_bf16) {
      __nv_bfloat16 *ust = reinterpret_cast<__nv_bfloat16 *>(sm + kOffS);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ust[(j0 + j) * 128 + v] = __float2bfloat16_rn(u0[j]);
        ust[(j0 + 16 + j) * 128 + v] = __float2bfloat16_rn(u1[j]);
      }
    } else {
      float *ust = reinterpret_cast<float *>(sm + kOffS);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ust[(j0 + j) * 128 + v] = u0[j];
        ust[(j0 + 16 + j) * 128 + v] = u1[j];
      }
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      const uint32_t orow = 128 * sizeof(Tout), urow = a.u_bf16 ? 256u : 512u;
      int j = 0;
      for (int i = 0; i < kRowMaps; ++i) {
        const int r = kTile >> i;
        if (n_nodes & r) {
          ptx::tma_store_3d(&tm_o.m[i], sbase + kOffA2 + j * orow, 0, h, lo + j);
          ptx::tma_store_3d(&tm_u.m[i], sbase + kOffS + j * urow, 0, h, lo + j);
          j += r;
        }
      }
      ptx::bulk_commit();
      ptx::bulk_wait_read();
    }
  }
}

// ---- host side ------------------------------------------------------------------------
template <bool kGdn, typename Tout, bool kFused>
cudaError_t launch_tc_t(const VerifyArgs &a, const FuseArgs &f, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  RowMaps mo, mu;
  // (a next tree with no nodes at all still gets maps over a one-row view: the kernel only
  // commits then)
  const int rows = a.T > 0 ? a.T : 1;
  if (!make_node_map(&mq, a.q, a.Hk, rows, kTile) || !make_node_map(&mk, a.k, a.Hk, rows, kTile) ||
      !make_node_map(&mv, a.v, a.H, rows, kTile))
    return cudaErrorInvalidValue;
  for (int i = 0; i < kRowMaps; ++i)
    if (!make_row_map(&mo.m[i], a.out, sizeof(Tout) == 2, a.H, rows, kTile >> i) ||
        !make_row_map(&mu.m[i], a.U, a.u_bf16 != 0, a.H, rows, kTile >> i))
      return cudaErrorInvalidValue;
  auto kern = verify_tc_kernel<kGdn, Tout, kFused>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the CTA one resident wave ahead (two per SM) gets its inputs prefetched into L2
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.H);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, mu, a, f, 2 * sms);
}

}  // namespace

int verify_tc_max_nodes() { return kTile; }
int fused_max_path() { return kFuseMax; }

cudaError_t launch_verify_tc(const VerifyArgs &a, int mode, int out_dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;   // every tree is empty
  const bool gdn = mode == TV_MODE_GDN;
  const FuseArgs f = {};
  if (out_dtype == TV_BF16)
    return gdn ? launch_tc_t<true, __nv_bfloat16, false>(a, f, st)
               : launch_tc_t<false, __nv_bfloat16, false>(a, f, st);
  return gdn ? launch_tc_t<true, float, false>(a, f, st) : launch_tc_t<false, float, false>(a, f, st);
}

cudaError_t launch_commit_verify_tc(const VerifyArgs &a, const FuseArgs &f, int mode,
                                    int out_dtype, cudaStream_t st) {
  const bool gdn = mode == TV_MODE_GDN;
  if (out_dtype == TV_BF16)
    return gdn ? launch_tc_t<true, __nv_bfloat16, true>(a, f, st)
               : launch_tc_t<false, __nv_bfloat16, true>(a, f, st);
  return gdn ? launch_tc_t<true, float, true>(a, f, st) : launch_tc_t<false, float, true>(a, f, st);
}

}  // namespace tv
