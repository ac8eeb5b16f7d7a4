// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// Notation for one (sequence, head) item: N <= 64 nodes in topological order, path(n) =
// strict ancestors anc(n) plus n (root first, indices increase along it), cl_n = fp32 sum
// of log_a over path(n) (root first), gamma_n = exp(cl_n), D[n][i] = exp(cl_n - cl_i).
//
// MMA 1 (tcgen05 kind::f16, 128 x 192 x 128, bf16 in, fp32 accumulate in TMEM):
//      [ Q ] . [ K ; S_root ]^T  ->  [ Q K^T | (S_root Q^T)^T ]   lanes 0..63
//      [ K ]                         [ K K^T | (S_root K^T)^T ]   lanes 64..127
// gives both path Gram blocks and both state products.  q, k, v arrive by TMA in the
// 128-byte swizzled layout the MMA reads; S_root (fp32 in HBM) is converted to bf16 by all
// threads straight into the same layout.
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
// MMA 2 (kind::tf32, 128 x 128 x 64, operands rounded to nearest tf32) accumulates
// [ W ; T ] . R onto accumulator columns 64..191, which by then hold gamma_n S_root q_n
// (q lanes, rescaled in place) and zeros (k lanes): the accumulator ends as [ O ; U ].
// It leaves through a swizzled shared tile as coalesced 512-byte rows.
//
// Two CTAs (about 104 KiB of shared memory each) share an SM so that one's loads overlap
// the other's math.  Every wait on an mbarrier is bounded; a wait that runs out records
// TV_ERR_TIMEOUT on the status word, the CTA drains what it issued, frees its tensor
// memory and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;                  // nodes per tree handled by this kernel
constexpr int kRegDepth = 8;               // deeper paths take the shared-memory recursion
constexpr uint32_t kTmemCols = 256;        // accumulator columns 0..191; two CTAs per SM
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out

// Dynamic shared memory, offsets from a 1024-byte aligned base.
//   [0, 64K)    MMA 1 operands: two 64-wide K halves of [Q ; K ; S_root] (256 rows x 128 B)
//               then  R^T (MMA 2 B operand, K-major, 128 x 64 fp32)       [0, 32K)
//                     [W ; T] (MMA 2 A operand, K-major, 128 x 64 fp32)   [32K, 64K)
//               then  O tile [0, 32K) and U tile [32K, 64K) (64 x 128 fp32 each)
//   [64K, 80K)  v tile (bf16, TMA swizzled), then q_n.k_i on paths (64 x 64 fp32)
//   [80K, 96K)  b_j k_j.k_i on paths (64 x 64 fp32)
//   [96K, 100K) root-first paths, position-major bytes: node m's a-th entry at a*64 + m
constexpr int kOpHalf = 256 * 128;
constexpr int kOffOp = 0;
constexpr int kOffB2 = 0;
constexpr int kOffA2 = 32768;
constexpr int kAtom2 = 16384;              // one 32-wide K atom of a 128-row MMA 2 operand
constexpr int kOffOt = 0;
constexpr int kOffUt = 32768;
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 65536;
constexpr int kOffGQ = 65536;
constexpr int kOffLK = 81920;
constexpr int kOffPath = 98304;
constexpr int kOffMisc = kOffPath + kTile * kTile;

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_mma1;
  unsigned long long bar_mma2;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int flag;                        // 0, or a tv_status to record for this item
  int maxdep;
  // trees no deeper than kRegDepth keep the path Gram entries by path position:
  float lpos[kTile][kRegDepth];    // b_j k_j.k_{a-th ancestor of j}
  float gpos[kTile][kRegDepth];    // q_n.k_{a-th node of path(n)}
  int par[kTile];
  int dep[kTile];
  float la[kTile];
  float bb[kTile];
  float cl[kTile];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;

// fp32 [64][128] tile in four 32-column slabs of 128-byte rows with 16-byte chunks
// XOR-swizzled by row: row-per-thread writes and row-per-warp reads are conflict-free.
__device__ __forceinline__ int tile_off(int n, int v) {
  return ((v >> 5) << 13) + (n << 7) + ((((v >> 2) & 7) ^ (n & 7)) << 4) + ((v & 3) << 2);
}
// fp32 element (row, k) of a K-major MMA 2 operand (128 rows, K = 64, 128-byte swizzle).
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
// fp32 -> nearest tf32 (ties away), kept in an fp32 container with the low 13 bits clear.
__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Row m of [W ; T] (A2 row `r2`): x_a for path positions a < d,
//   x_a = x0_a - sum_{c > a} x_c lk[p_c][p_a]   (x0 = e_{d-1}: T row; x0 = gq row: W row)
// (no recursion for scalar decay, where L = 0), times D[m][p_a], rounded to tf32 and
// stored at column p_a.  Trees deeper than kRegDepth run this in the A2 row itself on
// dense Gram matrices, out of line so that the register version below (compact,
// position-indexed Gram entries) stays small in the instruction cache.
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

template <bool kW, bool kGdn>
__device__ __forceinline__ void row_coefficients(unsigned char *sm, const uint8_t *paths,
                                                 const Misc &ms, int m, int d, int r2) {
  const float clm = ms.cl[m];
  int p[kRegDepth];
  float x[kRegDepth];
#pragma unroll
  for (int a = 0; a < kRegDepth; ++a) {
    p[a] = a < d ? paths[a * kTile + m] : m;
    x[a] = kW ? (a < d ? ms.gpos[m][a] : 0.f) : (a == d - 1 ? 1.f : 0.f);
  }
#pragma unroll
  for (int c = kRegDepth - 1; c >= 1; --c) {
    if (kGdn && c < d) {
      const float xc = x[c];
#pragma unroll
      for (int a = 0; a < c; ++a) x[a] = fmaf(-xc, ms.lpos[p[c]][a], x[a]);
    }
  }
#pragma unroll
  for (int a = 0; a < kRegDepth; ++a)
    if (a < d) sts(sm, kOffA2 + op2_off(r2, p[a]), tf32_rn(x[a] * __expf(clm - ms.cl[p[a]])));
}

__device__ __forceinline__ void release_tmem(int warp, uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool kGdn, typename Tout>
__global__ void __launch_bounds__(kThreads, 2)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, VerifyArgs a,
                     int prefetch_stride) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Misc &ms = *reinterpret_cast<Misc *>(sm + kOffMisc);
  uint8_t *paths = reinterpret_cast<uint8_t *>(sm + kOffPath);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int s = blockIdx.x / H, h = blockIdx.x % H;

  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes || hi - lo > kTile ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n_nodes = hi - lo;
  if (n_nodes == 0) return;

  const uint32_t sbase = ptx::smem_addr(sm);
  const uint32_t bar_tma = ptx::smem_addr(&ms.bar_tma);
  const uint32_t bar_mma1 = ptx::smem_addr(&ms.bar_mma1);
  const uint32_t bar_mma2 = ptx::smem_addr(&ms.bar_mma2);

  // ---- 1. TMA of q / k / v, tensor memory, S_root -> bf16 operand rows 128..255 --------
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_mma1, 1);
    ptx::mbar_init(bar_mma2, 1);
    ptx::fence_mbar_init();
    ms.flag = 0;
    ms.maxdep = 0;
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::mbar_arrive_expect_tx(bar_tma, 6 * kTile * 128);
    for (int half = 0; half < 2; ++half) {
      const uint32_t hb = sbase + kOffOp + half * kOpHalf;
      ptx::tma_load_3d(hb, &tm_q, bar_tma, half * 64, h, lo);
      ptx::tma_load_3d(hb + kTile * 128, &tm_k, bar_tma, half * 64, h, lo);
      ptx::tma_load_3d(sbase + kOffV + half * kVHalf, &tm_v, bar_tma, half * 64, h, lo);
    }
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&ms.tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  bool bad = false;
  {
    const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + ((size_t)s * H + h) * 128 * 128);
    const int kc = tid & 15;                 // 8-element chunk of k owned by this thread
    float4 r[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = (tid >> 4) + 16 * j;
      r[2 * j] = __ldcs(Sg + v * 32 + kc * 2);
      r[2 * j + 1] = __ldcs(Sg + v * 32 + kc * 2 + 1);
    }
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
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = (tid >> 4) + 16 * j, row = 128 + v;
      __nv_bfloat162 b0 = __floats2bfloat162_rn(r[2 * j].x, r[2 * j].y);
      __nv_bfloat162 b1 = __floats2bfloat162_rn(r[2 * j].z, r[2 * j].w);
      __nv_bfloat162 b2 = __floats2bfloat162_rn(r[2 * j + 1].x, r[2 * j + 1].y);
      __nv_bfloat162 b3 = __floats2bfloat162_rn(r[2 * j + 1].z, r[2 * j + 1].w);
      uint4 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&b0);
      pk.y = *reinterpret_cast<uint32_t *>(&b1);
      pk.z = *reinterpret_cast<uint32_t *>(&b2);
      pk.w = *reinterpret_cast<uint32_t *>(&b3);
      const int off = (kc >> 3) * kOpHalf + row * 128 + (((kc & 7) ^ (row & 7)) << 4);
      *reinterpret_cast<uint4 *>(sm + kOffOp + off) = pk;
    }
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  const bool bad_tree = __syncthreads_or(bad) != 0;
  ptx::tc_fence_after();
  const uint32_t tmem = ms.tmem_base;

  // ---- 2. MMA 1 (one thread) while the tree metadata is formed -------------------------
  if (tid == kThreads - 1) {
    if (!ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit)) {
      ms.flag = TV_ERR_TIMEOUT;
    } else if (!bad_tree) {
      ptx::tc_fence_after();
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 192);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t base = sbase + kOffOp + (kk >> 2) * kOpHalf + (kk & 3) * 32;
        ptx::mma_bf16(tmem, ptx::smem_desc_sw128(base, 1024),
                      ptx::smem_desc_sw128(base + kTile * 128, 1024), idesc, kk > 0 ? 1u : 0u);
      }
      ptx::mma_commit(bar_mma1);
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
    ms.anc[tid] = bits;
    ms.dep[tid] = d;
    ms.cl[tid] = cl;
    atomicMax(&ms.maxdep, d);
  }
  __syncthreads();
  if (bad_tree || ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, bad_tree ? TV_ERR_BAD_TREE : ms.flag, s);
      if (ms.flag == TV_ERR_TIMEOUT) ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit);
    }
    release_tmem(warp, tmem);
    return;
  }
  if (tid == 0 && !ptx::mbar_wait_bounded(bar_mma1, 0, kSpinLimit)) ms.flag = TV_ERR_TIMEOUT;
  __syncthreads();
  if (ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, ms.flag, s);
      ptx::mbar_wait_bounded(bar_mma1, 0, kSpinLimit);
    }
    release_tmem(warp, tmem);
    return;
  }
  ptx::tc_fence_after();
  const bool fast = ms.maxdep <= kRegDepth;   // compact Gram entries, register recursion

  // ---- 3. accumulator 1 -> R (k lanes), gamma S_root q in place (q lanes), Gram ---------
  if (tid == kThreads - 32) {
    // L2 prefetch for the CTA one resident wave ahead: its S_root block and q / k / v
    // tiles.  Issued once this CTA's own operands are consumed (MMA 1 done): earlier it
    // competes with this CTA's loads, later it arrives too late for the next CTA.
    const int nxt = blockIdx.x + prefetch_stride;
    if (nxt < a.B * H) {
      const int s2 = nxt / H, h2 = nxt % H;
      ptx::prefetch_l2(a.S_root + (size_t)nxt * 128 * 128, 128 * 128 * 4);
      const int lo2 = a.node_offsets[s2];
      if (lo2 >= 0 && lo2 < a.T)
        for (int half = 0; half < 2; ++half) {
          ptx::prefetch_tile_l2(&tm_q, half * 64, h2, lo2);
          ptx::prefetch_tile_l2(&tm_k, half * 64, h2, lo2);
          ptx::prefetch_tile_l2(&tm_v, half * 64, h2, lo2);
        }
    }
  }
  // warp w owns TMEM lanes 32*(w%4)..; warps 0-3 take value columns 0..63 and Gram
  // columns 0..31, warps 4-7 value columns 64..127 and Gram columns 32..63.
  const int quarter = warp & 3, set = warp >> 2;
  const int row = quarter * 32 + lane;
  const bool is_q = row < kTile;
  const int n = is_q ? row : row - kTile;
  const bool live = n < n_nodes;
  const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
  const unsigned long long ancn = ms.anc[n];
  {
    const float gam = __expf(ms.cl[n]);
    const float bn = ms.bb[n];
    const unsigned char *vt = sm + kOffV;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float x[16];
      const int v0 = set * 64 + c * 16;
      ptx::tmem_ld16(trow + 64 + v0, x);
      if (is_q) {
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) x[j] *= gam;
        ptx::tmem_st16(trow + 64 + v0, x);
      } else {
        const int half = v0 >> 6, ch = (v0 & 63) >> 3;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(
            vt + half * kVHalf + (n << 7) + ((ch ^ (n & 7)) << 4));
        const uint4 w1 = *reinterpret_cast<const uint4 *>(
            vt + half * kVHalf + (n << 7) + (((ch + 1) ^ (n & 7)) << 4));
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        ptx::tmem_wait_ld();
        const float bg = bn * gam;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float vn = __uint_as_float(((wv[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu) << 16);
          x[j] = live ? tf32_rn(kGdn ? fmaf(-bg, x[j], bn * vn) : vn) : 0.f;
        }
        // column n of R^T: a warp's 32 nodes fill one 128-byte swizzle row per value v
#pragma unroll
        for (int j = 0; j < 16; ++j) sts(sm, kOffB2 + op2_off(v0 + j, n), x[j]);
        float z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0.f;
        ptx::tmem_st16(trow + 64 + v0, z);
      }
    }
    // Gram entries: k lanes b_n k_n.k_i on anc(n) (gated delta only); q lanes (compact
    // form only) q_n.k_i on path(n).  Position of node i on a path = ancestors below i.
    if (is_q ? fast : kGdn) {
      const unsigned long long sel = !live ? 0ull : (is_q ? (ancn | (1ull << n)) : ancn);
      const float scale = is_q ? 1.f : bn;
      float *posrow = is_q ? &ms.gpos[n][0] : &ms.lpos[n][0];
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float g[16];
        const int i0 = set * 32 + c * 16;
        ptx::tmem_ld16(trow + i0, g);
        const unsigned bits = (unsigned)(sel >> i0) & 0xFFFFu;
        int pos = __popcll(sel & ((1ull << i0) - 1ull));   // path position of column i0
        ptx::tmem_wait_ld();
        if (!fast) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if ((bits >> j) & 1u) sts(sm, kOffLK + coef_off(n, i0 + j), scale * g[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if ((bits >> j) & 1u) posrow[pos++] = scale * g[j];
        }
      }
    }
    // [W ; T] starts as zeros
    const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4 *>(sm + kOffA2 + (tid + j * kThreads) * 16) = zf;
  }
  ptx::tmem_wait_st();
  ptx::tc_fence_before();
  __syncthreads();
  if (!fast) {
  if (is_q) {   // dense q_n.k_i on path(n), into the now free v tile
    ptx::tc_fence_after();
    const unsigned long long sel = live ? (ancn | (1ull << n)) : 0ull;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float g[16];
      const int i0 = set * 32 + c * 16;
      ptx::tmem_ld16(trow + i0, g);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if ((sel >> (i0 + j)) & 1ull) sts(sm, kOffGQ + coef_off(n, i0 + j), g[j]);
    }
  }
  __syncthreads();
  }

  // ---- 4. rows of W (warps 0-1) and T (warps 2-3) by the path recursion ---------------
  if (set == 0 && live) {
    const int d = ms.dep[n];
    if (fast) {
      if (is_q) row_coefficients<true, kGdn>(sm, paths, ms, n, d, n);
      else row_coefficients<false, kGdn>(sm, paths, ms, n, d, kTile + n);
    } else {
      if (is_q) row_coefficients_deep<true, kGdn>(sm, paths, ms, n, d, n);
      else row_coefficients_deep<false, kGdn>(sm, paths, ms, n, d, kTile + n);
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 5. MMA 2: accumulator columns 64..191 += [W ; T] . R  (tf32) --------------------
  if (tid == kThreads - 1) {
    ptx::tc_fence_after();
    constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t koff = (kk >> 2) * kAtom2 + (kk & 3) * 32;
      ptx::mma_tf32(tmem + 64, ptx::smem_desc_sw128(sbase + kOffA2 + koff, 1024),
                    ptx::smem_desc_sw128(sbase + kOffB2 + koff, 1024), idesc, 1u);
    }
    ptx::mma_commit(bar_mma2);
  }
  if (tid == 0 && !ptx::mbar_wait_bounded(bar_mma2, 0, kSpinLimit)) ms.flag = TV_ERR_TIMEOUT;
  __syncthreads();
  if (ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, ms.flag, s);
      ptx::mbar_wait_bounded(bar_mma2, 0, kSpinLimit);
    }
    release_tmem(warp, tmem);
    return;
  }
  ptx::tc_fence_after();

  // ---- 6. accumulator -> O / U tiles -> coalesced rows ---------------------------------
  {
    unsigned char *tile = sm + (is_q ? kOffOt : kOffUt);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float y[16];
      const int v0 = set * 64 + c * 16;
      ptx::tmem_ld16(trow + 64 + v0, y);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4 *>(tile + tile_off(n, v0 + j)) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
    }
  }
  release_tmem(warp, tmem);
  // coalesced rows: a warp writes one 512-byte row of o or U per instruction
  Tout *out = static_cast<Tout *>(a.out);
  const int v4 = lane * 4;
  for (int r = warp; r < 2 * n_nodes; r += kThreads / 32) {
    const bool is_u = r >= n_nodes;
    const int m = is_u ? r - n_nodes : r;
    const float4 x = *reinterpret_cast<const float4 *>(sm + (is_u ? kOffUt : kOffOt) + tile_off(m, v4));
    const size_t g = ((size_t)(lo + m) * H + h) * 128 + v4;
    if (is_u) {
      __stcs(reinterpret_cast<float4 *>(a.U + g), x);
    } else if (sizeof(Tout) == 4) {
      __stcs(reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + g), x);
    } else {
      __nv_bfloat162 l2 = __floats2bfloat162_rn(x.x, x.y), h2 = __floats2bfloat162_rn(x.z, x.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&l2);
      pk.y = *reinterpret_cast<uint32_t *>(&h2);
      *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(out) + g) = pk;
    }
  }
}

// ---- host side ------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [T][H][128] bf16 viewed as a 3-D tensor (128, H, T); box = 64 elements x 1 head x 64 nodes.
bool make_map(CUtensorMap *m, const void *ptr, int H, int T) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kGdn, typename Tout>
cudaError_t launch_tc_t(const VerifyArgs &a, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.H, a.T) || !make_map(&mk, a.k, a.H, a.T) ||
      !make_map(&mv, a.v, a.H, a.T))
    return cudaErrorInvalidValue;
  auto kern = verify_tc_kernel<kGdn, Tout>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the CTA one resident wave ahead (two per SM) gets its inputs prefetched into L2
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kern<<<a.B * a.H, kThreads, kSmemBytes, st>>>(mq, mk, mv, a, 2 * sms);
  return cudaGetLastError();
}

}  // namespace

int verify_tc_max_nodes() { return kTile; }

cudaError_t launch_verify_tc(const VerifyArgs &a, int mode, int out_dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;   // every tree is empty
  const bool gdn = mode == TV_MODE_GDN;
  if (out_dtype == TV_BF16)
    return gdn ? launch_tc_t<true, __nv_bfloat16>(a, st) : launch_tc_t<false, __nv_bfloat16>(a, st);
  return gdn ? launch_tc_t<true, float>(a, st) : launch_tc_t<false, float>(a, st);
}

}  // namespace tv
