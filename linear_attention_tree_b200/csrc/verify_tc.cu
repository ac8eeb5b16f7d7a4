// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// One CTA (256 threads, two per SM) per (sequence, head).  Notation: N <= 64 nodes in
// topological order, path(n) = strict ancestors anc(n) plus n, cl_n = fp32 sum of log_a
// over path(n) (root first), gamma_n = exp(cl_n), D[n][i] = exp(cl_n - cl_i).
//
// MMA 1 (tcgen05 kind::f16, 128 x 192 x 128, bf16 in, fp32 accumulate in TMEM):
//      [ Q ] . [ K ; S_root ]^T  ->  [ Q K^T | (S_root Q^T)^T ]   rows 0..63
//      [ K ]                         [ K K^T | (S_root K^T)^T ]   rows 64..127
// gives both path Gram blocks and both state products at once.  q, k, v arrive by TMA in
// the 128-byte swizzled layout the MMA reads; S_root (fp32 in HBM) is converted to bf16 by
// all threads straight into the same layout.
//
// The tree system (tree-structured WY form of the TreeWY abstract) is
//      (I + L) U = R,  L[n][i] = b_n D[n][i] k_n.k_i (i in anc(n)),  R_n = b_n (v_n - gamma_n S_root k_n)
// and the outputs (closed form of the Bole summary's worked example, "具体技术细节示例",
// extended to the delta rule) are  O = diag(gamma) S_root Q^T + P U  with
// P[n][i] = D[n][i] q_n.k_i on path(n).  With T = (I + L)^-1 and W = P T:
//      U = R + (T - I) R,      O = diag(gamma) S_root Q^T + W R .
// Rows of T and W live on the node's own path and follow from L alone by a backward
// recursion over that path (T (I + L) = I, W (I + L) = P), so every node's row is one
// thread's work with no synchronisation.  MMA 2 (kind::tf32, 128 x 128 x 64) then forms
//      [ W ; T - I ] . R   in TMEM, and the epilogue adds gamma S_root q_n and R.
// Scalar decay is the special case L = 0 (T = I, W = P, U = R = V).
//
// Every wait on an mbarrier is bounded; a wait that runs out records TV_ERR_TIMEOUT on
// the status word, the CTA frees its tensor memory and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;                  // nodes per tree handled by this kernel
constexpr uint32_t kTmemCols = 256;        // two CTAs per SM share the 512 columns
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out

// Dynamic shared memory, offsets from a 1024-byte aligned base.
//   [0, 64K)    MMA 1 operands: two 64-wide K halves of [Q ; K ; S_root] (256 rows x 128 B)
//               then B2 = R^T  [0, 32K)  and A2 = [W ; T - I]  [32K, 64K)   (MMA 2, fp32)
//               then the U tile in [32K, 64K)
//   [64K, 80K)  v tile (bf16, TMA swizzled)     then first half of the O tile
//   [80K, 96K)  L coefficients (64 x 64 fp32)   then second half of the O tile
constexpr int kOpHalf = 256 * 128;
constexpr int kOffOp = 0;
constexpr int kOffB2 = 0;
constexpr int kOffA2 = 32768;
constexpr int kAtom2 = 16384;              // one 32-wide K atom of a 128-row fp32 operand
constexpr int kOffUt = 32768;
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 2 * kOpHalf;
constexpr int kOffL = kOffV + 2 * kVHalf;
constexpr int kOffOt = kOffV;
constexpr int kOffMisc = kOffL + kTile * kTile * 4;

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_mma1;
  unsigned long long bar_mma2;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int flag;                        // 0 ok, else a tv_status to record
  int par[kTile];
  float la[kTile];
  float bb[kTile];
  float cl[kTile];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;

// fp32 [64][128] tile in four 32-column slabs of 128-byte rows with 16-byte chunks
// XOR-swizzled by row: row-per-thread and column-per-thread accesses are conflict-free.
__device__ __forceinline__ int tile_off(int n, int v) {
  return ((v >> 5) << 13) + (n << 7) + ((((v >> 2) & 7) ^ (n & 7)) << 4) + ((v & 3) << 2);
}
// fp32 element (row, k) of a 128-row K-major operand with 128-byte swizzle (32 fp32 per
// swizzle row, two K atoms for K = 64).
__device__ __forceinline__ int op2_off(int row, int k) {
  return ((k >> 5) * kAtom2) + (row << 7) + ((((k >> 2) & 7) ^ (row & 7)) << 4) + ((k & 3) << 2);
}
// [64][64] fp32 coefficients, column XOR-swizzled by row.
__device__ __forceinline__ int coef_off(int n, int i) { return (n << 6) + (i ^ (n & 31)); }

__device__ __forceinline__ float lds(const unsigned char *sm, int off) {
  return *reinterpret_cast<const float *>(sm + off);
}
__device__ __forceinline__ void sts(unsigned char *sm, int off, float x) {
  *reinterpret_cast<float *>(sm + off) = x;
}

__device__ __forceinline__ void cleanup_and_exit(Misc &ms, int warp, uint32_t tmem) {
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
                     const __grid_constant__ CUtensorMap tm_v, VerifyArgs a) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Misc &ms = *reinterpret_cast<Misc *>(sm + kOffMisc);
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

  const uint32_t bar_tma = ptx::smem_addr(&ms.bar_tma);
  const uint32_t bar_mma1 = ptx::smem_addr(&ms.bar_mma1);
  const uint32_t bar_mma2 = ptx::smem_addr(&ms.bar_mma2);
  const uint32_t sbase = ptx::smem_addr(sm);

  // ---- 1. barriers, TMA of q / k / v, TMEM allocation ---------------------------------
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_mma1, 1);
    ptx::mbar_init(bar_mma2, 1);
    ptx::fence_mbar_init();
    ms.flag = 0;
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

  // ---- 2. S_root fp32 -> bf16 into rows 128..255 of the operand tile -------------------
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
        if (p < -1 || p >= tid) ms.flag = TV_ERR_BAD_TREE;
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
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ms.tmem_base;

  // ---- 3. MMA 1 (one thread) while the tree metadata is formed -------------------------
  if (tid == kThreads - 1) {
    if (!ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit)) {
      ms.flag = TV_ERR_TIMEOUT;
    } else if (ms.flag == 0) {
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
    // strict ancestors by walking up; cl summed root first (ancestor indices increase with
    // depth, so ascending bit order is path order)
    unsigned long long bits = 0ull;
    float cl = 0.f;
    if (tid < n_nodes && ms.flag != TV_ERR_BAD_TREE) {
      for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) bits |= 1ull << x;
      for (unsigned long long b = bits; b; b &= b - 1) cl += ms.la[__ffsll((long long)b) - 1];
      cl += ms.la[tid];
    }
    ms.anc[tid] = bits;
    ms.cl[tid] = cl;
  }
  __syncthreads();
  if (ms.flag != 0) {
    if (tid == 0) set_status(a.ws, ms.flag, s);
    cleanup_and_exit(ms, warp, tmem);
    return;
  }
  if (tid == 0 && !ptx::mbar_wait_bounded(bar_mma1, 0, kSpinLimit)) ms.flag = TV_ERR_TIMEOUT;
  __syncthreads();
  if (ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, ms.flag, s);
      ptx::mbar_wait_bounded(bar_mma1, 0, kSpinLimit);
    }
    cleanup_and_exit(ms, warp, tmem);
    return;
  }
  ptx::tc_fence_after();

  // ---- 4. accumulator 1 -> R^T, L, P (row per thread) -------------------------------
  // Warp w reads TMEM lanes 32*(w%4).. ; warps 0-3 take value columns 0..63 and Gram
  // columns 0..31, warps 4-7 value columns 64..127 and Gram columns 32..63.
  const int quarter = warp & 3, set = warp >> 2;
  const int row = quarter * 32 + lane;
  const bool is_q = row < kTile;
  const int n = is_q ? row : row - kTile;
  const bool live = n < n_nodes;
  const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
  const float cln = ms.cl[n];
  const float gam = expf(cln);
  const unsigned long long ancn = ms.anc[n];
  const unsigned long long pathn = live ? (ancn | (1ull << n)) : 0ull;
  // A2 = [W ; T - I] starts as zeros; P is written into its top half below
  {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4 *>(sm + kOffA2 + (tid + j * kThreads) * 16) = z;
  }
  __syncthreads();
  if (!is_q) {
    // R_n = b_n (v_n - gamma_n S_root k_n) (scalar: v_n) -> column n of R^T
    const float bn = ms.bb[n];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float x[16];
      const int v0 = set * 64 + c * 16;
      ptx::tmem_ld16(trow + 64 + v0, x);
      // the 16 bf16 values v_n[v0 .. v0+15]: two swizzled 16-byte chunks of the v tile
      const int half = v0 >> 6, ch = (v0 & 63) >> 3;
      const uint4 w0 = *reinterpret_cast<const uint4 *>(
          sm + kOffV + half * kVHalf + (n << 7) + ((ch ^ (n & 7)) << 4));
      const uint4 w1 = *reinterpret_cast<const uint4 *>(
          sm + kOffV + half * kVHalf + (n << 7) + (((ch + 1) ^ (n & 7)) << 4));
      const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t bits16 = (wv[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu;
        const float vn = __uint_as_float(bits16 << 16);
        const float rr = kGdn ? bn * (vn - gam * x[j]) : vn;
        sts(sm, kOffB2 + op2_off(v0 + j, n), live ? rr : 0.f);
      }
    }
    if (kGdn) {
      // L row n on its strict ancestors
      float *L = reinterpret_cast<float *>(sm + kOffL);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float g[16];
        const int i0 = set * 32 + c * 16;
        ptx::tmem_ld16(trow + i0, g);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int i = i0 + j;
          if (live && ((ancn >> i) & 1ull)) L[coef_off(n, i)] = bn * expf(cln - ms.cl[i]) * g[j];
        }
      }
    }
  } else {
    // P row n on its path, into the W rows of A2
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float g[16];
      const int i0 = set * 32 + c * 16;
      ptx::tmem_ld16(trow + i0, g);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int i = i0 + j;
        if ((pathn >> i) & 1ull) sts(sm, kOffA2 + op2_off(n, i), expf(cln - ms.cl[i]) * g[j]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 5. rows of T - I and W by backward recursion along each node's own path ---------
  //   T[n][i] = -sum_{j in path(n), j > i} T[n][j] L[j][i]      (T[n][n] = 1)
  //   W[n][i] =  P[n][i] - sum_{j in path(n), j > i} W[n][j] L[j][i]
  // for i in anc(n), deepest first (ancestor indices increase with depth).
  if (kGdn && tid < 2 * kTile) {
    const float *L = reinterpret_cast<const float *>(sm + kOffL);
    const bool do_t = tid >= kTile;
    const int m = do_t ? tid - kTile : tid;
    if (m < n_nodes) {
      const unsigned long long am = ms.anc[m];
      const int r2 = do_t ? kTile + m : m;            // row of A2
      const float selfc = do_t ? 1.f : lds(sm, kOffA2 + op2_off(r2, m));
      for (unsigned long long bi = am; bi;) {
        const int i = 63 - __clzll((long long)bi);
        bi ^= 1ull << i;
        float acc = do_t ? 0.f : lds(sm, kOffA2 + op2_off(r2, i));
        acc = fmaf(-selfc, L[coef_off(m, i)], acc);
        // deeper ancestors j of m below i: bits of am above i
        for (unsigned long long bj = am & ~((2ull << i) - 1ull); bj; bj &= bj - 1) {
          const int j = __ffsll((long long)bj) - 1;
          acc = fmaf(-lds(sm, kOffA2 + op2_off(r2, j)), L[coef_off(j, i)], acc);
        }
        sts(sm, kOffA2 + op2_off(r2, i), acc);
      }
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 6. MMA 2: [W ; T - I] . R  (tf32) into TMEM columns 192..255 (v 0..63) and
  //         0..63 (v 64..127; the Gram columns, already read) -------------------------
  if (tid == kThreads - 1) {
    ptx::tc_fence_after();
    constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 64);
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {
      const uint32_t dcol = hv == 0 ? 192u : 0u;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * kAtom2 + (kk & 3) * 32;
        const uint64_t ad = ptx::smem_desc_sw128(sbase + kOffA2 + koff, 1024);
        const uint64_t bd = ptx::smem_desc_sw128(sbase + kOffB2 + koff + hv * 64 * 128, 1024);
        ptx::mma_tf32(tmem + dcol, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
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
    cleanup_and_exit(ms, warp, tmem);
    return;
  }
  ptx::tc_fence_after();

  // ---- 7. epilogue: o_n = gamma_n S_root q_n + (W R)_n,  u_n = R_n + ((T - I) R)_n ----
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    const int v0 = set * 64 + c * 16;
    const uint32_t col2 = set == 0 ? 192u + c * 16 : (uint32_t)c * 16;
    float y[16];
    ptx::tmem_ld16(trow + col2, y);
    if (is_q) {
      float x[16];
      ptx::tmem_ld16(trow + 64 + v0, x);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 o4 = make_float4(fmaf(gam, x[j], y[j]), fmaf(gam, x[j + 1], y[j + 1]),
                                      fmaf(gam, x[j + 2], y[j + 2]), fmaf(gam, x[j + 3], y[j + 3]));
        *reinterpret_cast<float4 *>(sm + kOffOt + tile_off(n, v0 + j)) = o4;
      }
    } else {
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        float4 u4;
        u4.x = lds(sm, kOffB2 + op2_off(v0 + j, n)) + y[j];
        u4.y = lds(sm, kOffB2 + op2_off(v0 + j + 1, n)) + y[j + 1];
        u4.z = lds(sm, kOffB2 + op2_off(v0 + j + 2, n)) + y[j + 2];
        u4.w = lds(sm, kOffB2 + op2_off(v0 + j + 3, n)) + y[j + 3];
        *reinterpret_cast<float4 *>(sm + kOffUt + tile_off(n, v0 + j)) = u4;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {  // accumulators fully read: hand the tensor memory back
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  // coalesced rows: a warp writes one 512-byte row of o or U per instruction
  Tout *out = static_cast<Tout *>(a.out);
  const int v4 = (tid & 31) * 4;
  for (int r = tid >> 5; r < 2 * n_nodes; r += kThreads / 32) {
    const bool is_u = r >= n_nodes;
    const int m = is_u ? r - n_nodes : r;
    const float4 x = *reinterpret_cast<const float4 *>(sm + (is_u ? kOffUt : kOffOt) + tile_off(m, v4));
    const size_t g = ((size_t)(lo + m) * H + h) * 128 + v4;
    if (is_u) {
      __stcs(reinterpret_cast<float4 *>(a.U + g), x);
    } else if (sizeof(Tout) == 4) {
      __stcs(reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + g), x);
    } else {
      __nv_bfloat162 lo2 = __floats2bfloat162_rn(x.x, x.y), hi2 = __floats2bfloat162_rn(x.z, x.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&lo2);
      pk.y = *reinterpret_cast<uint32_t *>(&hi2);
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
  kern<<<a.B * a.H, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
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
