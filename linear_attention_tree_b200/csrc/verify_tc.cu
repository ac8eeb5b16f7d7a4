// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// Notation for one (sequence, head) item: N <= 64 nodes in topological order, path(n) =
// strict ancestors anc(n) plus n, cl_n = fp32 sum of log_a over path(n) (root first),
// gamma_n = exp(cl_n), D[n][i] = exp(cl_n - cl_i).
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
//      U = T R,      O = diag(gamma) S_root Q^T + W R .
// Rows of T and W live on the node's own path and follow from L alone by a backward
// recursion along that path (T (I + L) = I, W (I + L) = P): one thread per row, no
// barriers.  MMA 2 (kind::tf32, 128 x 128 x 64, operands rounded to nearest tf32) forms
// [ W ; T ] . R in TMEM.  Scalar decay is the special case L = 0 (T = I, W = P, U = R = V).
//
// Scheduling: one persistent CTA per SM walks the items blockIdx.x, +gridDim.x, ...
// While item i is in its epilogue, item i+1's S_root is already streaming into registers
// and its q/k/v into a second set of buffers by TMA, so HBM stays busy across items.
//
// Every wait on an mbarrier is bounded; a wait that runs out records TV_ERR_TIMEOUT on
// the status word, the CTA drains what it issued, frees its tensor memory and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;                  // nodes per tree handled by this kernel
constexpr uint32_t kTmemCols = 512;        // accumulator 1: cols 0..191, accumulator 2: 256..383
constexpr uint32_t kAcc2 = 256;
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out

// Dynamic shared memory, offsets from a 1024-byte aligned base.
constexpr int kOpHalf = 256 * 128;         // one 64-wide K half of [Q ; K ; S_root]
constexpr int kOffOp = 0;                  // MMA 1 operands, 64 KiB
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 65536;               // two v tiles (bf16, TMA swizzled), 2 x 16 KiB
constexpr int kOffB2 = 98304;              // R^T, MMA 2 B operand (fp32); then the O tile
constexpr int kOffA2 = 131072;             // [W ; T], MMA 2 A operand (fp32); then the U tile
constexpr int kAtom2 = 16384;              // one 32-wide K atom of a 128-row fp32 operand
constexpr int kOffL = 163840;              // L coefficients, 64 x 64 fp32
constexpr int kOffMisc = kOffL + kTile * kTile * 4;

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_mma1;
  unsigned long long bar_mma2;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int timeout;
  int outstanding[3];              // an issued TMA / MMA 1 / MMA 2 whose barrier was not waited
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
// fp32 element (row, k) of a 128-row, K = 64 K-major operand with 128-byte swizzle.
__device__ __forceinline__ int op2_off(int row, int k) {
  return ((k >> 5) * kAtom2) + (row << 7) + ((((k >> 2) & 7) ^ (row & 7)) << 4) + ((k & 3) << 2);
}
// [64][64] fp32 coefficients, column XOR-swizzled by row.
__device__ __forceinline__ int coef_off(int n, int i) { return (n << 6) + (i ^ (n & 31)); }

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

struct Item {
  int s, h, lo, n;
  bool ok;     // node_offsets consistent for this sequence
};

__device__ __forceinline__ Item load_item(const VerifyArgs &a, int it) {
  Item r;
  r.s = it / a.H;
  r.h = it % a.H;
  const int lo = a.node_offsets[r.s], hi = a.node_offsets[r.s + 1];
  r.ok = !(lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes || hi - lo > kTile ||
           (r.s == 0 && lo != 0) || (r.s == a.B - 1 && hi != a.T));
  r.lo = r.ok ? lo : 0;
  r.n = r.ok ? hi - lo : 0;
  return r;
}

__device__ __forceinline__ void issue_tma(const Item &x, int buf, uint32_t sbase, uint32_t bar,
                                          const CUtensorMap *tq, const CUtensorMap *tk,
                                          const CUtensorMap *tvv) {
  ptx::mbar_arrive_expect_tx(bar, 6 * kTile * 128);
  for (int half = 0; half < 2; ++half) {
    const uint32_t hb = sbase + kOffOp + half * kOpHalf;
    ptx::tma_load_3d(hb, tq, bar, half * 64, x.h, x.lo);
    ptx::tma_load_3d(hb + kTile * 128, tk, bar, half * 64, x.h, x.lo);
    ptx::tma_load_3d(sbase + kOffV + buf * 2 * kVHalf + half * kVHalf, tvv, bar, half * 64, x.h,
                     x.lo);
  }
}

// S_root[s][h] as 16 float4 per thread: thread t owns 8-element k chunk (t & 15) of rows
// v = t/16 + 16 j.
__device__ __forceinline__ void load_state(const VerifyArgs &a, const Item &x, int tid,
                                           float4 (&r)[16]) {
  const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + ((size_t)x.s * a.H + x.h) * 128 * 128);
  const int kc = tid & 15;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int v = (tid >> 4) + 16 * j;
    r[2 * j] = __ldcs(Sg + v * 32 + kc * 2);
    r[2 * j + 1] = __ldcs(Sg + v * 32 + kc * 2 + 1);
  }
}

template <bool kGdn>
__device__ __forceinline__ void load_meta(const VerifyArgs &a, const Item &x, int tid, int &p,
                                          float &la, float &bb) {
  p = -1;
  la = 0.f;
  bb = 0.f;
  if (tid < x.n) {
    p = a.parent[x.lo + tid];
    la = a.log_a[(size_t)(x.lo + tid) * a.H + x.h];
    bb = kGdn ? a.b[(size_t)(x.lo + tid) * a.H + x.h] : 0.f;
  }
}

template <bool kGdn, typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, VerifyArgs a) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Misc &ms = *reinterpret_cast<Misc *>(sm + kOffMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_items = a.B * a.H;
  int it = blockIdx.x;
  if (it >= num_items) return;

  const uint32_t sbase = ptx::smem_addr(sm);
  const uint32_t bar_tma = ptx::smem_addr(&ms.bar_tma);
  const uint32_t bar_mma1 = ptx::smem_addr(&ms.bar_mma1);
  const uint32_t bar_mma2 = ptx::smem_addr(&ms.bar_mma2);

  // ---- prologue: barriers, tensor memory, first item's loads --------------------------
  Item cur = load_item(a, it);
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_mma1, 1);
    ptx::mbar_init(bar_mma2, 1);
    ptx::fence_mbar_init();
    ms.timeout = 0;
    ms.outstanding[0] = 1;
    ms.outstanding[1] = 0;
    ms.outstanding[2] = 0;
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    issue_tma(cur, 0, sbase, bar_tma, &tm_q, &tm_k, &tm_v);
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&ms.tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  float4 sreg[16];
  load_state(a, cur, tid, sreg);
  int p_reg;
  float la_reg, bb_reg;
  load_meta<kGdn>(a, cur, tid, p_reg, la_reg, bb_reg);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ms.tmem_base;

  const int quarter = warp & 3, set = warp >> 2;
  const int row = quarter * 32 + lane;             // TMEM lane of this thread
  const bool is_q = row < kTile;
  const int n = is_q ? row : row - kTile;          // node of this thread's accumulator row
  const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);

  uint32_t ph_tma = 0, ph_m1 = 0, ph_m2 = 0;
  for (int local = 0; it < num_items; ++local, it += gridDim.x) {
    const int buf = local & 1;
    const int nxt = it + gridDim.x;
    const bool has_next = nxt < num_items;
    Item nx;
    if (has_next) nx = load_item(a, nxt);
    const int n_nodes = cur.n;

    // ---- 1. state -> bf16 operand rows 128..255; tree metadata -> shared --------------
    {
      const int kc = tid & 15;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = (tid >> 4) + 16 * j, r = 128 + v;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(sreg[2 * j].x, sreg[2 * j].y);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(sreg[2 * j].z, sreg[2 * j].w);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(sreg[2 * j + 1].x, sreg[2 * j + 1].y);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(sreg[2 * j + 1].z, sreg[2 * j + 1].w);
        uint4 pk;
        pk.x = *reinterpret_cast<uint32_t *>(&b0);
        pk.y = *reinterpret_cast<uint32_t *>(&b1);
        pk.z = *reinterpret_cast<uint32_t *>(&b2);
        pk.w = *reinterpret_cast<uint32_t *>(&b3);
        const int off = (kc >> 3) * kOpHalf + r * 128 + (((kc & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(sm + kOffOp + off) = pk;
      }
      ptx::fence_proxy_async_smem();
    }
    bool bad = false;
    if (tid < kTile) {
      ms.par[tid] = p_reg;
      ms.la[tid] = la_reg;
      ms.bb[tid] = bb_reg;
      bad = tid < n_nodes && (p_reg < -1 || p_reg >= tid);
    }
    const bool bad_tree = __syncthreads_or(bad) != 0 || !cur.ok;
    const bool run = !bad_tree && n_nodes > 0;

    // ---- 2. MMA 1 (one thread); metadata walk; next item's state and metadata loads ---
    if (tid == kThreads - 1) {
      const bool landed = ptx::mbar_wait_bounded(bar_tma, ph_tma, kSpinLimit);
      if (landed) ms.outstanding[0] = 0;
      else ms.timeout = 1;
      if (landed && run) {
        ptx::tc_fence_after();
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 192);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t base = sbase + kOffOp + (kk >> 2) * kOpHalf + (kk & 3) * 32;
          ptx::mma_bf16(tmem, ptx::smem_desc_sw128(base, 1024),
                        ptx::smem_desc_sw128(base + kTile * 128, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        ms.outstanding[1] = 1;
        ptx::mma_commit(bar_mma1);
      }
    }
    ph_tma ^= 1u;
    if (tid < kTile) {
      // strict ancestors by walking up; cl summed root first (ancestor indices increase
      // with depth, so ascending bit order is path order)
      unsigned long long bits = 0ull;
      float cl = 0.f;
      if (run && tid < n_nodes) {
        for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) bits |= 1ull << x;
        for (unsigned long long b = bits; b; b &= b - 1) cl += ms.la[__ffsll((long long)b) - 1];
        cl += ms.la[tid];
      }
      ms.anc[tid] = bits;
      ms.cl[tid] = cl;
    }
    if (has_next) {
      load_state(a, nx, tid, sreg);
      load_meta<kGdn>(a, nx, tid, p_reg, la_reg, bb_reg);
    }
    __syncthreads();
    if (ms.timeout) break;
    if (bad_tree && tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, cur.s);

    // ---- 3. operands consumed: prefetch the next item's q / k / v ---------------------
    if (tid == 0) {
      if (run) {
        if (ptx::mbar_wait_bounded(bar_mma1, ph_m1, kSpinLimit)) ms.outstanding[1] = 0;
        else ms.timeout = 1;
      }
      if (has_next && !ms.timeout) {
        ms.outstanding[0] = 1;
        issue_tma(nx, buf ^ 1, sbase, bar_tma, &tm_q, &tm_k, &tm_v);
      }
    }
    if (run) ph_m1 ^= 1u;
    __syncthreads();
    if (ms.timeout) break;

    if (run) {
      ptx::tc_fence_after();
      const bool live = n < n_nodes;
      const float cln = ms.cl[n];
      const float gam = expf(cln);
      const unsigned long long ancn = ms.anc[n];
      const unsigned long long pathn = live ? (ancn | (1ull << n)) : 0ull;
      const unsigned char *vt = sm + kOffV + buf * 2 * kVHalf;

      // ---- 4. accumulator 1 -> R^T (B2), raw Gram on paths (L, and P in A2's W rows) --
      if (!is_q) {
        const float bn = ms.bb[n];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float x[16];
          const int v0 = set * 64 + c * 16;
          ptx::tmem_ld16(trow + 64 + v0, x);
          const int half = v0 >> 6, ch = (v0 & 63) >> 3;
          const uint4 w0 = *reinterpret_cast<const uint4 *>(
              vt + half * kVHalf + (n << 7) + ((ch ^ (n & 7)) << 4));
          const uint4 w1 = *reinterpret_cast<const uint4 *>(
              vt + half * kVHalf + (n << 7) + (((ch + 1) ^ (n & 7)) << 4));
          const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float vn = __uint_as_float(((wv[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu) << 16);
            const float rr = kGdn ? bn * (vn - gam * x[j]) : vn;
            sts(sm, kOffB2 + op2_off(v0 + j, n), live ? tf32_rn(rr) : 0.f);
          }
        }
        if (kGdn) {
          float *L = reinterpret_cast<float *>(sm + kOffL);
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float g[16];
            const int i0 = set * 32 + c * 16;
            ptx::tmem_ld16(trow + i0, g);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if ((ancn >> (i0 + j)) & 1ull) L[coef_off(n, i0 + j)] = g[j];
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float g[16];
          const int i0 = set * 32 + c * 16;
          ptx::tmem_ld16(trow + i0, g);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            sts(sm, kOffA2 + op2_off(n, i0 + j), ((pathn >> (i0 + j)) & 1ull) ? g[j] : 0.f);
        }
      }
      ptx::tc_fence_before();
      __syncthreads();

      // ---- 5. decays on L (one thread per node): L[m][i] = b_m D[m][i] k_m.k_i ---------
      float *L = reinterpret_cast<float *>(sm + kOffL);
      if (kGdn && tid < n_nodes) {
        const int m = tid;
        const float clm = ms.cl[m], bm = ms.bb[m];
        for (unsigned long long bi = ms.anc[m]; bi; bi &= bi - 1) {
          const int i = __ffsll((long long)bi) - 1;
          L[coef_off(m, i)] *= bm * expf(clm - ms.cl[i]);
        }
      }
      __syncthreads();

      // ---- 6. rows of W (tid < 64) and T (tid 64..127) by backward recursion ------------
      //   W[m][i] = P[m][i] - sum_{j in path(m), j > i} W[m][j] L[j][i]
      //   T[m][i] =  I[m][i] - sum_{j in path(m), j > i} T[m][j] L[j][i]
      // for i in anc(m), deepest first (ancestor indices increase with depth).
      if (tid < 2 * kTile) {
        const bool do_t = tid >= kTile;
        const int m = do_t ? tid - kTile : tid;
        const int r2 = do_t ? kTile + m : m;
        if (do_t) {
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            *reinterpret_cast<float4 *>(sm + kOffA2 + op2_off(r2, c * 4)) = z;
          if (m < n_nodes) sts(sm, kOffA2 + op2_off(r2, m), 1.f);
        }
        if (m < n_nodes) {
          const unsigned long long am = ms.anc[m];
          const float clm = ms.cl[m];
          if (!do_t)   // P[m][i] = D[m][i] q_m.k_i
            for (unsigned long long bi = am; bi; bi &= bi - 1) {
              const int i = __ffsll((long long)bi) - 1;
              const int o = kOffA2 + op2_off(r2, i);
              sts(sm, o, lds(sm, o) * expf(clm - ms.cl[i]));
            }
          if (kGdn) {
            const float selfc = lds(sm, kOffA2 + op2_off(r2, m));
            for (unsigned long long bi = am; bi;) {
              const int i = 63 - __clzll((long long)bi);
              bi ^= 1ull << i;
              float acc = do_t ? 0.f : lds(sm, kOffA2 + op2_off(r2, i));
              acc = fmaf(-selfc, L[coef_off(m, i)], acc);
              for (unsigned long long bj = am & ~((2ull << i) - 1ull); bj; bj &= bj - 1) {
                const int j = __ffsll((long long)bj) - 1;
                acc = fmaf(-lds(sm, kOffA2 + op2_off(r2, j)), L[coef_off(j, i)], acc);
              }
              sts(sm, kOffA2 + op2_off(r2, i), acc);
            }
          }
          // operands of the tf32 MMA, rounded to nearest
          for (unsigned long long bi = am | (1ull << m); bi; bi &= bi - 1) {
            const int o = kOffA2 + op2_off(r2, __ffsll((long long)bi) - 1);
            sts(sm, o, tf32_rn(lds(sm, o)));
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ---- 7. MMA 2: [W ; T] . R  (tf32, 128 x 128 x 64) -> TMEM columns 256..383 ------
      if (tid == kThreads - 1) {
        ptx::tc_fence_after();
        constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * kAtom2 + (kk & 3) * 32;
          ptx::mma_tf32(tmem + kAcc2, ptx::smem_desc_sw128(sbase + kOffA2 + koff, 1024),
                        ptx::smem_desc_sw128(sbase + kOffB2 + koff, 1024), idesc,
                        kk > 0 ? 1u : 0u);
        }
        ms.outstanding[2] = 1;
        ptx::mma_commit(bar_mma2);
      }
      __syncthreads();
      if (tid == 0) {
        if (ptx::mbar_wait_bounded(bar_mma2, ph_m2, kSpinLimit)) ms.outstanding[2] = 0;
        else ms.timeout = 1;
      }
      ph_m2 ^= 1u;
      __syncthreads();
      if (ms.timeout) break;
      ptx::tc_fence_after();

      // ---- 8. epilogue: o = gamma S_root q + (W R), u = (T R) -> O / U tiles ------------
      unsigned char *tile = sm + (is_q ? kOffB2 : kOffA2);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int v0 = set * 64 + c * 16;
        float y[16];
        ptx::tmem_ld16(trow + kAcc2 + v0, y);
        if (is_q) {
          float x[16];
          ptx::tmem_ld16(trow + 64 + v0, x);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = fmaf(gam, x[j], y[j]);
        } else {
          ptx::tmem_wait_ld();
        }
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4 *>(tile + tile_off(n, v0 + j)) =
              make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
      }
      ptx::tc_fence_before();
      __syncthreads();

      // ---- 9. coalesced rows out: a warp writes one 512-byte row per instruction ---------
      Tout *out = static_cast<Tout *>(a.out);
      const int v4 = lane * 4;
      for (int r = warp; r < 2 * n_nodes; r += kThreads / 32) {
        const bool is_u = r >= n_nodes;
        const int m = is_u ? r - n_nodes : r;
        const float4 x = *reinterpret_cast<const float4 *>(sm + (is_u ? kOffA2 : kOffB2) + tile_off(m, v4));
        const size_t g = ((size_t)(cur.lo + m) * a.H + cur.h) * 128 + v4;
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
    if (has_next) cur = nx;
  }

  // ---- teardown: drain an issued copy, record a timeout, free tensor memory ----------
  if (ms.timeout && tid == 0) {
    set_status(a.ws, TV_ERR_TIMEOUT, blockIdx.x);
    if (ms.outstanding[0]) ptx::mbar_wait_bounded(bar_tma, ph_tma, kSpinLimit);
    if (ms.outstanding[1]) ptx::mbar_wait_bounded(bar_mma1, ph_m1, kSpinLimit);
    if (ms.outstanding[2]) ptx::mbar_wait_bounded(bar_mma2, ph_m2, kSpinLimit);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
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

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
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
  const int items = a.B * a.H;
  const int grid = items < sm_count() ? items : sm_count();
  kern<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
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
