// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// Notation for one (sequence, head) item: N <= 64 nodes in topological order, path(n) =
// strict ancestors anc(n) plus n (root first, indices increase along it), cl_n = fp32 sum
// of log_a over path(n) (root first), gamma_n = exp(cl_n), D[n][i] = exp(cl_n - cl_i).
//
// MMA (tcgen05 kind::f16, 128 x 192 x 128, bf16 in, fp32 accumulate in TMEM):
//      [ Q ] . [ K ; S_root ]^T  ->  [ Q K^T | (S_root Q^T)^T ]   rows 0..63
//      [ K ]                         [ K K^T | (S_root K^T)^T ]   rows 64..127
// gives both path Gram blocks and both state products -- the only dense contraction of
// the method.  q, k, v arrive by TMA in the 128-byte swizzled layout the MMA reads;
// S_root (fp32 in HBM) is converted to bf16 by all threads straight into the same layout.
//
// The tree system (tree-structured WY form of the TreeWY abstract) is
//      (I + L) U = R,  L[n][i] = b_n D[n][i] k_n.k_i (i in anc(n)),  R_n = b_n (v_n - gamma_n S_root k_n)
// and the outputs (closed form of the Bole summary's worked example, "具体技术细节示例",
// extended to the delta rule) are  o_n = gamma_n S_root q_n + sum_i P[n][i] u_i  with
// P[n][i] = D[n][i] q_n.k_i on path(n).  With T = (I + L)^-1 and W = P T:
//      u_n = sum_{i in path(n)} T[n][i] R_i,      o_n = gamma_n S_root q_n + sum_{i in path(n)} W[n][i] R_i .
// The decays factor out of both rows: T[n][i] = D[n][i] tau_i, W[n][i] = D[n][i] omega_i,
// where along path(n) = p_0 .. p_{d-1} = n (right-looking, deepest first)
//      tau_{d-1} = 1,             tau_a   = - sum_{c > a} tau_c   b_{p_c} k_{p_c}.k_{p_a}
//      omega_a = q_n.k_{p_a}                - sum_{c > a} omega_c b_{p_c} k_{p_c}.k_{p_a}
// so each row is one thread's short register recursion, and the path sums are fp32 FMAs
// with one warp per node row, written straight to HBM.  Scalar decay: tau = e_{d-1}
// (u_n = v_n), omega_a = q_n.k_{p_a}.
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
constexpr int kRegDepth = 16;              // deeper paths take the shared-memory recursion
constexpr uint32_t kTmemCols = 256;        // accumulator: columns 0..191
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out

// Dynamic shared memory, offsets from a 1024-byte aligned base.
//   [0, 64K)      MMA operands: two 64-wide K halves of [Q ; K ; S_root] (256 rows x 128 B).
//                 Once the MMA is done, the next item's q/k land in rows 0..127 of each
//                 half while rows 128..255 (the S_root rows) hold the T and W rows:
//                 T at [16K, 32K), W at [48K, 64K) (64 x 64 fp32 each).
//   [64K, 96K)    two v tiles (bf16, TMA swizzled)
//   [96K, 128K)   R tile, 64 x 128 fp32
//   [128K, 160K)  gamma_n S_root q_n tile, 64 x 128 fp32
//   [160K, 176K)  b_j k_j.k_i on paths, 64 x 64 fp32
//   [176K, 192K)  q_n.k_i on paths, 64 x 64 fp32
//   [192K, 196K)  root-first path of every node (bytes)
constexpr int kOpHalf = 256 * 128;
constexpr int kOffOp = 0;
constexpr int kOffT = 16384;
constexpr int kOffW = 49152;
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 65536;
constexpr int kOffR = 98304;
constexpr int kOffSQ = 131072;
constexpr int kOffLK = 163840;
constexpr int kOffGQ = 180224;
constexpr int kOffPath = 196608;
constexpr int kOffMisc = kOffPath + kTile * kTile;

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_mma;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int timeout;
  int outstanding[2];              // an issued TMA / MMA whose barrier was not waited
  int par[kTile];
  int dep[kTile];
  float la[kTile];
  float bb[kTile];
  float cl[kTile];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;

// fp32 [64][128] tile in four 32-column slabs of 128-byte rows with 16-byte chunks
// XOR-swizzled by row: row-per-thread and row-per-warp accesses are conflict-free.
__device__ __forceinline__ int tile_off(int n, int v) {
  return ((v >> 5) << 13) + (n << 7) + ((((v >> 2) & 7) ^ (n & 7)) << 4) + ((v & 3) << 2);
}
// [64][64] fp32 matrix, column XOR-swizzled by row.
__device__ __forceinline__ int coef_off(int n, int i) { return ((n << 6) + (i ^ (n & 31))) << 2; }

__device__ __forceinline__ float lds(const unsigned char *p, int off) {
  return *reinterpret_cast<const float *>(p + off);
}
__device__ __forceinline__ void sts(unsigned char *p, int off, float x) {
  *reinterpret_cast<float *>(p + off) = x;
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

// Row recursion of node m (d = depth, path bytes `pth`): x_a for a < d with
//   x_a = x0_a - sum_{c > a} x_c b_{p_c} k_{p_c}.k_{p_a}   (x0 = e_{d-1} for T, q_m.k for W)
// then stores D[m][p_a] x_a into `dst` row m.  Register version for d <= kRegDepth.
template <bool kW>
__device__ __forceinline__ void row_recursion(unsigned char *sm, const uint8_t *pth, int m, int d,
                                              const Misc &ms, int dst) {
  const float clm = ms.cl[m];
  if (d <= kRegDepth) {
    int p[kRegDepth];
    float x[kRegDepth];
#pragma unroll
    for (int a = 0; a < kRegDepth; ++a) {
      p[a] = a < d ? pth[a] : 0;
      x[a] = kW ? (a < d ? lds(sm, kOffGQ + coef_off(m, p[a])) : 0.f) : (a == d - 1 ? 1.f : 0.f);
    }
#pragma unroll
    for (int c = kRegDepth - 1; c >= 1; --c) {
      if (c < d) {
        const float xc = x[c];
#pragma unroll
        for (int a = 0; a < c; ++a)
          x[a] = fmaf(-xc, lds(sm, kOffLK + coef_off(p[c], p[a])), x[a]);
      }
    }
#pragma unroll
    for (int a = 0; a < kRegDepth; ++a)
      if (a < d) sts(sm, dst + coef_off(m, p[a]), x[a] * expf(clm - ms.cl[p[a]]));
  } else {
    // deep path: the row itself is the working storage (other rows are only read from LK)
    for (int a = 0; a < d; ++a)
      sts(sm, dst + coef_off(m, pth[a]),
          kW ? lds(sm, kOffGQ + coef_off(m, pth[a])) : (a == d - 1 ? 1.f : 0.f));
    for (int c = d - 1; c >= 1; --c) {
      const float xc = lds(sm, dst + coef_off(m, pth[c]));
      for (int a = 0; a < c; ++a) {
        const int o = dst + coef_off(m, pth[a]);
        sts(sm, o, fmaf(-xc, lds(sm, kOffLK + coef_off(pth[c], pth[a])), lds(sm, o)));
      }
    }
    for (int a = 0; a < d; ++a) {
      const int o = dst + coef_off(m, pth[a]);
      sts(sm, o, lds(sm, o) * expf(clm - ms.cl[pth[a]]));
    }
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
  uint8_t *paths = reinterpret_cast<uint8_t *>(sm + kOffPath);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_items = a.B * a.H;
  int it = blockIdx.x;
  if (it >= num_items) return;

  const uint32_t sbase = ptx::smem_addr(sm);
  const uint32_t bar_tma = ptx::smem_addr(&ms.bar_tma);
  const uint32_t bar_mma = ptx::smem_addr(&ms.bar_mma);

  // ---- prologue: barriers, tensor memory, first item's loads --------------------------
  Item cur = load_item(a, it);
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_mma, 1);
    ptx::fence_mbar_init();
    ms.timeout = 0;
    ms.outstanding[0] = 1;
    ms.outstanding[1] = 0;
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

  uint32_t ph_tma = 0, ph_mma = 0;
  for (int local = 0; it < num_items; ++local, it += gridDim.x) {
    const int buf = local & 1;
    const int nxt = it + gridDim.x;
    const bool has_next = nxt < num_items;
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

    // ---- 2. MMA (one thread); paths and decays; the next item's loads -----------------
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
        ptx::mma_commit(bar_mma);
      }
    }
    ph_tma ^= 1u;
    Item nx;
    if (has_next) nx = load_item(a, nxt);
    if (has_next) load_state(a, nx, tid, sreg);
    if (tid < kTile) {
      // walk up: ancestor bits, depth, root-first path bytes; cl summed root first
      unsigned long long bits = 0ull;
      int d = 0;
      float cl = 0.f;
      if (run && tid < n_nodes) {
        d = 1;
        for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) {
          bits |= 1ull << x;
          ++d;
        }
        uint8_t *pth = paths + tid * kTile;
        pth[d - 1] = (uint8_t)tid;
        int pos = d - 2;
        for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) pth[pos--] = (uint8_t)x;
        for (int t = 0; t < d; ++t) cl += ms.la[pth[t]];
      }
      ms.anc[tid] = bits;
      ms.dep[tid] = d;
      ms.cl[tid] = cl;
    }
    if (has_next) load_meta<kGdn>(a, nx, tid, p_reg, la_reg, bb_reg);
    __syncthreads();
    if (ms.timeout) break;
    if (bad_tree && tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, cur.s);

    // ---- 3. operands consumed: prefetch the next item's q / k / v ---------------------
    if (tid == 0) {
      if (run) {
        if (ptx::mbar_wait_bounded(bar_mma, ph_mma, kSpinLimit)) ms.outstanding[1] = 0;
        else ms.timeout = 1;
      }
      if (has_next && !ms.timeout) {
        ms.outstanding[0] = 1;
        issue_tma(nx, buf ^ 1, sbase, bar_tma, &tm_q, &tm_k, &tm_v);
      }
    }
    if (run) ph_mma ^= 1u;
    __syncthreads();
    if (ms.timeout) break;

    if (run) {
      ptx::tc_fence_after();
      const bool live = n < n_nodes;
      const float gam = expf(ms.cl[n]);
      const unsigned long long ancn = ms.anc[n];
      const unsigned long long pathn = live ? (ancn | (1ull << n)) : 0ull;
      const unsigned char *vt = sm + kOffV + buf * 2 * kVHalf;

      // ---- 4. accumulator -> R and gamma S_root q tiles, path Gram entries -------------
      // warp w reads TMEM lanes 32*(w%4)..; warps 0-3 take value columns 0..63 and Gram
      // columns 0..31, warps 4-7 value columns 64..127 and Gram columns 32..63.
      {
        const float bn = ms.bb[n];
        unsigned char *tile = sm + (is_q ? kOffSQ : kOffR);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float x[16];
          const int v0 = set * 64 + c * 16;
          ptx::tmem_ld16(trow + 64 + v0, x);
          if (is_q) {
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] *= gam;
          } else {
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
              x[j] = live ? (kGdn ? bn * (vn - gam * x[j]) : vn) : 0.f;
            }
          }
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4 *>(tile + tile_off(n, v0 + j)) =
                make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
        }
        // Gram on paths: K rows -> b_n k_n.k_i (i in anc(n)), Q rows -> q_n.k_i (i in path(n))
        const int gbase = is_q ? kOffGQ : kOffLK;
        const unsigned long long sel = is_q ? pathn : (live ? ancn : 0ull);
        const float scale = is_q ? 1.f : bn;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float g[16];
          const int i0 = set * 32 + c * 16;
          ptx::tmem_ld16(trow + i0, g);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if ((sel >> (i0 + j)) & 1ull) sts(sm, gbase + coef_off(n, i0 + j), scale * g[j]);
        }
      }
      ptx::tc_fence_before();
      __syncthreads();

      // ---- 5. T rows (threads 0..63) and W rows (threads 64..127) ----------------------
      if (tid < 2 * kTile) {
        const int m = tid & (kTile - 1);
        if (m < n_nodes) {
          const int d = ms.dep[m];
          const uint8_t *pth = paths + m * kTile;
          if (tid < kTile) {
            if (kGdn) {
              row_recursion<false>(sm, pth, m, d, ms, kOffT);
            } else {
              for (int a2 = 0; a2 < d; ++a2) sts(sm, kOffT + coef_off(m, pth[a2]), a2 == d - 1 ? 1.f : 0.f);
            }
          } else {
            if (kGdn) {
              row_recursion<true>(sm, pth, m, d, ms, kOffW);
            } else {
              const float clm = ms.cl[m];
              for (int a2 = 0; a2 < d; ++a2) {
                const int i = pth[a2];
                sts(sm, kOffW + coef_off(m, i), lds(sm, kOffGQ + coef_off(m, i)) * expf(clm - ms.cl[i]));
              }
            }
          }
        }
      }
      __syncthreads();

      // ---- 6. path sums, one warp per node row, straight to HBM -----------------------
      //   u_m = sum_{i in path(m)} T[m][i] R_i,   o_m = gamma_m S_root q_m + sum_i W[m][i] R_i
      Tout *out = static_cast<Tout *>(a.out);
      const int v4 = lane * 4;
      for (int m = warp; m < n_nodes; m += kThreads / 32) {
        const int d = ms.dep[m];
        const uint8_t *pth = paths + m * kTile;
        float4 o4 = *reinterpret_cast<const float4 *>(sm + kOffSQ + tile_off(m, v4));
        float4 u4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int a2 = 0; a2 < d; ++a2) {
          const int i = pth[a2];
          const float ct = lds(sm, kOffT + coef_off(m, i));
          const float cw = lds(sm, kOffW + coef_off(m, i));
          const float4 r4 = *reinterpret_cast<const float4 *>(sm + kOffR + tile_off(i, v4));
          u4.x = fmaf(ct, r4.x, u4.x); u4.y = fmaf(ct, r4.y, u4.y);
          u4.z = fmaf(ct, r4.z, u4.z); u4.w = fmaf(ct, r4.w, u4.w);
          o4.x = fmaf(cw, r4.x, o4.x); o4.y = fmaf(cw, r4.y, o4.y);
          o4.z = fmaf(cw, r4.z, o4.z); o4.w = fmaf(cw, r4.w, o4.w);
        }
        const size_t g = ((size_t)(cur.lo + m) * a.H + cur.h) * 128 + v4;
        __stcs(reinterpret_cast<float4 *>(a.U + g), u4);
        if (sizeof(Tout) == 4) {
          __stcs(reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + g), o4);
        } else {
          __nv_bfloat162 l2 = __floats2bfloat162_rn(o4.x, o4.y), h2 = __floats2bfloat162_rn(o4.z, o4.w);
          uint2 pk;
          pk.x = *reinterpret_cast<uint32_t *>(&l2);
          pk.y = *reinterpret_cast<uint32_t *>(&h2);
          *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(out) + g) = pk;
        }
      }
      // the next item's state conversion overwrites the T / W rows read above
      __syncthreads();
    }
    if (has_next) cur = nx;
  }

  // ---- teardown: drain an issued copy, record a timeout, free tensor memory ----------
  if (ms.timeout && tid == 0) {
    set_status(a.ws, TV_ERR_TIMEOUT, blockIdx.x);
    if (ms.outstanding[0]) ptx::mbar_wait_bounded(bar_tma, ph_tma, kSpinLimit);
    if (ms.outstanding[1]) ptx::mbar_wait_bounded(bar_mma, ph_mma, kSpinLimit);
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
