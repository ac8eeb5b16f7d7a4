// Tensor-core tree verification of wide trees for sm_100a: bf16 q/k/v, dk = dv = 128,
// 1..256 nodes per tree, gated delta rule or scalar decay.  Trees of up to 64 nodes have
// their own kernel (verify_tc.cu); this one takes the batches whose largest tree is wider.
//
// The method is the one of the 64-node kernel (notation there): with the tree system
// (I + L) U = R of the TreeWY abstract's tree-structured WY form and the closed form of
// the Bole summary's worked example ("具体技术细节示例"),
//      U = T R,   O = diag(gamma) S_root Q^T + W R,   T = (I + L)^-1,  W = P T,
// and the rows of T and W are short recursions over each node's own root-first path.
//
// A tree of N nodes is processed in tiles of 64 nodes in index order.  Indices are
// topological (parent[i] < i), so the path of a node in tile c only visits tiles 0..c: in
// a 4-word ancestor bitmask, word c' holds exactly the path nodes that lie in tile c'.
// One CTA of 256 threads per (sequence, head), one CTA per SM:
//   0. TMA: S_root (four 32-column fp32 chunks) and the q / k / v tiles of tiles 0 and 1.
//      Tree walk (one thread per node): ancestor bits, depth, root-first paths, cl, gamma,
//      and per tile the set of tiles holding path nodes of its nodes (warp OR-reductions).
//   1. S_root fp32 -> bf16, row v into tensor-memory lane v (the state MMA's A operand);
//      then the k tiles of tiles 0..N/64-2 into the freed staging area, where the Gram
//      blocks of later tiles read them.
//   for every tile c:
//   2. Gram blocks [Q_c ; K_c] . K_c'^T (tcgen05 kind::f16) for every c' <= c in one batch:
//      the earlier tiles' k rows lie back to back in shared memory, so they form one operand
//      of 64 c rows (one MMA chain, N = 64 c), and the tile's own k rows another (N = 64);
//      three threads issue the chains.  Each thread stages its row's 32 values of a block in
//      shared memory and picks out its path columns: q_n.k_i for i on path(n) (this tile's
//      rows), b_n k_n.k_i for i in anc(n) (kept for all nodes), stored by path position.
//   3. state MMA S_root . [Q_c ; K_c]^T (kind::f16, A = S_root from tensor memory), in the
//      same batch as the Gram chains when their columns do not overlap its own.
//   4. warps 4-7, per value lane and all 64 node columns: o columns scaled by gamma_n,
//      R^T_c[v][j] = b_j v_j[v] - b_j gamma_j (S_root k_j)[v] (tf32) into tensor memory next
//      to the R^T of earlier tiles, U zeroed; meanwhile warps 0-3 run the T and W rows of
//      the tile's nodes (register recursions, paths up to kDepth deep).
//   5. path MMAs, one per tile c' <= c holding path nodes: [o ; U]_c^T += R^T_c' . [W ; T]_c,c'^T
//      (kind::tf32, A = R^T_c' from tensor memory, B = the coefficient block in shared
//      memory, built from each row's path positions in tile c'; two N = 64 chains).
//   6. o_c and U_c from tensor memory: a full tile as node rows in shared memory and two TMA
//      tensor stores (read out before the next tile's extraction, after which that buffer
//      takes the tile two ahead), a ragged last tile as 128-byte row segments.
// Tensor memory (512 columns): [0, 256) R^T of the four tiles, [256, 384) o^T | U^T of the
// current tile, [384, 448) S_root in bf16, [448, 512) the Gram block of the tile's own k rows.
// The Gram blocks of tile c against tiles 0..c-1 go to [64 c, 128 c): R^T columns of tiles
// c.. (written later, in step 4) and, for c = 3, the o^T | U^T columns (the state MMA then
// waits until they are read).  Shared memory holds two q / k / v buffers (tile c in buffer
// c & 1), one coefficient buffer and the k rows of tiles 0..2.
// Trees deeper than kDepth are verified by the CUDA-core algorithm in the same CTA.
//
// Every wait is bounded: a wait that runs out records TV_ERR_TIMEOUT on the status word; the
// CTA then lets its copies and MMAs finish (bounded), frees tensor memory and returns.
#include "simt_item.cuh"
#include "tc_ptx.cuh"
#include "tmaps.cuh"

namespace tv {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;
constexpr int kTiles = 4;
constexpr int kNodes = kTile * kTiles;     // 256
constexpr int kDepth = 16;                 // deepest path the tensor-core path takes
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColR = 0;              // R^T of tile c at 64 c .. 64 c + 63
constexpr uint32_t kColD = 256;            // o^T (64 columns) then U^T (64 columns)
constexpr uint32_t kColA = 384;            // S_root in bf16 (64 columns)
constexpr uint32_t kColG = 448;            // one Gram block (64 columns)
constexpr uint32_t kSpinLimit = 1u << 22;

// Dynamic shared memory, offsets from a 1024-byte aligned base.
constexpr int kHalf = 128 * 128;            // one 64-wide K half of a 128-row bf16 operand
constexpr int kQKBytes = 2 * kHalf;         // [Q_c ; K_c]
constexpr int kKHalf = kTile * 128;         // one K half of a 64-row bf16 tile
constexpr int kKBytes = 2 * kKHalf;         // one k (or v) tile
constexpr int kAtom2 = 16384;               // one 32-wide K atom of the 128-row fp32 operand
constexpr int kOffQK = 0;                   // two buffers (tile c in buffer c & 1)
constexpr int kOffV = 2 * kQKBytes;         // two buffers
constexpr int kOffWT = kOffV + 2 * kKBytes; // [W ; T] block: 128 rows x 64 fp32, two K atoms
constexpr int kOffKS = kOffWT + 2 * kAtom2; // k tiles 0..2 for the Gram blocks of later tiles
constexpr int kKSHalf = 3 * kKHalf;         // K half h of those tiles: rows of tiles 0..2 in order
constexpr int kOffS = kOffWT;               // S_root fp32 staging (64 KiB) before steps 2..7
constexpr int kOffMeta = kOffKS + 3 * kKBytes;

struct Meta {
  unsigned long long bar_s, bar_t[2], bar_ks, bar_mma, bar_g, bar_pm;
  uint32_t tmem_base;
  int flag;
  int maxdep;
  unsigned blkm[kTiles];              // tile c: bit c' set if tile c' holds path nodes of its nodes
  unsigned long long anc[kNodes][4];  // strict-ancestor bits, word w = nodes 64 w .. 64 w + 63
  int par[kNodes];
  int dep[kNodes];
  float la[kNodes];
  float bb[kNodes];
  float cl[kNodes];
  __align__(16) float gam[kNodes];    // gamma_n (0 past the last node)
  __align__(16) float bg[kNodes];     // b_n gamma_n
  __align__(16) float bq[kNodes];     // b_n
  float lpos[kDepth][kNodes];         // b_j k_j.k_{a-th ancestor of j}, every node
  float gpos[kDepth][kTile];          // q_n.k_{a-th node of path(n)}, then W, current tile
  float tpos[kDepth][kTile];          // T[n][p_a], current tile
  uint8_t paths[kDepth][kNodes];      // a-th node of path(n), root first
};
constexpr int kSmemBytes = kOffMeta + (int)sizeof(Meta) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(simt_smem_bytes(128, 128) <= (size_t)kOffMeta, "deep-tree fallback workspace");

__device__ __forceinline__ int op2_off(int row, int k) {
  return ((k >> 5) * kAtom2) + (row << 7) + ((((k >> 2) & 7) ^ (row & 7)) << 4) + ((k & 3) << 2);
}
__device__ __forceinline__ float tf32_rn(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void st_out(float *p, float x) { __stcs(p, x); }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

// Thread 0 waits on `bar`; every thread learns whether it completed (and leaves the
// tcgen05 fence for the caller).  A time-out is recorded once.
__device__ __forceinline__ bool wait_all(Meta &mt, uint32_t bar, uint32_t parity, int *ws, int s) {
  if (threadIdx.x == 0 && !ptx::mbar_wait_bounded(bar, parity, kSpinLimit)) {
    mt.flag = TV_ERR_TIMEOUT;
    set_status(ws, TV_ERR_TIMEOUT, s);
  }
  __syncthreads();
  return mt.flag == 0;
}

// Row r of T (kW false) or W (kW true) for node n by path position a < d, decayed and
// rounded to tf32, into tpos / gpos column r.
template <bool kW, bool kGdn>
__device__ __forceinline__ void row_coefficients(Meta &mt, int n, int r, int d) {
  const float cln = mt.cl[n];
  int p[kDepth];
  float x[kDepth];
#pragma unroll
  for (int a = 0; a < kDepth; ++a) {
    p[a] = a < d ? mt.paths[a][n] : n;
    x[a] = kW ? (a < d ? mt.gpos[a][r] : 0.f) : (a == d - 1 ? 1.f : 0.f);
  }
#pragma unroll
  for (int c = kDepth - 1; c >= 1; --c) {
    if (kGdn && c < d) {
      const float xc = x[c];
#pragma unroll
      for (int a = 0; a < c; ++a) x[a] = fmaf(-xc, mt.lpos[a][p[c]], x[a]);
    }
  }
  float(*dst)[kTile] = kW ? mt.gpos : mt.tpos;
#pragma unroll
  for (int a = 0; a < kDepth; ++a)
    if (a < d) dst[a][r] = tf32_rn(x[a] * __expf(cln - mt.cl[p[a]]));
}

// q, k and v of tile t (64 node rows from lo + 64 t) into buffer t & 1; out-of-range rows
// of the box are zero-filled or belong to the next sequence, and are never used.
__device__ __forceinline__ void issue_tile(uint32_t sbase, Meta &mt, const CUtensorMap *tq,
                                           const CUtensorMap *tk, const CUtensorMap *tv_, int h,
                                           int kh, int lo, int t) {
  const int b = t & 1;
  const uint32_t bar = ptx::smem_addr(&mt.bar_t[b]);
  ptx::mbar_arrive_expect_tx(bar, 6 * kKHalf);
  for (int half = 0; half < 2; ++half) {
    const uint32_t hb = sbase + kOffQK + b * kQKBytes + half * kHalf;
    ptx::tma_load_3d(hb, tq, bar, half * 64, kh, lo + kTile * t);
    ptx::tma_load_3d(hb + kKHalf, tk, bar, half * 64, kh, lo + kTile * t);
    ptx::tma_load_3d(sbase + kOffV + b * kKBytes + half * kKHalf, tv_, bar, half * 64, h,
                     lo + kTile * t);
  }
}

// Leave after a time-out or a malformed tree: let issued copies and MMAs finish, free
// tensor memory.  `t_issued` tiles were issued (tile t on buffer t & 1, phase t >> 1).
__device__ void bail_out(Meta &mt, uint32_t tmem, bool tmem_held, int t_issued, bool ks_issued,
                         bool s_issued) {
  if (threadIdx.x == 0) {
    if (s_issued) ptx::mbar_wait_bounded(ptx::smem_addr(&mt.bar_s), 0, kSpinLimit);
    if (ks_issued) ptx::mbar_wait_bounded(ptx::smem_addr(&mt.bar_ks), 0, kSpinLimit);
    for (int t = t_issued > 2 ? t_issued - 2 : 0; t < t_issued; ++t)
      ptx::mbar_wait_bounded(ptx::smem_addr(&mt.bar_t[t & 1]), (t >> 1) & 1, kSpinLimit);
  }
  if (threadIdx.x == 0) ptx::bulk_wait();   // output rows still being copied out
  ptx::tc_fence_before();
  __syncthreads();
  if (tmem_held && (threadIdx.x >> 5) == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool kGdn, typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
    verify_tcw_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_s,
                      const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_u, VerifyArgs a) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Meta &mt = *reinterpret_cast<Meta *>(sm + kOffMeta);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int H = a.H;
  const int s = blockIdx.x / H, h = blockIdx.x % H, kh = qk_head(h, H, a.Hk);
  // Launched with programmatic stream serialisation: the kernel before this one on the
  // stream may still be finishing.  Until it has (griddepcontrol.wait), this CTA only asks
  // L2 for its S_root block and node range: a prefetch moves nothing into the CTA, and a
  // write by that kernel to the same lines lands in L2 after it, so this is correct
  // whatever it writes.  Then the kernel after this one may get its CTAs resident early.
  if (threadIdx.x == 0) {
    ptx::prefetch_l2(a.S_root + (size_t)blockIdx.x * 128 * 128, 128 * 128 * 4);
    ptx::prefetch_line_l2(a.node_offsets + blockIdx.x / a.H);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes || hi - lo > kNodes ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n = hi - lo;
  if (n == 0) return;
  const int n_tiles = (n + kTile - 1) / kTile;
  const uint32_t sbase = ptx::smem_addr(sm);

  // ---- 0. tree inputs, copies out, tensor memory, walk -------------------------------------
  // the tree's small loads go out first, ahead of the bulk copies in the memory queues
  int p_in = -1;
  float la_in = 0.f, bb_in = 0.f;
  if (tid < n) {
    p_in = a.parent[lo + tid];
    la_in = a.log_a[(size_t)(lo + tid) * H + h];
    bb_in = kGdn ? a.b[(size_t)(lo + tid) * H + h] : 0.f;
  }
  if (tid == 0) {
    ptx::mbar_init(ptx::smem_addr(&mt.bar_s), 1);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_t[0]), 1);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_t[1]), 1);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_ks), 1);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_mma), 1);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_g), 3);
    ptx::mbar_init(ptx::smem_addr(&mt.bar_pm), 2);
    ptx::fence_mbar_init();
    mt.flag = 0;
    mt.maxdep = 0;
    for (int t = 0; t < kTiles; ++t) mt.blkm[t] = 0u;
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_s);
    ptx::prefetch_tmap(&tm_o);
    ptx::prefetch_tmap(&tm_u);
    const uint32_t bs = ptx::smem_addr(&mt.bar_s);
    ptx::mbar_arrive_expect_tx(bs, 4 * kAtom2);
    for (int c = 0; c < 4; ++c)
      ptx::tma_load_2d(sbase + kOffS + c * kAtom2, &tm_s, bs, c * 32, blockIdx.x * 128);
    for (int t = 0; t < 2 && t < n_tiles; ++t) issue_tile(sbase, mt, &tm_q, &tm_k, &tm_v, h, kh, lo, t);
  }
  int t_issued = n_tiles < 2 ? n_tiles : 2;
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&mt.tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  const bool bad = tid < n && (p_in < -1 || p_in >= tid);
  mt.par[tid] = p_in;
  mt.la[tid] = la_in;
  mt.bb[tid] = bb_in;
  ptx::tc_fence_before();
  const bool bad_tree = __syncthreads_or(bad) != 0;
  ptx::tc_fence_after();
  const uint32_t tmem = mt.tmem_base;
  if (bad_tree) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    bail_out(mt, tmem, true, t_issued, false, true);
    return;
  }
  {
    // one thread per node: its ancestors in ascending order are its root-first path
    unsigned long long bits[4] = {0ull, 0ull, 0ull, 0ull};
    int d = 0;
    float cl = 0.f;
    if (tid < n) {
      for (int x = mt.par[tid]; x >= 0; x = mt.par[x]) bits[x >> 6] |= 1ull << (x & 63);
#pragma unroll
      for (int w = 0; w < 4; ++w)
        for (unsigned long long b = bits[w]; b; b &= b - 1) {
          const int x = w * 64 + __ffsll((long long)b) - 1;
          if (d < kDepth) mt.paths[d][tid] = (uint8_t)x;
          cl += mt.la[x];
          ++d;
        }
      if (d < kDepth) mt.paths[d][tid] = (uint8_t)tid;
      cl += mt.la[tid];
      ++d;
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) mt.anc[tid][w] = bits[w];
    const float gam = tid < n ? __expf(cl) : 0.f;
    mt.dep[tid] = d;
    mt.cl[tid] = cl;
    mt.gam[tid] = gam;
    mt.bg[tid] = mt.bb[tid] * gam;
    mt.bq[tid] = mt.bb[tid];
    atomicMax(&mt.maxdep, d);
    // tiles holding path nodes (ancestors and the node itself), OR-ed over each warp: the
    // 32 nodes of a warp lie in one tile
    unsigned tm = tid < n ? 1u << (tid >> 6) : 0u;
#pragma unroll
    for (int w = 0; w < 4; ++w) tm |= bits[w] ? 1u << w : 0u;
    tm = __reduce_or_sync(0xffffffffu, tm);
    if ((tid & 31) == 0 && tm) atomicOr(&mt.blkm[tid >> 6], tm);
  }
  __syncthreads();
  if (mt.maxdep > kDepth) {
    // deeper than the path registers: verify this item on CUDA cores, in the same CTA
    bail_out(mt, tmem, true, t_issued, false, true);
    simt_item<__nv_bfloat16, Tout, kGdn, kThreads>(a, s, h, sm);
    return;
  }

  // ---- 1. S_root -> bf16 A operand (lane v = value row v) -----------------------------------
  if (!wait_all(mt, ptx::smem_addr(&mt.bar_s), 0, a.ws, s)) {
    bail_out(mt, tmem, true, t_issued, false, true);
    return;
  }
  const int row = tid & 127, ch = tid >> 7;
  const uint32_t tlane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  if (tid < 128) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      const unsigned char *rp = sm + kOffS + c * kAtom2 + row * 128;
      uint32_t pk[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 f = *reinterpret_cast<const float4 *>(rp + ((u ^ (row & 7)) << 4));
        pk[2 * u] = pack_bf16(f.x, f.y);
        pk[2 * u + 1] = pack_bf16(f.z, f.w);
      }
      ptx::tmem_st16(tlane + kColA + c * 16, reinterpret_cast<const float(&)[16]>(pk));
    }
    ptx::tmem_wait_st();
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const bool ks_issued = n_tiles > 1;
  if (tid == 0 && ks_issued) {
    // k of tiles 0 .. n_tiles - 2 over the staging area, for the Gram blocks of later tiles
    const uint32_t bk = ptx::smem_addr(&mt.bar_ks);
    ptx::mbar_arrive_expect_tx(bk, (n_tiles - 1) * kKBytes);
    for (int t = 0; t < n_tiles - 1; ++t)
      for (int half = 0; half < 2; ++half)
        ptx::tma_load_3d(sbase + kOffKS + half * kKSHalf + t * kKHalf, &tm_k, bk, half * 64, kh,
                         lo + kTile * t);
  }

  uint32_t mma_phase = 0, gphase = 0, pm_phase = 0;
  for (int c = 0; c < n_tiles; ++c) {
    const int b = c & 1, node0 = c * kTile;
    const int nc = n - node0 < kTile ? n - node0 : kTile;
    const uint32_t qk = sbase + kOffQK + b * kQKBytes;
    bool ok = wait_all(mt, ptx::smem_addr(&mt.bar_t[b]), (c >> 1) & 1, a.ws, s);
    if (ok && c == 1) ok = wait_all(mt, ptx::smem_addr(&mt.bar_ks), 0, a.ws, s);
    if (!ok) {
      bail_out(mt, tmem, true, t_issued, ks_issued, false);
      return;
    }
    const unsigned blkm = mt.blkm[c];       // tiles holding path nodes of this tile's nodes

    // ---- 2. Gram blocks and their entries by path position (+ 3. the state MMA) ----------
    const bool g_is_q = row < kTile;
    const int gr = row & (kTile - 1);
    const int gn = node0 + gr;               // node of this Gram row
    const bool g_live = gr < nc;
    const uint32_t col_early = kTile * c;    // Gram blocks against tiles 0..c-1
    const bool state_early = 2 * kTile * c <= (int)kColD;
    // Three chains into separate columns, issued by one thread each of warps 0-2 (the issue
    // of a tcgen05.mma takes tens of cycles); every issuer commits to bar_g.
    if ((tid & 31) == 0 && warp < 3) {
      ptx::tc_fence_after();
      if (warp == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16(tmem + kColG,
                        ptx::smem_desc_sw128(qk + (kk >> 2) * kHalf + (kk & 3) * 32, 1024),
                        ptx::smem_desc_sw128(qk + kKHalf + (kk >> 2) * kHalf + (kk & 3) * 32, 1024),
                        ptx::idesc_bf16_f32(128, kTile), kk > 0 ? 1u : 0u);
      } else if (warp == 1 && c > 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16(tmem + col_early,
                        ptx::smem_desc_sw128(qk + (kk >> 2) * kHalf + (kk & 3) * 32, 1024),
                        ptx::smem_desc_sw128(sbase + kOffKS + (kk >> 2) * kKSHalf + (kk & 3) * 32, 1024),
                        ptx::idesc_bf16_f32(128, kTile * c), kk > 0 ? 1u : 0u);
      } else if (warp == 2 && state_early) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_tmem_a(tmem + kColD, tmem + kColA + kk * 8,
                               ptx::smem_desc_sw128(qk + (kk >> 2) * kHalf + (kk & 3) * 32, 1024),
                               ptx::idesc_bf16_f32(128, 128), kk > 0 ? 1u : 0u);
      }
      ptx::mma_commit(ptx::smem_addr(&mt.bar_g));
    }
    // The previous tile's output rows must have been read out of shared memory before the
    // extraction below writes its slots; then that tile's buffer takes the tile two ahead.
    if (tid == 0) ptx::bulk_wait_read();
    if (!wait_all(mt, ptx::smem_addr(&mt.bar_g), gphase++ & 1, a.ws, s)) {
      bail_out(mt, tmem, true, t_issued, ks_issued, false);
      return;
    }
    if (c >= 1 && c + 1 < n_tiles) {
      if (tid == 0) issue_tile(sbase, mt, &tm_q, &tm_k, &tm_v, h, kh, lo, c + 1);
      t_issued = c + 2;
    }
    ptx::tc_fence_after();
    // Each thread stages its 32 Gram values of a block in its own 128-byte slot of the
    // (idle) coefficient buffer, then visits only the columns on its row's path.
    unsigned char *slot = sm + kOffWT + (row * 2 + ch) * 128;
    for (int c2 = 0; c2 <= c; ++c2) {
      if (!((blkm >> c2) & 1u)) continue;
      if (g_is_q || kGdn) {   // uniform per warp: rows 0..63 are q rows
        const uint32_t gcol = c2 < c ? col_early + kTile * c2 : kColG;
        float g[2][16];
        ptx::tmem_ld16(tlane + gcol + 32 * ch, g[0]);
        ptx::tmem_ld16(tlane + gcol + 32 * ch + 16, g[1]);
        ptx::tmem_wait_ld();
        if (g_live) {
          // bits of path(gn) (q rows) or anc(gn) (k rows) in tile c2, and the number of path
          // entries before tile c2 and before this thread's 32 columns
          int pos = 0;
          for (int w = 0; w < c2; ++w) pos += __popcll(mt.anc[gn][w]);
          unsigned long long wb = mt.anc[gn][c2];
          if (g_is_q && c2 == c) wb |= 1ull << gr;
          pos += __popcll(wb & ((1ull << (32 * ch)) - 1ull));
          unsigned bits = (unsigned)(wb >> (32 * ch));
          if (bits) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4 *>(slot + ((q4 ^ (row & 7)) << 4)) =
                  make_float4(g[q4 >> 2][(q4 & 3) * 4], g[q4 >> 2][(q4 & 3) * 4 + 1],
                              g[q4 >> 2][(q4 & 3) * 4 + 2], g[q4 >> 2][(q4 & 3) * 4 + 3]);
            const float scale = g_is_q ? 1.f : mt.bb[gn];
            while (bits) {
              const int j = __ffs(bits) - 1;
              bits &= bits - 1u;
              const float val =
                  *reinterpret_cast<const float *>(slot + ((((j >> 2) ^ (row & 7)) << 4) | ((j & 3) << 2)));
              if (g_is_q) mt.gpos[pos][gr] = val;
              else mt.lpos[pos][gn] = scale * val;
              ++pos;
            }
          }
        }
      }
    }
    ptx::tc_fence_before();
    __syncthreads();

    if (!state_early) {
      // ---- 3. state MMA: [o^T | U^T] columns = S_root . [Q_c ; K_c]^T ---------------------
      if (tid == 0) {
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_tmem_a(tmem + kColD, tmem + kColA + kk * 8,
                               ptx::smem_desc_sw128(qk + (kk >> 2) * kHalf + (kk & 3) * 32, 1024),
                               ptx::idesc_bf16_f32(128, 128), kk > 0 ? 1u : 0u);
        ptx::mma_commit(ptx::smem_addr(&mt.bar_mma));
      }
      if (!wait_all(mt, ptx::smem_addr(&mt.bar_mma), mma_phase++ & 1, a.ws, s)) {
        bail_out(mt, tmem, true, t_issued, ks_issued, false);
        return;
      }
    }
    ptx::tc_fence_after();

    // ---- 4. warps 4-7 form gamma o^T, R^T_c and U^T = 0 for all 64 node columns of their
    // lanes (lane v = tid - 128) while warps 0-3 run the W rows (threads 0..63) and T rows
    // (threads 64..127) of the tile's nodes.
    if (tid >= 128) {
      const int v = row;
      const unsigned char *vt = sm + kOffV + b * kKBytes + (v >> 6) * kKHalf + (v & 7) * 2;
      const int vc = (v & 63) >> 3;
#pragma unroll 1
      for (int j0 = 0; j0 < kTile; j0 += 32) {
        float o0[16], o1[16], k0[16], k1[16];
        ptx::tmem_ld16(tlane + kColD + j0, o0);
        ptx::tmem_ld16(tlane + kColD + j0 + 16, o1);
        ptx::tmem_ld16(tlane + kColD + kTile + j0, k0);
        ptx::tmem_ld16(tlane + kColD + kTile + j0 + 16, k1);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int ja = j0 + j, jb = j0 + 16 + j;
          o0[j] *= mt.gam[node0 + ja];
          o1[j] *= mt.gam[node0 + jb];
          const float va = __bfloat162float(
              *reinterpret_cast<const __nv_bfloat16 *>(vt + ja * 128 + ((vc ^ (ja & 7)) << 4)));
          const float vb = __bfloat162float(
              *reinterpret_cast<const __nv_bfloat16 *>(vt + jb * 128 + ((vc ^ (jb & 7)) << 4)));
          k0[j] = ja < nc ? tf32_rn(kGdn ? fmaf(-mt.bg[node0 + ja], k0[j], mt.bq[node0 + ja] * va) : va) : 0.f;
          k1[j] = jb < nc ? tf32_rn(kGdn ? fmaf(-mt.bg[node0 + jb], k1[j], mt.bq[node0 + jb] * vb) : vb) : 0.f;
        }
        ptx::tmem_st16(tlane + kColD + j0, o0);
        ptx::tmem_st16(tlane + kColD + j0 + 16, o1);
        ptx::tmem_st16(tlane + kColR + kTile * c + j0, k0);
        ptx::tmem_st16(tlane + kColR + kTile * c + j0 + 16, k1);
#pragma unroll
        for (int j = 0; j < 16; ++j) k0[j] = 0.f;
        ptx::tmem_st16(tlane + kColD + kTile + j0, k0);
        ptx::tmem_st16(tlane + kColD + kTile + j0 + 16, k0);
      }
      ptx::tmem_wait_st();
    } else if ((tid & 63) < nc) {
      const int r = tid & 63, nn = node0 + r, d = mt.dep[nn];
      if (tid < kTile) row_coefficients<true, kGdn>(mt, nn, r, d);
      else row_coefficients<false, kGdn>(mt, nn, r, d);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    // ---- 5. path MMAs, one coefficient block per tile c' holding path nodes -----------------
    for (int c2 = 0; c2 <= c; ++c2) {
      if (!((blkm >> c2) & 1u)) continue;
      {
        // thread t writes K atom t / 128 (node columns 32 atom .. 32 atom + 31 of tile c2) of
        // operand row t % 128: zeros, then its path coefficients that fall there
        const int r2 = row, atom = ch;
        const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<float4 *>(sm + kOffWT + op2_off(r2, atom * 32 + q4 * 4)) = zf;
        const int r = r2 & 63;
        if (r < nc) {
          // the path positions that fall in tile c2: after the ones in tiles 0..c2-1
          const int nn = node0 + r;
          const float(*cf)[kTile] = r2 < kTile ? mt.gpos : mt.tpos;
          int a0 = 0;
          for (int w = 0; w < c2; ++w) a0 += __popcll(mt.anc[nn][w]);
          const int a1 = a0 + __popcll(mt.anc[nn][c2]) + (c2 == c ? 1 : 0);
          for (int a2 = a0; a2 < a1; ++a2) {
            const int i = mt.paths[a2][nn];
            if (((i >> 5) & 1) == atom)
              *reinterpret_cast<float *>(sm + kOffWT + op2_off(r2, i & 63)) = cf[a2][r];
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      // two chains of N = 64 from two threads: W rows into the o columns, T rows into the U
      // columns (rows 64.. of each K atom start 8 KiB into it)
      if (tid == 0 || tid == 32) {
        ptx::tc_fence_after();
        const uint32_t hf = tid == 0 ? 0u : 1u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_tf32_tmem_a(tmem + kColD + hf * kTile, tmem + kColR + kTile * c2 + kk * 8,
                               ptx::smem_desc_sw128(sbase + kOffWT + hf * (kTile * 128) + (kk >> 2) * kAtom2 + (kk & 3) * 32, 1024),
                               ptx::idesc_tf32_f32(128, kTile), 1u);
        ptx::mma_commit(ptx::smem_addr(&mt.bar_pm));
      }
      if (!wait_all(mt, ptx::smem_addr(&mt.bar_pm), pm_phase++ & 1, a.ws, s)) {
        bail_out(mt, tmem, true, t_issued, ks_issued, false);
        return;
      }
    }
    ptx::tc_fence_after();

    // ---- 6. o_c and U_c (lane v, node columns 32 ch .. 32 ch + 31) --------------------------
    {
      const int v = row, j0 = 32 * ch;
      float o0[16], o1[16], u0[16], u1[16];
      ptx::tmem_ld16(tlane + kColD + j0, o0);
      ptx::tmem_ld16(tlane + kColD + j0 + 16, o1);
      ptx::tmem_ld16(tlane + kColD + kTile + j0, u0);
      ptx::tmem_ld16(tlane + kColD + kTile + j0 + 16, u1);
      ptx::tmem_wait_ld();
      if (nc == kTile) {
        // a full tile: node rows into shared memory (o over the coefficient buffer, U over
        // this tile's dead q / k buffer), then one tensor store each; both buffers are read
        // out before the next tile touches them
        Tout *ost = reinterpret_cast<Tout *>(sm + kOffWT);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          ost[(j0 + j) * 128 + v] = from_f32<Tout>(o0[j]);
          ost[(j0 + 16 + j) * 128 + v] = from_f32<Tout>(o1[j]);
        }
        unsigned char *ust = sm + kOffQK + b * kQKBytes;
        if (a.u_bf16) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            reinterpret_cast<__nv_bfloat16 *>(ust)[(j0 + j) * 128 + v] = __float2bfloat16_rn(u0[j]);
            reinterpret_cast<__nv_bfloat16 *>(ust)[(j0 + 16 + j) * 128 + v] = __float2bfloat16_rn(u1[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            reinterpret_cast<float *>(ust)[(j0 + j) * 128 + v] = u0[j];
            reinterpret_cast<float *>(ust)[(j0 + 16 + j) * 128 + v] = u1[j];
          }
        }
        ptx::fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
          ptx::tma_store_3d(&tm_o, sbase + kOffWT, 0, h, lo + node0);
          ptx::tma_store_3d(&tm_u, ptx::smem_addr(ust), 0, h, lo + node0);
          ptx::bulk_commit();
        }
      } else {
        Tout *out = static_cast<Tout *>(a.out) + ((size_t)(lo + node0) * H + h) * 128 + v;
        const size_t ub = ((size_t)(lo + node0) * H + h) * 128 + v;
        const size_t rs = (size_t)H * 128;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j0 + j < nc) {
            st_out(out + (j0 + j) * rs, o0[j]);
            store_u(a.U, ub + (j0 + j) * rs, u0[j], a.u_bf16);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j0 + 16 + j < nc) {
            st_out(out + (j0 + 16 + j) * rs, o1[j]);
            store_u(a.U, ub + (j0 + 16 + j) * rs, u1[j], a.u_bf16);
          }
        }
      }
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (tid == 0) ptx::bulk_wait();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool kGdn, typename Tout>
cudaError_t launch_tcw_t(const VerifyArgs &a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, ms, mo, mu;
  if (!make_node_map(&mq, a.q, a.Hk, a.T, kTile) || !make_node_map(&mk, a.k, a.Hk, a.T, kTile) ||
      !make_node_map(&mv, a.v, a.H, a.T, kTile) ||
      !make_state_map(&ms, a.S_root, (long long)a.B * a.H * 128) ||
      !make_row_map(&mo, a.out, sizeof(Tout) == 2, a.H, a.T, kTile) ||
      !make_row_map(&mu, a.U, a.u_bf16 != 0, a.H, a.T, kTile))
    return cudaErrorInvalidValue;
  auto kern = verify_tcw_kernel<kGdn, Tout>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
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
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, ms, mo, mu, a);
}

}  // namespace

int verify_tcw_max_nodes() { return kNodes; }

cudaError_t launch_verify_tcw(const VerifyArgs &a, int mode, int out_dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const bool gdn = mode == TV_MODE_GDN;
  if (out_dtype == TV_BF16)
    return gdn ? launch_tcw_t<true, __nv_bfloat16>(a, st) : launch_tcw_t<false, __nv_bfloat16>(a, st);
  return gdn ? launch_tcw_t<true, float>(a, st) : launch_tcw_t<false, float>(a, st);
}

}  // namespace tv
