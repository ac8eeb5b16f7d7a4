// Tensor-core tree verification for sm_100a: bf16 q/k/v, dk = dv = 128, up to 64 nodes
// per tree, gated delta rule or scalar decay.
//
// One CTA (256 threads, two per SM) per (sequence, head).  The only dense contraction of
// the method runs on the 5th-generation tensor cores as ONE 128 x 192 x 128 MMA:
//
//      [ Q ]                     [ Q K^T | S_root Q^T ... ]     rows 0..63   : q_n
//      [ K ] . [ K ; S_root ]^T = [ K K^T | S_root K^T ... ]    rows 64..127 : k_n
//
// so a single accumulator in tensor memory (TMEM) holds the path Gram terms q_n.k_i and
// k_n.k_i (columns 0..63) and the state products S_root q_n and S_root k_n (columns
// 64..191).  q, k and v arrive by TMA in the 128-byte swizzled layout the MMA reads;
// S_root (fp32 in HBM) is converted to bf16 by all threads straight into the same layout.
//
// With cl_n the fp32 cumulative log-decay of the root->n path and gamma_n = exp(cl_n):
//   pseudo-values (tree-structured WY form, TreeWY abstract): forward substitution
//     u_n = b_n (v_n - gamma_n S_root k_n) - sum_{i in anc(n)} b_n exp(cl_n-cl_i)(k_n.k_i) u_i
//   level by level over depth (nodes of one depth are independent), every value column
//   in parallel;
//   outputs (closed form of the Bole summary's worked example, "具体技术细节示例",
//   extended to the delta rule):
//     o_n = gamma_n S_root q_n + sum_{i in path(n)} exp(cl_n-cl_i) (q_n.k_i) u_i .
// Scalar decay has u_n = v_n.  o and U leave with coalesced stores.
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
constexpr uint32_t kTmemCols = 256;        // 192 used; two CTAs per SM share the 512
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait is declared timed out

// Dynamic shared memory (offsets from a 1024-byte aligned base).
constexpr int kOpHalf = 256 * 128;         // one 64-wide K half of [Q;K;S]: 256 rows x 128 B
constexpr int kOffOp = 0;                  // operand tile, 2 halves = 64 KiB
constexpr int kVHalf = kTile * 128;
constexpr int kOffV = 2 * kOpHalf;         // v tile (bf16, TMA-swizzled), 2 halves = 16 KiB
constexpr int kOffLc = kOffV + 2 * kVHalf; // b_n exp(cl_n-cl_i) k_n.k_i, 64 x 64 fp32
constexpr int kOffMisc = kOffLc + kTile * kTile * 4;
// after the MMA has consumed the operands:
constexpr int kOffU = kOffOp;              // pseudo-values, 64 x 128 fp32 (swizzled)
constexpr int kOffSQ = kOffOp + 32768;     // gamma_n S_root q_n, 64 x 128 fp32 (swizzled)
constexpr int kOffP = kOffV;               // exp(cl_n-cl_i) q_n.k_i, 64 x 64 fp32

struct Misc {
  unsigned long long bar_tma;
  unsigned long long bar_mma;
  unsigned long long anc[kTile];   // strict-ancestor bitmask
  uint32_t tmem_base;
  int flag;                        // 0 ok, else a tv_status to record
  int maxdep;
  int par[kTile];
  int dep[kTile];
  int lvl_start[kTile + 2];
  int lvl_nodes[kTile];
  float la[kTile];
  float bb[kTile];
  float cl[kTile];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;

// fp32 [64 rows][128 cols] in four 32-column slabs of 128-byte rows, 16-byte chunks
// XOR-swizzled by row: both row-per-thread and column-per-thread access are conflict-free.
__device__ __forceinline__ int f32_tile_off(int n, int v) {
  return ((v >> 5) << 13) + (n << 7) + ((((v >> 2) & 7) ^ (n & 7)) << 4) + ((v & 3) << 2);
}
// [64][64] fp32 coefficient matrix, column XOR-swizzled by row (conflict-free row writes).
__device__ __forceinline__ int coef_off(int n, int i) { return (n << 6) + (i ^ (n & 31)); }

__device__ __forceinline__ float bf16_tile_ld(const unsigned char *vt, int n, int v) {
  const int half = v >> 6, chunk = (v & 63) >> 3;
  const int off = half * kVHalf + (n << 7) + ((chunk ^ (n & 7)) << 4) + ((v & 7) << 1);
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(vt + off));
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
  const uint32_t bar_mma = ptx::smem_addr(&ms.bar_mma);
  const uint32_t op = ptx::smem_addr(sm + kOffOp);

  // ---- 1. barriers, TMA of q / k / v, TMEM allocation ---------------------------------
  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_mma, 1);
    ptx::fence_mbar_init();
    ms.flag = 0;
    ms.maxdep = 0;
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::mbar_arrive_expect_tx(bar_tma, 6 * kTile * 128);
    for (int half = 0; half < 2; ++half) {
      const uint32_t hb = op + half * kOpHalf;
      ptx::tma_load_3d(hb, &tm_q, bar_tma, half * 64, h, lo);
      ptx::tma_load_3d(hb + kTile * 128, &tm_k, bar_tma, half * 64, h, lo);
      ptx::tma_load_3d(ptx::smem_addr(sm + kOffV + half * kVHalf), &tm_v, bar_tma, half * 64, h, lo);
    }
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&ms.tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }

  // ---- 2. S_root fp32 -> bf16, rows 128..255 of the operand tile ----------------------
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
      if (tid < n_nodes) {
        const int p = a.parent[lo + tid];
        if (p < -1 || p >= tid) ms.flag = TV_ERR_BAD_TREE;
        ms.par[tid] = p;
        ms.la[tid] = a.log_a[(size_t)(lo + tid) * H + h];
        ms.bb[tid] = kGdn ? a.b[(size_t)(lo + tid) * H + h] : 0.f;
      } else {
        ms.par[tid] = -1;
        ms.la[tid] = 0.f;
        ms.bb[tid] = 0.f;
      }
      ms.anc[tid] = 0ull;
      ms.dep[tid] = 0;
      ms.cl[tid] = 0.f;
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

  // ---- 3. one thread waits for the tiles and issues the MMA chain --------------------
  if (tid == kThreads - 1) {
    const bool loaded = ptx::mbar_wait_bounded(bar_tma, 0, kSpinLimit);
    if (!loaded) {
      ms.flag = TV_ERR_TIMEOUT;
    } else if (ms.flag == 0) {
      ptx::tc_fence_after();
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 192);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t base = op + (kk >> 2) * kOpHalf + (kk & 3) * 32;
        const uint64_t ad = ptx::smem_desc_sw128(base, 1024);
        const uint64_t bd = ptx::smem_desc_sw128(base + kTile * 128, 1024);
        ptx::mma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      ptx::mma_commit(bar_mma);
    }
  }
  // tree metadata while the tensor core works: depth and strict-ancestor bits
  if (tid < n_nodes && ms.flag == 0) {
    unsigned long long bits = 0ull;
    int d = 1;
    for (int x = ms.par[tid]; x >= 0; x = ms.par[x]) {
      bits |= 1ull << x;
      ++d;
    }
    ms.anc[tid] = bits;
    ms.dep[tid] = d;
    atomicMax(&ms.maxdep, d);
  }
  __syncthreads();
  const int flag0 = ms.flag;
  if (flag0 != 0) {
    // nothing was issued to the tensor core; the tiles have landed (or timed out)
    if (tid == 0) set_status(a.ws, flag0, s);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      ptx::tc_fence_after();
      ptx::tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  const int maxdep = ms.maxdep;
  for (int lvl = 1; lvl <= maxdep; ++lvl) {
    if (tid < n_nodes && ms.dep[tid] == lvl)
      ms.cl[tid] = (ms.par[tid] < 0 ? 0.f : ms.cl[ms.par[tid]]) + ms.la[tid];
    __syncthreads();
  }
  if (tid == 0) {
    // nodes grouped by depth (counting sort), for the level-by-level solve
    int cnt[kTile + 2];
    for (int d = 0; d <= maxdep + 1; ++d) cnt[d] = 0;
    for (int i = 0; i < n_nodes; ++i) ++cnt[ms.dep[i]];
    int acc = 0;
    for (int d = 0; d <= maxdep + 1; ++d) {
      ms.lvl_start[d] = acc;
      acc += cnt[d];
      cnt[d] = ms.lvl_start[d];
    }
    for (int i = 0; i < n_nodes; ++i) ms.lvl_nodes[cnt[ms.dep[i]]++] = i;
    if (!ptx::mbar_wait_bounded(bar_mma, 0, kSpinLimit)) ms.flag = TV_ERR_TIMEOUT;
  }
  __syncthreads();
  if (ms.flag != 0) {
    if (tid == 0) {
      set_status(a.ws, ms.flag, s);
      ptx::mbar_wait_bounded(bar_mma, 0, kSpinLimit);  // give the MMA one more chance
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      ptx::tc_fence_after();
      ptx::tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  ptx::tc_fence_after();

  // ---- 4. accumulator -> shared memory (row per thread) -------------------------------
  // warp w reads TMEM lanes 32*(w%4).. (rows); warps 0-3 take Gram columns 0..31 and value
  // columns 0..63, warps 4-7 Gram columns 32..63 and value columns 64..127.
  const int quarter = warp & 3, set = warp >> 2;
  const int row = quarter * 32 + lane;
  const bool is_q = row < kTile;
  const int n = is_q ? row : row - kTile;
  const bool live = n < n_nodes;
  const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
  const float cln = ms.cl[n];
  const float gam = expf(cln);
  const unsigned long long ancn = ms.anc[n];
  const float bn = ms.bb[n];
  float *Lc = reinterpret_cast<float *>(sm + kOffLc);
  {
    const unsigned char *vt = sm + kOffV;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float x[16];
      const int v0 = set * 64 + c * 16;
      ptx::tmem_ld16(trow + 64 + v0, x);
      ptx::tmem_wait_ld();
      if (is_q) {
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const float4 o4 = make_float4(gam * x[j], gam * x[j + 1], gam * x[j + 2], gam * x[j + 3]);
          *reinterpret_cast<float4 *>(sm + kOffSQ + f32_tile_off(n, v0 + j)) = o4;
        }
      } else {
        float4 u4[4];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float vn = live ? bf16_tile_ld(vt, n, v0 + j) : 0.f;
          const float u = kGdn ? bn * (vn - gam * x[j]) : vn;
          reinterpret_cast<float *>(u4)[j] = u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float4 *>(sm + kOffU + f32_tile_off(n, v0 + 4 * j)) = u4[j];
      }
    }
    if (kGdn && !is_q) {
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float g[16];
        const int i0 = set * 32 + c * 16;
        ptx::tmem_ld16(trow + i0, g);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int i = i0 + j;
          const bool on = live && ((ancn >> i) & 1ull);
          Lc[coef_off(n, i)] = on ? bn * expf(cln - ms.cl[i]) * g[j] : 0.f;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();   // v tile consumed: the P coefficients may now overwrite it
  float *P = reinterpret_cast<float *>(sm + kOffP);
  if (is_q) {
    ptx::tc_fence_after();
    const unsigned long long pathn = live ? (ancn | (1ull << n)) : 0ull;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float g[16];
      const int i0 = set * 32 + c * 16;
      ptx::tmem_ld16(trow + i0, g);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int i = i0 + j;
        const bool on = (pathn >> i) & 1ull;
        P[coef_off(n, i)] = on ? expf(cln - ms.cl[i]) * g[j] : 0.f;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {  // accumulator fully read: hand the tensor memory back early
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }

  // ---- 5. tree solve, level by level, one value column per thread ---------------------
  const int v = tid & 127, part = tid >> 7;
  if (kGdn) {
    for (int lvl = 2; lvl <= maxdep; ++lvl) {
      const int b0 = ms.lvl_start[lvl], b1 = ms.lvl_start[lvl + 1];
      for (int idx = b0 + part; idx < b1; idx += 2) {
        const int m = ms.lvl_nodes[idx];
        float acc = *reinterpret_cast<const float *>(sm + kOffU + f32_tile_off(m, v));
        unsigned long long bits = ms.anc[m];
        while (bits) {
          const int i = __ffsll((long long)bits) - 1;
          bits &= bits - 1;
          acc = fmaf(-Lc[coef_off(m, i)],
                     *reinterpret_cast<const float *>(sm + kOffU + f32_tile_off(i, v)), acc);
        }
        *reinterpret_cast<float *>(sm + kOffU + f32_tile_off(m, v)) = acc;
      }
      __syncthreads();
    }
  }

  // ---- 6. outputs and pseudo-values, coalesced rows -----------------------------------
  Tout *out = static_cast<Tout *>(a.out);
  for (int m = part; m < n_nodes; m += 2) {
    float o = *reinterpret_cast<const float *>(sm + kOffSQ + f32_tile_off(m, v));
    unsigned long long bits = ms.anc[m] | (1ull << m);
    while (bits) {
      const int i = __ffsll((long long)bits) - 1;
      bits &= bits - 1;
      o = fmaf(P[coef_off(m, i)], *reinterpret_cast<const float *>(sm + kOffU + f32_tile_off(i, v)), o);
    }
    const size_t g = ((size_t)(lo + m) * H + h) * 128 + v;
    out[g] = from_f32<Tout>(o);
    a.U[g] = *reinterpret_cast<const float *>(sm + kOffU + f32_tile_off(m, v));
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
