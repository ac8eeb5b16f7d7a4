// Commit of the accepted path: rebuild one state per (sequence, head) from pseudo-values.
//
// Along the accepted root-first path p_1..p_m the state is the closed form
//     S_new = exp(c_m) S_root + sum_j exp(c_m - c_j) u_{p_j} k_{p_j}^T,  c_j = sum_{l<=j} log_a_{p_l}
// (the Bole summary's worked example rebuilds S_c3 this way for scalar decay; with the
// pseudo-values of the tree solve the same form holds for the gated delta rule).
//
// One CTA per (sequence, head, slice of kRows state rows).  The kernel is HBM bound (one
// read and one write of the state), so everything that depends on the path is kept to
// two sets of dependent global loads, overlapped with the state loads:
//   first loads: the state slice (registers), node_offsets, the accepted_path row (warp 0,
//            checked with one ballot per 32 entries);
//   second loads: parent and log_a of the path nodes and their u and k rows, all at once.
// Then one thread forms the fp32 prefix sums c_j (root first, the order the verify
// kernels use for cl), the u rows are scaled, and S_new streams out with 128-bit stores.
//
// For dk = dv = 128 a streaming form replaces it: persistent CTAs (one per SM) walk a
// contiguous range of (sequence, head) states.  Each 64 KiB state arrives by bulk copy into
// a two-stage shared-memory ring one item ahead, and a loader warp gathers the next item's
// path (the two dependent load sets above) while sixteen warps rebuild and store the current
// one, so the state stream never waits on the path gather.
#include <algorithm>
#include <cstddef>

#include "tc_ptx.cuh"
#include "tv_internal.cuh"

namespace tv {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = 32;                            // state rows (v) per CTA
constexpr int kChunk = 16;                           // path entries staged at a time
constexpr int kMaxVec = kRows * 128 / 4 / kThreads;  // float4 slots per thread at dk=128
constexpr int kMaxPathWidth = 1024;

struct CommitSmem {
  float cu[kChunk][kRows]; // exp(c_m - c_j) u_{p_j}, this CTA's rows
  float kk[kChunk][128];   // k_{p_j}
  int prow[kMaxNodes];     // root-first path nodes
  float la[kMaxNodes];     // log_a of the path nodes
  float e[kMaxNodes];      // exp(c_m - c_j)
  int m;
  int lo;
  int bad;
};

// kD128: dk == 128, so thread t always owns column block 4*(t%32) and rows t/32 + 4r.
template <typename Tk, bool kD128>
__global__ void __launch_bounds__(kThreads) commit_kernel(CommitArgs a) {
  __shared__ __align__(16) CommitSmem sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, dk = a.dk, dv = a.dv;
  const int slices = (dv + kRows - 1) / kRows;
  const int s = blockIdx.x / (H * slices), h = (blockIdx.x / slices) % H;
  const int Hk = a.Hk, kh = qk_head(h, H, Hk);
  const int r0 = (blockIdx.x % slices) * kRows;           // first state row of the slice
  const int rows = min(kRows, dv - r0);
  const Tk *k = static_cast<const Tk *>(a.k);

  // ---- first loads -----------------------------------------------------------------
  const size_t base = (((size_t)s * H + h) * dv + r0) * dk;
  const float4 *Sg = reinterpret_cast<const float4 *>(a.S_root + base);
  const int nvec = rows * dk / 4;
  float4 acc[kMaxVec];
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) acc[r] = __ldcs(Sg + e);
  }
  if (warp == 0) {
    const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
    const bool tree_ok = !(lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
                           (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T));
    const int n_nodes = hi - lo;
    const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
    // m = number of leading non-negative entries; after them only -1 may follow
    int m = -1;
    bool bad = false;
    for (int t0 = 0; t0 < a.max_path; t0 += 32) {
      const int t = t0 + lane;
      const int p = t < a.max_path ? row[t] : -1;
      const unsigned neg = __ballot_sync(0xffffffffu, t < a.max_path && p < 0);
      if (m < 0 && neg) m = t0 + __ffs(neg) - 1;
      const bool in_path = m < 0 || t < m;
      if (t < a.max_path) {
        if (in_path) {
          if (p < 0 || p >= n_nodes || t >= kMaxNodes) bad = true;
          else sm.prow[t] = p;
        } else if (p != -1) {
          bad = true;
        }
      }
    }
    if (m < 0) m = a.max_path;
    bad = __any_sync(0xffffffffu, bad) || !tree_ok;
    if (lane == 0) {
      sm.m = bad ? 0 : m;
      sm.lo = lo;
      sm.bad = bad ? (tree_ok ? TV_ERR_BAD_PATH : TV_ERR_BAD_TREE) : 0;
    }
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0 && r0 == 0) set_status(a.ws, sm.bad, s);
    return;
  }
  const int m = sm.m, lo = sm.lo;

  // ---- second loads: parent / log_a of the path, the first chunk of u and k rows -----
  int chain_bad = 0;
  for (int t = tid; t < m; t += kThreads) {
    const int p = sm.prow[t];
    sm.la[t] = a.log_a[(size_t)(lo + p) * H + h];
    if (a.parent && a.parent[lo + p] != (t == 0 ? -1 : sm.prow[t - 1])) chain_bad = 1;
  }
  const int cnt0 = min(kChunk, m);
  for (int e = tid; e < cnt0 * 128; e += kThreads) {
    const int j = e >> 7, x = e & 127;
    const int row = lo + sm.prow[j];
    if (x < rows) sm.cu[j][x] = load_u(a.U, ((size_t)row * H + h) * dv + r0 + x, a.u_bf16);
    if (x < dk) sm.kk[j][x] = to_f32(k[((size_t)row * Hk + kh) * dk + x]);
  }
  if (__syncthreads_or(chain_bad)) {
    if (tid == 0 && r0 == 0) set_status(a.ws, TV_ERR_BAD_PATH, s);
    return;
  }
  if (tid == 0) {
    float c = 0.f;
    for (int j = 0; j < m; ++j) {
      c += sm.la[j];
      sm.la[j] = c;                    // now c_j
    }
    for (int j = 0; j < m; ++j) sm.e[j] = expf(c - sm.la[j]);
  }
  __syncthreads();
  for (int e = tid; e < cnt0 * kRows; e += kThreads) sm.cu[e / kRows][e % kRows] *= sm.e[e / kRows];
  __syncthreads();
  const float gam = m ? expf(sm.la[m - 1]) : 1.f;
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    acc[r].x *= gam; acc[r].y *= gam; acc[r].z *= gam; acc[r].w *= gam;
  }

  // ---- rank-one terms of the path, kChunk entries at a time --------------------------
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    const int cnt = min(kChunk, m - j0);
    if (j0) {
      __syncthreads();
      for (int e = tid; e < cnt * 128; e += kThreads) {
        const int j = e >> 7, x = e & 127;
        const int row = lo + sm.prow[j0 + j];
        if (x < rows)
          sm.cu[j][x] = sm.e[j0 + j] * load_u(a.U, ((size_t)row * H + h) * dv + r0 + x, a.u_bf16);
        if (x < dk) sm.kk[j][x] = to_f32(k[((size_t)row * Hk + kh) * dk + x]);
      }
      __syncthreads();
    }
    if (kD128) {
      // fixed column block per thread: one k chunk per path entry serves all its rows
      const int col = (tid & 31) * 4, rb = tid >> 5;
      for (int j = 0; j < cnt; ++j) {
        const float4 kv = *reinterpret_cast<const float4 *>(&sm.kk[j][col]);
#pragma unroll
        for (int r = 0; r < kMaxVec; ++r) {
          const float cu = sm.cu[j][rb + 4 * r];
          acc[r].x = fmaf(cu, kv.x, acc[r].x);
          acc[r].y = fmaf(cu, kv.y, acc[r].y);
          acc[r].z = fmaf(cu, kv.z, acc[r].z);
          acc[r].w = fmaf(cu, kv.w, acc[r].w);
        }
      }
    } else {
#pragma unroll
      for (int r = 0; r < kMaxVec; ++r) {
        const int e = tid + r * kThreads;
        if (e < nvec) {
          const int rr = (e * 4) / dk, col = (e * 4) % dk;
          for (int j = 0; j < cnt; ++j) {
            const float cu = sm.cu[j][rr];
            const float4 kv = *reinterpret_cast<const float4 *>(&sm.kk[j][col]);
            acc[r].x = fmaf(cu, kv.x, acc[r].x);
            acc[r].y = fmaf(cu, kv.y, acc[r].y);
            acc[r].z = fmaf(cu, kv.z, acc[r].z);
            acc[r].w = fmaf(cu, kv.w, acc[r].w);
          }
        }
      }
    }
  }

  // ---- stream the state slice out ------------------------------------------------------
  float4 *Sn = reinterpret_cast<float4 *>(a.S_new + base);
#pragma unroll
  for (int r = 0; r < kMaxVec; ++r) {
    const int e = tid + r * kThreads;
    if (e < nvec) __stcs(Sn + e, acc[r]);
  }
}


// ---- streaming form (dk = dv = 128) --------------------------------------------------
// Warp roles in one persistent CTA per SM, linked by mbarriers:
//   warps 0-15  read an item's state from its stage (releasing the stage at once), rebuild
//               it in registers and stream it out with 128-bit stores,
//   warp 16     bulk-copies states into the two-stage ring as stages are released,
//   warps 17-20 gather paths, item li by warp 17 + li % 4 (eight path buffers, two each: a
//               gather is one or two dependent round trips to memory that is busy with the
//               state stream, so four are kept in flight).
constexpr int kSCompute = 512;
constexpr int kSMoverWarp = 16;
constexpr int kSGatherWarp = 17;
constexpr int kGatherers = 4;
constexpr int kSThreads = (17 + kGatherers) * 32;
constexpr int kPathBufs = 2 * kGatherers;
constexpr int kPathRows = 8;                   // path entries staged in shared memory
constexpr uint32_t kStateBytes = 128 * 128 * 4;
constexpr uint32_t kSSpinLimit = 1u << 22;

struct __align__(16) PathBuf {
  float cu[kPathRows][128];   // exp(c_m - c_j) u_{p_j}, all 128 state rows
  float kk[kPathRows][128];   // k_{p_j} in its input type (bf16 rows use the first half)
  int prow[kMaxNodes];        // root-first path nodes
  float e[kMaxNodes];         // log_a of the path nodes, then exp(c_m - c_j)
  float gam;                  // exp(c_m)
  int m;                      // path length (0 if the item is bad)
  int m_row;                  // length of the checked accepted-path row, -1 if it is bad
  int lo;                     // first node of the sequence
  int status;                 // 0, TV_ERR_BAD_TREE or TV_ERR_BAD_PATH
};
struct StreamSmem {
  float S[2][128 * 128];                      // state ring
  PathBuf pb[kPathBufs];
  unsigned long long s_full[2], s_empty[2];   // state loaded / stage read
  unsigned long long p_full[kPathBufs], p_empty[kPathBufs];
  int fail;
};
constexpr int kStreamSmemBytes = (int)sizeof(StreamSmem) + 1024;
// bulk copies, cp.async and float4 accesses need 16-byte aligned buffers
static_assert(sizeof(PathBuf) % 16 == 0 && offsetof(StreamSmem, pb) % 16 == 0, "alignment");

// Asynchronous global -> shared copies of 16 and 8 bytes (both sides aligned to the size).
__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_addr(sdst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void *sdst, const void *gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(ptx::smem_addr(sdst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_k(float *sdst, const float *gsrc) { cp_async16(sdst, gsrc); }
__device__ __forceinline__ void cp_async_k(__nv_bfloat16 *sdst, const __nv_bfloat16 *gsrc) {
  cp_async8(sdst, gsrc);
}

__device__ __forceinline__ float4 load_k4(const float *k, size_t off) {
  return *reinterpret_cast<const float4 *>(k + off);
}
__device__ __forceinline__ float4 load_k4(const __nv_bfloat16 *k, size_t off) {
  const uint2 r = *reinterpret_cast<const uint2 *>(k + off);
  return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                     __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
}

template <typename Tk>
__device__ void gather_rows(const CommitArgs &a, int it, PathBuf &pb, int m, int lo, int lane);

// Gatherer warp: the path of item `it` into `pb` -- node range, accepted-path row (checked),
// log_a and the parent chain, the decay weights, and the first kPathRows u and k rows.
template <typename Tk>
__device__ void gather_path(const CommitArgs &a, int it, PathBuf &pb, const PathBuf *prev,
                            int prev_it, int lane) {
  const int H = a.H, s = it / H;
  if (prev && prev_it / H == s && prev->m_row >= 0) {
    // same sequence as the item `prev` holds: its node range and checked path row carry
    // over (a chain error found for that head is found again below)
    const int m = prev->m_row;
    for (int t = lane; t < m; t += 32) pb.prow[t] = prev->prow[t];
    if (lane == 0) {
      pb.m_row = m;
      pb.lo = prev->lo;
    }
    __syncwarp();
    gather_rows<Tk>(a, it, pb, m, prev->lo, lane);
    return;
  }
  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  const bool tree_ok = !(lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
                         (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T));
  const int n_nodes = hi - lo;
  const int32_t *row = a.accepted_path + (size_t)s * a.max_path;
  // m = number of leading non-negative entries; after them only -1 may follow
  int m = -1;
  bool bad = false;
  for (int t0 = 0; t0 < a.max_path; t0 += 32) {
    const int t = t0 + lane;
    const int p = t < a.max_path ? row[t] : -1;
    const unsigned neg = __ballot_sync(0xffffffffu, t < a.max_path && p < 0);
    if (m < 0 && neg) m = t0 + __ffs(neg) - 1;
    const bool in_path = m < 0 || t < m;
    if (t < a.max_path) {
      if (in_path) {
        if (p < 0 || p >= n_nodes || t >= kMaxNodes) bad = true;
        else pb.prow[t] = p;
      } else if (p != -1) {
        bad = true;
      }
    }
  }
  if (m < 0) m = a.max_path;
  bad = __any_sync(0xffffffffu, bad) || !tree_ok;
  if (bad) {
    if (lane == 0) {
      pb.status = tree_ok ? TV_ERR_BAD_PATH : TV_ERR_BAD_TREE;
      pb.m = 0;
      pb.m_row = -1;
    }
    __syncwarp();
    return;
  }
  if (lane == 0) {
    pb.m_row = m;
    pb.lo = lo;
  }
  __syncwarp();
  gather_rows<Tk>(a, it, pb, m, lo, lane);
}

// Gatherer warp, second load set: log_a and the parent chain of the m path entries (row already
// in pb.prow), decay weights, and the u and k rows of the first kPathRows entries.
template <typename Tk>
__device__ void gather_rows(const CommitArgs &a, int it, PathBuf &pb, int m, int lo, int lane) {
  const int H = a.H, h = it % H, kh = qk_head(h, H, a.Hk);
  // log_a and the parent chain of every path entry; the u and k rows of the first
  // kPathRows entries go straight into the buffer by asynchronous copies (bf16 u rows land
  // in the first half of their row and are widened when they are scaled)
  const Tk *k = static_cast<const Tk *>(a.k);
  Tk *kk = reinterpret_cast<Tk *>(&pb.kk[0][0]);
  const int staged = min(m, kPathRows);
  for (int j = 0; j < staged; ++j) {
    const int row = lo + pb.prow[j];
    const size_t node = (size_t)row * H + h;
    if (a.u_bf16)
      cp_async8(reinterpret_cast<__nv_bfloat16 *>(&pb.cu[j][0]) + 4 * lane,
                static_cast<const __nv_bfloat16 *>(a.U) + node * 128 + 4 * lane);
    else
      cp_async16(&pb.cu[j][4 * lane], static_cast<const float *>(a.U) + node * 128 + 4 * lane);
    cp_async_k(kk + j * 128 + 4 * lane, k + ((size_t)row * a.Hk + kh) * 128 + 4 * lane);
  }
  int chain_bad = 0;
  for (int t = lane; t < m; t += 32) {
    const int p = pb.prow[t];
    pb.e[t] = a.log_a[(size_t)(lo + p) * H + h];
    if (a.parent && a.parent[lo + p] != (t == 0 ? -1 : pb.prow[t - 1])) chain_bad = 1;
  }
  chain_bad = __any_sync(0xffffffffu, chain_bad);
  __syncwarp();
  if (lane == 0) {
    if (chain_bad) {
      pb.status = TV_ERR_BAD_PATH;
      pb.m = 0;
    } else {
      // fp32 prefix sums c_j, root first (the order the verify kernels use for cl)
      float c = 0.f;
      for (int j = 0; j < m; ++j) {
        c += pb.e[j];
        pb.e[j] = c;
      }
      for (int j = 0; j < m; ++j) pb.e[j] = expf(c - pb.e[j]);
      pb.gam = m ? expf(c) : 1.f;
      pb.m = m;
      pb.lo = lo;
      pb.status = 0;
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncwarp();
  if (!chain_bad)
    for (int j = 0; j < staged; ++j) {
      // each lane scales the 4 columns it copied
      float4 *c4 = reinterpret_cast<float4 *>(&pb.cu[j][4 * lane]);
      const float e = pb.e[j];
      float4 u;
      if (a.u_bf16) {
        const uint2 r = reinterpret_cast<const uint2 *>(&pb.cu[j][0])[lane];
        u = make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                        __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
        __syncwarp();   // every lane has read its bf16 values before the row is widened
      } else {
        u = *c4;
      }
      *c4 = make_float4(e * u.x, e * u.y, e * u.z, e * u.w);
    }
  __syncwarp();
}

// Bounded wait on phase `par` of `bar`; on a time-out the CTA-wide failure flag is raised.
__device__ __forceinline__ bool stream_wait(StreamSmem &sm, uint32_t bar, uint32_t par, int *ws,
                                            int detail) {
  for (uint32_t i = 0; i < kSSpinLimit; ++i) {
    if (ptx::mbar_try_wait(bar, par)) return true;
    if (*reinterpret_cast<volatile int *>(&sm.fail)) return false;
  }
  if (atomicExch(&sm.fail, 1) == 0) set_status(ws, TV_ERR_TIMEOUT, detail);
  return false;
}

template <typename Tk>
__global__ void __launch_bounds__(kSThreads, 1) commit_stream_kernel(CommitArgs a) {
  extern __shared__ unsigned char smem_raw[];
  StreamSmem &sm = *reinterpret_cast<StreamSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = a.B * a.H;
  // a contiguous range of items per CTA: the heads of a sequence share its path row
  const int first = (int)((long long)blockIdx.x * n_items / gridDim.x);
  const int n = (int)((long long)(blockIdx.x + 1) * n_items / gridDim.x) - first;
  // Launched with programmatic stream serialisation.  Before the grid dependency resolves
  // the mover only asks L2 to prefetch its first two S_root blocks: a prefetch moves no
  // data into this CTA, and a write by the previous kernel to the same lines lands in L2
  // after it, so this is correct whatever that kernel writes (another commit's S_new
  // included).  Every load and store waits for the previous kernel to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(ptx::smem_addr(&sm.s_full[i]), 1);
      ptx::mbar_init(ptx::smem_addr(&sm.s_empty[i]), kSCompute / 32);
    }
    for (int i = 0; i < kPathBufs; ++i) {
      ptx::mbar_init(ptx::smem_addr(&sm.p_full[i]), 1);
      ptx::mbar_init(ptx::smem_addr(&sm.p_empty[i]), kSCompute / 32);
    }
    ptx::fence_mbar_init();
    sm.fail = 0;
  }
  __syncthreads();

  if (warp == kSMoverWarp && lane == 0)
    for (int li = 0; li < n && li < 2; ++li)
      ptx::prefetch_l2(a.S_root + (size_t)(first + li) * 128 * 128, kStateBytes);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (warp == kSMoverWarp) {
    if (lane == 0) {
      // item li goes into stage li & 1 once the compute warps have read item li - 2 from it
      int loaded = 0;
      for (int li = 0; li < n; ++li) {
        const int st = li & 1;
        if (li >= 2 &&
            !stream_wait(sm, ptx::smem_addr(&sm.s_empty[st]), ((li - 2) >> 1) & 1, a.ws, first / a.H))
          break;
        const uint32_t full = ptx::smem_addr(&sm.s_full[st]);
        ptx::mbar_arrive_expect_tx(full, kStateBytes);
        ptx::bulk_load(ptx::smem_addr(sm.S[st]), a.S_root + (size_t)(first + li) * 128 * 128,
                       kStateBytes, full);
        loaded = li + 1;
      }
      if (*reinterpret_cast<volatile int *>(&sm.fail))
        // after a time-out: let the state copies still in flight land before the CTA's
        // shared memory is released (bounded)
        for (int li = loaded > 2 ? loaded - 2 : 0; li < loaded; ++li)
          ptx::mbar_wait_bounded(ptx::smem_addr(&sm.s_full[li & 1]), (li >> 1) & 1, kSSpinLimit);
    }
  } else if (warp >= kSGatherWarp) {
    const int g = warp - kSGatherWarp;
    for (int li = g; li < n; li += kGatherers) {
      const int b = li & (kPathBufs - 1), use = li / kPathBufs;
      if (use > 0 &&
          !__all_sync(0xffffffffu, stream_wait(sm, ptx::smem_addr(&sm.p_empty[b]), (use - 1) & 1,
                                               a.ws, (first + li) / a.H)))
        break;
      // this warp's previous item is still in its other buffer
      const int pl = li - kGatherers;
      gather_path<Tk>(a, first + li, sm.pb[b], pl >= 0 ? &sm.pb[pl & (kPathBufs - 1)] : nullptr,
                      first + pl, lane);
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&sm.p_full[b]));
    }
  } else {
    // compute thread t: 4 state columns from 4 (t % 32), rows t / 32 + 16 i
    const int col = (tid & 31) * 4, rb = tid >> 5;
    const Tk *k = static_cast<const Tk *>(a.k);
    for (int li = 0; li < n; ++li) {
      const int it = first + li, st = li & 1, b = li & (kPathBufs - 1);
      bool ok = stream_wait(sm, ptx::smem_addr(&sm.s_full[st]), (li >> 1) & 1, a.ws, it / a.H);
      ok = ok && stream_wait(sm, ptx::smem_addr(&sm.p_full[b]), (li / kPathBufs) & 1, a.ws, it / a.H);
      if (!__all_sync(0xffffffffu, ok)) break;
      const PathBuf &pb = sm.pb[b];
      const float *Ss = sm.S[st];
      // the state into registers, then the stage goes back to the mover
      float4 acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        acc[i] = *reinterpret_cast<const float4 *>(Ss + (rb + 16 * i) * 128 + col);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&sm.s_empty[st]));
      if (pb.status) {
        if (tid == 0) set_status(a.ws, pb.status, it / a.H);
      } else {
        const int m = pb.m;
        const float gam = pb.gam;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc[i].x *= gam; acc[i].y *= gam; acc[i].z *= gam; acc[i].w *= gam;
        }
        const int staged = min(m, kPathRows);
        const Tk *kk = reinterpret_cast<const Tk *>(&pb.kk[0][0]);
        for (int j = 0; j < staged; ++j) {
          const float4 kv = load_k4(kk, (size_t)j * 128 + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float cu = pb.cu[j][rb + 16 * i];
            acc[i].x = fmaf(cu, kv.x, acc[i].x);
            acc[i].y = fmaf(cu, kv.y, acc[i].y);
            acc[i].z = fmaf(cu, kv.z, acc[i].z);
            acc[i].w = fmaf(cu, kv.w, acc[i].w);
          }
        }
        // path entries past the staged ones come straight from HBM
        const int h = it % a.H, kh = qk_head(h, a.H, a.Hk);
        for (int j = staged; j < m; ++j) {
          const int row = pb.lo + pb.prow[j];
          const size_t node = (size_t)row * a.H + h;
          const float4 kv = load_k4(k, ((size_t)row * a.Hk + kh) * 128 + col);
          const float e = pb.e[j];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float cu = e * load_u(a.U, node * 128 + rb + 16 * i, a.u_bf16);
            acc[i].x = fmaf(cu, kv.x, acc[i].x);
            acc[i].y = fmaf(cu, kv.y, acc[i].y);
            acc[i].z = fmaf(cu, kv.z, acc[i].z);
            acc[i].w = fmaf(cu, kv.w, acc[i].w);
          }
        }
        float *Sn = a.S_new + (size_t)it * 128 * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          __stcs(reinterpret_cast<float4 *>(Sn + (rb + 16 * i) * 128 + col), acc[i]);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&sm.p_empty[b]));
    }
  }
  __syncthreads();
}

}  // namespace

int commit_max_path_width() { return kMaxPathWidth; }

template <typename Tk>
cudaError_t launch_stream(const CommitArgs &a, cudaStream_t st) {
  auto kern = commit_stream_kernel<Tk>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kStreamSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(a.B * a.H, sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = kStreamSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_commit(const CommitArgs &a, int in_dtype, cudaStream_t st) {
  if (a.dk == 128 && a.dv == 128 && a.B * a.H > 0)
    return in_dtype == TV_F32 ? launch_stream<float>(a, st) : launch_stream<__nv_bfloat16>(a, st);
  const int grid = a.B * a.H * ((a.dv + kRows - 1) / kRows);
  const bool d128 = a.dk == 128 && a.dv % kRows == 0;
  if (in_dtype == TV_F32) {
    if (d128) commit_kernel<float, true><<<grid, kThreads, 0, st>>>(a);
    else commit_kernel<float, false><<<grid, kThreads, 0, st>>>(a);
  } else {
    if (d128) commit_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, st>>>(a);
    else commit_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace tv
