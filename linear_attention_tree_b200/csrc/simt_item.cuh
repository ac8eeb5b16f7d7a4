// The CUDA-core verification of one (sequence, head) item, shared by the CUDA-core kernel
// and by the wide tensor-core kernel (which hands it the trees deeper than its path
// registers).  Included by the kernels' translation units only.
//
// Thread v owns value column v of everything the method produces for that column: S_root
// row v (staged in shared memory), the column-v entries of S_root q_n and S_root k_n, the
// pseudo-value column u_n[v] and the output column o_n[v].  The only quantities shared
// across columns are per-node scalars: the path Gram terms q_n.k_i and k_n.k_i and the path
// decays exp(cl_n - cl_i); warps compute those cooperatively before the column phase of
// each node.
//
// Nodes are processed in index order, which is topological (parent[i] < i), so when node
// n is reached every ancestor's u_i column is final.  This is the forward substitution of
// the unit-lower-triangular tree system (TreeWY abstract, tree-structured WY form):
//     u_n = b_n (v_n - exp(cl_n) S_root k_n) - sum_{i in anc(n)} b_n exp(cl_n-cl_i)(k_n.k_i) u_i
// and the output is the closed form of the Bole summary's worked example ("具体技术细节示例")
// extended to the delta rule:
//     o_n = exp(cl_n) S_root q_n + sum_{i in path(n)} exp(cl_n-cl_i) (q_n.k_i) u_i .
// Scalar decay has u_n = v_n.
#pragma once

#include "tv_internal.cuh"

namespace tv {

struct SimtSmem {
  int par[kMaxNodes];
  int dep[kMaxNodes];
  int plist[kMaxNodes];       // path of the current node: ancestors ascending, then itself
  float la[kMaxNodes];
  float bb[kMaxNodes];
  float cl[kMaxNodes];
  float cq[kMaxNodes];        // exp(cl_n - cl_i) q_n.k_i      for i = plist[e]
  float ck[kMaxNodes];        // b_n exp(cl_n - cl_i) k_n.k_i  for strict ancestors
  unsigned long long anc[kMaxNodes][kAncWords];
  float qn[128];
  float kn[128];
  int flag;
  int maxdep;
  int plen;
  // followed by S_root: dv rows of (dk + 1) floats (the pad keeps column reads conflict-free)
};

// Bytes of shared memory simt_item needs for value width dv and key width dk.
__host__ __device__ constexpr size_t simt_smem_bytes(int dk, int dv) {
  return sizeof(SimtSmem) + (size_t)dv * (dk + 1) * sizeof(float);
}

// Every thread of the CTA calls this (it synchronises the CTA); the first kNT threads do
// the work.  Errors in the item's data are recorded on the status word.
template <typename Tin, typename Tout, bool kGdn, int kNT>
__device__ void simt_item(const VerifyArgs &a, int s, int h, unsigned char *smem_raw) {
  SimtSmem &sm = *reinterpret_cast<SimtSmem *>(smem_raw);
  float *S = reinterpret_cast<float *>(smem_raw + sizeof(SimtSmem));
  const int tid = threadIdx.x;
  const int H = a.H, dk = a.dk, dv = a.dv, ldS = a.dk + 1;
  const int Hk = a.Hk, kh = qk_head(h, H, Hk);
  const Tin *q = static_cast<const Tin *>(a.q);
  const Tin *k = static_cast<const Tin *>(a.k);
  const Tin *vv = static_cast<const Tin *>(a.v);
  Tout *out = static_cast<Tout *>(a.out);

  const int lo = a.node_offsets[s], hi = a.node_offsets[s + 1];
  if (lo < 0 || hi < lo || hi > a.T || hi - lo > a.max_nodes ||
      (s == 0 && lo != 0) || (s == a.B - 1 && hi != a.T)) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  const int n_nodes = hi - lo;
  if (n_nodes == 0) return;

  if (tid == 0) { sm.flag = 0; sm.maxdep = 0; }
  __syncthreads();
  for (int i = tid; i < n_nodes; i += kNT) {
    const int p = a.parent[lo + i];
    if (p < -1 || p >= i) sm.flag = 1;
    sm.par[i] = p;
    sm.la[i] = a.log_a[(size_t)(lo + i) * H + h];
    sm.bb[i] = kGdn ? a.b[(size_t)(lo + i) * H + h] : 0.f;
    for (int w = 0; w < kAncWords; ++w) sm.anc[i][w] = 0ull;
  }
  __syncthreads();
  if (sm.flag) {
    if (tid == 0) set_status(a.ws, TV_ERR_BAD_TREE, s);
    return;
  }
  // depth and strict-ancestor bits: each thread walks its own node's parent chain
  for (int i = tid; i < n_nodes; i += kNT) {
    int d = 1;
    for (int x = sm.par[i]; x >= 0; x = sm.par[x]) {
      sm.anc[i][x >> 6] |= 1ull << (x & 63);
      ++d;
    }
    sm.dep[i] = d;
    atomicMax(&sm.maxdep, d);
  }
  // S_root row v -> shared memory (fp32, padded rows)
  const float *Sg = a.S_root + ((size_t)s * H + h) * dv * dk;
  for (int e = tid; e < dv * dk; e += kNT) S[(e / dk) * ldS + e % dk] = Sg[e];
  __syncthreads();
  // cumulative path log-decay, level by level from the root: cl_n = cl_parent + log_a_n
  for (int lvl = 1; lvl <= sm.maxdep; ++lvl) {
    for (int i = tid; i < n_nodes; i += kNT)
      if (sm.dep[i] == lvl) sm.cl[i] = (sm.par[i] < 0 ? 0.f : sm.cl[sm.par[i]]) + sm.la[i];
    __syncthreads();
  }

  const int warp = tid >> 5, lane = tid & 31;
  for (int n = 0; n < n_nodes; ++n) {
    const size_t rowq = ((size_t)(lo + n) * Hk + kh) * dk;
    for (int j = tid; j < dk; j += kNT) {
      sm.qn[j] = to_f32(q[rowq + j]);
      sm.kn[j] = to_f32(k[rowq + j]);
    }
    if (tid == 0) {
      int e = 0;
      for (int w = 0; w < kAncWords; ++w) {
        unsigned long long bits = sm.anc[n][w];
        while (bits) {
          const int bit = __ffsll((long long)bits) - 1;
          sm.plist[e++] = w * 64 + bit;
          bits &= bits - 1;
        }
      }
      sm.plist[e++] = n;
      sm.plen = e;
    }
    __syncthreads();
    const int plen = sm.plen;
    const float cln = sm.cl[n], bn = sm.bb[n];
    // path Gram terms, one warp per path entry
    for (int e = warp; e < plen; e += kNT / 32) {
      const int i = sm.plist[e];
      const size_t rowk = ((size_t)(lo + i) * Hk + kh) * dk;
      float gq = 0.f, gk = 0.f;
      for (int j = lane; j < dk; j += 32) {
        const float ki = to_f32(k[rowk + j]);
        gq = fmaf(sm.qn[j], ki, gq);
        gk = fmaf(sm.kn[j], ki, gk);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        gq += __shfl_xor_sync(0xffffffffu, gq, o);
        gk += __shfl_xor_sync(0xffffffffu, gk, o);
      }
      if (lane == 0) {
        const float dec = expf(cln - sm.cl[i]);
        sm.cq[e] = dec * gq;
        sm.ck[e] = bn * dec * gk;
      }
    }
    __syncthreads();
    // column phase
    for (int col = tid; col < dv; col += kNT) {
      const float *Srow = S + col * ldS;
      float sq = 0.f, sk = 0.f;
      for (int j = 0; j < dk; ++j) {
        sq = fmaf(Srow[j], sm.qn[j], sq);
        sk = fmaf(Srow[j], sm.kn[j], sk);
      }
      const float gam = expf(cln);
      const size_t rowv = ((size_t)(lo + n) * H + h) * dv;
      const float vn = to_f32(vv[rowv + col]);
      float u;
      if (kGdn) {
        u = bn * (vn - gam * sk);
        for (int e = 0; e < plen - 1; ++e)
          u = fmaf(-sm.ck[e], load_u(a.U, ((size_t)(lo + sm.plist[e]) * H + h) * dv + col, a.u_bf16), u);
      } else {
        u = vn;
      }
      float o = gam * sq;
      for (int e = 0; e < plen - 1; ++e)
        o = fmaf(sm.cq[e], load_u(a.U, ((size_t)(lo + sm.plist[e]) * H + h) * dv + col, a.u_bf16), o);
      o = fmaf(sm.cq[plen - 1], u, o);
      store_u(a.U, rowv + col, u, a.u_bf16);
      out[rowv + col] = from_f32<Tout>(o);
    }
    __syncthreads();
  }
}

}  // namespace tv
