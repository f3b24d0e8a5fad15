// tree_expand_topb kernels: one round of SpecExec's batched best-first
// expansion (SpecExec page, "Approach": build the tree from the highest
// cumulative-probability continuations by a batched Dijkstra-style search).
//
// Candidate representation.  Within one parent the candidates' order is the
// order of its draft logits (score = logp + z/tau - lse is increasing in z),
// so the taken children of a node always form a prefix of its row sorted by
// (z desc, token asc).  The pool is therefore kept implicitly: each expanded
// node owns a sorted list of its best K = min(V, budget - n_nodes) tokens
// and a cursor; the candidate set of a round is the union of the lists from
// their cursors.  (Tokens past the remaining budget can never be taken.)
//
//   expand_rows_kernel   one CTA per row: lse of the row and a radix select
//                        of its top-K logits (three histogram passes on the
//                        order-preserving 32-bit key), then a bitonic sort
//                        of those K into the node's list;
//   expand_merge_kernel  one CTA: repeatedly take the best s <= 128
//                        candidates of the union.  The s-th best list head
//                        bounds the s-th best candidate, so only the <= s
//                        lists whose head ranks within the first s can
//                        contribute, each with at most s entries; a radix
//                        select over those <= s*s composite keys (score,
//                        parent, token) and a sort of the winners append the
//                        next nodes in rank order.
#include "tv_common.cuh"

namespace tv {

struct NodeMeta {
  int32_t len;        // entries in the node's sorted list (0: not expanded)
  int32_t cursor;     // first entry not yet taken
  int32_t expanded;   // set once a row for the node has been consumed
  int32_t pad;
  double lse;         // logsumexp of the node's row / tau
};

struct ListEntry {
  float z;
  int32_t tok;
};

constexpr int kRowThreads = 1024;
constexpr int kRowWarps = kRowThreads / kWarp;
constexpr int kMergeThreads = 1024;
constexpr int kMergeWarps = kMergeThreads / kWarp;
constexpr int kMergeStep = 128;                     // nodes taken per sub-step
constexpr int kMergeCap = kMergeStep * kMergeStep;  // candidate capacity
constexpr int kSegE = 128;

__host__ __device__ inline int64_t expand_kcap(int budget, int V) {
  int64_t k = budget - 1;
  if (k > V) k = V;
  return k < 1 ? 1 : k;
}
__host__ __device__ inline size_t expand_lists_offset(int budget) {
  const size_t m = static_cast<size_t>(budget) * sizeof(NodeMeta);
  return (m + 255) & ~static_cast<size_t>(255);
}

struct ExpandParams {
  int V, R, Bsel, budget;
  float tau;
  const float* logits; int64_t ld;
  const int32_t* row_node;
  int32_t* n_nodes;
  int32_t* parent;
  int32_t* token;
  double* logp;
  NodeMeta* meta;
  ListEntry* lists;
  int64_t kcap;
  int32_t* frontier;
  int32_t* n_appended;
  uint32_t* status;
};

// descending-score key: smaller key = larger value
__device__ __forceinline__ uint32_t zdesc_key(float z) { return ~f32_key(z); }
__device__ __forceinline__ uint64_t sdesc_key(double s) { return ~f64_key(s); }
__device__ __forceinline__ double sdesc_val(uint64_t k) { return key_f64(~k); }

// Cumulative log-probability of a list entry (same expression everywhere).
__device__ __forceinline__ double entry_score(double logp_n, float z, float tau, double lse) {
  return (logp_n + static_cast<double>(z) / static_cast<double>(tau)) - lse;
}

// ------------------------------------------------------------ block helpers

struct RowShared {
  double red_d[kRowWarps];
  float red_f[kRowWarps];
  int red_i[kRowWarps];
  int bc[8];
  double bcd[2];
};

// Find the bin holding the rank-th smallest element (rank 1-based) of a
// histogram; returns the bin and the count of elements in lower bins.
__device__ void find_rank_bin(const uint32_t* hist, int nbins, int rank, int* bin,
                              int* before, RowShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) { sh.bc[0] = 0; sh.bc[1] = 0; }
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int lo = min(tid * per, nbins), hi = min(lo + per, nbins);
  int ls = 0;
  for (int i = lo; i < hi; ++i) ls += static_cast<int>(hist[i]);
  int incl = ls;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) sh.red_i[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const int v = (lane < nw) ? sh.red_i[lane] : 0;
    int wi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < nw) sh.red_i[lane] = wi - v;     // exclusive warp offsets
  }
  __syncthreads();
  const int excl = sh.red_i[warp] + incl - ls;
  if (excl < rank && rank <= excl + ls) {
    int cum = excl;
    for (int i = lo; i < hi; ++i) {
      const int h = static_cast<int>(hist[i]);
      if (rank <= cum + h) { sh.bc[0] = i; sh.bc[1] = cum; break; }
      cum += h;
    }
  }
  __syncthreads();
  *bin = sh.bc[0];
  *before = sh.bc[1];
  __syncthreads();
}

// ------------------------------------------------------------ row kernel

__global__ void __launch_bounds__(kRowThreads)
expand_rows_kernel(ExpandParams p) {
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ RowShared sh;
  __shared__ uint32_t hist[2048];
  __shared__ int s_count;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int node = p.row_node[r];
  if (node < 0) return;
  const int n0 = *p.n_nodes;
  if (node >= n0) {
    if (tid == 0) set_status(p.status, TV_DEV_BAD_ROW);
    return;
  }
  if (tid == 0) sh.bc[2] = atomicExch(&p.meta[node].expanded, 1);
  __syncthreads();
  if (sh.bc[2] != 0) {
    if (tid == 0) set_status(p.status, TV_DEV_BAD_ROW);
    return;
  }
  const int V = p.V;
  const int K = min(V, p.budget - n0);
  if (K <= 0) return;
  const float* row = p.logits + static_cast<int64_t>(r) * p.ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  const int nseg = (V + kSegE - 1) / kSegE;
  const int P = 1 << (32 - __clz(K - 1 | 1));      // next power of two >= K (>= 2)
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(dsm);
  double* seg_s = reinterpret_cast<double*>(sbuf + P);
  float* seg_m = reinterpret_cast<float*>(seg_s + nseg);
  const double invtau = 1.0 / static_cast<double>(p.tau);

  for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  // pass 1: segment max / exp sums, finiteness, histogram of the top 11 key bits
  bool bad = false;
  float lmax = -INFINITY;
  for (int s = warp; s < nseg; s += kRowWarps) {
    const int e0 = s * kSegE + lane * 4;
    const float4 v = load4(row, e0, V, vec, 0.f);
    const float xs[4] = {v.x, v.y, v.z, v.w};
    float m4 = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (e0 + k < V) {
        if (!isfinite(xs[k])) bad = true;
        else {
          m4 = fmaxf(m4, xs[k]);
          atomicAdd(&hist[zdesc_key(xs[k]) >> 21], 1u);
        }
      }
    const float wm = warp_max(m4);
    double a = 0.0;
    // double-precision exponentials: the row's lse enters every cumulative
    // score, and cross-row ranks must not move by more than fp64 rounding
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (e0 + k < V && isfinite(xs[k]))
        a += exp((static_cast<double>(xs[k]) - static_cast<double>(wm)) * invtau);
    a = warp_sum(a);
    if (lane == 0) { seg_m[s] = wm; seg_s[s] = a; }
    lmax = fmaxf(lmax, wm);
  }
  const int any_bad = __syncthreads_or(bad ? 1 : 0);
  if (any_bad) {
    if (tid == 0) set_status(p.status, TV_DEV_NONFINITE);
    return;
  }
  // row maximum and lse = M/tau + log sum exp((z - M)/tau)
  float M = warp_max(lmax);
  if (lane == 0) sh.red_f[warp] = M;
  __syncthreads();
  if (warp == 0) {
    float t = (lane < kRowWarps) ? sh.red_f[lane] : -INFINITY;
    t = warp_max(t);
    if (lane == 0) sh.red_f[0] = t;
  }
  __syncthreads();
  M = sh.red_f[0];
  double part = 0.0;
  for (int s = tid; s < nseg; s += blockDim.x)
    part += seg_s[s] * exp((static_cast<double>(seg_m[s]) - static_cast<double>(M)) * invtau);
  part = warp_sum(part);
  __syncthreads();
  if (lane == 0) sh.red_d[warp] = part;
  __syncthreads();
  if (warp == 0) {
    double t = (lane < kRowWarps) ? sh.red_d[lane] : 0.0;
    t = warp_sum(t);
    if (lane == 0) sh.bcd[0] = t;
  }
  __syncthreads();
  const double lse = static_cast<double>(M) * invtau + log(sh.bcd[0]);

  // radix select of the K-th smallest descending key (11 + 11 + 10 bits)
  int b1, before;
  find_rank_bin(hist, 2048, K, &b1, &before, sh);
  int need = K - before;
  for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int e = tid; e < V; e += blockDim.x) {
    const uint32_t k = zdesc_key(__ldg(row + e));
    if ((k >> 21) == static_cast<uint32_t>(b1)) atomicAdd(&hist[(k >> 10) & 0x7FFu], 1u);
  }
  __syncthreads();
  int b2;
  find_rank_bin(hist, 2048, need, &b2, &before, sh);
  need -= before;
  const uint32_t pre2 = (static_cast<uint32_t>(b1) << 11) | static_cast<uint32_t>(b2);
  for (int i = tid; i < 1024; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int e = tid; e < V; e += blockDim.x) {
    const uint32_t k = zdesc_key(__ldg(row + e));
    if ((k >> 10) == pre2) atomicAdd(&hist[k & 0x3FFu], 1u);
  }
  __syncthreads();
  int b3;
  find_rank_bin(hist, 1024, need, &b3, &before, sh);
  need -= before;                                    // ties at theta to take
  const uint32_t theta = (pre2 << 10) | static_cast<uint32_t>(b3);
  const int n_eq = static_cast<int>(hist[b3]);

  // collect: keys below theta, then the first `need` ties by token index
  if (tid == 0) s_count = 0;
  __syncthreads();
  for (int e = tid; e < V; e += blockDim.x) {
    const uint32_t k = zdesc_key(__ldg(row + e));
    if (k < theta || (k == theta && n_eq == need)) {
      const int pos = atomicAdd(&s_count, 1);
      if (pos < K) sbuf[pos] = (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(e);
    }
  }
  __syncthreads();
  if (n_eq != need) {
    // ordered pass over the row for the ties
    int taken = 0;
    for (int base = 0; base < V && taken < need; base += blockDim.x) {
      const int e = base + tid;
      const bool is = (e < V) && zdesc_key(__ldg(row + e)) == theta;
      const unsigned m = __ballot_sync(0xffffffffu, is);
      if (lane == 0) sh.red_i[warp] = __popc(m);
      __syncthreads();
      if (warp == 0) {
        const int v = (lane < kRowWarps) ? sh.red_i[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (lane < kRowWarps) sh.red_i[lane] = incl - v;
        if (lane == 31) sh.bc[3] = incl;
      }
      __syncthreads();
      const int rank = taken + sh.red_i[warp] + __popc(m & ((1u << lane) - 1u));
      if (is && rank < need) {
        const int pos = atomicAdd(&s_count, 1);
        if (pos < K) sbuf[pos] = (static_cast<uint64_t>(theta) << 32) | static_cast<uint32_t>(e);
      }
      taken += sh.bc[3];
      __syncthreads();
    }
  }
  for (int i = K + tid; i < P; i += blockDim.x) sbuf[i] = ~0ull;
  __syncthreads();
  // bitonic sort ascending: (z desc, token asc)
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = sbuf[i], b = sbuf[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) { sbuf[i] = b; sbuf[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  ListEntry* lst = p.lists + static_cast<int64_t>(node) * p.kcap;
  for (int i = tid; i < K; i += blockDim.x) {
    const uint64_t v = sbuf[i];
    ListEntry le;
    le.z = key_f32(~static_cast<uint32_t>(v >> 32));
    le.tok = static_cast<int32_t>(v & 0xFFFFFFFFu);
    lst[i] = le;
  }
  if (tid == 0) {
    p.meta[node].len = K;
    p.meta[node].cursor = 0;
    p.meta[node].lse = lse;
  }
}

// ------------------------------------------------------------ merge kernel

struct MergeShared {
  int red_i[kMergeWarps];
  int bc[8];
  uint32_t hist[256];
  uint64_t selA[kMergeStep];
  uint32_t selB[kMergeStep];
  int qlist[kMergeStep];
  int cnt[4];
};

__device__ __forceinline__ bool comp_le(uint64_t a, uint32_t b, uint64_t ta, uint32_t tb) {
  return a < ta || (a == ta && b <= tb);
}

// rank-th smallest (1-based) composite (A, B) among N entries in smem.
__device__ void radix_select_ab(const uint64_t* A, const uint32_t* Bk, int N, int rank,
                                uint64_t* thA, uint32_t* thB, MergeShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t pA = 0, mA = 0;
  uint32_t pB = 0, mB = 0;
  int need = rank;
  for (int pass = 0; pass < 12; ++pass) {
    for (int i = tid; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    const int shA = 56 - 8 * pass, shB = 24 - 8 * (pass - 8);
    for (int i = tid; i < N; i += blockDim.x) {
      if ((A[i] & mA) == pA && (Bk[i] & mB) == pB) {
        const uint32_t dg = pass < 8 ? static_cast<uint32_t>(A[i] >> shA) & 255u
                                     : (Bk[i] >> shB) & 255u;
        atomicAdd(&sh.hist[dg], 1u);
      }
    }
    __syncthreads();
    if (warp == 0) {
      int ls = 0;
      for (int k = 0; k < 8; ++k) ls += static_cast<int>(sh.hist[lane * 8 + k]);
      int incl = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int excl = incl - ls;
      if (excl < need && need <= incl) {
        int cum = excl;
        for (int k = 0; k < 8; ++k) {
          const int h = static_cast<int>(sh.hist[lane * 8 + k]);
          if (need <= cum + h) { sh.bc[0] = lane * 8 + k; sh.bc[1] = cum; sh.bc[2] = h; break; }
          cum += h;
        }
      }
    }
    __syncthreads();
    const int dg = sh.bc[0], bef = sh.bc[1], cnt = sh.bc[2];
    need -= bef;
    if (pass < 8) { pA |= static_cast<uint64_t>(dg) << shA; mA |= 0xFFull << shA; }
    else { pB |= static_cast<uint32_t>(dg) << shB; mB |= 0xFFu << shB; }
    __syncthreads();
    if (cnt == 1) {
      // a single entry carries this prefix: it is the answer
      for (int i = tid; i < N; i += blockDim.x)
        if ((A[i] & mA) == pA && (Bk[i] & mB) == pB) { sh.selA[0] = A[i]; sh.selB[0] = Bk[i]; }
      __syncthreads();
      *thA = sh.selA[0];
      *thB = sh.selB[0];
      __syncthreads();
      return;
    }
  }
  *thA = pA;
  *thB = pB;
}

__global__ void __launch_bounds__(kMergeThreads)
expand_merge_kernel(ExpandParams p) {
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ MergeShared sh;
  uint64_t* A = reinterpret_cast<uint64_t*>(dsm);
  uint32_t* Bk = reinterpret_cast<uint32_t*>(A + kMergeCap);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n0 = *p.n_nodes;
  const int rem = p.budget - n0;
  const int total = rem > 0 ? min(p.Bsel, rem) : 0;
  int appended = 0;
  while (appended < total) {
    const int s = min(kMergeStep, total - appended);
    // 1. list heads of every expanded node with entries left
    if (tid == 0) { sh.cnt[0] = 0; sh.cnt[1] = 0; sh.cnt[2] = 0; }
    __syncthreads();
    for (int nd = tid; nd < n0; nd += blockDim.x) {
      const int len = __ldcg(&p.meta[nd].len);
      const int cur = __ldcg(&p.meta[nd].cursor);
      if (cur < len) {
        const ListEntry e = p.lists[static_cast<int64_t>(nd) * p.kcap + cur];
        const double sc = entry_score(p.logp[nd], e.z, p.tau, __ldcg(&p.meta[nd].lse));
        const int i = atomicAdd(&sh.cnt[0], 1);
        A[i] = sdesc_key(sc);
        Bk[i] = (static_cast<uint32_t>(nd) << 18) | static_cast<uint32_t>(e.tok);
      }
    }
    __syncthreads();
    const int H = sh.cnt[0];
    if (H == 0) break;
    uint64_t tA = ~0ull;
    uint32_t tB = ~0u;
    if (H > s) radix_select_ab(A, Bk, H, s, &tA, &tB, sh);
    __syncthreads();
    for (int i = tid; i < H; i += blockDim.x)
      if (comp_le(A[i], Bk[i], tA, tB)) {
        const int k = atomicAdd(&sh.cnt[1], 1);
        if (k < kMergeStep) sh.qlist[k] = static_cast<int>(Bk[i] >> 18);
      }
    __syncthreads();
    const int Q = min(sh.cnt[1], kMergeStep);
    // 2. candidates ranked within the first s heads' bound, <= s per list
    for (int qi = warp; qi < Q; qi += kMergeWarps) {
      const int nd = sh.qlist[qi];
      const int len = __ldcg(&p.meta[nd].len);
      const int cur = __ldcg(&p.meta[nd].cursor);
      const double lse = __ldcg(&p.meta[nd].lse);
      const double lp = p.logp[nd];
      const ListEntry* lst = p.lists + static_cast<int64_t>(nd) * p.kcap;
      for (int base = 0; base < s; base += 32) {
        const int pos = cur + base + lane;
        bool ok = (base + lane < s) && pos < len;
        uint64_t a = 0;
        uint32_t bb = 0;
        if (ok) {
          const ListEntry e = lst[pos];
          a = sdesc_key(entry_score(lp, e.z, p.tau, lse));
          bb = (static_cast<uint32_t>(nd) << 18) | static_cast<uint32_t>(e.tok);
          ok = comp_le(a, bb, tA, tB);
        }
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        const int c = __popc(m);
        int off = 0;
        if (lane == 0 && c > 0) off = atomicAdd(&sh.cnt[2], c);
        off = __shfl_sync(0xffffffffu, off, 0);
        if (ok) {
          const int k = __popc(m & ((1u << lane) - 1u));
          if (off + k < kMergeCap) {
            A[off + k] = a;   // heads are no longer needed
            Bk[off + k] = bb;
          }
        }
        if (c < 32) break;
      }
    }
    __syncthreads();
    const int C = min(sh.cnt[2], kMergeCap);
    uint64_t uA = ~0ull;
    uint32_t uB = ~0u;
    if (C > s) radix_select_ab(A, Bk, C, s, &uA, &uB, sh);
    if (tid == 0) sh.cnt[3] = 0;
    __syncthreads();
    for (int i = tid; i < C; i += blockDim.x)
      if (comp_le(A[i], Bk[i], uA, uB)) {
        const int k = atomicAdd(&sh.cnt[3], 1);
        if (k < kMergeStep) {
          sh.selA[k] = A[i];
          sh.selB[k] = Bk[i];
        }
      }
    __syncthreads();
    const int S = min(sh.cnt[3], kMergeStep);
    for (int i = S + tid; i < kMergeStep; i += blockDim.x) { sh.selA[i] = ~0ull; sh.selB[i] = ~0u; }
    __syncthreads();
    // 3. sort the winners by (score desc, parent asc, token asc)
    for (int k = 2; k <= kMergeStep; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (tid < kMergeStep) {
          const int i = tid, ixj = i ^ j;
          if (ixj > i) {
            const uint64_t a0 = sh.selA[i], a1 = sh.selA[ixj];
            const uint32_t b0 = sh.selB[i], b1 = sh.selB[ixj];
            const bool gt = a0 > a1 || (a0 == a1 && b0 > b1);
            const bool up = (i & k) == 0;
            if (gt == up) {
              sh.selA[i] = a1; sh.selA[ixj] = a0;
              sh.selB[i] = b1; sh.selB[ixj] = b0;
            }
          }
        }
        __syncthreads();
      }
    }
    // 4. append in rank order and advance the source lists' cursors
    if (tid < S) {
      const int node = n0 + appended + tid;
      const int nd = static_cast<int>(sh.selB[tid] >> 18);
      p.parent[node] = nd;
      p.token[node] = static_cast<int32_t>(sh.selB[tid] & 0x3FFFFu);
      p.logp[node] = sdesc_val(sh.selA[tid]);
      p.frontier[appended + tid] = node;
      atomicAdd(&p.meta[nd].cursor, 1);
    }
    __threadfence_block();
    __syncthreads();
    appended += S;
    if (S < s) break;
  }
  for (int i = appended + tid; i < p.Bsel; i += blockDim.x) p.frontier[i] = -1;
  if (tid == 0) {
    *p.n_nodes = n0 + appended;
    *p.n_appended = appended;
  }
}

__global__ void expand_init_kernel(ExpandParams p, int root_token) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < p.budget) {
    NodeMeta m;
    m.len = 0; m.cursor = 0; m.expanded = 0; m.pad = 0; m.lse = 0.0;
    p.meta[i] = m;
  }
  if (i == 0) {
    *p.n_nodes = 1;
    p.parent[0] = -1;
    p.token[0] = root_token;
    p.logp[0] = 0.0;
  }
}

// ------------------------------------------------------------ host side

size_t expand_pool_bytes(int budget, int V) {
  return expand_lists_offset(budget) +
         static_cast<size_t>(budget) * static_cast<size_t>(expand_kcap(budget, V)) * sizeof(ListEntry);
}

static ExpandParams make_params(const tv_expand_args* a) {
  ExpandParams p;
  p.V = a->V; p.R = a->R; p.Bsel = a->Bsel; p.budget = a->budget;
  p.tau = a->draft_temperature;
  p.logits = a->draft_logits; p.ld = a->ld_logits;
  p.row_node = a->row_node;
  p.n_nodes = a->n_nodes; p.parent = a->parent; p.token = a->token; p.logp = a->logp;
  p.meta = static_cast<NodeMeta*>(a->pool);
  p.lists = reinterpret_cast<ListEntry*>(static_cast<unsigned char*>(a->pool) + expand_lists_offset(a->budget));
  p.kcap = expand_kcap(a->budget, a->V);
  p.frontier = a->frontier; p.n_appended = a->n_appended;
  p.status = a->dev_status;
  return p;
}

cudaError_t launch_expand_init(const tv_expand_args* a, int root_token, cudaStream_t stream) {
  ExpandParams p = make_params(a);
  const int threads = 256;
  expand_init_kernel<<<(a->budget + threads - 1) / threads, threads, 0, stream>>>(p, root_token);
  return cudaGetLastError();
}

cudaError_t launch_expand(const tv_expand_args* a, cudaStream_t stream) {
  ExpandParams p = make_params(a);
  if (a->R > 0) {
    const int nseg = (a->V + kSegE - 1) / kSegE;
    const int K = static_cast<int>(expand_kcap(a->budget, a->V));
    int P = 2;
    while (P < K) P <<= 1;
    const size_t smem = static_cast<size_t>(P) * 8 + static_cast<size_t>(nseg) * 12 + 16;
    cudaError_t e = cudaFuncSetAttribute(expand_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    expand_rows_kernel<<<a->R, kRowThreads, smem, stream>>>(p);
  }
  const size_t msmem = static_cast<size_t>(kMergeCap) * (sizeof(uint64_t) + sizeof(uint32_t));
  cudaError_t e = cudaFuncSetAttribute(expand_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(msmem));
  if (e != cudaSuccess) return e;
  expand_merge_kernel<<<1, kMergeThreads, msmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tv
