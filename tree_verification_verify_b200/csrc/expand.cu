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
//   expand_rows_kernel   one CTA per row: the row's maximum and minimum,
//                        then its lse with a histogram of 2048 value bins
//                        over [min, max] (monotone in the logit, so the
//                        boundary bin of the top K follows by a prefix
//                        count), then the bins above the boundary plus an
//                        exact sort of the boundary bin's members, and a
//                        bitonic sort of the K into the node's list (a
//                        boundary bin too crowded for shared memory falls
//                        back to a radix select on the 32-bit key);
// Beam mode (the SpecExec page's ablation: standard beam search) ranks only
// the children of the call's own rows: each row's list holds its best
// min(V, Bsel) tokens and the merge reads the lists stamped by this call.
//
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
  int32_t stamp;      // number of the call whose row built the list
  double lse;         // logsumexp of the node's row / tau
};

// Pool header: calls made since tree_expand_init (stamps the lists, so
// that beam mode takes only the lists its own rows built).
struct PoolHeader {
  int32_t calls;
};
constexpr size_t kPoolHeaderBytes = 256;

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
constexpr int kCandCap = 4096;                      // boundary-bin candidates in shared memory

__host__ __device__ inline int64_t expand_kcap(int budget, int V) {
  int64_t k = budget - 1;
  if (k > V) k = V;
  return k < 1 ? 1 : k;
}
__host__ __device__ inline size_t expand_lists_offset(int budget) {
  const size_t m = kPoolHeaderBytes + static_cast<size_t>(budget) * sizeof(NodeMeta);
  return (m + 255) & ~static_cast<size_t>(255);
}

struct ExpandParams {
  int V, R, Bsel, budget;
  int beam;               // TV_EXPAND_BEAM: rank this call's rows only
  float tau;
  const float* logits; int64_t ld;
  const int32_t* row_node;
  int32_t* n_nodes;
  int32_t* parent;
  int32_t* token;
  double* logp;
  PoolHeader* header;
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

// Ascending bitonic sort of P (a power of two, 2 <= P) keys in shared
// memory by the whole block.  Stages whose partners lie within a 64-key
// block run in registers (warp w, lane l holds keys 64b + l and 64b + 32 + l
// of its blocks b): the partner 32 apart is the thread's other key, closer
// partners come by shuffle.  Wider stages compare in shared memory.
__device__ __forceinline__ uint64_t cas_u64(uint64_t v, uint64_t pv, bool keep_min) {
  return keep_min ? (v < pv ? v : pv) : (v > pv ? v : pv);
}

__device__ void bitonic_block64(uint64_t* buf, int P, int k, int jmax) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  for (int blk = warp; blk * 64 < P; blk += nw) {
    const int i0 = blk * 64 + lane, i1 = i0 + 32;
    uint64_t v0 = buf[i0], v1 = buf[i1];
    for (int kk = (k <= 64 ? 2 : k); kk <= (k <= 64 ? 64 : k); kk <<= 1) {
      const int jtop = (k <= 64) ? (kk >> 1) : jmax;
      for (int j = jtop; j > 0; j >>= 1) {
        if (kk > P) break;
        const bool up0 = (i0 & kk) == 0, up1 = (i1 & kk) == 0;
        if (j == 32) {
          // partners i0 and i1 = i0 + 32: i0 is the lower index
          const uint64_t a = v0, b = v1;
          v0 = cas_u64(a, b, up0);
          v1 = cas_u64(b, a, !up1);
        } else {
          const uint64_t p0 = __shfl_xor_sync(0xffffffffu, v0, j);
          const uint64_t p1 = __shfl_xor_sync(0xffffffffu, v1, j);
          const bool low0 = (i0 & j) == 0, low1 = (i1 & j) == 0;
          v0 = cas_u64(v0, p0, low0 == up0);
          v1 = cas_u64(v1, p1, low1 == up1);
        }
      }
      if (k > 64) break;
    }
    buf[i0] = v0;
    buf[i1] = v1;
  }
}

__device__ void bitonic_sort_u64(uint64_t* buf, int P) {
  const int tid = threadIdx.x;
  if (P < 64) {
    // small: plain shared-memory stages
    for (int k = 2; k <= P; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < P; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint64_t a = buf[i], b = buf[ixj];
            const bool up = (i & k) == 0;
            if ((a > b) == up) { buf[i] = b; buf[ixj] = a; }
          }
        }
        __syncthreads();
      }
    return;
  }
  // k = 2 .. 64 entirely in registers
  bitonic_block64(buf, P, 64, 32);
  __syncthreads();
  for (int k = 128; k <= P; k <<= 1) {
    for (int j = k >> 1; j >= 64; j >>= 1) {
      for (int i = tid; i < P; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = buf[i], b = buf[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) { buf[i] = b; buf[ixj] = a; }
        }
      }
      __syncthreads();
    }
    bitonic_block64(buf, P, k, 32);
    __syncthreads();
  }
}

// ------------------------------------------------------------ row kernel

__device__ __forceinline__ float warp_min_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// The elements of a row pass: iteration it of a thread covers elements
// 4 (it * blockDim + tid) .. + 3; every thread runs the same number of
// iterations (ballots stay warp-uniform), four loads in flight per batch.
template <class F>
__device__ __forceinline__ void row_pass(const float* row, int V, bool vec, F&& f) {
  const int tid = threadIdx.x;
  const int per = 4 * static_cast<int>(blockDim.x);
  const int iters = (V + per - 1) / per;
  for (int it0 = 0; it0 < iters; it0 += 4) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e0 = ((it0 + u) * static_cast<int>(blockDim.x) + tid) * 4;
      v[u] = (it0 + u < iters) ? load4(row, e0, V, vec, 0.f) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (it0 + u >= iters) break;
      const int e0 = ((it0 + u) * static_cast<int>(blockDim.x) + tid) * 4;
      const float xs[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) f(e0 + k, xs[k], e0 + k < V);
    }
  }
}

// Appends the lanes' flagged 64-bit entries at buf[*count ..] (one shared
// atomic per warp); entries past cap are dropped (the count still grows).
__device__ __forceinline__ void warp_append(bool take, uint64_t v, uint64_t* buf, int* count, int cap) {
  const int lane = threadIdx.x & 31;
  const unsigned m = __ballot_sync(0xffffffffu, take);
  if (m == 0u) return;
  int off = 0;
  if (lane == 0) off = atomicAdd(count, __popc(m));
  off = __shfl_sync(0xffffffffu, off, 0);
  if (take) {
    const int pos = off + __popc(m & ((1u << lane) - 1u));
    if (pos < cap) buf[pos] = v;
  }
}

__global__ void __launch_bounds__(kRowThreads)
expand_rows_kernel(ExpandParams p) {
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ RowShared sh;
  __shared__ uint32_t hist[2048];
  __shared__ int s_count, s_cand;
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
  // best-first: every candidate that can still be taken; beam: this call
  // takes at most Bsel, and its lists are not used later
  const int K = p.beam ? min(min(V, p.Bsel), p.budget - n0) : min(V, p.budget - n0);
  if (K <= 0) return;
  const float* row = p.logits + static_cast<int64_t>(r) * p.ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  const int P = 1 << (32 - __clz(K - 1 | 1));      // next power of two >= K (>= 2)
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(dsm);
  uint64_t* cbuf = sbuf + P;                         // boundary-bin candidates
  const double invtau = 1.0 / static_cast<double>(p.tau);

  // pass 1: finiteness, row maximum and minimum
  bool bad = false;
  float lmax = -INFINITY, lmin = INFINITY;
  row_pass(row, V, vec, [&](int, float x, bool in) {
    if (!in) return;
    if (!isfinite(x)) bad = true;
    else { lmax = fmaxf(lmax, x); lmin = fminf(lmin, x); }
  });
  const int any_bad = __syncthreads_or(bad ? 1 : 0);
  if (any_bad) {
    if (tid == 0) set_status(p.status, TV_DEV_NONFINITE);
    return;
  }
  lmax = warp_max(lmax);
  lmin = warp_min_f(lmin);
  if (lane == 0) { sh.red_f[warp] = lmax; sh.red_d[warp] = static_cast<double>(lmin); }
  for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  float M = -INFINITY, mn = INFINITY;
  for (int w = 0; w < kRowWarps; ++w) { M = fmaxf(M, sh.red_f[w]); mn = fminf(mn, static_cast<float>(sh.red_d[w])); }
  __syncthreads();
  // pass 2: value bins (M - z) * 2047 / (M - min), non-decreasing as z
  // falls, so bin order is rank order; and the row's sum of exponentials
  const float range = M - mn;
  const float sc = (range > 0.f && isfinite(range)) ? 2047.f / range : 0.f;
  double es = 0.0;
  row_pass(row, V, vec, [&](int, float x, bool in) {
    if (!in) return;
    const int bin = static_cast<int>(fminf((M - x) * sc, 2047.f));
    atomicAdd(&hist[bin], 1u);
    // double-precision exponentials: the row's lse enters every cumulative
    // score, and cross-row ranks must not move by more than fp64 rounding
    es += exp((static_cast<double>(x) - static_cast<double>(M)) * invtau);
  });
  es = warp_sum(es);
  if (lane == 0) sh.red_d[warp] = es;
  __syncthreads();
  if (warp == 0) {
    double t = (lane < kRowWarps) ? sh.red_d[lane] : 0.0;
    t = warp_sum(t);
    if (lane == 0) sh.bcd[0] = t;
  }
  __syncthreads();
  const double lse = static_cast<double>(M) * invtau + log(sh.bcd[0]);

  int b1, before;
  find_rank_bin(hist, 2048, K, &b1, &before, sh);
  const int n1 = static_cast<int>(hist[b1]);
  const int need = K - before;                     // taken from the boundary bin
  if (n1 <= kCandCap) {
    // pass 3: the bins above the boundary go to the list, the boundary bin
    // to the candidates, whose exact order (key, token) decides the rest
    if (tid == 0) { s_count = 0; s_cand = 0; }
    __syncthreads();
    row_pass(row, V, vec, [&](int e, float x, bool in) {
      const int bin = in ? static_cast<int>(fminf((M - x) * sc, 2047.f)) : 2048;
      const uint64_t v = (static_cast<uint64_t>(zdesc_key(x)) << 32) | static_cast<uint32_t>(e);
      warp_append(bin < b1, v, sbuf, &s_count, K);
      warp_append(bin == b1, v, cbuf, &s_cand, kCandCap);
    });
    __syncthreads();
    const int nc = min(s_cand, kCandCap);
    const int Pc = 1 << (32 - __clz(nc - 1 | 1));
    for (int i = nc + tid; i < Pc; i += blockDim.x) cbuf[i] = ~0ull;
    __syncthreads();
    bitonic_sort_u64(cbuf, Pc);
    for (int i = tid; i < need; i += blockDim.x) sbuf[before + i] = cbuf[i];
    __syncthreads();
  } else {
    // a crowded boundary bin: radix select on the 32-bit key instead
    // (11 + 11 + 10 bits), then the keys below the threshold and the first
    // ties by token index
    __syncthreads();
    for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    row_pass(row, V, vec, [&](int, float x, bool in) {
      if (in) atomicAdd(&hist[zdesc_key(x) >> 21], 1u);
    });
    __syncthreads();
    int kb1, kbefore;
    find_rank_bin(hist, 2048, K, &kb1, &kbefore, sh);
    int kneed = K - kbefore;
    for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int e = tid; e < V; e += blockDim.x) {
      const uint32_t k = zdesc_key(__ldg(row + e));
      if ((k >> 21) == static_cast<uint32_t>(kb1)) atomicAdd(&hist[(k >> 10) & 0x7FFu], 1u);
    }
    __syncthreads();
    int b2;
    find_rank_bin(hist, 2048, kneed, &b2, &kbefore, sh);
    kneed -= kbefore;
    const uint32_t pre2 = (static_cast<uint32_t>(kb1) << 11) | static_cast<uint32_t>(b2);
    for (int i = tid; i < 1024; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int e = tid; e < V; e += blockDim.x) {
      const uint32_t k = zdesc_key(__ldg(row + e));
      if ((k >> 10) == pre2) atomicAdd(&hist[k & 0x3FFu], 1u);
    }
    __syncthreads();
    int b3;
    find_rank_bin(hist, 1024, kneed, &b3, &kbefore, sh);
    const int need3 = kneed - kbefore;                 // ties at theta to take
    const uint32_t theta = (pre2 << 10) | static_cast<uint32_t>(b3);
    const int n_eq = static_cast<int>(hist[b3]);

    // collect: keys below theta, then the first `need` ties by token index
    if (tid == 0) s_count = 0;
    __syncthreads();
    for (int base = warp * 32; base < V; base += blockDim.x) {
      const int e = base + lane;
      const uint32_t k = (e < V) ? zdesc_key(__ldg(row + e)) : ~0u;
      const bool take = (e < V) && (k < theta || (k == theta && n_eq == need3));
      const unsigned m = __ballot_sync(0xffffffffu, take);
      int off = 0;
      if (lane == 0 && m) off = atomicAdd(&s_count, __popc(m));
      off = __shfl_sync(0xffffffffu, off, 0);
      if (take) {
        const int pos = off + __popc(m & ((1u << lane) - 1u));
        if (pos < K) sbuf[pos] = (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(e);
      }
    }
    __syncthreads();
    if (n_eq != need3) {
      // ordered pass over the row for the ties
      int taken = 0;
      for (int base = 0; base < V && taken < need3; base += blockDim.x) {
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
        if (is && rank < need3) {
          const int pos = atomicAdd(&s_count, 1);
          if (pos < K) sbuf[pos] = (static_cast<uint64_t>(theta) << 32) | static_cast<uint32_t>(e);
        }
        taken += sh.bc[3];
        __syncthreads();
      }
    }
  }
  for (int i = K + tid; i < P; i += blockDim.x) sbuf[i] = ~0ull;
  __syncthreads();
  bitonic_sort_u64(sbuf, P);
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
    p.meta[node].stamp = __ldcg(&p.header->calls) + 1;
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
  const int stamp = __ldcg(&p.header->calls) + 1;    // this call's number
  int appended = 0;
  while (appended < total) {
    const int s = min(kMergeStep, total - appended);
    // 1. list heads of every expanded node with entries left
    if (tid == 0) { sh.cnt[0] = 0; sh.cnt[1] = 0; sh.cnt[2] = 0; }
    __syncthreads();
    // best-first: every expanded node's list; beam: only the lists built by
    // this call's rows (each node once)
    const int nh = p.beam ? p.R : n0;
    for (int h = tid; h < nh; h += blockDim.x) {
      int nd = h;
      if (p.beam) {
        nd = p.row_node[h];
        if (nd < 0 || nd >= n0 || __ldcg(&p.meta[nd].stamp) != stamp) continue;
        bool dup = false;
        for (int h2 = 0; h2 < h && !dup; ++h2) dup = (p.row_node[h2] == nd);
        if (dup) continue;
      }
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
  __syncthreads();
  if (tid == 0) {
    *p.n_nodes = n0 + appended;
    *p.n_appended = appended;
    p.header->calls = stamp;
  }
}

__global__ void expand_init_kernel(ExpandParams p, int root_token) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < p.budget) {
    NodeMeta m;
    m.len = 0; m.cursor = 0; m.expanded = 0; m.stamp = 0; m.lse = 0.0;
    p.meta[i] = m;
  }
  if (i == 0) {
    p.header->calls = 0;
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
  p.beam = a->mode == TV_EXPAND_BEAM;
  p.tau = a->draft_temperature;
  p.logits = a->draft_logits; p.ld = a->ld_logits;
  p.row_node = a->row_node;
  p.n_nodes = a->n_nodes; p.parent = a->parent; p.token = a->token; p.logp = a->logp;
  p.header = static_cast<PoolHeader*>(a->pool);
  p.meta = reinterpret_cast<NodeMeta*>(static_cast<unsigned char*>(a->pool) + kPoolHeaderBytes);
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
    const int K = static_cast<int>(expand_kcap(a->budget, a->V));
    int P = 2;
    while (P < K) P <<= 1;
    const size_t smem = (static_cast<size_t>(P) + kCandCap) * sizeof(uint64_t);
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
