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
// One launch per round, one CTA per row (expand_round_kernel):
//   row      the row is copied into shared memory at kernel entry (bulk
//            copies in 16 KB chunks, when it fits).  The first chunk gives
//            the frame of a 2048-bin value histogram (its maximum and
//            minimum; values outside share the first or last bin, and bin
//            order is rank order) and a collection threshold.  Pass 1, chunk
//            by chunk as the copies land: finiteness, the row maximum, the
//            histogram, and the collection of the elements at or above the
//            threshold (about 1.5 K of them).  Pass 2: the row's lse in fp64
//            (a table-driven exponential).  The bin of the K-th largest
//            follows from one scan of the histogram; the collected elements
//            above it are scattered bin by bin into the node's list and
//            ordered inside their bin by counting, the boundary bin's best
//            members likewise.  Crowded bins fall back to a bitonic sort of
//            the whole list, a boundary bin too crowded for shared memory to
//            a radix select on the 32-bit key, a collection that missed part
//            of the top K to a scatter from the row.
//   merge    the last CTA to finish its row (a ticket) takes the best
//            s <= 128 candidates of the union, repeatedly: the s-th best
//            list head (heads are cached in the node metadata) bounds the
//            s-th best candidate, so only entries at least as good as the
//            worst head in the first s (found with a histogram of the
//            heads' scores; with fewer than s heads, the s-th best of the
//            first ceil(s / H) entries of every list) can be taken; they are
//            gathered, a histogram of their scores isolates the s winners
//            (exact (score, parent, token) ranks inside the boundary bin),
//            the winners are ordered by counting and appended.  When a
//            bound leaves too many candidates it falls back to a radix
//            select over <= s lists of <= s entries.
// A call with no rows runs the merge alone (expand_merge_kernel).
// Beam mode (the SpecExec page's ablation: standard beam search) ranks only
// the children of the call's own rows: each row's list holds its best
// min(V, Bsel) tokens and the merge reads the lists stamped by this call.
#include "tc_prims.cuh"

namespace tv {

// Test hook (tv_expand_set_wait_limit): when nonzero, a staged row waits
// for its first chunk with this many non-blocking tests of a barrier that
// nothing arrives on (as if the copy were lost), so the wait expires.
__device__ uint32_t g_row_wait_polls = 0u;

struct NodeMeta {
  int32_t len;        // entries in the node's sorted list (0: not expanded)
  int32_t cursor;     // first entry not yet taken
  int32_t expanded;   // set once a row for the node has been consumed
  int32_t stamp;      // number of the call whose row built the list
  double lse;         // logsumexp of the node's row / tau
  uint64_t head;      // descending-score key of the entry at the cursor (~0: none)
};

// Pool header: calls made since tree_expand_init (stamps the lists, so
// that beam mode takes only the lists its own rows built) and the ticket
// of the round's row CTAs.
struct PoolHeader {
  int32_t calls;
  int32_t rows_done;
};
constexpr size_t kPoolHeaderBytes = 256;

struct ListEntry {
  float z;
  int32_t tok;
};

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / kWarp;
constexpr int kBins = 2048;
constexpr int kCandCap = 2048;       // boundary-bin members kept in shared memory
constexpr int kCollCap = 4096;       // likely members of the top K collected during the first pass
constexpr int kRankMax = 256;        // groups up to this size are ordered by counting
constexpr int kChunkFloats = 4 * kThreads;   // one staged chunk: a float4 per thread
constexpr int kChunkBytes = kChunkFloats * 4;
constexpr int kMaxChunks = 14;
constexpr int kMergeStep = 128;                     // nodes taken per sub-step
constexpr int kMergeCap = kMergeStep * kMergeStep;  // candidates of the radix fallback
constexpr int kHeadCap = 8192;                      // heads (one per expanded node)
constexpr int kFastCap = 3072;                      // candidates of the threshold path
constexpr int kQCap = 1024;                         // lists that can contribute to one sub-step
// offset of the per-list metadata (lse, log-probability, node, length,
// cursor) of the threshold path in its shared memory
constexpr size_t kQMetaOff = static_cast<size_t>(kHeadCap) * 12 + static_cast<size_t>(kFastCap) * 16;
constexpr size_t kMergeDyn = static_cast<size_t>(kMergeCap) * (sizeof(uint64_t) + sizeof(uint32_t));

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
  int stage;              // rows are staged in shared memory
  int stage_bytes;        // shared memory of a staged row (16-byte multiple)
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

struct ExpandShared {
  uint32_t hist[kBins];
  uint32_t boff[kBins];
  uint32_t bfill[kBins];
  uint64_t bar[kMaxChunks];
  uint64_t lost_bar;  // never arrived on (the wait-expiry test hook)
  double etab[256];   // 2^(j/256)
  double red_d[kWarps];
  float red_f[kWarps];
  float red_g[kWarps];
  int red_i[kWarps];
  int bc[8];
  int cnt[4];
  double bcd[2];
  unsigned long long kmin, kmax, kthr;
  uint64_t selA[kMergeStep];
  uint32_t selB[kMergeStep];
  int selP[kMergeStep];       // (list slot << 13 | list position) of a winner, threshold path
  uint64_t ordA[kMergeStep];
  uint32_t ordB[kMergeStep];
  int ordP[kMergeStep];
  int haveP;
  int qlist[kMergeStep];
  int flag;
  int last;
  int abort;
};

// descending-score key: smaller key = larger value
__device__ __forceinline__ uint32_t zdesc_key(float z) { return ~f32_key(z); }
__device__ __forceinline__ uint64_t sdesc_key(double s) { return ~f64_key(s); }
__device__ __forceinline__ double sdesc_val(uint64_t k) { return key_f64(~k); }

// Cumulative log-probability of a list entry (same expression everywhere).
__device__ __forceinline__ double entry_score(double logp_n, float z, float tau, double lse) {
  return (logp_n + static_cast<double>(z) / static_cast<double>(tau)) - lse;
}

// e^t for t <= 0, table driven (P. T. P. Tang, "Table-driven implementation
// of the exponential function in IEEE floating-point arithmetic", ACM TOMS
// 15(2), 1989): t = k ln2/256 + r with k the nearest integer to t 256/ln2
// and |r| <= ln2/512, so e^t = 2^(k >> 8) 2^((k & 255)/256) e^r; e^r - 1 is
// its degree-4 Taylor polynomial (truncation below 4e-17 relative), ln2/256
// is split into a double and its remainder, and the power of two is added
// to the exponent field.  Terms below e^-700 are returned as 0 (next to the
// row maximum's 1 they are below 1e-300).  T[j] = 2^(j/256).
__device__ __forceinline__ double exp_neg(double t, const double* T) {
  constexpr double kInvL = 369.3299304675746;          // 256 / ln 2
  constexpr double kLhi = 0.0027076061740622863;       // ln 2 / 256, rounded
  constexpr double kLlo = 9.058776616587108e-20;       // ln 2 / 256 - kLhi
  if (!(t >= -700.0)) return 0.0;
  const double kd = rint(t * kInvL);
  double r = fma(-kd, kLhi, t);
  r = fma(-kd, kLlo, r);
  const double em1 = r * (1.0 + r * (0.5 + r * (1.0 / 6.0 + r * (1.0 / 24.0))));
  const int k = static_cast<int>(kd);
  const double tj = T[k & 255];
  const double v = fma(tj, em1, tj);
  return __longlong_as_double(__double_as_longlong(v) + (static_cast<long long>(k >> 8) << 52));
}

// Value bin of a logit in the frame [top - 2047/sc, top]: (top - z) * sc
// clamped to [0, 2047], non-decreasing as z falls (one function, so every
// pass bins an element identically; values outside the frame share the
// first or the last bin).
__device__ __forceinline__ int vbin(float x, float top, float sc) {
  return static_cast<int>(fmaxf(fminf((top - x) * sc, 2047.f), 0.f));
}
// Score bin: (best - score) * scale in fp64, non-decreasing as the score falls.
__device__ __forceinline__ int sbin(double s, double best, double scale) {
  const double b = (best - s) * scale;
  return b >= 2047.0 ? 2047 : static_cast<int>(b);
}

__device__ __forceinline__ ListEntry entry_of(uint64_t v) {
  ListEntry le;
  le.z = key_f32(~static_cast<uint32_t>(v >> 32));
  le.tok = static_cast<int32_t>(v & 0xFFFFFFFFu);
  return le;
}

__device__ __forceinline__ ListEntry load_entry(const ListEntry* e) {
  const int2 v = __ldcg(reinterpret_cast<const int2*>(e));
  ListEntry le;
  le.z = __int_as_float(v.x);
  le.tok = v.y;
  return le;
}

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t t = __shfl_xor_sync(0xffffffffu, v, o);
    v = t < v ? t : v;
  }
  return v;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t t = __shfl_xor_sync(0xffffffffu, v, o);
    v = t > v ? t : v;
  }
  return v;
}
__device__ __forceinline__ float warp_min_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------ block helpers

// Find the bin holding the rank-th smallest element (rank 1-based) of a
// histogram; returns the bin and the count of elements in lower bins.
__device__ void find_rank_bin(const uint32_t* hist, int nbins, int rank, int* bin, int* before,
                              ExpandShared& sh) {
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

// One scan of a histogram for the bin holding the rank-th smallest element
// (rank 1-based): exclusive prefix offsets of every bin into boff, bfill
// zeroed; returns the bin, the count before it and the largest count among
// the bins before it.
__device__ void boundary_scan(const uint32_t* hist, uint32_t* boff, uint32_t* bfill, int rank, int* bin,
                              int* before, int* maxc, ExpandShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = kBins / kThreads;                   // 2 bins per thread
  const int lo = tid * per;
  int ls = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) ls += static_cast<int>(hist[lo + i]);
  int incl = ls;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh.red_i[warp] = incl;
  if (tid == 0) sh.bc[4] = 0;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < kWarps ? sh.red_i[lane] : 0;
    int wi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kWarps) sh.red_i[lane] = wi - v;
  }
  __syncthreads();
  int cum = sh.red_i[warp] + incl - ls;
  int mx = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int h = static_cast<int>(hist[lo + i]);
    boff[lo + i] = static_cast<uint32_t>(cum);
    bfill[lo + i] = 0u;
    if (cum < rank && rank <= cum + h) { sh.bc[0] = lo + i; sh.bc[1] = cum; }
    if (cum + h < rank) mx = max(mx, h);              // bins before the boundary
    cum += h;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0 && mx > 0) atomicMax(&sh.bc[4], mx);
  __syncthreads();
  *bin = sh.bc[0];
  *before = sh.bc[1];
  *maxc = sh.bc[4];
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

// ------------------------------------------------------------ row passes

// The elements of a row in global memory: iteration it of a thread covers
// elements 4 (it * blockDim + tid) .. + 3; every thread runs the same
// number of iterations (ballots stay warp-uniform), four loads in flight.
template <class F>
__device__ __forceinline__ void global_pass(const float* row, int V, bool vec, F&& f) {
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

// The same visit order over a row staged in shared memory (16-byte aligned).
__device__ __forceinline__ float4 smem4(const float* srow, int e0, int V) {
  if (e0 + 3 < V) return *reinterpret_cast<const float4*>(srow + e0);
  float4 v;
  v.x = (e0 + 0 < V) ? srow[e0 + 0] : 0.f;
  v.y = (e0 + 1 < V) ? srow[e0 + 1] : 0.f;
  v.z = (e0 + 2 < V) ? srow[e0 + 2] : 0.f;
  v.w = (e0 + 3 < V) ? srow[e0 + 3] : 0.f;
  return v;
}
template <class F>
__device__ __forceinline__ void smem_pass(const float* srow, int V, F&& f) {
  const int per = 4 * static_cast<int>(blockDim.x);
  for (int base = 0; base < V; base += per) {
    const int e0 = base + 4 * static_cast<int>(threadIdx.x);
    const float4 v = smem4(srow, e0, V);
    f(e0 + 0, v.x, e0 + 0 < V);
    f(e0 + 1, v.y, e0 + 1 < V);
    f(e0 + 2, v.z, e0 + 2 < V);
    f(e0 + 3, v.w, e0 + 3 < V);
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

// ------------------------------------------------------------ row

// The sorted list of one row's best K tokens (without the crowded-bin
// shortcuts): the bins above the boundary and the boundary bin's best
// members gathered in sbuf, then one bitonic sort.
template <bool STAGED>
__device__ void row_list_sorted(const ExpandParams& p, const float* src, bool vec, int V, int K, int P, float M,
                                float sc, int b1, int before, uint64_t* sbuf, uint64_t* cbuf, ListEntry* lst,
                                ExpandShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n1 = static_cast<int>(sh.hist[b1]);
  const int need = K - before;
  auto pass = [&](auto&& f) {
    if (STAGED) smem_pass(src, V, f);
    else global_pass(src, V, vec, f);
  };
  if (n1 <= kCandCap) {
    if (tid == 0) { sh.cnt[0] = 0; sh.cnt[1] = 0; }
    __syncthreads();
    pass([&](int e, float x, bool in) {
      const int bin = in ? vbin(x, M, sc) : kBins;
      const uint64_t v = (static_cast<uint64_t>(zdesc_key(x)) << 32) | static_cast<uint32_t>(e);
      warp_append(bin < b1, v, sbuf, &sh.cnt[0], K);
      warp_append(bin == b1, v, cbuf, &sh.cnt[1], kCandCap);
    });
    __syncthreads();
    const int nc = min(sh.cnt[1], kCandCap);
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
    uint32_t* hist = sh.hist;
    __syncthreads();
    for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    pass([&](int, float x, bool in) {
      if (in) atomicAdd(&hist[zdesc_key(x) >> 21], 1u);
    });
    __syncthreads();
    int kb1, kbefore;
    find_rank_bin(hist, kBins, K, &kb1, &kbefore, sh);
    int kneed = K - kbefore;
    for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    pass([&](int, float x, bool in) {
      const uint32_t k = zdesc_key(x);
      if (in && (k >> 21) == static_cast<uint32_t>(kb1)) atomicAdd(&hist[(k >> 10) & 0x7FFu], 1u);
    });
    __syncthreads();
    int b2;
    find_rank_bin(hist, kBins, kneed, &b2, &kbefore, sh);
    kneed -= kbefore;
    const uint32_t pre2 = (static_cast<uint32_t>(kb1) << 11) | static_cast<uint32_t>(b2);
    for (int i = tid; i < 1024; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    pass([&](int, float x, bool in) {
      const uint32_t k = zdesc_key(x);
      if (in && (k >> 10) == pre2) atomicAdd(&hist[k & 0x3FFu], 1u);
    });
    __syncthreads();
    int b3;
    find_rank_bin(hist, 1024, kneed, &b3, &kbefore, sh);
    const int need3 = kneed - kbefore;                 // ties at theta to take
    const uint32_t theta = (pre2 << 10) | static_cast<uint32_t>(b3);
    const int n_eq = static_cast<int>(hist[b3]);

    // collect: keys below theta, then the first `need3` ties by token index
    if (tid == 0) sh.cnt[0] = 0;
    __syncthreads();
    pass([&](int e, float x, bool in) {
      const uint32_t k = zdesc_key(x);
      const bool take = in && (k < theta || (k == theta && n_eq == need3));
      warp_append(take, (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(e), sbuf, &sh.cnt[0], K);
    });
    __syncthreads();
    if (n_eq != need3) {
      // ordered pass over the row for the ties
      int taken = 0;
      for (int base = 0; base < V && taken < need3; base += blockDim.x) {
        const int e = base + tid;
        const float x = (e < V) ? (STAGED ? src[e] : __ldg(src + e)) : 0.f;
        const bool is = (e < V) && zdesc_key(x) == theta;
        const unsigned m = __ballot_sync(0xffffffffu, is);
        if (lane == 0) sh.red_i[warp] = __popc(m);
        __syncthreads();
        if (warp == 0) {
          const int v = (lane < kWarps) ? sh.red_i[lane] : 0;
          int incl = v;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          if (lane < kWarps) sh.red_i[lane] = incl - v;
          if (lane == 31) sh.bc[3] = incl;
        }
        __syncthreads();
        const int rank = taken + sh.red_i[warp] + __popc(m & ((1u << lane) - 1u));
        if (is && rank < need3) {
          const int pos = atomicAdd(&sh.cnt[0], 1);
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
  for (int i = tid; i < K; i += blockDim.x) lst[i] = entry_of(sbuf[i]);
}

template <bool STAGED>
__device__ void row_lists(const ExpandParams& p, const float* src, bool vec, int V, int K, int P, float M, float sc,
                          uint64_t* sbuf, uint64_t* cbuf, const uint64_t* coll, int ncoll, int bcoll, ListEntry* lst,
                          ExpandShared& sh) {
  const int tid = threadIdx.x;
  int b1, before, maxc;
  boundary_scan(sh.hist, sh.boff, sh.bfill, K, &b1, &before, &maxc, sh);
  const int n1 = static_cast<int>(sh.hist[b1]);
  const int need = K - before;
  if (maxc > kRankMax || n1 > kCandCap) {
    row_list_sorted<STAGED>(p, src, vec, V, K, P, M, sc, b1, before, sbuf, cbuf, lst, sh);
    return;
  }
  // scatter: the bins above the boundary bin by bin into sbuf (unordered
  // inside a bin), the boundary bin's members into cbuf -- from the
  // elements collected in the first pass when they hold every bin up to
  // the boundary, else from the row
  if (tid == 0) sh.cnt[1] = 0;
  __syncthreads();
  if (b1 <= bcoll && ncoll <= kCollCap) {
    for (int i = tid; i < ncoll; i += blockDim.x) {
      const uint64_t v = coll[i];
      const int bin = vbin(key_f32(~static_cast<uint32_t>(v >> 32)), M, sc);
      if (bin < b1) {
        sbuf[sh.boff[bin] + atomicAdd(&sh.bfill[bin], 1u)] = v;
      } else if (bin == b1) {
        const int c = atomicAdd(&sh.cnt[1], 1);
        if (c < kCandCap) cbuf[c] = v;
      }
    }
  } else if (STAGED) {
    smem_pass(src, V, [&](int e, float x, bool in) {
      if (!in) return;
      const int bin = vbin(x, M, sc);
      if (bin > b1) return;
      const uint64_t v = (static_cast<uint64_t>(zdesc_key(x)) << 32) | static_cast<uint32_t>(e);
      if (bin < b1) {
        sbuf[sh.boff[bin] + atomicAdd(&sh.bfill[bin], 1u)] = v;
      } else {
        const int c = atomicAdd(&sh.cnt[1], 1);
        if (c < kCandCap) cbuf[c] = v;
      }
    });
  } else {
    global_pass(src, V, vec, [&](int e, float x, bool in) {
      if (!in) return;
      const int bin = vbin(x, M, sc);
      if (bin > b1) return;
      const uint64_t v = (static_cast<uint64_t>(zdesc_key(x)) << 32) | static_cast<uint32_t>(e);
      if (bin < b1) {
        sbuf[sh.boff[bin] + atomicAdd(&sh.bfill[bin], 1u)] = v;
      } else {
        const int c = atomicAdd(&sh.cnt[1], 1);
        if (c < kCandCap) cbuf[c] = v;
      }
    });
  }
  __syncthreads();
  // every element of a bin above the boundary: its place is the bin's
  // offset plus the number of the bin's members ahead of it (keys are
  // unique: the token is part of the key)
  for (int i = tid; i < before; i += blockDim.x) {
    const uint64_t v = sbuf[i];
    const int bin = vbin(key_f32(~static_cast<uint32_t>(v >> 32)), M, sc);
    const int st = static_cast<int>(sh.boff[bin]), c = static_cast<int>(sh.hist[bin]);
    int rank = 0;
    for (int j = st; j < st + c; ++j) rank += (sbuf[j] < v) ? 1 : 0;
    lst[st + rank] = entry_of(v);
  }
  // the boundary bin: its `need` best members, in order
  if (n1 <= kRankMax) {
    for (int i = tid; i < n1; i += blockDim.x) {
      const uint64_t v = cbuf[i];
      int rank = 0;
      for (int j = 0; j < n1; ++j) rank += (cbuf[j] < v) ? 1 : 0;
      if (rank < need) lst[before + rank] = entry_of(v);
    }
  } else {
    const int Pc = 1 << (32 - __clz(n1 - 1 | 1));
    for (int i = n1 + tid; i < Pc; i += blockDim.x) cbuf[i] = ~0ull;
    __syncthreads();
    bitonic_sort_u64(cbuf, Pc);
    for (int i = tid; i < need; i += blockDim.x) lst[before + i] = entry_of(cbuf[i]);
  }
}

// Row r of the call: consume the row of node row_node[r] into the node's
// sorted list.  Every return is uniform across the CTA.
__device__ void row_body(const ExpandParams& p, int r, unsigned char* dsm, ExpandShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int V = p.V;
  const float* row = p.logits + static_cast<int64_t>(r) * p.ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  const bool staged = p.stage != 0;
  float* srow = reinterpret_cast<float*>(dsm);
  const int nchunks = (V + kChunkFloats - 1) / kChunkFloats;
  const int nbytes = (V * 4) & ~15;                  // bulk-copied part of a staged row
  const int ncopy = (nbytes + kChunkBytes - 1) / kChunkBytes;

  // a staged row is copied at once, in chunks, before the row is checked
  // (the copies overlap those checks); the passes below take each chunk as
  // it lands
  int issued = 0;                                    // thread 0's count of copies issued
  if (staged && tid == 0) {
    sh.abort = 0;
    for (int c = 0; c < ncopy; ++c) tc::mbar_init(&sh.bar[c], 1);
    tc::mbar_init(&sh.lost_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    for (; issued < ncopy; ++issued) {
      const int b = min(kChunkBytes, nbytes - issued * kChunkBytes);
      tc::mbar_expect_tx(&sh.bar[issued], static_cast<uint32_t>(b));
      tc::bulk_g2s(tc::smem_u32(srow + issued * kChunkFloats), row + issued * kChunkFloats,
                   static_cast<uint32_t>(b), &sh.bar[issued]);
    }
  }
  // a row that is dropped before its passes: its copies land first
  auto leave = [&]() {
    if (tid == 0)
      for (int c = 0; c < issued; ++c) tc::mbar_drain(&sh.bar[c], 0);
    __syncthreads();
  };
  const int node = p.row_node[r];
  if (node < 0) { leave(); return; }
  const int n0 = *p.n_nodes;
  if (node >= n0) {
    if (tid == 0) set_status(p.status, TV_DEV_BAD_ROW);
    leave();
    return;
  }
  if (tid == 0) sh.flag = atomicExch(&p.meta[node].expanded, 1);
  __syncthreads();
  const int was = sh.flag;
  __syncthreads();
  if (was != 0) {
    if (tid == 0) set_status(p.status, TV_DEV_BAD_ROW);
    leave();
    return;
  }
  // best-first: every candidate that can still be taken; beam: this call
  // takes at most Bsel, and its lists are not used later
  const int K = p.beam ? min(min(V, p.Bsel), p.budget - n0) : min(V, p.budget - n0);
  if (K <= 0) { leave(); return; }
  const int P = 1 << (32 - __clz(K - 1 | 1));      // next power of two >= K (>= 2)
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(dsm + (staged ? p.stage_bytes : 0));
  uint64_t* cbuf = sbuf + P;                         // boundary-bin candidates
  uint64_t* coll = cbuf + kCandCap;                  // likely top-K members
  const double invtau = 1.0 / static_cast<double>(p.tau);
  if (staged) {
    const int tail0 = nbytes / 4;                    // the last V % 4 elements: plain loads
    if (tid < V - tail0) srow[tail0 + tid] = __ldg(row + tail0 + tid);
  }
  if (tid < 256) sh.etab[tid] = exp2(static_cast<double>(tid) * (1.0 / 256.0));
  for (int i = tid; i < kBins; i += blockDim.x) { sh.hist[i] = 0; sh.boff[i] = 0; }
  if (tid == 0) sh.cnt[2] = 0;
  __syncthreads();

  // a copy that did not land in time: wait (bounded) for every copy issued,
  // then drop the row
  auto give_up = [&]() {
    if (tid == 0) {
      for (int c = 0; c < issued; ++c) tc::mbar_drain(&sh.bar[c], 0);
      set_status(p.status, TV_DEV_TIMEOUT);
    }
    __syncthreads();
  };
  bool ok = true;

  // every lane waits for a staged chunk itself (measured faster than one
  // lane per warp followed by a warp barrier)
  const uint32_t lost = g_row_wait_polls;
  auto wait_chunk = [&](int c) {
    bool w = true;
    if (lane == 0 || lost == 0u) {
      if (c == 0 && lost != 0u) {
        // the test hook: the first phase of a barrier nothing arrives on
        w = false;
        for (uint32_t it = 0; it < lost && !w; ++it) w = tc::mbar_test(&sh.lost_bar, 0);
        if (!w) sh.abort = 1;
      } else {
        w = tc::mbar_wait(&sh.bar[c], 0, &sh.abort);
      }
    }
    return __all_sync(0xffffffffu, w);
  };

  // the histogram frame: maximum and minimum of the first chunk
  // (later elements outside it share the first or the last bin)
  float4 f0;
  if (staged) {
    if (ncopy > 0) ok = wait_chunk(0);
    f0 = smem4(srow, 4 * tid, V);
  } else {
    f0 = load4(row, 4 * tid, V, vec, 0.f);
  }
  const float x0[4] = {f0.x, f0.y, f0.z, f0.w};
  {
    float hi = -INFINITY, lo = INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (4 * tid + k < V && isfinite(x0[k])) { hi = fmaxf(hi, x0[k]); lo = fminf(lo, x0[k]); }
    hi = warp_max(hi);
    lo = warp_min_f(lo);
    if (lane == 0) { sh.red_f[warp] = hi; sh.red_g[warp] = lo; }
  }
  if (__syncthreads_or(ok ? 0 : 1)) { give_up(); return; }
  float top = -INFINITY, bot = INFINITY;
  for (int w = 0; w < kWarps; ++w) { top = fmaxf(top, sh.red_f[w]); bot = fminf(bot, sh.red_g[w]); }
  const float range = top - bot;
  const float sc = (range > 0.f && isfinite(range)) ? 2047.f / range : 0.f;
  // the bin bcoll holding about the (1.5 K n0 / V)-th largest of those n0
  // elements: the first pass collects every element binned at or above it
  // (about 1.5 K elements), which then holds the top K unless the first
  // elements misrepresent the row
  const int n0c = min(V, kChunkFloats);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (4 * tid + k < V) atomicAdd(&sh.boff[vbin(x0[k], top, sc)], 1u);
  __syncthreads();
  int bcoll = -1, bbef;
  {
    const long long want = (3ll * K * n0c + 2ll * V - 1) / (2ll * V) + 8;
    const int r0 = want < n0c ? static_cast<int>(want) : n0c;
    find_rank_bin(sh.boff, kBins, r0, &bcoll, &bbef, sh);
  }

  // pass 1 (a staged row chunk by chunk as its copy lands): finiteness, the
  // row maximum, the histogram of value bins and the collection (one slot
  // claim per warp and step)
  bool bad = false;
  float lm = -INFINITY;
  auto p1 = [&](int e0, float4 v) {
    const float xs[4] = {v.x, v.y, v.z, v.w};
    int nt = 0;
    unsigned tk = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool in = e0 + k < V;
      if (in) {
        if (isfinite(xs[k])) lm = fmaxf(lm, xs[k]);
        else bad = true;
      }
      const int bin = in ? vbin(xs[k], top, sc) : kBins;
      if (in) atomicAdd(&sh.hist[bin], 1u);
      if (bin <= bcoll) { tk |= 1u << k; ++nt; }
    }
    int incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int wtot = __shfl_sync(0xffffffffu, incl, 31);
    int base = 0;
    if (lane == 0 && wtot > 0) base = atomicAdd(&sh.cnt[2], wtot);
    base = __shfl_sync(0xffffffffu, base, 0) + incl - nt;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (tk & (1u << k)) {
        if (base < kCollCap)
          coll[base] = (static_cast<uint64_t>(zdesc_key(xs[k])) << 32) | static_cast<uint32_t>(e0 + k);
        ++base;
      }
  };
  if (staged) {
    for (int c = 0; c < nchunks; ++c) {
      if (c < ncopy && ok) ok = wait_chunk(c);
      const int e0 = c * kChunkFloats + 4 * tid;
      p1(e0, smem4(srow, e0, V));
    }
    if (__syncthreads_or(ok ? 0 : 1)) { give_up(); return; }
  } else {
    const int per = 4 * static_cast<int>(blockDim.x);
    for (int b = 0; b < V; b += per) p1(b + 4 * tid, load4(row, b + 4 * tid, V, vec, 0.f));
  }
  const int any_bad = __syncthreads_or(bad ? 1 : 0);
  if (any_bad) {
    if (tid == 0) set_status(p.status, TV_DEV_NONFINITE);
    return;
  }
  {
    const float wm = warp_max(lm);
    if (lane == 0) sh.red_f[warp] = wm;
  }
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh.red_f[w]);
  const double md = static_cast<double>(M);

  // pass 2: the sum of e^((x - M)/tau) (independent exponentials)
  const double* T = sh.etab;
  double ls = 0.0;
  auto p2 = [&](int e0, float4 v) {
    const float xs[4] = {v.x, v.y, v.z, v.w};
    double e[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      e[k] = e0 + k < V ? exp_neg((static_cast<double>(xs[k]) - md) * invtau, T) : 0.0;
    ls += (e[0] + e[1]) + (e[2] + e[3]);
  };
  {
    const int per = 4 * static_cast<int>(blockDim.x);
    for (int b = 0; b < V; b += per)
      p2(b + 4 * tid, staged ? smem4(srow, b + 4 * tid, V) : load4(row, b + 4 * tid, V, vec, 0.f));
  }
  ls = warp_sum(ls);
  if (lane == 0) sh.red_d[warp] = ls;
  __syncthreads();
  if (warp == 0) {
    double t = lane < kWarps ? sh.red_d[lane] : 0.0;
    t = warp_sum(t);
    if (lane == 0) sh.bcd[0] = t;
  }
  __syncthreads();
  const double lse = static_cast<double>(M) * invtau + log(sh.bcd[0]);

  ListEntry* lst = p.lists + static_cast<int64_t>(node) * p.kcap;
  const int ncoll = sh.cnt[2];
  if (staged) row_lists<true>(p, srow, vec, V, K, P, top, sc, sbuf, cbuf, coll, ncoll, bcoll, lst, sh);
  else row_lists<false>(p, row, vec, V, K, P, top, sc, sbuf, cbuf, coll, ncoll, bcoll, lst, sh);
  if (tid == 0) {
    NodeMeta m;
    m.len = K;
    m.cursor = 0;
    m.expanded = 1;
    m.stamp = __ldcg(&p.header->calls) + 1;
    m.lse = lse;
    // the list's first entry is the row maximum
    m.head = sdesc_key(entry_score(__ldcg(&p.logp[node]), M, p.tau, lse));
    p.meta[node] = m;
  }
}

// ------------------------------------------------------------ merge

// A slot per flagged lane of the warp (one shared atomic per warp); every
// lane of the warp calls it.  -1 for lanes not flagged.
__device__ __forceinline__ int warp_claim(bool take, int* count) {
  const int lane = threadIdx.x & 31;
  const unsigned m = __ballot_sync(0xffffffffu, take);
  int off = 0;
  if (lane == 0 && m != 0u) off = atomicAdd(count, __popc(m));
  off = __shfl_sync(0xffffffffu, off, 0);
  return take ? off + __popc(m & ((1u << lane) - 1u)) : -1;
}

__device__ __forceinline__ bool comp_le(uint64_t a, uint32_t b, uint64_t ta, uint32_t tb) {
  return a < ta || (a == ta && b <= tb);
}
__device__ __forceinline__ bool comp_lt(uint64_t a, uint32_t b, uint64_t ta, uint32_t tb) {
  return a < ta || (a == ta && b < tb);
}

// The head of node nd's list (false when the list is used up or, in beam
// mode, not this call's).
__device__ __forceinline__ bool list_head(const ExpandParams& p, int h, int n0, int stamp, uint64_t* a,
                                          uint32_t* b) {
  int nd = h;
  if (p.beam) {
    nd = p.row_node[h];
    if (nd < 0 || nd >= n0 || __ldcg(&p.meta[nd].stamp) != stamp) return false;
    for (int h2 = 0; h2 < h; ++h2)
      if (p.row_node[h2] == nd) return false;
  }
  const int len = __ldcg(&p.meta[nd].len);
  const int cur = __ldcg(&p.meta[nd].cursor);
  if (cur >= len) return false;
  const ListEntry e = load_entry(p.lists + static_cast<int64_t>(nd) * p.kcap + cur);
  *a = sdesc_key(entry_score(__ldcg(&p.logp[nd]), e.z, p.tau, __ldcg(&p.meta[nd].lse)));
  *b = (static_cast<uint32_t>(nd) << 18) | static_cast<uint32_t>(e.tok);
  return true;
}

// rank-th smallest (1-based) composite (A, B) among N entries in smem.
__device__ void radix_select_ab(const uint64_t* A, const uint32_t* Bk, int N, int rank, uint64_t* thA,
                                uint32_t* thB, ExpandShared& sh) {
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
        const uint32_t dg = pass < 8 ? static_cast<uint32_t>(A[i] >> shA) & 255u : (Bk[i] >> shB) & 255u;
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

// Threshold path of one sub-step: the s best candidates of the union into
// sh.selA/selB (unordered); returns their number, or -1 when a bound leaves
// more candidates than it handles.
__device__ int merge_select_fast(const ExpandParams& p, unsigned char* dsm, ExpandShared& sh, int n0, int stamp,
                                 int s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* hA = reinterpret_cast<uint64_t*>(dsm);                 // head keys
  int* hN = reinterpret_cast<int*>(hA + kHeadCap);                 // their nodes
  uint64_t* cA = reinterpret_cast<uint64_t*>(hN + kHeadCap);       // candidates
  uint32_t* cB = reinterpret_cast<uint32_t*>(cA + kFastCap);
  int* cP = reinterpret_cast<int*>(cB + kFastCap);                 // list slot << 13 | position
  double* qLse = reinterpret_cast<double*>(cP + kFastCap);         // lists that can contribute
  double* qLp = qLse + kQCap;
  int* qN = reinterpret_cast<int*>(qLp + kQCap);
  int* qLen = qN + kQCap;
  int* qCur = qLen + kQCap;
  int* act = qCur + kQCap;                                         // lists still open, two buffers
  const int nh = p.beam ? p.R : n0;
  if (nh > kHeadCap) return -1;
  // 1. the cached head of every list with entries left
  if (tid == 0) { sh.cnt[0] = 0; sh.kmin = ~0ull; sh.kmax = 0ull; sh.kthr = 0ull; }
  __syncthreads();
  uint64_t kmin = ~0ull, kmax = 0ull;
  for (int base = 0; base < nh; base += blockDim.x) {
    const int h = base + tid;
    int nd = h;
    bool ok = h < nh;
    if (ok && p.beam) {
      nd = p.row_node[h];
      ok = nd >= 0 && nd < n0 && __ldcg(&p.meta[nd].stamp) == stamp;
      for (int h2 = 0; ok && h2 < h; ++h2) ok = p.row_node[h2] != nd;
    }
    const uint64_t a = ok ? __ldcg(reinterpret_cast<const unsigned long long*>(&p.meta[nd].head)) : ~0ull;
    const int i = warp_claim(a != ~0ull, &sh.cnt[0]);
    if (i >= 0) {
      hA[i] = a;
      hN[i] = nd;
      kmin = a < kmin ? a : kmin;
      kmax = a > kmax ? a : kmax;
    }
  }
  kmin = warp_min_u64(kmin);
  kmax = warp_max_u64(kmax);
  if (lane == 0) { atomicMin(&sh.kmin, kmin); atomicMax(&sh.kmax, kmax); }
  __syncthreads();
  const int H = sh.cnt[0];
  if (H == 0) return 0;
  // 2. bound: with more than s heads, the worst head among the bins holding
  //    the s best heads (every candidate that can win is at least as good);
  //    with fewer, the s-th best of the first ceil(s / H) entries of every
  //    list (any s candidates bound the s-th best from below)
  uint64_t tA = ~0ull;
  if (H <= s) {
    const int m = (s + H - 1) / H;
    if (tid == 0) { sh.cnt[1] = 0; sh.kthr = ~0ull; }
    __syncthreads();
    for (int hi = warp; hi < H; hi += kWarps) {
      const int nd = hN[hi];
      const int len = __ldcg(&p.meta[nd].len);
      const int cur = __ldcg(&p.meta[nd].cursor);
      const double lse = __ldcg(&p.meta[nd].lse);
      const double lp = __ldcg(&p.logp[nd]);
      const ListEntry* lst = p.lists + static_cast<int64_t>(nd) * p.kcap;
      for (int base = 0; base < m; base += 32) {
        const int pos = cur + base + lane;
        if (base + lane < m && pos < len) {
          const ListEntry e = load_entry(lst + pos);
          const int k = atomicAdd(&sh.cnt[1], 1);
          cA[k] = sdesc_key(entry_score(lp, e.z, p.tau, lse));     // k < H * m < 2 s
        }
      }
    }
    __syncthreads();
    const int ns = sh.cnt[1];
    if (ns >= s) {
      // the s-th smallest key: the smallest key with at least s keys <= it
      for (int i = tid; i < ns; i += blockDim.x) {
        const uint64_t a = cA[i];
        int le = 0;
        for (int j = 0; j < ns; ++j) le += (cA[j] <= a) ? 1 : 0;
        if (le >= s) atomicMin(&sh.kthr, a);
      }
      __syncthreads();
      tA = sh.kthr;
    }
    __syncthreads();
  } else {
    const double best = sdesc_val(sh.kmin), worst = sdesc_val(sh.kmax);
    const double scale = best > worst ? 2047.0 / (best - worst) : 0.0;
    for (int i = tid; i < kBins; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < H; i += blockDim.x) atomicAdd(&sh.hist[sbin(sdesc_val(hA[i]), best, scale)], 1u);
    __syncthreads();
    int hb, hbef, hmx;
    boundary_scan(sh.hist, sh.boff, sh.bfill, s, &hb, &hbef, &hmx, sh);
    uint64_t t = 0ull;
    for (int i = tid; i < H; i += blockDim.x)
      if (sbin(sdesc_val(hA[i]), best, scale) <= hb) t = hA[i] > t ? hA[i] : t;
    t = warp_max_u64(t);
    if (lane == 0) atomicMax(&sh.kthr, t);
    __syncthreads();
    tA = sh.kthr;
  }
  // 3. the lists that can contribute (head within the bound) with their
  //    metadata, one thread per list
  if (tid == 0) { sh.cnt[1] = 0; sh.cnt[2] = 0; sh.kmin = ~0ull; sh.kmax = 0ull; }
  __syncthreads();
  for (int base = 0; base < H; base += blockDim.x) {
    const int i = base + tid;
    const int q = warp_claim(i < H && hA[i] <= tA, &sh.cnt[2]);
    if (q >= 0 && q < kQCap) qN[q] = hN[i];
  }
  __syncthreads();
  const int Q = sh.cnt[2];
  if (Q > kQCap) return -1;
  for (int q = tid; q < Q; q += blockDim.x) {
    const int nd = qN[q];
    qLen[q] = __ldcg(&p.meta[nd].len);
    qCur[q] = __ldcg(&p.meta[nd].cursor);
    qLse[q] = __ldcg(&p.meta[nd].lse);
    qLp[q] = __ldcg(&p.logp[nd]);
    act[q] = q;
  }
  __syncthreads();
  // 4. gather every list entry at least as good as the bound, 32 positions
  //    of each open list per round (<= s per list: a list's (s+1)-th entry
  //    is beaten by its first s); a warp takes four lists at a time with
  //    their loads in flight together; a list stays open while all 32 pass
  uint64_t cmin = ~0ull, cmax = 0ull;
  int nact = Q;
  int* cur_act = act;
  int* nxt_act = act + kQCap;
  for (int rb = 0; rb * 32 < s && nact > 0; ++rb) {
    if (tid == 0) sh.cnt[3] = 0;
    __syncthreads();
    for (int a0 = warp; a0 < nact; a0 += 4 * kWarps) {
      ListEntry e[4];
      bool v[4];
      int ql[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ai = a0 + u * kWarps;
        ql[u] = ai < nact ? cur_act[ai] : -1;
        v[u] = false;
        if (ql[u] >= 0) {
          const int q = ql[u];
          const int pos = qCur[q] + rb * 32 + lane;
          v[u] = rb * 32 + lane < s && pos < qLen[q];
          if (v[u]) e[u] = load_entry(p.lists + static_cast<int64_t>(qN[q]) * p.kcap + pos);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (ql[u] < 0) continue;                      // warp-uniform
        const int q = ql[u];
        uint64_t a = ~0ull;
        uint32_t b = 0u;
        bool ok = v[u];
        if (ok) {
          a = sdesc_key(entry_score(qLp[q], e[u].z, p.tau, qLse[q]));
          b = (static_cast<uint32_t>(qN[q]) << 18) | static_cast<uint32_t>(e[u].tok);
          ok = a <= tA;
        }
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        const int c = __popc(m);
        int off = 0;
        if (lane == 0 && c > 0) off = atomicAdd(&sh.cnt[1], c);
        off = __shfl_sync(0xffffffffu, off, 0);
        if (ok) {
          const int k = off + __popc(m & ((1u << lane) - 1u));
          if (k < kFastCap) { cA[k] = a; cB[k] = b; cP[k] = (q << 13) | (qCur[q] + rb * 32 + lane); }
          cmin = a < cmin ? a : cmin;
          cmax = a > cmax ? a : cmax;
        }
        if (c == 32 && lane == 0) nxt_act[atomicAdd(&sh.cnt[3], 1)] = q;
      }
    }
    __syncthreads();
    nact = sh.cnt[3];
    int* t = cur_act;
    cur_act = nxt_act;
    nxt_act = t;
  }
  cmin = warp_min_u64(cmin);
  cmax = warp_max_u64(cmax);
  if (lane == 0) { atomicMin(&sh.kmin, cmin); atomicMax(&sh.kmax, cmax); }
  __syncthreads();
  const int C = sh.cnt[1];
  if (C > kFastCap) return -1;
  // 5. the s best of the C: bins of their scores, then exact ranks inside
  //    the boundary bin
  if (C <= s) {
    for (int i = tid; i < C; i += blockDim.x) { sh.selA[i] = cA[i]; sh.selB[i] = cB[i]; sh.selP[i] = cP[i]; }
    __syncthreads();
    return C;
  }
  const double best = sdesc_val(sh.kmin), worst = sdesc_val(sh.kmax);
  const double scale = best > worst ? 2047.0 / (best - worst) : 0.0;
  for (int i = tid; i < kBins; i += blockDim.x) sh.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < C; i += blockDim.x) atomicAdd(&sh.hist[sbin(sdesc_val(cA[i]), best, scale)], 1u);
  __syncthreads();
  int hc, cbef, cmx;
  boundary_scan(sh.hist, sh.boff, sh.bfill, s, &hc, &cbef, &cmx, sh);
  const int nb = static_cast<int>(sh.hist[hc]);
  if (nb > kRankMax) return -1;
  if (tid == 0) { sh.cnt[2] = 0; sh.cnt[3] = 0; }
  __syncthreads();
  uint64_t* bA = hA;           // the heads are no longer needed
  uint32_t* bB = reinterpret_cast<uint32_t*>(hN);
  int* bP = hN + kHeadCap / 2;
  for (int base = 0; base < C; base += blockDim.x) {
    const int i = base + tid;
    const int bn = i < C ? sbin(sdesc_val(cA[i]), best, scale) : kBins;
    const int k = warp_claim(bn < hc, &sh.cnt[2]);
    const int kb = warp_claim(bn == hc, &sh.cnt[3]);
    if (k >= 0) {
      sh.selA[k] = cA[i];
      sh.selB[k] = cB[i];
      sh.selP[k] = cP[i];
    } else if (kb >= 0) {
      bA[kb] = cA[i];
      bB[kb] = cB[i];
      bP[kb] = cP[i];
    }
  }
  __syncthreads();
  const int take = s - cbef;
  for (int i = tid; i < nb; i += blockDim.x) {
    const uint64_t a = bA[i];
    const uint32_t b = bB[i];
    int rank = 0;
    for (int j = 0; j < nb; ++j) rank += comp_lt(bA[j], bB[j], a, b) ? 1 : 0;
    if (rank < take) {
      sh.selA[cbef + rank] = a;
      sh.selB[cbef + rank] = b;
      sh.selP[cbef + rank] = bP[i];
    }
  }
  __syncthreads();
  return s;
}

// Radix fallback of one sub-step (any bound): the s best heads, then <= s
// entries of each of their lists, then a radix select of the s best.
__device__ int merge_select_radix(const ExpandParams& p, unsigned char* dsm, ExpandShared& sh, int n0, int stamp,
                                  int s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* A = reinterpret_cast<uint64_t*>(dsm);
  uint32_t* Bk = reinterpret_cast<uint32_t*>(A + kMergeCap);
  if (tid == 0) { sh.cnt[0] = 0; sh.cnt[1] = 0; sh.cnt[2] = 0; sh.cnt[3] = 0; }
  __syncthreads();
  const int nh = p.beam ? p.R : n0;
  for (int h = tid; h < nh; h += blockDim.x) {
    uint64_t a;
    uint32_t b;
    if (list_head(p, h, n0, stamp, &a, &b)) {
      const int i = atomicAdd(&sh.cnt[0], 1);
      if (i < kMergeCap) { A[i] = a; Bk[i] = b; }
    }
  }
  __syncthreads();
  const int H = min(sh.cnt[0], kMergeCap);
  if (H == 0) return 0;
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
  for (int qi = warp; qi < Q; qi += kWarps) {
    const int nd = sh.qlist[qi];
    const int len = __ldcg(&p.meta[nd].len);
    const int cur = __ldcg(&p.meta[nd].cursor);
    const double lse = __ldcg(&p.meta[nd].lse);
    const double lp = __ldcg(&p.logp[nd]);
    const ListEntry* lst = p.lists + static_cast<int64_t>(nd) * p.kcap;
    for (int base = 0; base < s; base += 32) {
      const int pos = cur + base + lane;
      bool ok = (base + lane < s) && pos < len;
      uint64_t a = 0;
      uint32_t bb = 0;
      if (ok) {
        const ListEntry e = load_entry(lst + pos);
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
  __syncthreads();
  return S;
}

__device__ void merge_body(const ExpandParams& p, unsigned char* dsm, ExpandShared& sh) {
  const int tid = threadIdx.x;
  const int n0 = __ldcg(p.n_nodes);
  const int rem = p.budget - n0;
  const int total = rem > 0 ? min(p.Bsel, rem) : 0;
  const int stamp = __ldcg(&p.header->calls) + 1;    // this call's number
  int appended = 0;
  while (appended < total) {
    const int s = min(kMergeStep, total - appended);
    int S = merge_select_fast(p, dsm, sh, n0, stamp, s);
    const bool haveP = S >= 0;               // winners carry their list slot and position
    __syncthreads();
    if (S < 0) S = merge_select_radix(p, dsm, sh, n0, stamp, s);
    if (S == 0) break;
    // order the winners by (score desc, parent asc, token asc): each one's
    // place is the number of winners ahead of it, counted by eight threads
    for (int i0 = 0; i0 < S; i0 += kThreads / 8) {
      const int i = i0 + (tid >> 3), part = tid & 7;
      int rank = 0;
      uint64_t a = 0;
      uint32_t b = 0;
      if (i < S) {
        a = sh.selA[i];
        b = sh.selB[i];
        for (int j = part; j < S; j += 8) rank += comp_lt(sh.selA[j], sh.selB[j], a, b) ? 1 : 0;
      }
      rank += __shfl_xor_sync(0xffffffffu, rank, 1);
      rank += __shfl_xor_sync(0xffffffffu, rank, 2);
      rank += __shfl_xor_sync(0xffffffffu, rank, 4);
      if (i < S && part == 0) {
        sh.ordA[rank] = a;
        sh.ordB[rank] = b;
        sh.ordP[rank] = haveP ? sh.selP[i] : -1;
      }
    }
    __syncthreads();
    // append in rank order; the last winner of each source list advances
    // the list's cursor past its winners and refreshes the cached head
    if (tid < S) {
      const int node = n0 + appended + tid;
      const int nd = static_cast<int>(sh.ordB[tid] >> 18);
      p.parent[node] = nd;
      p.token[node] = static_cast<int32_t>(sh.ordB[tid] & 0x3FFFFu);
      p.logp[node] = sdesc_val(sh.ordA[tid]);
      p.frontier[appended + tid] = node;
      int taken = 0;
      bool last = true;
      for (int j = 0; j < S; ++j)
        if (static_cast<int>(sh.ordB[j] >> 18) == nd) {
          ++taken;
          if (j > tid) last = false;
        }
      if (last) {
        // the threshold path knows the winner's list slot (its length, lse
        // and parent log-probability are in shared memory) and position
        const int pp = sh.ordP[tid];
        int cur, len;
        double lse, lp;
        if (pp >= 0) {
          const double* qLse = reinterpret_cast<const double*>(dsm + kQMetaOff);
          const int q = pp >> 13;
          cur = (pp & 0x1FFF) + 1;
          len = reinterpret_cast<const int*>(qLse + 2 * kQCap)[kQCap + q];
          lse = qLse[q];
          lp = qLse[kQCap + q];
        } else {
          cur = __ldcg(&p.meta[nd].cursor) + taken;
          len = __ldcg(&p.meta[nd].len);
          lse = __ldcg(&p.meta[nd].lse);
          lp = __ldcg(&p.logp[nd]);
        }
        uint64_t head = ~0ull;
        if (cur < len) {
          const ListEntry e = load_entry(p.lists + static_cast<int64_t>(nd) * p.kcap + cur);
          head = sdesc_key(entry_score(lp, e.z, p.tau, lse));
        }
        p.meta[nd].cursor = cur;
        p.meta[nd].head = head;
      }
    }
    if (appended + S < total && S == s) __threadfence();   // another sub-step reads them
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

// ------------------------------------------------------------ kernels

__global__ void __launch_bounds__(kThreads, 1)
expand_round_kernel(ExpandParams p) {
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ ExpandShared sh;
  row_body(p, blockIdx.x, dsm, sh);
  // the last CTA to finish its row runs the merge (the CTA's writes are
  // ordered before the ticket by the barrier and thread 0's fence)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int t = atomicAdd(&p.header->rows_done, 1);
    sh.last = (t == static_cast<int>(gridDim.x) - 1) ? 1 : 0;
    if (sh.last) {
      __threadfence();
      p.header->rows_done = 0;
    }
  }
  __syncthreads();
  if (!sh.last) return;
  merge_body(p, dsm, sh);
}

__global__ void __launch_bounds__(kThreads, 1)
expand_merge_kernel(ExpandParams p) {
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ ExpandShared sh;
  merge_body(p, dsm, sh);
}

__global__ void expand_init_kernel(ExpandParams p, int root_token) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < p.budget) {
    NodeMeta m;
    m.len = 0; m.cursor = 0; m.expanded = 0; m.stamp = 0; m.lse = 0.0; m.head = ~0ull;
    p.meta[i] = m;
  }
  if (i == 0) {
    p.header->calls = 0;
    p.header->rows_done = 0;
    *p.n_nodes = 1;
    p.parent[0] = -1;
    p.token[0] = root_token;
    p.logp[0] = 0.0;
  }
}

__global__ void expand_exp_kernel(const double* t, double* out, int n) {
  __shared__ double T[256];
  for (int j = threadIdx.x; j < 256; j += blockDim.x) T[j] = exp2(static_cast<double>(j) * (1.0 / 256.0));
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = exp_neg(t[i], T);
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
  p.stage = 0;
  p.stage_bytes = 0;
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

cudaError_t expand_set_wait_limit(uint32_t polls) {
  return cudaMemcpyToSymbol(g_row_wait_polls, &polls, sizeof(polls));
}

cudaError_t launch_expand_exp(const double* t, double* out, int n, cudaStream_t stream) {
  expand_exp_kernel<<<(n + 255) / 256, 256, 0, stream>>>(t, out, n);
  return cudaGetLastError();
}

cudaError_t launch_expand_init(const tv_expand_args* a, int root_token, cudaStream_t stream) {
  ExpandParams p = make_params(a);
  const int threads = 256;
  expand_init_kernel<<<(a->budget + threads - 1) / threads, threads, 0, stream>>>(p, root_token);
  return cudaGetLastError();
}

cudaError_t launch_expand(const tv_expand_args* a, cudaStream_t stream) {
  ExpandParams p = make_params(a);
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (a->R > 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, expand_round_kernel);
    if (e != cudaSuccess) return e;
    const size_t maxdyn = static_cast<size_t>(optin) - fa.sharedSizeBytes;
    const int K = static_cast<int>(p.kcap);
    int P = 2;
    while (P < K) P <<= 1;
    const size_t lists = (static_cast<size_t>(P) + kCandCap + kCollCap) * sizeof(uint64_t);
    const size_t row_bytes = (static_cast<size_t>(a->V) * 4 + 15) & ~static_cast<size_t>(15);
    const bool aligned = (reinterpret_cast<uintptr_t>(a->draft_logits) & 15u) == 0 && (a->ld_logits % 4) == 0;
    const int ncopy = static_cast<int>((((static_cast<size_t>(a->V) * 4) & ~static_cast<size_t>(15)) +
                                        kChunkBytes - 1) / kChunkBytes);
    if (aligned && ncopy <= kMaxChunks && row_bytes + lists <= maxdyn) {
      p.stage = 1;
      p.stage_bytes = static_cast<int>(row_bytes);
    }
    size_t smem = (p.stage ? row_bytes : 0) + lists;
    if (smem < kMergeDyn) smem = kMergeDyn;
    if (smem > maxdyn) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(expand_round_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    expand_round_kernel<<<a->R, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(expand_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMergeDyn));
  if (e != cudaSuccess) return e;
  expand_merge_kernel<<<1, kThreads, kMergeDyn, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tv
