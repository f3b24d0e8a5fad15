// tree_accept kernel: per-node decisions over vocabulary rows, then a walk
// from the root along the accepted children.
//
// Acceptance rules (SpecExec page, "Approach" and "Builds on": speculative
// sampling / SpecInfer; greedy longest match at temperature 0):
//   GREEDY      descend to the lowest-index child carrying argmax z_c;
//   SPECSAMPLE  child j accepted when u_j < r(x_j) / q(x_j), r the current
//               (residual) target distribution, r <- (r - q)^+ / sum on
//               rejection, inverse-CDF sample of r when all are rejected;
//   SPECEXEC    x ~ softmax(z_c / tau) by inverse CDF, descend to a child
//               carrying x.
// Every node's decision depends only on its own rows and its own Philox
// draws, so all nodes decide in parallel; the last node of a sequence to
// finish (an atomic ticket, no waiting) walks the decisions from the root.
//
// Layout of a row pass.  A thread-block cluster of C CTAs (C <= 8) owns one
// node row; CTA rank r owns a contiguous slice of 512-element segments.  A
// warp owns a segment at a time, lane l holding elements 128k + 4l ..
// 128k + 4l + 3 (k = 0..3).  Aligned rows are streamed by bulk copies: each
// warp keeps three segments (z and q) in flight in its own shared-memory
// ring; other rows are read with plain loads.  Cross-CTA sums and maxima go
// through distributed shared memory (double-buffered slots, one cluster
// barrier per reduction); every CTA computes the same reduced values and so
// takes the same branches.
//
// Arithmetic.  Every element weight is e_t = 2^(z_t * k - M * k) with
// k = log2(e) / tau and M the row maximum (one FFMA and one ex2.approx), the
// unnormalised softmax.  The first pass keeps, per segment, the maximum m_s
// and the sum of 2^((z - m_s) k); once the per-CTA maxima are gathered, the
// row sum and the segment sums are brought to the frame of M.  Residuals are parametrised as
// r = (p - c q)^+ / D with p = e / s: rejecting a child with the current
// (c, D) gives c' = c + D and D' = sum_t (p_t - c' q_t)^+, one pass.
// Weights are fp32; each lane's four weights are summed in fp32, segment
// sums are fp32 warp reductions and everything above that is fp64.  The
// segment sums are kept in shared memory, so an inverse-CDF sample re-reads
// one segment only.
#include <cooperative_groups.h>

#include <cfloat>
#include <mutex>

#include "tv_common.cuh"

namespace cg = cooperative_groups;

namespace tv {

struct AcceptDec {
  int32_t child;   // accepted child, or -1
  int32_t token;   // bonus token when child == -1; kNonFiniteRow when the
                   // node's rows were not finite (reported only if visited)
  double margin;   // smallest decision margin at this node (+inf if none)
};
constexpr int32_t kNonFiniteRow = -2;

struct AcceptParams {
  int B, T, V;
  const float* z; int64_t z_sb, z_st;
  const float* q; int64_t q_sb, q_st;
  const int32_t* tok; int64_t tok_sb;
  const int32_t* parent; int64_t par_sb;
  const int32_t* n_nodes;
  int mode;                 // resolved: 1 greedy, 2 specsample, 3 specexec
  float tau;
  uint64_t seed, step;
  uint32_t* status;
  AcceptDec* dec;           // [B][T]
  int32_t* ticket;          // [B], zero between calls
  int32_t* n_acc;
  int32_t* acc_nodes;
  int32_t* out_tokens;
  double* min_margin;
  int C;                    // CTAs per row (cluster size)
  int seg_per_cta;          // 512-element segments per CTA
};

constexpr int kAcceptThreads = 256;
constexpr int kAcceptWarps = kAcceptThreads / kWarp;
constexpr int kSeg = 512;               // elements per segment
constexpr int kSub = 128;               // elements of one warp-wide float4 load
constexpr int kMaxSegPerCta = 128;      // 65536 elements per CTA
constexpr int kRing = 3;                // segments in flight per warp (bulk copies)
constexpr uint32_t kSegBytes = kSeg * 4;
constexpr uint32_t kStageBytes = 2 * kSegBytes;               // z then q
constexpr size_t kRingBytes = static_cast<size_t>(kAcceptWarps) * kRing * kStageBytes;   // 96 KB
constexpr uint32_t kRingWait = 1u << 22;

// ------------------------------------------------------------ shared state

struct Slot {            // one CTA's contribution to a cluster reduction
  double a, b;
  float f;
  int i, j;
};

struct AcceptShared {
  double red_d[kAcceptWarps];
  float red_f[kAcceptWarps];
  int red_i[kAcceptWarps];
  int wofs[kAcceptWarps];
  int clist[kAcceptThreads];
  int ctok[kAcceptThreads];     // first window of children: tokens, z and q at them
  float cz[kAcceptThreads];
  float cq[kAcceptThreads];
  int bc_int[4];
  double bc_dbl[4];
  Slot slot[2];
  double cu[kAcceptThreads];    // first window of children: their uniforms
  double rank_tot[8];           // per-CTA totals of the current weights
  float seg_a[kMaxSegPerCta];   // segment sums of the current weights
  float seg_b[kMaxSegPerCta];   // scratch for a residual pass (first pass: segment maxima)
  uint64_t ring_bar[kAcceptWarps * kRing];
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Element weight: e = 2^(z k + zoff) (zoff = -M k), or the residual
// (e * inv_s - c q)^+.
__device__ __forceinline__ float weight(float z, float q, float k, float zoff, float inv_s, float c, bool resid) {
  const float e = ex2_approx(fmaf(z, k, zoff));
  return resid ? fmaxf(fmaf(-c, q, e * inv_s), 0.f) : e;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double block_sum_d(double v, AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh.red_d[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kAcceptWarps; ++w) t += sh.red_d[w];
  return t;
}

__device__ __forceinline__ int block_min_i(int v, AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh.red_i[warp] = v;
  __syncthreads();
  int t = INT_MAX;
#pragma unroll
  for (int w = 0; w < kAcceptWarps; ++w) t = min(t, sh.red_i[w]);
  return t;
}

// Cluster all-gather of one Slot per CTA: after the call every thread of
// every CTA sees the C slots in `out` (rank order).  `k` counts the
// reductions so that consecutive ones use alternate slots.
__device__ __forceinline__ void cluster_gather(cg::cluster_group& cl, AcceptShared& sh, const Slot& mine,
                                               int C, int& k, Slot* out) {
  Slot* s = &sh.slot[k & 1];
  if (threadIdx.x == 0) *s = mine;
  cl.sync();
  for (int r = 0; r < C; ++r) out[r] = *cl.map_shared_rank(s, r);
  ++k;
}

// Lowest-index child of c (c < j < n) that carries token x, or -1.
__device__ int first_child_with_token(const int32_t* par, const int32_t* tok, int c, int n, int x,
                                      AcceptShared& sh) {
  int best = INT_MAX;
  for (int j = c + 1 + threadIdx.x; j < n; j += blockDim.x)
    if (par[j] == c && tok[j] == x) { best = j; break; }
  best = block_min_i(best, sh);
  return best == INT_MAX ? -1 : best;
}

struct Frame {
  float k, zoff, inv_s, c;   // weight parameters
  bool resid;
};

// The four float4 of segment start s0 held by this lane (elements
// s0 + 128k + 4l ..); positions past the row end read `fill`.
__device__ __forceinline__ void load_seg(const float* __restrict__ row, int s0, int V, bool vec, float fill,
                                         float4 (&v)[4]) {
  const int lane = threadIdx.x & 31;
  if (vec && s0 + kSeg <= V) {
    const float4* p = reinterpret_cast<const float4*>(row + s0) + lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __ldg(p + 32 * k);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = load4(row, s0 + k * kSub + 4 * lane, V, vec, fill);
  }
}

// ---------------------------------------------------------- segment streams
// A warp visits its segments s = warp, warp + 8, ... of the CTA's slice in
// order.  When the rows allow it (16-byte aligned rows, V a multiple of 4)
// lane 0 keeps kRing segments in flight with bulk copies into the warp's
// ring in shared memory (one mbarrier per ring stage); otherwise the lanes
// load each segment directly.  The same slice is streamed once per pass.

__device__ __forceinline__ void ring_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void ring_copy(uint32_t dst, const float* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Bounded wait on phase `parity` of a ring barrier; false when it expired.
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_addr(bar);
  for (uint32_t it = 0; it < kRingWait; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

struct SegStream {
  const float* zr;
  const float* qr;
  bool zvec, qvec;      // 16-byte aligned rows (plain loads)
  bool readq;           // stream q as well
  bool bulk;            // bulk copies into the ring
  int V, seg0, nloc;
  uint32_t ring;        // shared address of this warp's ring
  uint64_t* bar;        // this warp's kRing barriers
  uint32_t count;       // segments this warp has streamed (all passes)
  bool dead;            // a ring wait expired: the stream delivers fill values,
                        // and the kernel raises TV_DEV_TIMEOUT before it exits
};

__device__ __forceinline__ void seg_issue(const SegStream& st, int sl, uint32_t stage) {
  const int s0 = (st.seg0 + sl) * kSeg;
  const uint32_t bytes = static_cast<uint32_t>(min(kSeg, st.V - s0)) * 4u;
  uint64_t* bar = st.bar + stage;
  ring_expect(bar, st.readq ? 2u * bytes : bytes);
  ring_copy(st.ring + stage * kStageBytes, st.zr + s0, bytes, bar);
  if (st.readq) ring_copy(st.ring + stage * kStageBytes + kSegBytes, st.qr + s0, bytes, bar);
}

// One pass over the warp's segments: f(sl, s0, z[4], q[4]) per segment
// (sl the segment's index in the slice, s0 its first element; the lane
// holds elements s0 + 128k + 4l ..; past the row end z reads zfill and q 0).
template <class F>
__device__ __forceinline__ void stream_pass(SegStream& st, float zfill, F&& f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ns = warp < st.nloc ? (st.nloc - warp + kAcceptWarps - 1) / kAcceptWarps : 0;
  if (!st.bulk) {
    for (int i = 0; i < ns; ++i) {
      const int sl = warp + i * kAcceptWarps;
      const int s0 = (st.seg0 + sl) * kSeg;
      float4 zv[4], qv[4];
      load_seg(st.zr, s0, st.V, st.zvec, zfill, zv);
      if (st.readq) load_seg(st.qr, s0, st.V, st.qvec, 0.f, qv);
      else {
#pragma unroll
        for (int k = 0; k < 4; ++k) qv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      f(sl, s0, zv, qv);
    }
    return;
  }
  const uint32_t c0 = st.count;
  if (lane == 0 && !st.dead)
    for (int i = 0; i < min(kRing, ns); ++i) seg_issue(st, warp + i * kAcceptWarps, (c0 + i) % kRing);
  for (int i = 0; i < ns; ++i) {
    const uint32_t g = c0 + i, stage = g % kRing;
    const int sl = warp + i * kAcceptWarps;
    const int s0 = (st.seg0 + sl) * kSeg;
    if (!st.dead && !__all_sync(0xffffffffu, ring_wait(st.bar + stage, (g / kRing) & 1))) {
      // expired: issue nothing more, let the copies in flight land (bounded)
      st.dead = true;
      if (lane == 0)
        for (int j = i; j < min(i + kRing, ns); ++j) ring_wait(st.bar + (c0 + j) % kRing, ((c0 + j) / kRing) & 1);
      __syncwarp();
    }
    float4 zv[4], qv[4];
    if (!st.dead) {
      const uint8_t* stg = reinterpret_cast<const uint8_t*>(__cvta_shared_to_generic(st.ring + stage * kStageBytes));
      const float4* z4 = reinterpret_cast<const float4*>(stg) + lane;
      const float4* q4 = reinterpret_cast<const float4*>(stg + kSegBytes) + lane;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        zv[k] = z4[32 * k];
        qv[k] = st.readq ? q4[32 * k] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (s0 + kSeg > st.V) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e0 = s0 + k * kSub + 4 * lane;
          if (e0 + 0 >= st.V) { zv[k].x = zfill; qv[k].x = 0.f; }
          if (e0 + 1 >= st.V) { zv[k].y = zfill; qv[k].y = 0.f; }
          if (e0 + 2 >= st.V) { zv[k].z = zfill; qv[k].z = 0.f; }
          if (e0 + 3 >= st.V) { zv[k].w = zfill; qv[k].w = 0.f; }
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        zv[k] = make_float4(zfill, zfill, zfill, zfill);
        qv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    f(sl, s0, zv, qv);
    __syncwarp();
    if (!st.dead && i + kRing < ns && lane == 0) {
      // the lanes' reads of this stage are done before the copy overwrites it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      seg_issue(st, warp + (i + kRing) * kAcceptWarps, stage);
    }
  }
  st.count = c0 + ns;
}

// One pass over this CTA's slice: segment sums of the current weights into
// seg_out; returns the slice total (fp64).  Past the row end the logits read
// -FLT_MAX, whose weight is 0.
__device__ double weight_pass(SegStream& st, const Frame& f, float* seg_out, AcceptShared& sh) {
  const int lane = threadIdx.x & 31;
  double tot = 0.0;
  stream_pass(st, -FLT_MAX, [&](int sl, int, const float4 (&zv)[4], const float4 (&qv)[4]) {
    float g = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      g += weight(zv[k].x, qv[k].x, f.k, f.zoff, f.inv_s, f.c, f.resid);
      g += weight(zv[k].y, qv[k].y, f.k, f.zoff, f.inv_s, f.c, f.resid);
      g += weight(zv[k].z, qv[k].z, f.k, f.zoff, f.inv_s, f.c, f.resid);
      g += weight(zv[k].w, qv[k].w, f.k, f.zoff, f.inv_s, f.c, f.resid);
    }
    const float ss = warp_sum_f(g);
    if (lane == 0) seg_out[sl] = ss;
    tot += static_cast<double>(ss);
  });
  return block_sum_d(lane == 0 ? tot : 0.0, sh);
}

// Inverse-CDF search inside this CTA's slice (run by warp 0): the first
// element where the running sum, starting at `base`, exceeds `target`.
// Returns t (or the slice's last positive element when rounding leaves the
// crossing past the end) and the relative margin.
__device__ void slice_search(const float* zr, const float* qr, bool zvec, bool qvec, int V, int seg0, int nloc,
                             const float* seg_w, const Frame& f, double base, double target, double W, int* out_t,
                             double* out_margin) {
  const int lane = threadIdx.x & 31;
  const int per = (nloc + 31) / 32;
  const int lo = min(lane * per, nloc), hi = min(lo + per, nloc);
  double ls = 0.0;
  for (int s = lo; s < hi; ++s) ls += static_cast<double>(seg_w[s]);
  const double incl = base + warp_incl_scan(ls);
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = base;
  const unsigned m = __ballot_sync(0xffffffffu, incl > target);
  int seg = -1;
  double cb = 0.0;
  bool found = false;
  if (m != 0u) {
    const int L = __ffs(m) - 1;
    if (lane == L) {
      double cum = excl;
      int s = lo;
      for (; s < hi; ++s) {
        if (cum + static_cast<double>(seg_w[s]) > target) break;
        cum += static_cast<double>(seg_w[s]);
      }
      seg = (s < hi) ? s : hi - 1;
      cb = (s < hi) ? cum : cum - static_cast<double>(seg_w[hi - 1]);
    }
    seg = __shfl_sync(0xffffffffu, seg, L);
    cb = __shfl_sync(0xffffffffu, cb, L);
    found = true;
  } else {
    int last = -1;
    for (int s = lo; s < hi; ++s) if (seg_w[s] > 0.f) last = s;
    const unsigned mm = __ballot_sync(0xffffffffu, last >= 0);
    const int L = mm ? 31 - __clz(mm) : 0;
    seg = __shfl_sync(0xffffffffu, last, L);
    if (seg < 0) seg = 0;
  }
  const int s0 = (seg0 + seg) * kSeg;
  float4 zv[4], qv[4];
  load_seg(zr, s0, V, zvec, -FLT_MAX, zv);
  if (f.resid) load_seg(qr, s0, V, qvec, 0.f, qv);
  else {
#pragma unroll
    for (int k = 0; k < 4; ++k) qv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  int t = -1;
  double margin = 0.0;
  int lastpos = -1;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e0 = s0 + k * kSub + lane * 4;
    double w[4];
    w[0] = weight(zv[k].x, qv[k].x, f.k, f.zoff, f.inv_s, f.c, f.resid);
    w[1] = weight(zv[k].y, qv[k].y, f.k, f.zoff, f.inv_s, f.c, f.resid);
    w[2] = weight(zv[k].z, qv[k].z, f.k, f.zoff, f.inv_s, f.c, f.resid);
    w[3] = weight(zv[k].w, qv[k].w, f.k, f.zoff, f.inv_s, f.c, f.resid);
    for (int e = 0; e < 4; ++e) if (w[e] > 0.0 && e0 + e < V) lastpos = e0 + e;
    if (found && t < 0) {
      const double lsum = ((w[0] + w[1]) + w[2]) + w[3];
      const double li = cb + warp_incl_scan(lsum);
      double le = __shfl_up_sync(0xffffffffu, li, 1);
      if (lane == 0) le = cb;
      const unsigned m2 = __ballot_sync(0xffffffffu, li > target);
      if (m2 != 0u) {
        const int L = __ffs(m2) - 1;
        int tt = -1;
        double mg = 0.0;
        if (lane == L) {
          double cum = le;
          for (int e = 0; e < 4; ++e) {
            if (cum + w[e] > target) {
              tt = e0 + e;
              mg = fmin(cum + w[e] - target, target - cum) / W;
              break;
            }
            cum += w[e];
          }
        }
        t = __shfl_sync(0xffffffffu, tt, L);
        margin = __shfl_sync(0xffffffffu, mg, L);
      }
      cb = __shfl_sync(0xffffffffu, li, 31);
    }
  }
  if (t < 0) {
    // rounding put the crossing past this segment: its last positive element
    const unsigned mm = __ballot_sync(0xffffffffu, lastpos >= 0);
    int best = lastpos;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    t = mm ? best : s0;
    margin = 0.0;
  }
  *out_t = t;
  *out_margin = margin;
}

// ------------------------------------------------------------ the walk

// Called by every thread of one CTA: thread 0 follows the accepted children
// from the root, then the block pads the outputs with -1.  When they fit,
// the sequence's decisions are first copied to `scratch` (shared memory) by
// the whole block, so that the walk's dependent reads stay on chip.
__device__ void accept_walk(const AcceptParams& p, int b, int n, AcceptShared& sh, AcceptDec* scratch,
                            int scratch_cap) {
  const int T = p.T;
  int32_t* acc = p.acc_nodes + static_cast<int64_t>(b) * T;
  int32_t* out = p.out_tokens + static_cast<int64_t>(b) * (T + 1);
  const int32_t* tok = p.tok + b * p.tok_sb;
  const bool walk = (n > 0 && n <= T);
  const AcceptDec* dsrc = p.dec + static_cast<int64_t>(b) * T;
  const bool local = walk && n <= scratch_cap;
  if (local) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      AcceptDec d;
      d.child = __ldcg(&dsrc[i].child);
      d.token = __ldcg(&dsrc[i].token);
      d.margin = __ldcg(&dsrc[i].margin);
      scratch[i] = d;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int len = 0;
    double mg = INFINITY;
    if (walk) {
      int c = 0;
      int bonus = -1;
      for (int step = 0; step < n; ++step) {
        int child, token;
        if (local) {
          child = scratch[c].child;
          token = scratch[c].token;
          mg = fmin(mg, scratch[c].margin);
        } else {
          const AcceptDec* dp = dsrc + c;
          child = __ldcg(&dp->child);
          token = __ldcg(&dp->token);
          mg = fmin(mg, __ldcg(&dp->margin));
        }
        if (child >= 0 && child < n) {
          acc[len] = child;
          out[len] = tok[child];
          ++len;
          c = child;
        } else {
          bonus = token;
          if (bonus == kNonFiniteRow) {
            set_status(p.status, TV_DEV_NONFINITE);
            bonus = -1;
          }
          break;
        }
      }
      out[len] = bonus;
    }
    p.n_acc[b] = len;
    if (p.min_margin) p.min_margin[b] = mg;
    sh.bc_int[1] = len;
  }
  __syncthreads();
  const int len = sh.bc_int[1];
  for (int i = len + threadIdx.x; i < T; i += blockDim.x) acc[i] = -1;
  for (int i = len + (walk ? 1 : 0) + threadIdx.x; i < T + 1; i += blockDim.x) out[i] = -1;
}

// ------------------------------------------------------------ node kernel

__global__ void __launch_bounds__(kAcceptThreads, 2)
accept_node_kernel(AcceptParams p) {
  __shared__ AcceptShared sh;
  extern __shared__ __align__(128) uint8_t ring_smem[];
  cg::cluster_group cl = cg::this_cluster();
  const int C = p.C;
  const int rank = static_cast<int>(cl.block_rank());
  const int c = blockIdx.x / C, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n <= 0 || n > p.T) {
    // nothing to decide: the first CTA writes the empty result
    if (c == 0 && rank == 0) {
      if (n != 0 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
      accept_walk(p, b, n, sh, nullptr, 0);
    }
    return;                                  // the whole cluster leaves together
  }
  if (c >= n) return;
  const int32_t* par = p.parent + b * p.par_sb;
  const int32_t* tok = p.tok + b * p.tok_sb;
  if (rank == 0 && tid == 0) {
    uint32_t bits = 0;
    const int pc = par[c];
    if (c == 0 ? (pc != -1) : (pc < 0 || pc >= c)) bits |= TV_DEV_BAD_PARENT;
    if (c > 0) {
      const int t = tok[c];
      if (t < 0 || t >= p.V) bits |= TV_DEV_BAD_TOKEN;
    }
    set_status(p.status, bits);
  }
  const int V = p.V;
  const int nseg = (V + kSeg - 1) / kSeg;
  const int seg0 = min(rank * p.seg_per_cta, nseg);
  const int nloc = min(p.seg_per_cta, nseg - seg0);
  const float* zr = p.z + b * p.z_sb + c * p.z_st;
  const bool zvec = (reinterpret_cast<uintptr_t>(zr) & 15u) == 0;
  int kred = 0;
  Slot all[8];
  AcceptDec d;
  d.child = -1; d.token = -1; d.margin = INFINITY;
  const bool greedy = (p.mode == TV_ACCEPT_GREEDY);
  const bool specsample = (p.mode == TV_ACCEPT_SPECSAMPLE);
  int has_child = 0;
  int cnt0 = 0;                 // children in the first window [c + 1, c + 1 + blockDim)
  if (specsample) {
    // the first window of children, in node order, and whether more follow
    const int j = c + 1 + tid;
    const bool is = (j < n) && par[j] == c;
    const unsigned m = __ballot_sync(0xffffffffu, is);
    if (lane == 0) sh.red_i[warp] = __popc(m);
    __syncthreads();
    if (tid == 0) {
      int acc = 0;
      for (int w = 0; w < kAcceptWarps; ++w) { sh.wofs[w] = acc; acc += sh.red_i[w]; }
      sh.bc_int[3] = acc;
    }
    __syncthreads();
    if (is) sh.clist[sh.wofs[warp] + __popc(m & ((1u << lane) - 1u))] = j;
    cnt0 = sh.bc_int[3];
    int fl = cnt0 > 0;
    for (int jj = c + 1 + static_cast<int>(blockDim.x) + tid; jj < n && !fl; jj += blockDim.x) fl = (par[jj] == c);
    has_child = __syncthreads_or(fl);
  }
  const bool read_q = specsample && has_child;
  const float* qr = read_q ? p.q + b * p.q_sb + c * p.q_st : nullptr;
  const bool qvec = read_q && ((reinterpret_cast<uintptr_t>(qr) & 15u) == 0);
  if (read_q && tid < cnt0) {
    // the first window's point values, loaded while the first pass streams
    const int x = tok[sh.clist[tid]];
    const bool okx = x >= 0 && x < V;
    sh.ctok[tid] = x;
    sh.cz[tid] = okx ? zr[x] : 0.f;
    sh.cq[tid] = okx ? qr[x] : 0.f;
    sh.cu[tid] = accept_uniform(p.seed, p.step, b, c, tid, kTagChild);
  }
  if (!greedy && tid == kAcceptThreads - 1)
    sh.bc_dbl[3] = accept_uniform(p.seed, p.step, b, c, 0, specsample ? kTagResidual : kTagSpecExec);

  SegStream st;
  st.zr = zr; st.qr = qr; st.zvec = zvec; st.qvec = qvec; st.readq = read_q;
  st.bulk = zvec && (V % 4 == 0) && (!read_q || qvec);
  st.V = V; st.seg0 = seg0; st.nloc = nloc;
  st.ring = smem_addr(ring_smem) + warp * kRing * kStageBytes;
  st.bar = sh.ring_bar + warp * kRing;
  st.count = 0;
  st.dead = false;
  if (st.bulk) {
    if (lane == 0) {
      for (int r = 0; r < kRing; ++r)
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(st.bar + r)) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
  }

  float M = -INFINITY;
  int gbad = 0;
  double ssum = 0.0;
  if (greedy) {
    // ---- the row maximum and its first index; NaN makes the row non-finite
    float bv = -INFINITY;
    int bi = INT_MAX;
    bool bad = false;
    stream_pass(st, -INFINITY, [&](int, int s0, const float4 (&v)[4], const float4 (&)[4]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e0 = s0 + k * kSub + lane * 4;
        const float xs[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = xs[e];
          if (e0 + e < V) {
            if (x != x) bad = true;
            else if (x > bv || (x == bv && e0 + e < bi)) { bv = x; bi = e0 + e; }
          }
        }
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    const int any_bad = __syncthreads_or(bad ? 1 : 0);
    if (lane == 0) { sh.red_f[warp] = bv; sh.red_i[warp] = bi; }
    __syncthreads();
    {
      float v = -INFINITY;
      int i = INT_MAX;
#pragma unroll
      for (int w = 0; w < kAcceptWarps; ++w)
        if (sh.red_f[w] > v || (sh.red_f[w] == v && sh.red_i[w] < i)) { v = sh.red_f[w]; i = sh.red_i[w]; }
      Slot mine;
      mine.a = 0.0; mine.b = 0.0; mine.f = v; mine.i = i; mine.j = any_bad;
      cluster_gather(cl, sh, mine, C, kred, all);
    }
    int am = INT_MAX;
    for (int r = 0; r < C; ++r) {
      gbad |= all[r].j;
      if (all[r].f > M || (all[r].f == M && all[r].i < am)) { M = all[r].f; am = all[r].i; }
    }
    if (gbad) {
      d.token = kNonFiniteRow;
    } else if (rank == 0) {
      d.child = first_child_with_token(par, tok, c, n, am, sh);
      d.token = (d.child >= 0) ? -1 : am;
    }
  }
  const double k_d = 1.4426950408889634 / static_cast<double>(p.tau);
  Frame f;
  f.k = static_cast<float>(k_d);
  f.inv_s = 1.f;
  f.c = 0.f;
  f.resid = false;
  if (!greedy) {
    // ---- one pass: per-segment maximum m_s and sum of 2^((z - m_s) k),
    // finiteness (and q >= 0); the row frame follows from the gathered
    // per-CTA maxima
    bool bad = false;
    float nf = 0.f;                 // x * 0 turns any non-finite x into NaN
    float qmin = 0.f;
    float wmax = -INFINITY;         // running maximum of this warp's segments
    const float k = f.k;
    stream_pass(st, -FLT_MAX, [&](int sl, int, const float4 (&v)[4], const float4 (&qv)[4]) {
      float m = -FLT_MAX;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        m = fmaxf(fmaxf(m, v[kk].x), fmaxf(v[kk].y, fmaxf(v[kk].z, v[kk].w)));
        nf = fmaf(v[kk].x, 0.f, nf); nf = fmaf(v[kk].y, 0.f, nf);
        nf = fmaf(v[kk].z, 0.f, nf); nf = fmaf(v[kk].w, 0.f, nf);
        if (read_q) {
          qmin = fminf(qmin, fminf(fminf(qv[kk].x, qv[kk].y), fminf(qv[kk].z, qv[kk].w)));
          nf = fmaf(qv[kk].x, 0.f, nf); nf = fmaf(qv[kk].y, 0.f, nf);
          nf = fmaf(qv[kk].z, 0.f, nf); nf = fmaf(qv[kk].w, 0.f, nf);
        }
      }
      m = warp_max(m);
      wmax = fmaxf(wmax, m);
      const float off = -m * k;
      float g = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        g += ex2_approx(fmaf(v[kk].x, k, off)) + ex2_approx(fmaf(v[kk].y, k, off));
        g += ex2_approx(fmaf(v[kk].z, k, off)) + ex2_approx(fmaf(v[kk].w, k, off));
      }
      g = warp_sum_f(g);
      if (lane == 0) { sh.seg_b[sl] = m; sh.seg_a[sl] = g; }
    });
    if (nf != nf || qmin < 0.f) bad = true;
    if (lane == 0) sh.red_f[warp] = wmax;
    const int any_bad = __syncthreads_or(bad ? 1 : 0);
    // this CTA's maximum and its sum in that frame
    float mr = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAcceptWarps; ++w) mr = fmaxf(mr, sh.red_f[w]);
    double sr = 0.0;
    for (int sl = tid; sl < nloc; sl += blockDim.x)
      sr += static_cast<double>(sh.seg_a[sl]) * exp2(static_cast<double>(sh.seg_b[sl] - mr) * k_d);
    sr = block_sum_d(sr, sh);
    {
      Slot mine;
      mine.a = sr; mine.b = 0.0; mine.f = mr; mine.i = 0; mine.j = any_bad;
      cluster_gather(cl, sh, mine, C, kred, all);
    }
    for (int r = 0; r < C; ++r) { gbad |= all[r].j; M = fmaxf(M, all[r].f); }
    if (gbad) d.token = kNonFiniteRow;
    else {
      for (int r = 0; r < C; ++r) {
        const double tr = (all[r].f == -INFINITY) ? 0.0 : all[r].a * exp2(static_cast<double>(all[r].f - M) * k_d);
        ssum += tr;
        if (tid == 0) sh.rank_tot[r] = tr;
      }
      // segment sums in the row frame
      for (int sl = tid; sl < nloc; sl += blockDim.x)
        sh.seg_a[sl] = sh.seg_a[sl] * ex2_approx((sh.seg_b[sl] - M) * k);
      __syncthreads();
    }
  }

  if (!greedy && !gbad) {
    f.zoff = -M * f.k;
    float* seg_w = sh.seg_a;
    float* seg_r = sh.seg_b;
    const double inv_s = 1.0 / ssum;
    // the weights e_t carry the fp32 frame offset zoff; point values use the
    // same offset in fp64: p(x) = 2^(z_x k + zoff) / s
    const double zoff_d = static_cast<double>(f.zoff);
    const double k_f = static_cast<double>(f.k);
    double margin = INFINITY;
    bool decided = false;
    double cpar = 0.0, D = 1.0;
    if (read_q) {
      const float* q = qr;
      int kk = 0;   // child ordinal = draw index
      for (int base = c + 1, win = 0; base < n && !decided; base += blockDim.x, ++win) {
        int cnt = cnt0;           // the first window was listed before the first pass
        if (win > 0) {
          const int j = base + tid;
          const bool is = (j < n) && par[j] == c;
          const unsigned m = __ballot_sync(0xffffffffu, is);
          if (lane == 0) sh.red_i[warp] = __popc(m);
          __syncthreads();
          if (tid == 0) {
            int acc = 0;
            for (int w = 0; w < kAcceptWarps; ++w) { sh.wofs[w] = acc; acc += sh.red_i[w]; }
            sh.bc_int[3] = acc;
          }
          __syncthreads();
          if (is) sh.clist[sh.wofs[warp] + __popc(m & ((1u << lane) - 1u))] = j;
          cnt = sh.bc_int[3];
          __syncthreads();
        }
        for (int ci = 0; ci < cnt && !decided; ++ci, ++kk) {
          const int jc = sh.clist[ci];
          const int x = (win == 0) ? sh.ctok[ci] : tok[jc];
          if (x < 0 || x >= V) continue;
          const float zx = (win == 0) ? sh.cz[ci] : zr[x];
          const double px = exp2(static_cast<double>(zx) * k_f + zoff_d) * inv_s;
          const double qx = static_cast<double>((win == 0) ? sh.cq[ci] : q[x]);
          const double num = px - cpar * qx;
          const double rx = num > 0.0 ? num / D : 0.0;
          const double ratio = qx > 0.0 ? rx / qx : (rx > 0.0 ? INFINITY : 0.0);
          const double u = (win == 0) ? sh.cu[ci] : accept_uniform(p.seed, p.step, b, c, kk, kTagChild);
          if (isfinite(ratio)) margin = fmin(margin, fabs(u - ratio));
          if (u < ratio) {
            d.child = jc;
            decided = true;
            break;
          }
          // residual pass with c' = c + D
          const double cn = cpar + D;
          Frame fr = f;
          fr.inv_s = static_cast<float>(inv_s);
          fr.c = static_cast<float>(cn);
          fr.resid = true;
          const double S_loc = weight_pass(st, fr, seg_r, sh);
          Slot ms;
          ms.a = S_loc; ms.b = 0.0; ms.f = 0.f; ms.i = 0; ms.j = 0;
          cluster_gather(cl, sh, ms, C, kred, all);
          double S = 0.0;
          for (int r = 0; r < C; ++r) S += all[r].a;
          if (S > 0.0) {
            cpar = cn; D = S; f = fr;
            float* t = seg_w; seg_w = seg_r; seg_r = t;
            for (int r = 0; r < C; ++r) sh.rank_tot[r] = all[r].a;
          }
          __syncthreads();
        }
      }
    }
    if (!decided) {
      // inverse-CDF sample over the current weights: find the CTA whose
      // slice holds the crossing, search inside it, gather the result
      const double u = sh.bc_dbl[3];
      double W = 0.0;
      for (int r = 0; r < C; ++r) W += sh.rank_tot[r];
      const double target = u * W;
      int owner = -1, last_pos = -1;
      double base = 0.0, cum = 0.0;
      for (int r = 0; r < C; ++r) {
        if (sh.rank_tot[r] > 0.0) last_pos = r;
        if (owner < 0 && cum + sh.rank_tot[r] > target) { owner = r; base = cum; }
        if (owner < 0) cum += sh.rank_tot[r];
      }
      if (owner < 0) {                         // rounding: the last slice with weight
        owner = last_pos < 0 ? 0 : last_pos;
        base = 0.0;
        for (int r = 0; r < owner; ++r) base += sh.rank_tot[r];
      }
      if (rank == owner && warp == 0) {
        int t;
        double mg;
        slice_search(zr, qr, zvec, qvec, V, seg0, nloc, seg_w, f, base, target, W, &t, &mg);
        if (lane == 0) { sh.bc_int[2] = t; sh.bc_dbl[2] = mg; }
      }
      __syncthreads();
      Slot res;
      res.a = 0.0; res.b = 0.0; res.f = 0.f; res.i = -1; res.j = 0;
      if (rank == owner) { res.i = sh.bc_int[2]; res.b = sh.bc_dbl[2]; }
      cluster_gather(cl, sh, res, C, kred, all);
      const int t = all[owner].i;
      margin = fmin(margin, all[owner].b);
      if (specsample) {
        d.token = t;
      } else if (rank == 0) {
        d.child = first_child_with_token(par, tok, c, n, t, sh);
        d.token = (d.child >= 0) ? -1 : t;
      }
    }
    d.margin = margin;
  }
  // rank 0 publishes the decision; the last node of the sequence walks
  if (rank == 0) {
    if (tid == 0) {
      p.dec[static_cast<int64_t>(b) * p.T + c] = d;
      __threadfence();
      const int done = atomicAdd(&p.ticket[b], 1);
      sh.bc_int[2] = (done == n - 1);
    }
    __syncthreads();
    if (sh.bc_int[2]) {
      __threadfence();
      // the rings are idle now: their shared memory holds the decisions
      accept_walk(p, b, n, sh, reinterpret_cast<AcceptDec*>(ring_smem),
                  static_cast<int>(kRingBytes / sizeof(AcceptDec)));
      if (tid == 0) p.ticket[b] = 0;           // ready for the next call
    }
  }
  // a ring wait that expired left this warp's passes on fill values
  if (st.dead && lane == 0) set_status(p.status, TV_DEV_TIMEOUT);
  cl.sync();                                   // no CTA leaves while others may read its slots
}

// ------------------------------------------------------------ host side

// Workspace: [0, 64 KB) ticket counters (zero between calls), then the
// per-node decisions.
constexpr size_t kAcceptTicketBytes = 64 * 1024;

size_t accept_workspace_bytes(int B, int T) {
  return kAcceptTicketBytes + static_cast<size_t>(B) * static_cast<size_t>(T) * sizeof(AcceptDec);
}

cudaError_t launch_accept(const tv_accept_args* a, int mode, void* ws, cudaStream_t stream) {
  AcceptParams p;
  p.B = a->B; p.T = a->T; p.V = a->V;
  p.z = a->target_logits; p.z_sb = a->tl_sb; p.z_st = a->tl_st;
  p.q = a->draft_probs; p.q_sb = a->dp_sb; p.q_st = a->dp_st;
  p.tok = a->draft_tokens; p.tok_sb = a->tok_sb;
  p.parent = a->parent; p.par_sb = a->parent_sb;
  p.n_nodes = a->n_nodes;
  p.mode = mode;
  p.tau = a->temperature;
  p.seed = a->seed; p.step = a->step;
  p.status = a->dev_status;
  p.ticket = static_cast<int32_t*>(ws);
  p.dec = reinterpret_cast<AcceptDec*>(static_cast<unsigned char*>(ws) + kAcceptTicketBytes);
  p.n_acc = a->n_accepted; p.acc_nodes = a->accepted_nodes; p.out_tokens = a->out_tokens;
  p.min_margin = a->min_margin;
  if (a->B == 0) return cudaSuccess;
  // CTAs per row: few rows need several CTAs per row (the sampling modes
  // make sequential passes over a row); many rows already fill the GPU and
  // extra CTAs only add cluster synchronisation.  The sampling modes keep
  // per-segment sums in shared memory, which bounds the slice length.
  const int nseg = (a->V + kSeg - 1) / kSeg;
  const int64_t rows_total = static_cast<int64_t>(a->B) * (a->T > 0 ? a->T : 1);
  int C;
  if (mode == TV_ACCEPT_GREEDY) C = rows_total >= 256 ? 1 : (rows_total >= 64 ? 2 : 4);
  else C = rows_total >= 256 ? 2 : 4;
  if (mode != TV_ACCEPT_GREEDY) C = max(C, (nseg + kMaxSegPerCta - 1) / kMaxSegPerCta);
  C = min(C, max(1, nseg));
  if (C > 8) return cudaErrorInvalidValue;
  p.C = C;
  p.seg_per_cta = (nseg + C - 1) / C;
  const int rows = a->T > 0 ? a->T : 1;        // T == 0: one cluster writes the empty result
  cudaError_t e = cudaFuncSetAttribute(accept_node_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kRingBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * C, a->B, 1);
  cfg.blockDim = dim3(kAcceptThreads, 1, 1);
  cfg.dynamicSmemBytes = kRingBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, accept_node_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------ no-allocation entry

int resolve_mode(const tv_accept_args* a);
tv_status check_accept(const tv_accept_args* a);

// Scratch of tree_accept_noalloc: the ticket region then the decisions of
// at most kNoAllocMaxRows node rows.  Every GPU that loads the library holds
// this array until the process exits.
constexpr int kNoAllocMaxRows = 32768;
constexpr size_t kNoAllocBytes = kAcceptTicketBytes + static_cast<size_t>(kNoAllocMaxRows) * sizeof(AcceptDec);
static __device__ __align__(256) unsigned char g_accept_scratch[kNoAllocBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

}  // namespace tv

// tree_accept for callers that cannot allocate device memory (see
// include/tree_verify.h).  The first call on a device resolves the device
// address of the file-scope scratch array with cudaGetSymbolAddress; later
// calls reuse it.
extern "C" tv_status tree_accept_noalloc(const tv_accept_args* a, tv_stream_t stream) {
  using namespace tv;
  const tv_status st = check_accept(a);
  if (st != TV_OK) return st;
  if (a->B == 0) return TV_OK;
  if (static_cast<int64_t>(a->B) * a->T > kNoAllocMaxRows) return TV_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TV_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* sym = nullptr;
      if (cudaGetSymbolAddress(&sym, g_accept_scratch) != cudaSuccess || sym == nullptr) return TV_ERR_CUDA;
      g_scratch_ptr[dev] = sym;
    }
    ptr = g_scratch_ptr[dev];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the tickets must start at zero whatever an earlier call left behind
  if (cudaMemsetAsync(ptr, 0, static_cast<size_t>(a->B) * sizeof(int32_t), s) != cudaSuccess) return TV_ERR_CUDA;
  return launch_accept(a, resolve_mode(a), ptr, s) == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}
