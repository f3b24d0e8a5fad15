// tree_accept kernels: per-node decisions over vocabulary rows, then a walk
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
// draws, so all nodes decide in parallel (one CTA per node row) and a
// second, tiny kernel follows the decisions from the root.
//
// Data layout of a row pass: the row is cut into 128-element segments; a
// warp owns a segment (lane l holds elements 4l..4l+3, one 16-byte load).
// Per segment the first pass keeps the segment maximum wm and the sum of
// exp((z - wm)/tau); element weights are always recomputed in that same
// segment frame, scaled by f_seg = exp((wm - M)/tau) (M the row maximum),
// so segment sums and element values agree to rounding order.  Residuals
// are parametrised as r = (p - c q)^+ / D: rejecting a child with the
// current (c, D) gives c' = c + D and D' = sum_t (p - c' q)^+, one pass.
#include "tv_common.cuh"

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
  int32_t* n_acc;
  int32_t* acc_nodes;
  int32_t* out_tokens;
  double* min_margin;
};

constexpr int kAcceptThreads = 512;
constexpr int kAcceptWarps = kAcceptThreads / kWarp;
constexpr int kSeg = 128;

// ------------------------------------------------------------ block helpers

struct AcceptShared {
  double red_d[kAcceptWarps];
  float red_f[kAcceptWarps];
  int red_i[kAcceptWarps];
  int wofs[kAcceptWarps];
  int clist[kAcceptThreads];
  int bc_int[4];
  double bc_dbl[4];
};

__device__ __forceinline__ double block_sum_d(double v, AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh.red_d[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (warp == 0) {
    t = (lane < kAcceptWarps) ? sh.red_d[lane] : 0.0;
    t = warp_sum(t);
    if (lane == 0) sh.bc_dbl[0] = t;
  }
  __syncthreads();
  return sh.bc_dbl[0];
}

__device__ __forceinline__ float block_max_f(float v, AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) sh.red_f[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = (lane < kAcceptWarps) ? sh.red_f[lane] : -INFINITY;
    t = warp_max(t);
    if (lane == 0) sh.red_f[0] = t;
  }
  __syncthreads();
  return sh.red_f[0];
}

__device__ __forceinline__ int block_min_i(int v, AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh.red_i[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int t = (lane < kAcceptWarps) ? sh.red_i[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = min(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (lane == 0) sh.bc_int[0] = t;
  }
  __syncthreads();
  return sh.bc_int[0];
}

// Lowest-index child of c (c < j < n) that carries token x, or -1.
__device__ int first_child_with_token(const int32_t* par, const int32_t* tok, int c, int n,
                                      int x, AcceptShared& sh) {
  int best = INT_MAX;
  for (int j = c + 1 + threadIdx.x; j < n; j += blockDim.x)
    if (par[j] == c && tok[j] == x) { best = j; break; }
  best = block_min_i(best, sh);
  return best == INT_MAX ? -1 : best;
}

// Weight of one element in the current distribution: e = exp((z-wm)/tau) *
// f_seg (unnormalised softmax), or the residual (e/s - c q)^+.
__device__ __forceinline__ double elem_weight(float z, float q, float wm, double fseg,
                                              double invtau, double inv_s, double cpar,
                                              bool resid) {
  const double e = exp_neg((static_cast<double>(z) - static_cast<double>(wm)) * invtau) * fseg;
  if (!resid) return e;
  const double w = e * inv_s - cpar * static_cast<double>(q);
  return w > 0.0 ? w : 0.0;
}

// Inverse-CDF sample: smallest t with sum_{s<=t} w_s > u * W over the
// current weights (segment sums in seg_w).  Returns t and the relative
// margin min(cum_t - uW, uW - cum_{t-1}) / W.  Called by the whole block.
__device__ void sample_row(const float* zr, const float* qr, bool zvec, bool qvec, int V,
                           int nseg, const float* seg_m, const double* seg_f,
                           const double* seg_w, double invtau, double inv_s, double cpar,
                           bool resid, double u, int* out_t, double* out_margin,
                           AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double part = 0.0;
  for (int s = threadIdx.x; s < nseg; s += blockDim.x) part += seg_w[s];
  const double W = block_sum_d(part, sh);
  const double target = u * W;
  if (warp == 0) {
    // 1. the segment where the running sum first exceeds target
    const int per = (nseg + 31) / 32;
    const int lo = min(lane * per, nseg), hi = min(lo + per, nseg);
    double ls = 0.0;
    for (int s = lo; s < hi; ++s) ls += seg_w[s];
    const double incl = warp_incl_scan(ls);
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const unsigned m = __ballot_sync(0xffffffffu, incl > target);
    int seg = -1;
    double base = 0.0;
    if (m != 0u) {
      const int L = __ffs(m) - 1;
      if (lane == L) {
        double cum = excl;
        int s = lo;
        for (; s < hi; ++s) {
          if (cum + seg_w[s] > target) break;
          cum += seg_w[s];
        }
        seg = (s < hi) ? s : hi - 1;
        base = (s < hi) ? cum : cum - seg_w[hi - 1];
      }
      seg = __shfl_sync(0xffffffffu, seg, L);
      base = __shfl_sync(0xffffffffu, base, L);
    } else {
      // target >= total by rounding: the last segment with weight
      int last = -1;
      for (int s = lo; s < hi; ++s) if (seg_w[s] > 0.0) last = s;
      const unsigned mm = __ballot_sync(0xffffffffu, last >= 0);
      const int L = mm ? 31 - __clz(mm) : 0;
      seg = __shfl_sync(0xffffffffu, last, L);
      if (seg < 0) seg = 0;
      base = -1.0;           // marks "take the last positive element"
    }
    // 2. inside the segment
    const int e0 = seg * kSeg + lane * 4;
    const float4 zv = load4(zr, e0, V, zvec, -INFINITY);
    float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (resid) qv = load4(qr, e0, V, qvec, 0.f);
    const float wm = seg_m[seg];
    const double fs = seg_f[seg];
    double w[4];
    w[0] = (e0 + 0 < V) ? elem_weight(zv.x, qv.x, wm, fs, invtau, inv_s, cpar, resid) : 0.0;
    w[1] = (e0 + 1 < V) ? elem_weight(zv.y, qv.y, wm, fs, invtau, inv_s, cpar, resid) : 0.0;
    w[2] = (e0 + 2 < V) ? elem_weight(zv.z, qv.z, wm, fs, invtau, inv_s, cpar, resid) : 0.0;
    w[3] = (e0 + 3 < V) ? elem_weight(zv.w, qv.w, wm, fs, invtau, inv_s, cpar, resid) : 0.0;
    int t = -1;
    double margin = 0.0;
    if (base >= 0.0) {
      const double lsum = ((w[0] + w[1]) + w[2]) + w[3];
      const double li = warp_incl_scan(lsum);
      double le = __shfl_up_sync(0xffffffffu, li, 1);
      if (lane == 0) le = 0.0;
      const unsigned m2 = __ballot_sync(0xffffffffu, base + li > target);
      if (m2 != 0u) {
        const int L = __ffs(m2) - 1;
        if (lane == L) {
          double cum = base + le;
          for (int k = 0; k < 4; ++k) {
            if (cum + w[k] > target) {
              t = e0 + k;
              margin = fmin(cum + w[k] - target, target - cum) / W;
              break;
            }
            cum += w[k];
          }
        }
        t = __shfl_sync(0xffffffffu, t, L);
        margin = __shfl_sync(0xffffffffu, margin, L);
      }
    }
    if (t < 0) {
      // rounding put the crossing at the segment's end: last positive element
      int lp = -1;
      for (int k = 0; k < 4; ++k) if (w[k] > 0.0) lp = e0 + k;
      const unsigned mm = __ballot_sync(0xffffffffu, lp >= 0);
      const int L = mm ? 31 - __clz(mm) : 0;
      t = __shfl_sync(0xffffffffu, lp, L);
      margin = 0.0;
    }
    if (lane == 0) { sh.bc_int[1] = t; sh.bc_dbl[1] = margin; }
  }
  __syncthreads();
  *out_t = sh.bc_int[1];
  *out_margin = sh.bc_dbl[1];
  __syncthreads();
}

// One pass over the row computing the segment sums of the residual
// weights (e/s - c q)^+; returns their total.
__device__ double residual_pass(const float* zr, const float* qr, bool zvec, bool qvec, int V,
                                int nseg, const float* seg_m, const double* seg_f,
                                double* seg_out, double invtau, double inv_s, double cpar,
                                AcceptShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double tot = 0.0;
  for (int s = warp; s < nseg; s += kAcceptWarps) {
    const int e0 = s * kSeg + lane * 4;
    const float4 zv = load4(zr, e0, V, zvec, -INFINITY);
    const float4 qv = load4(qr, e0, V, qvec, 0.f);
    const float wm = seg_m[s];
    const double fs = seg_f[s];
    double a = 0.0;
    if (e0 + 0 < V) a += elem_weight(zv.x, qv.x, wm, fs, invtau, inv_s, cpar, true);
    if (e0 + 1 < V) a += elem_weight(zv.y, qv.y, wm, fs, invtau, inv_s, cpar, true);
    if (e0 + 2 < V) a += elem_weight(zv.z, qv.z, wm, fs, invtau, inv_s, cpar, true);
    if (e0 + 3 < V) a += elem_weight(zv.w, qv.w, wm, fs, invtau, inv_s, cpar, true);
    a = warp_sum(a);
    if (lane == 0) seg_out[s] = a;
    tot += a;
  }
  return block_sum_d(lane == 0 ? tot : 0.0, sh);
}

// ------------------------------------------------------------ node kernel

__global__ void __launch_bounds__(kAcceptThreads)
accept_node_kernel(AcceptParams p) {
  extern __shared__ double dyn_smem[];
  __shared__ AcceptShared sh;
  const int c = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) {
    if (c == 0 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
    return;
  }
  if (c >= n) return;
  const int32_t* par = p.parent + b * p.par_sb;
  const int32_t* tok = p.tok + b * p.tok_sb;
  if (tid == 0) {
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
  const float* zr = p.z + b * p.z_sb + c * p.z_st;
  const bool zvec = (reinterpret_cast<uintptr_t>(zr) & 15u) == 0;
  AcceptDec d;
  d.child = -1; d.token = -1; d.margin = INFINITY;

  if (p.mode == TV_ACCEPT_GREEDY) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    bool nan = false;
    for (int s = warp; s < nseg; s += kAcceptWarps) {
      const int e0 = s * kSeg + lane * 4;
      const float4 v = load4(zr, e0, V, zvec, -INFINITY);
      const float xs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = e0 + k;
        if (idx < V) {
          const float x = xs[k];
          if (isnan(x)) nan = true;
          else if (x > bv || (x == bv && idx < bi)) { bv = x; bi = idx; }
        }
      }
    }
    // block argmax, ties to the lower index
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    const int any_nan = __syncthreads_or(nan ? 1 : 0);
    if (lane == 0) { sh.red_f[warp] = bv; sh.red_i[warp] = bi; }
    __syncthreads();
    if (warp == 0) {
      bv = (lane < kAcceptWarps) ? sh.red_f[lane] : -INFINITY;
      bi = (lane < kAcceptWarps) ? sh.red_i[lane] : INT_MAX;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (lane == 0) sh.bc_int[2] = bi;
    }
    __syncthreads();
    const int a = sh.bc_int[2];
    if (any_nan) {
      d.token = kNonFiniteRow;
    } else {
      d.child = first_child_with_token(par, tok, c, n, a, sh);
      d.token = (d.child >= 0) ? -1 : a;
    }
  } else {
    const bool specsample = (p.mode == TV_ACCEPT_SPECSAMPLE);
    int has_child = 0;
    if (specsample) {
      int f = 0;
      for (int j = c + 1 + tid; j < n && !f; j += blockDim.x) f = (par[j] == c);
      has_child = __syncthreads_or(f);
    }
    const bool read_q = specsample && has_child;
    const float* qr = read_q ? p.q + b * p.q_sb + c * p.q_st : nullptr;
    const bool qvec = read_q && ((reinterpret_cast<uintptr_t>(qr) & 15u) == 0);
    // dynamic shared memory: seg_f, seg_w, seg_r (double) then seg_m (float)
    double* seg_f = dyn_smem;
    double* seg_w = seg_f + nseg;
    double* seg_r = seg_w + nseg;
    float* seg_m = reinterpret_cast<float*>(seg_r + nseg);
    const double invtau = 1.0 / static_cast<double>(p.tau);

    // pass 1: segment maxima and segment-frame exponential sums
    bool bad = false, qbad = false;
    float lmax = -INFINITY;
    for (int s = warp; s < nseg; s += kAcceptWarps) {
      const int e0 = s * kSeg + lane * 4;
      const float4 v = load4(zr, e0, V, zvec, -INFINITY);
      const float xs[4] = {v.x, v.y, v.z, v.w};
      float m4 = -INFINITY;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (e0 + k < V) {
          if (!isfinite(xs[k])) bad = true;
          else m4 = fmaxf(m4, xs[k]);
        }
      if (read_q) {
        const float4 qv = load4(qr, e0, V, qvec, 0.f);
        const float qs[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (e0 + k < V && !(qs[k] >= 0.f && isfinite(qs[k]))) qbad = true;
      }
      const float wm = warp_max(m4);
      double a = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (e0 + k < V && isfinite(xs[k]))
          a += exp_neg((static_cast<double>(xs[k]) - static_cast<double>(wm)) * invtau);
      a = warp_sum(a);
      if (lane == 0) { seg_m[s] = wm; seg_w[s] = a; }
      lmax = fmaxf(lmax, wm);
    }
    const int any_bad = __syncthreads_or(bad ? 1 : 0);
    const int any_qbad = __syncthreads_or(qbad ? 1 : 0);
    const float M = block_max_f(lmax, sh);
    if (any_bad || any_qbad) {
      d.token = kNonFiniteRow;
    } else {
      double part = 0.0;
      for (int s = tid; s < nseg; s += blockDim.x) {
        const double f = exp((static_cast<double>(seg_m[s]) - static_cast<double>(M)) * invtau);
        seg_f[s] = f;
        seg_w[s] *= f;
        part += seg_w[s];
      }
      const double ssum = block_sum_d(part, sh);   // syncs: seg_f / seg_w visible
      const double inv_s = 1.0 / ssum;
      double margin = INFINITY;
      bool decided = false;
      double cpar = 0.0, D = 1.0;
      bool resid = false;
      if (specsample && has_child) {
        const float* q = qr;
        int k = 0;   // child ordinal = draw index
        for (int base = c + 1; base < n && !decided; base += blockDim.x) {
          const int j = base + tid;
          const bool is = (j < n) && par[j] == c;
          const unsigned m = __ballot_sync(0xffffffffu, is);
          if (lane == 0) sh.red_i[warp] = __popc(m);
          __syncthreads();
          if (warp == 0) {
            const int v = (lane < kAcceptWarps) ? sh.red_i[lane] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int t = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += t;
            }
            if (lane < kAcceptWarps) sh.wofs[lane] = incl - v;
            if (lane == 31) sh.bc_int[3] = incl;
          }
          __syncthreads();
          if (is) sh.clist[sh.wofs[warp] + __popc(m & ((1u << lane) - 1u))] = j;
          const int cnt = sh.bc_int[3];
          __syncthreads();
          for (int ci = 0; ci < cnt && !decided; ++ci, ++k) {
            const int jc = sh.clist[ci];
            const int x = tok[jc];
            if (x < 0 || x >= V) continue;
            // point value of the current distribution at x
            const int sx = x / kSeg;
            const double ex = exp_neg((static_cast<double>(zr[x]) - static_cast<double>(seg_m[sx])) * invtau) * seg_f[sx];
            const double px = ex * inv_s;
            const double qx = static_cast<double>(q[x]);
            const double num = px - cpar * qx;
            const double rx = num > 0.0 ? num / D : 0.0;
            const double ratio = qx > 0.0 ? rx / qx : (rx > 0.0 ? INFINITY : 0.0);
            const double u = accept_uniform(p.seed, p.step, b, c, k, kTagChild);
            if (isfinite(ratio)) margin = fmin(margin, fabs(u - ratio));
            if (u < ratio) {
              d.child = jc;
              decided = true;
              break;
            }
            const double cn = cpar + D;
            const double S = residual_pass(zr, q, zvec, qvec, V, nseg, seg_m, seg_f, seg_r,
                                           invtau, inv_s, cn, sh);
            if (S > 0.0) {
              cpar = cn; D = S; resid = true;
              double* t = seg_w; seg_w = seg_r; seg_r = t;
            }
          }
        }
      }
      if (!decided) {
        int t = -1;
        double mg = 0.0;
        const int tag = specsample ? kTagResidual : kTagSpecExec;
        const double u = accept_uniform(p.seed, p.step, b, c, 0, tag);
        sample_row(zr, qr, zvec, qvec, V, nseg, seg_m, seg_f, seg_w, invtau, inv_s, cpar,
                   resid, u, &t, &mg, sh);
        margin = fmin(margin, mg);
        if (specsample) {
          d.token = t;
        } else {
          d.child = first_child_with_token(par, tok, c, n, t, sh);
          d.token = (d.child >= 0) ? -1 : t;
        }
      }
      d.margin = margin;
    }
  }
  if (tid == 0) p.dec[static_cast<int64_t>(b) * p.T + c] = d;
}

// ------------------------------------------------------------ walk kernel

__global__ void accept_walk_kernel(AcceptParams p) {
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int T = p.T;
  const int n = p.n_nodes ? p.n_nodes[b] : T;
  int32_t* acc = p.acc_nodes + static_cast<int64_t>(b) * T;
  int32_t* out = p.out_tokens + static_cast<int64_t>(b) * (T + 1);
  const int32_t* tok = p.tok + b * p.tok_sb;
  int len = 0;
  double mg = INFINITY;
  if (lane == 0 && n > 0 && n <= T) {
    int c = 0;
    int bonus = -1;
    for (int step = 0; step < n; ++step) {
      const AcceptDec d = p.dec[static_cast<int64_t>(b) * T + c];
      mg = fmin(mg, d.margin);
      if (d.child >= 0 && d.child < n) {
        acc[len] = d.child;
        out[len] = tok[d.child];
        ++len;
        c = d.child;
      } else {
        bonus = d.token;
        if (bonus == kNonFiniteRow) {
          set_status(p.status, TV_DEV_NONFINITE);
          bonus = -1;
        }
        break;
      }
    }
    out[len] = bonus;
  }
  len = __shfl_sync(0xffffffffu, len, 0);
  const bool wrote_bonus = (n > 0 && n <= T);
  for (int i = len + lane; i < T; i += 32) acc[i] = -1;
  for (int i = len + (wrote_bonus ? 1 : 0) + lane; i < T + 1; i += 32) out[i] = -1;
  if (lane == 0) {
    p.n_acc[b] = len;
    if (p.min_margin) p.min_margin[b] = mg;
  }
}

// ------------------------------------------------------------ host side

size_t accept_workspace_bytes(int B, int T) {
  return static_cast<size_t>(B) * static_cast<size_t>(T) * sizeof(AcceptDec);
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
  p.dec = static_cast<AcceptDec*>(ws);
  p.n_acc = a->n_accepted; p.acc_nodes = a->accepted_nodes; p.out_tokens = a->out_tokens;
  p.min_margin = a->min_margin;
  if (a->B == 0) return cudaSuccess;
  if (a->T > 0) {
    const int nseg = (a->V + kSeg - 1) / kSeg;
    const size_t smem = (mode == TV_ACCEPT_GREEDY) ? 0 : static_cast<size_t>(nseg) * (3 * sizeof(double) + sizeof(float));
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(accept_node_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    dim3 grid(a->T, a->B);
    accept_node_kernel<<<grid, kAcceptThreads, smem, stream>>>(p);
  }
  accept_walk_kernel<<<a->B, 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tv
