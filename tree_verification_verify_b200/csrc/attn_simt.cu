// tree_verify_attn, CUDA-core kernels.
//
// The attention of draft node i covers K(i) = the shared prefix plus the
// nodes on its root path (tree attention; SpecExec page, "Approach": the
// whole tree is verified in one target pass).  The prefix part is dense
// (every node sees every prefix key) and the tree part is a short ancestor
// path, so the two are computed separately and combined by their
// log-sum-exp:
//
//   attn_prefix_simt_kernel  split-KV over the prefix: a CTA owns a tile of
//                            nodes x the G query heads of one kv head and a
//                            chunk of prefix positions; K/V tiles of 32 keys
//                            are staged in shared memory (fp32) and reused
//                            by every query row of the tile;
//   attn_tree_kernel         one CTA per (sequence, node, kv head): the
//                            root path of the node is collected once from
//                            parent[] into shared memory, then each warp
//                            runs the online softmax of one query head over
//                            the path's keys (the node itself included);
//   attn_merge_kernel        one warp per (sequence, node, query head):
//                            O = sum_c e^{lse_c - M} O_c / sum_c e^{lse_c - M}.
//
// Partials hold the normalised output and the natural-log lse of each chunk
// (lse = -inf for a chunk with no keys).
#include "attn.cuh"

namespace tv {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / kWarp;
constexpr int kSimtMaxRows = 64;
constexpr int kSimtKeys = 32;

template <typename T>
__device__ __forceinline__ float ld_elt(const void* base, int64_t off) {
  return to_f32(static_cast<const T*>(base)[off]);
}

// ------------------------------------------------------------ prefix (CUDA cores)

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
attn_prefix_simt_kernel(AttnParams p) {
  extern __shared__ __align__(16) float smem_f[];
  constexpr int DL = D / 32;                       // dims per lane
  const int chunk = blockIdx.x;
  const int tile = blockIdx.y;
  const int b = blockIdx.z / p.Hkv, g = blockIdx.z % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) return;
  const int i0 = tile * p.node_tile;
  if (i0 >= n) return;
  const int G = p.G;
  const int rows = min(p.node_tile, n - i0) * G;
  float* qs = smem_f;                               // [kSimtMaxRows][D]
  float* ks = qs + kSimtMaxRows * D;                // [32][D+1]
  float* vs = ks + kSimtKeys * (D + 1);             // [32][D]

  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;                   // flagged by the merge
  const int k0 = chunk * p.chunk_len;
  const int k1 = min(k0 + p.chunk_len, L);

  for (int e = tid; e < rows * D; e += blockDim.x) {
    const int r = e / D, dd = e % D;
    const int i = i0 + r / G, h = g * G + r % G;
    qs[r * D + dd] = ld_elt<T>(p.q, b * p.q_sb + i * p.q_st + h * p.q_sh + dd) * p.scale;
  }
  constexpr int MR = kSimtMaxRows / kSimtWarps;     // rows per warp (max)
  float m[MR], l[MR], acc[MR][DL];
#pragma unroll
  for (int rr = 0; rr < MR; ++rr) {
    m[rr] = -INFINITY; l[rr] = 0.f;
#pragma unroll
    for (int k = 0; k < DL; ++k) acc[rr][k] = 0.f;
  }
  __syncthreads();
  for (int kb = k0; kb < k1; kb += kSimtKeys) {
    const int nk = min(kSimtKeys, k1 - kb);
    for (int e = tid; e < kSimtKeys * D; e += blockDim.x) {
      const int j = e / D, dd = e % D;
      float kv = 0.f, vv = 0.f;
      if (j < nk) {
        const int64_t off = b * p.kv_sb + static_cast<int64_t>(kb + j) * p.kv_sl + g * p.kv_sh + dd;
        kv = ld_elt<T>(p.kc, off);
        vv = ld_elt<T>(p.vc, off);
      }
      ks[j * (D + 1) + dd] = kv;
      vs[j * D + dd] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < MR; ++rr) {
      const int r = warp + rr * kSimtWarps;
      if (r < rows) {
        float s = 0.f;
        const float* qr = qs + r * D;
        const float* kr = ks + lane * (D + 1);
#pragma unroll 8
        for (int dd = 0; dd < D; ++dd) s = fmaf(qr[dd], kr[dd], s);
        if (lane >= nk) s = -INFINITY;
        const float mx = warp_max(s);
        const float mn = fmaxf(m[rr], mx);
        const float corr = expf(m[rr] - mn);         // m = -inf at start: corr = 0
        const float pj = (lane < nk) ? expf(s - mn) : 0.f;
        l[rr] = l[rr] * corr + warp_sumf(pj);
#pragma unroll
        for (int k = 0; k < DL; ++k) acc[rr][k] *= corr;
        for (int j = 0; j < nk; ++j) {
          const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
          for (int k = 0; k < DL; ++k) acc[rr][k] = fmaf(pb, vs[j * D + lane + 32 * k], acc[rr][k]);
        }
        m[rr] = mn;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int rr = 0; rr < MR; ++rr) {
    const int r = warp + rr * kSimtWarps;
    if (r < rows) {
      const int i = i0 + r / G, h = g * G + r % G;
      const int64_t pr = part_row(p, chunk, b, i, h);
      const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
#pragma unroll
      for (int k = 0; k < DL; ++k) p.part_o[pr * D + lane + 32 * k] = acc[rr][k] * inv;
      if (lane == 0) p.part_lse[pr] = l[rr] > 0.f ? m[rr] + logf(l[rr]) : -INFINITY;
    }
  }
}

// ------------------------------------------------------------ tree ancestors

constexpr int kTreeThreads = 128;
constexpr int kTreeWarps = kTreeThreads / kWarp;
constexpr int kTreeStage = 32;                    // path rows staged per round

template <typename T, int D>
__global__ void __launch_bounds__(kTreeThreads)
attn_tree_kernel(AttnParams p) {
  extern __shared__ int path_smem[];              // [T] ancestor list
  __shared__ float ks[kTreeStage][D];
  __shared__ float vs[kTreeStage][D];
  __shared__ int s_len, s_ok;
  constexpr int DL = D / 32;
  const int i = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T || i >= n) return;
  const int32_t* par = p.parent + b * p.par_sb;
  if (p.prefix_only) {
    // a prefix-only partial: no tree keys (parent[] is not read)
    if (threadIdx.x == 0 && g == 0) p.node_ok[static_cast<int64_t>(b) * p.T + i] = 1;
    for (int hg = warp; hg < p.G; hg += kTreeWarps) {
      const int64_t pr = part_row(p, p.nchunk, b, i, g * p.G + hg);
      for (int k = lane; k < D; k += 32) p.part_o[pr * D + k] = 0.f;
      if (lane == 0) p.part_lse[pr] = -INFINITY;
    }
    return;
  }
  if (threadIdx.x == 0) {
    // root path of node i (i first, root last); malformed chains stop early
    int len = 0, ok = (par[0] == -1) ? 1 : 0;
    int j = i;
    while (ok) {
      path_smem[len++] = j;
      if (j == 0) break;
      const int pj = par[j];
      if (pj < 0 || pj >= j) { ok = 0; break; }
      j = pj;
    }
    s_len = len;
    s_ok = ok;
    if (g == 0) p.node_ok[static_cast<int64_t>(b) * p.T + i] = ok;
  }
  __syncthreads();
  const int len = s_ok ? s_len : 0;
  const int G = p.G;
  float qv[kTreeWarps > 0 ? 8 : 1][DL];            // up to 8 heads per warp
  float acc[8][DL], m[8], l[8];
  const int nh = (G + kTreeWarps - 1) / kTreeWarps;   // heads per warp (<= 16 for G <= 64)
  for (int h0 = 0; h0 < nh; h0 += 8) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int hg = warp + (h0 + r) * kTreeWarps;
      m[r] = -INFINITY; l[r] = 0.f;
#pragma unroll
      for (int k = 0; k < DL; ++k) {
        acc[r][k] = 0.f;
        qv[r][k] = (hg < G) ? ld_elt<T>(p.q, b * p.q_sb + i * p.q_st + (g * G + hg) * p.q_sh + lane + 32 * k) * p.scale
                            : 0.f;
      }
    }
    for (int t0 = 0; t0 < len; t0 += kTreeStage) {
      const int nt = min(kTreeStage, len - t0);
      __syncthreads();
      for (int e = threadIdx.x; e < nt * D; e += blockDim.x) {
        const int t = e / D, dd = e % D;
        const int64_t off = b * p.kt_sb + static_cast<int64_t>(path_smem[t0 + t]) * p.kt_st + g * p.kt_sh + dd;
        ks[t][dd] = ld_elt<T>(p.kt, off);
        vs[t][dd] = ld_elt<T>(p.vt, off);
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int hg = warp + (h0 + r) * kTreeWarps;
        if (hg >= G) break;
        for (int t = 0; t < nt; ++t) {
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < DL; ++k) s = fmaf(qv[r][k], ks[t][lane + 32 * k], s);
          s = warp_sumf(s);
          const float mn = fmaxf(m[r], s);
          const float corr = expf(m[r] - mn);
          const float pj = expf(s - mn);
          l[r] = l[r] * corr + pj;
#pragma unroll
          for (int k = 0; k < DL; ++k) acc[r][k] = fmaf(pj, vs[t][lane + 32 * k], acc[r][k] * corr);
          m[r] = mn;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int hg = warp + (h0 + r) * kTreeWarps;
      if (hg >= G) break;
      const int64_t pr = part_row(p, p.nchunk, b, i, g * G + hg);
      const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
#pragma unroll
      for (int k = 0; k < DL; ++k) p.part_o[pr * D + lane + 32 * k] = acc[r][k] * inv;
      if (lane == 0) p.part_lse[pr] = l[r] > 0.f ? m[r] + logf(l[r]) : -INFINITY;
    }
  }
}

// ------------------------------------------------------------ merge

template <typename T, int D>
__global__ void __launch_bounds__(256)
attn_merge_kernel(AttnParams p) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nrows = static_cast<int64_t>(p.B) * p.T * p.Hq;
  if (row >= nrows) return;
  const int h = static_cast<int>(row % p.Hq);
  const int i = static_cast<int>((row / p.Hq) % p.T);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.Hq) * p.T));
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) {
    if (i == 0 && h == 0 && lane == 0) set_status(p.status, TV_DEV_BAD_LEN);
    return;
  }
  if (i >= n) return;
  const int L = p.prefix_len[b];
  const bool bad_len = (L < 0 || L > p.Lmax);
  const bool ok = p.node_ok[static_cast<int64_t>(b) * p.T + i] != 0;
  if (lane == 0 && h == 0) {
    if (bad_len && i == 0) set_status(p.status, TV_DEV_BAD_LEN);
    if (!ok) set_status(p.status, TV_DEV_BAD_PARENT);
  }
  T* o = static_cast<T*>(p.out) + b * p.o_sb + i * p.o_st + h * p.o_sh;
  if (bad_len || !ok) {
#pragma unroll
    for (int k = 0; k < DL; ++k) o[lane + 32 * k] = static_cast<T>(NAN);
    if (p.lse && lane == 0) p.lse[row] = NAN;
    return;
  }
  // partial c's lse in lane c (at most 32 partials), weights by warp max
  const int np = p.nchunk + 1;
  float lc = -INFINITY;
  for (int c = lane; c < np; c += 32) lc = fmaxf(lc, p.part_lse[part_row(p, c, b, i, h)]);
  const float M = warp_max(lc);
  float wl = (lane < np && lc > -INFINITY) ? expf(lc - M) : 0.f;
  float den = warp_sumf(wl);
  float acc[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) acc[k] = 0.f;
  for (int c = 0; c < np; ++c) {
    const float w = __shfl_sync(0xffffffffu, wl, c & 31);
    if (w == 0.f) continue;
    const int64_t pr = part_row(p, c, b, i, h);
#pragma unroll
    for (int k = 0; k < DL; ++k) acc[k] = fmaf(w, p.part_o[pr * D + lane + 32 * k], acc[k]);
  }
  // no keys at all (an empty slice of a prefix-only partial): O = 0, lse = -inf
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int k = 0; k < DL; ++k) o[lane + 32 * k] = static_cast<T>(acc[k] * inv);
  if (p.lse && lane == 0) p.lse[row] = den > 0.f ? M + logf(den) : -INFINITY;
}

// Log-sum-exp merge of N stacked partials (tree_verify_attn_merge): one
// warp per output row.
template <typename T, int D>
__global__ void __launch_bounds__(256)
attn_partial_merge_kernel(const T* __restrict__ o_parts, const float* __restrict__ lse_parts, T* out, float* lse,
                          int N, int64_t nrows) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= nrows) return;
  float lc = -INFINITY;
  bool bad = false;
  for (int c = lane; c < N; c += 32) {
    const float v = lse_parts[static_cast<int64_t>(c) * nrows + row];
    bad |= (v != v);
    lc = fmaxf(lc, v);
  }
  bad = __any_sync(0xffffffffu, bad);
  const float M = warp_max(lc);
  float wsum = 0.f;
  for (int c = lane; c < N; c += 32) {
    const float v = lse_parts[static_cast<int64_t>(c) * nrows + row];
    wsum += (v > -INFINITY) ? expf(v - M) : 0.f;
  }
  const float den = warp_sumf(wsum);
  float acc[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) acc[k] = 0.f;
  if (!bad && den > 0.f) {
    for (int c = 0; c < N; ++c) {
      const float v = lse_parts[static_cast<int64_t>(c) * nrows + row];
      if (!(v > -INFINITY)) continue;
      const float w = expf(v - M);
      const T* src = o_parts + (static_cast<int64_t>(c) * nrows + row) * D;
#pragma unroll
      for (int k = 0; k < DL; ++k) acc[k] = fmaf(w, to_f32(src[lane + 32 * k]), acc[k]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* dst = out + row * D;
#pragma unroll
  for (int k = 0; k < DL; ++k) dst[lane + 32 * k] = static_cast<T>(bad ? NAN : acc[k] * inv);
  if (lse && lane == 0) lse[row] = bad ? NAN : (den > 0.f ? M + logf(den) : -INFINITY);
}

// ------------------------------------------------------------ launchers

template <typename T, int D>
static cudaError_t launch_prefix_t(const AttnParams& p, cudaStream_t s) {
  if (p.nchunk == 0 || p.B == 0 || p.T == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * (kSimtMaxRows * D + kSimtKeys * (D + 1) + kSimtKeys * D);
  cudaError_t e = cudaFuncSetAttribute(attn_prefix_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + p.node_tile - 1) / p.node_tile;
  dim3 grid(p.nchunk, ntiles, p.B * p.Hkv);
  attn_prefix_simt_kernel<T, D><<<grid, kSimtThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_tree_t(const AttnParams& p, cudaStream_t s) {
  if (p.B == 0 || p.T == 0) return cudaSuccess;
  const size_t smem = sizeof(int) * static_cast<size_t>(p.T);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_tree_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.T, p.B * p.Hkv);
  attn_tree_kernel<T, D><<<grid, kTreeThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_merge_t(const AttnParams& p, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.T * p.Hq;
  if (rows == 0) return cudaSuccess;
  const int per = 256 / 32;
  attn_merge_kernel<T, D><<<static_cast<unsigned>((rows + per - 1) / per), 256, 0, s>>>(p);
  return cudaGetLastError();
}

#define TV_DISPATCH_D(FN, T_, p, s)                         \
  switch ((p).d) {                                          \
    case 32: return FN<T_, 32>(p, s);                       \
    case 64: return FN<T_, 64>(p, s);                       \
    case 128: return FN<T_, 128>(p, s);                     \
    default: return cudaErrorInvalidValue;                  \
  }

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s) {
  if (p.dtype == TV_BF16) { TV_DISPATCH_D(launch_prefix_t, __nv_bfloat16, p, s) }
  TV_DISPATCH_D(launch_prefix_t, float, p, s)
}
cudaError_t launch_attn_tree(const AttnParams& p, cudaStream_t s) {
  if (p.dtype == TV_BF16) { TV_DISPATCH_D(launch_tree_t, __nv_bfloat16, p, s) }
  TV_DISPATCH_D(launch_tree_t, float, p, s)
}
cudaError_t launch_attn_merge(const AttnParams& p, cudaStream_t s) {
  if (p.dtype == TV_BF16) { TV_DISPATCH_D(launch_merge_t, __nv_bfloat16, p, s) }
  TV_DISPATCH_D(launch_merge_t, float, p, s)
}

template <typename T, int D>
static cudaError_t launch_partial_merge_t(const tv_attn_merge_args* a, cudaStream_t s) {
  const int64_t nrows = static_cast<int64_t>(a->B) * a->T * a->Hq;
  const int64_t blocks = (nrows + 7) / 8;
  attn_partial_merge_kernel<T, D><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const T*>(a->o_parts), a->lse_parts, static_cast<T*>(a->out), a->lse, a->N, nrows);
  return cudaGetLastError();
}

cudaError_t launch_attn_partial_merge(const tv_attn_merge_args* a, cudaStream_t s) {
  if (a->dtype == TV_BF16) {
    if (a->d == 128) return launch_partial_merge_t<__nv_bfloat16, 128>(a, s);
    if (a->d == 64) return launch_partial_merge_t<__nv_bfloat16, 64>(a, s);
    return launch_partial_merge_t<__nv_bfloat16, 32>(a, s);
  }
  if (a->d == 128) return launch_partial_merge_t<float, 128>(a, s);
  if (a->d == 64) return launch_partial_merge_t<float, 64>(a, s);
  return launch_partial_merge_t<float, 32>(a, s);
}

}  // namespace tv
