// Block top-k sparse verification attention ("Accelerate Speculative Decoding
// with Sparse Computation in Verification", "Methodology" 3, attention
// sparsity: keep only the top-k keys/values per query in structured blocks,
// chosen by a cheap relevance score).
//
//   block_means_kernel   kbar[b][j][g] = mean of the valid keys of prefix
//                        block j (one read of the K cache);
//   block_select_kernel  one CTA per (sequence, node, kv head): the cheap
//                        score of every block, sum over the group's query
//                        heads of <q_h, kbar_j> (computed as <sum_h q_h,
//                        kbar_j>), and a radix select of the top-k by
//                        (score desc, block asc); the kept ids are written
//                        in ascending order;
//   attn_sparse_kernel   the online softmax of the group's query heads over
//                        the kept blocks' keys (its partial joins the tree
//                        path's partial in the log-sum-exp merge).
#include "attn.cuh"

namespace tv {

template <typename T>
__device__ __forceinline__ float lde(const void* base, int64_t off) {
  return to_f32(static_cast<const T*>(base)[off]);
}

template <typename T>
__global__ void block_means_kernel(AttnParams p, float* kbar) {
  const int j = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int dd = threadIdx.x;
  if (dd >= p.d) return;
  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;
  const int lo = j * p.block_size, hi = min(lo + p.block_size, L);
  float* out = kbar + ((static_cast<int64_t>(b) * p.nblk_max + j) * p.Hkv + g) * p.d + dd;
  if (lo >= hi) { *out = 0.f; return; }
  float s = 0.f;
  for (int t = lo; t < hi; ++t)
    s += lde<T>(p.kc, b * p.kv_sb + static_cast<int64_t>(t) * p.kv_sl + g * p.kv_sh + dd);
  *out = s / static_cast<float>(hi - lo);
}

constexpr int kSelThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSelThreads) block_select_kernel(AttnParams p) {
  extern __shared__ float sc[];                    // [nblk] scores, then qsum[d]
  __shared__ uint32_t hist[256];
  __shared__ int bc[4];
  __shared__ int cnt;
  const int i = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T || i >= n) return;
  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;
  const int nblk = (L + p.block_size - 1) / p.block_size;
  const int k = p.topk;
  int32_t* sel = p.sel + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * k;
  float* qsum = sc + p.nblk_max;
  for (int dd = tid; dd < p.d; dd += blockDim.x) {
    float s = 0.f;
    for (int hg = 0; hg < p.G; ++hg)
      s += lde<T>(p.q, b * p.q_sb + i * p.q_st + (g * p.G + hg) * p.q_sh + dd);
    qsum[dd] = s;
  }
  __syncthreads();
  // one warp per block score
  for (int j = warp; j < nblk; j += blockDim.x >> 5) {
    const float* kb = p.kbar + ((static_cast<int64_t>(b) * p.nblk_max + j) * p.Hkv + g) * p.d;
    float s = 0.f;
    for (int dd = lane; dd < p.d; dd += 32) s = fmaf(qsum[dd], kb[dd], s);
    s = warp_sumf(s);
    if (lane == 0) sc[j] = s;
  }
  __syncthreads();
  if (nblk <= k) {
    for (int t = tid; t < k; t += blockDim.x) sel[t] = t < nblk ? t : -1;
  } else {
    // radix select of the k-th smallest descending key; ties by block index
    uint32_t prefix = 0, mask = 0;
    int need = k;
    for (int pass = 0; pass < 4; ++pass) {
      const int sh = 24 - 8 * pass;
      for (int t = tid; t < 256; t += blockDim.x) hist[t] = 0;
      __syncthreads();
      for (int j = tid; j < nblk; j += blockDim.x) {
        const uint32_t key = ~f32_key(sc[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        int ls = 0;
        for (int q = 0; q < 8; ++q) ls += static_cast<int>(hist[lane * 8 + q]);
        int incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const int excl = incl - ls;
        if (excl < need && need <= incl) {
          int cum = excl;
          for (int q = 0; q < 8; ++q) {
            const int h = static_cast<int>(hist[lane * 8 + q]);
            if (need <= cum + h) { bc[0] = lane * 8 + q; bc[1] = cum; bc[2] = h; break; }
            cum += h;
          }
        }
      }
      __syncthreads();
      need -= bc[1];
      prefix |= static_cast<uint32_t>(bc[0]) << sh;
      mask |= 0xFFu << sh;
      __syncthreads();
    }
    // keep keys below the threshold and the first `need` ties by block index:
    // mark in the score array (ascending scan keeps ids ordered)
    const uint32_t theta = prefix;
    if (tid == 0) {
      int taken = 0, w = 0, ties = 0;
      for (int j = 0; j < nblk; ++j) {
        const uint32_t key = ~f32_key(sc[j]);
        if ((key < theta || (key == theta && ties < need)) && w < k) {
          if (key == theta) ++ties;
          sel[w++] = j;
          ++taken;
        }
      }
      cnt = taken;
    }
    __syncthreads();
  }
  if (p.sel_out) {
    int32_t* so = p.sel_out + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * k;
    __syncthreads();
    for (int t = tid; t < k; t += blockDim.x) so[t] = sel[t];
  }
}

// Online softmax of the G query heads of (b, i, g) over the kept blocks.
template <typename T, int D>
__global__ void __launch_bounds__(128) attn_sparse_kernel(AttnParams p) {
  constexpr int DL = D / 32;
  const int i = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T || i >= n) return;
  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;
  const int32_t* sel = p.sel + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * p.topk;
  for (int hg = warp; hg < p.G; hg += blockDim.x >> 5) {
    const int h = g * p.G + hg;
    float qv[DL], acc[DL];
#pragma unroll
    for (int q = 0; q < DL; ++q) {
      qv[q] = lde<T>(p.q, b * p.q_sb + i * p.q_st + h * p.q_sh + lane + 32 * q) * p.scale;
      acc[q] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < p.topk; ++t) {
      const int j = sel[t];
      if (j < 0) break;
      const int lo = j * p.block_size, hi = min(lo + p.block_size, L);
      for (int pos = lo; pos < hi; ++pos) {
        const int64_t off = b * p.kv_sb + static_cast<int64_t>(pos) * p.kv_sl + g * p.kv_sh;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < DL; ++q) s = fmaf(qv[q], lde<T>(p.kc, off + lane + 32 * q), s);
        s = warp_sumf(s);
        const float mn = fmaxf(m, s);
        const float corr = expf(m - mn);
        const float pj = expf(s - mn);
        l = l * corr + pj;
#pragma unroll
        for (int q = 0; q < DL; ++q) acc[q] = fmaf(pj, lde<T>(p.vc, off + lane + 32 * q), acc[q] * corr);
        m = mn;
      }
    }
    const int64_t pr = part_row(p, 0, b, i, h);
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int q = 0; q < DL; ++q) p.part_o[pr * D + lane + 32 * q] = acc[q] * inv;
    if (lane == 0) p.part_lse[pr] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

cudaError_t launch_block_means(const AttnParams& p, float* kbar, cudaStream_t s) {
  if (p.nblk_max == 0) return cudaSuccess;
  dim3 grid(p.nblk_max, p.B * p.Hkv);
  if (p.dtype == TV_BF16) block_means_kernel<__nv_bfloat16><<<grid, p.d, 0, s>>>(p, kbar);
  else block_means_kernel<float><<<grid, p.d, 0, s>>>(p, kbar);
  return cudaGetLastError();
}

cudaError_t launch_block_select(const AttnParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (static_cast<size_t>(p.nblk_max) + p.d);
  dim3 grid(p.T, p.B * p.Hkv);
  cudaError_t e;
  if (p.dtype == TV_BF16) {
    e = cudaFuncSetAttribute(block_select_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_select_kernel<__nv_bfloat16><<<grid, kSelThreads, smem, s>>>(p);
  } else {
    e = cudaFuncSetAttribute(block_select_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_select_kernel<float><<<grid, kSelThreads, smem, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_sparse_t(const AttnParams& p, cudaStream_t s) {
  dim3 grid(p.T, p.B * p.Hkv);
  switch (p.d) {
    case 32: attn_sparse_kernel<T, 32><<<grid, 128, 0, s>>>(p); break;
    case 64: attn_sparse_kernel<T, 64><<<grid, 128, 0, s>>>(p); break;
    case 128: attn_sparse_kernel<T, 128><<<grid, 128, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_sparse(const AttnParams& p, cudaStream_t s) {
  if (p.dtype == TV_BF16) return launch_sparse_t<__nv_bfloat16>(p, s);
  return launch_sparse_t<float>(p, s);
}

}  // namespace tv
