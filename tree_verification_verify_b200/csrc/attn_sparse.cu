// Block top-k sparse verification attention ("Accelerate Speculative Decoding
// with Sparse Computation in Verification", "Methodology" 3, attention
// sparsity: keep only the top-k keys/values per query in structured blocks,
// chosen by a cheap relevance score).
//
//   block_means_kernel   kbar[b][j][g] = mean of the valid keys of prefix
//                        block j (one read of the K cache);
//   block_scores_kernel  the cheap score of every (node, block): the sum
//                        over the group's query heads of <q_h, kbar_j>,
//                        computed as <sum_h q_h, kbar_j>, as a tiled
//                        [nodes x d] x [d x blocks] product per (sequence,
//                        kv head);
//   block_select_kernel  one CTA per (sequence, node, kv head): a radix
//                        select of the top-k scores by (score desc, block
//                        asc); the kept ids are written in ascending order;
//   attn_sparse_kernel   the online softmax of the group's query heads over
//                        the kept blocks' keys, streamed through shared
//                        memory in tiles of 64 keys (its partial joins the
//                        tree path's partial in the log-sum-exp merge).
#include "attn.cuh"

namespace tv {

__device__ __forceinline__ float ex2_approx_f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T>
__device__ __forceinline__ float lde(const void* base, int64_t off) {
  return to_f32(static_cast<const T*>(base)[off]);
}

// One CTA of 256 threads per (block, sequence, kv head): thread t sums the
// 16-byte chunk t % nch of the keys t / nch, t / nch + 256 / nch, ... (plain
// element loads when the rows are not 16-byte aligned), then the partial
// sums of each chunk are added in shared memory in key-group order.
template <typename T>
__global__ void __launch_bounds__(256) block_means_kernel(AttnParams p, float* kbar) {
  __shared__ float part[256 * 8];
  const int j = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int tid = threadIdx.x;
  constexpr int E = 16 / sizeof(T);              // elements per 16-byte chunk
  const int nch = p.d / E;                        // chunks per key row (d = 32, 64, 128)
  const int groups = 256 / nch;
  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;
  const int lo = j * p.block_size, hi = min(lo + p.block_size, L);
  float* out = kbar + ((static_cast<int64_t>(b) * p.nblk_max + j) * p.Hkv + g) * p.d;
  const T* kc = static_cast<const T*>(p.kc);
  const bool vec = (reinterpret_cast<uintptr_t>(kc) & 15u) == 0 &&
                   ((p.kv_sb | p.kv_sl | p.kv_sh) * static_cast<int64_t>(sizeof(T))) % 16 == 0;
  const int c = tid % nch, kg = tid / nch;
  float acc[E];
#pragma unroll
  for (int x = 0; x < E; ++x) acc[x] = 0.f;
  if (kg < groups) {
    // four keys' loads in flight per batch (added in key order)
    for (int t0 = lo + kg; t0 < hi; t0 += 4 * groups) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * groups;
        const int64_t off = b * p.kv_sb + static_cast<int64_t>(t) * p.kv_sl + g * p.kv_sh + c * E;
        if (t < hi && vec) raw[u] = __ldg(reinterpret_cast<const uint4*>(kc + off));
        else raw[u] = make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * groups;
        if (t >= hi) break;
        if (vec) {
          const T* ev = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
          for (int x = 0; x < E; ++x) acc[x] += to_f32(ev[x]);
        } else {
          const int64_t off = b * p.kv_sb + static_cast<int64_t>(t) * p.kv_sl + g * p.kv_sh + c * E;
#pragma unroll
          for (int x = 0; x < E; ++x) acc[x] += to_f32(kc[off + x]);
        }
      }
    }
  }
#pragma unroll
  for (int x = 0; x < E; ++x) part[tid * E + x] = acc[x];
  __syncthreads();
  for (int dd = tid; dd < p.d; dd += blockDim.x) {
    const int cc = dd / E, x = dd % E;
    float sum = 0.f;
    for (int q = 0; q < groups; ++q) sum += part[(q * nch + cc) * E + x];
    out[dd] = (lo < hi) ? sum / static_cast<float>(hi - lo) : 0.f;
  }
}

// Cheap block scores of every (node, block) of a (sequence, kv head): the
// [nodes x d] matrix of summed group queries times the [d x blocks] block
// means, in tiles of 64 nodes x 64 blocks (256 threads, 4 x 4 outputs per
// thread, operands d-major in shared memory).  Each score is one fp32 dot
// product over d in order.
constexpr int kScTile = 64;
constexpr int kScPad = kScTile + 4;        // row stride of the d-major operands (fewer bank conflicts)

template <typename T>
__global__ void __launch_bounds__(256) block_scores_kernel(AttnParams p) {
  extern __shared__ float scs[];                     // Qs[d][kScPad], Ks[d][kScPad]
  float* Qs = scs;
  float* Ks = scs + p.d * kScPad;
  const int j0 = blockIdx.x * kScTile;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int i0 = blockIdx.z * kScTile;
  const int tid = threadIdx.x;
  constexpr int E = 16 / sizeof(T);
  const T* qp = static_cast<const T*>(p.q);
  const bool qvec = (reinterpret_cast<uintptr_t>(qp) & 15u) == 0 &&
                    ((p.q_sb | p.q_st | p.q_sh) * static_cast<int64_t>(sizeof(T))) % 16 == 0;
  const int nch = p.d / E;
  for (int e = tid; e < kScTile * nch; e += blockDim.x) {
    const int r = e % kScTile, c = e / kScTile;     // consecutive threads: consecutive rows
    float qsum[E];
#pragma unroll
    for (int x = 0; x < E; ++x) qsum[x] = 0.f;
    if (i0 + r < p.T)
      for (int hg = 0; hg < p.G; ++hg) {
        const int64_t off = b * p.q_sb + static_cast<int64_t>(i0 + r) * p.q_st + (g * p.G + hg) * p.q_sh + c * E;
        if (qvec) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qp + off));
          const T* ev = reinterpret_cast<const T*>(&raw);
#pragma unroll
          for (int x = 0; x < E; ++x) qsum[x] += to_f32(ev[x]);
        } else {
#pragma unroll
          for (int x = 0; x < E; ++x) qsum[x] += to_f32(qp[off + x]);
        }
      }
#pragma unroll
    for (int x = 0; x < E; ++x) Qs[(c * E + x) * kScPad + r] = qsum[x];
  }
  for (int e = tid; e < kScTile * p.d; e += blockDim.x) {
    const int r = e / p.d, dd = e % p.d;
    float kb = 0.f;
    if (j0 + r < p.nblk_max) kb = p.kbar[((static_cast<int64_t>(b) * p.nblk_max + j0 + r) * p.Hkv + g) * p.d + dd];
    Ks[dd * kScPad + r] = kb;
  }
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
  for (int dd = 0; dd < p.d; ++dd) {
    const float4 qa = *reinterpret_cast<const float4*>(Qs + dd * kScPad + ty * 4);
    const float4 kb = *reinterpret_cast<const float4*>(Ks + dd * kScPad + tx * 4);
    const float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(qv[a], kv[c], acc[a][c]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty * 4 + a;
    if (i >= p.T) continue;
    float* dst = p.scores + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * p.nblk_max;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j < p.nblk_max) dst[j] = acc[a][c];
    }
  }
}

constexpr int kSelThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSelThreads) block_select_kernel(AttnParams p) {
  extern __shared__ float sc[];                    // [nblk] scores, then qsum[d]
  __shared__ uint32_t hist[256];
  __shared__ int bc[4];
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
  const float* srow = p.scores + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * p.nblk_max;
  for (int j = tid; j < nblk; j += blockDim.x) sc[j] = srow[j];
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
    // ordered compaction, one block-wide pass per 256 blocks: ties are
    // ranked by block index, the kept ids keep ascending order
    const uint32_t theta = prefix;
    const unsigned lanemask = (1u << lane) - 1u;
    int ties_before = 0, taken_before = 0;
    for (int base = 0; base < nblk; base += blockDim.x) {
      const int j = base + tid;
      const uint32_t key = (j < nblk) ? ~f32_key(sc[j]) : ~0u;
      const bool lt = (j < nblk) && key < theta;
      const bool tie = (j < nblk) && key == theta;
      const unsigned mt = __ballot_sync(0xffffffffu, tie);
      if (lane == 0) hist[warp] = __popc(mt);
      __syncthreads();
      if (tid == 0) {
        int a = 0;
        for (int w = 0; w < (kSelThreads >> 5); ++w) { const int c = hist[w]; hist[w] = a; a += c; }
        hist[32] = a;
      }
      __syncthreads();
      const bool take = lt || (tie && ties_before + static_cast<int>(hist[warp]) + __popc(mt & lanemask) < need);
      const int tie_total = hist[32];
      const unsigned mk = __ballot_sync(0xffffffffu, take);
      __syncthreads();
      if (lane == 0) hist[64 + warp] = __popc(mk);
      __syncthreads();
      if (tid == 0) {
        int a = 0;
        for (int w = 0; w < (kSelThreads >> 5); ++w) { const int c = hist[64 + w]; hist[64 + w] = a; a += c; }
        hist[96] = a;
      }
      __syncthreads();
      if (take) {
        const int pos = taken_before + static_cast<int>(hist[64 + warp]) + __popc(mk & lanemask);
        if (pos < k) sel[pos] = j;
      }
      taken_before += hist[96];
      ties_before += tie_total;
      __syncthreads();
    }
  }
  if (p.sel_out) {
    int32_t* so = p.sel_out + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * k;
    __syncthreads();
    for (int t = tid; t < k; t += blockDim.x) so[t] = sel[t];
  }
}

// Online softmax of the G query heads of (b, i, g) over the kept blocks.
// The kept blocks are streamed in tiles of up to 64 keys: K and V rows go to
// shared memory with cp.async (two buffers, 16-byte chunks XOR-swizzled by
// row), then each warp scores its heads' 64 keys lane-per-key (lane l: keys
// l and l + 32), updates the base-2 online softmax once per tile and adds
// P V with lane l owning dimensions [l D/32, (l + 1) D/32).
constexpr int kSpTile = 64;

template <typename T, int D>
struct SpTile {
  static constexpr int kNch = D * static_cast<int>(sizeof(T)) / 16;     // 16-byte chunks per row
  static constexpr int kSwz = (kNch < 8 ? kNch : 8) - 1;
  static constexpr int kRowBytes = D * static_cast<int>(sizeof(T));
  static constexpr int kBytes = kSpTile * kRowBytes;                    // one of K or V
};

template <typename T, int D, int HPW>
__global__ void __launch_bounds__(512) attn_sparse_kernel(AttnParams p) {
  using TL = SpTile<T, D>;
  constexpr int DL = D / 32;
  extern __shared__ __align__(16) uint8_t sp_smem[];
  uint8_t* kv = sp_smem;                                      // [2][K tile, V tile]
  float* qs = reinterpret_cast<float*>(sp_smem + 4 * TL::kBytes);   // [G][D] scaled queries
  const int i = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T || i >= n) return;
  int L = p.prefix_len[b];
  if (L < 0 || L > p.Lmax) L = 0;
  const int32_t* sel = p.sel + ((static_cast<int64_t>(b) * p.T + i) * p.Hkv + g) * p.topk;
  const float sl2 = p.scale * 1.4426950408889634f;
  for (int e = tid; e < p.G * D; e += blockDim.x) {
    const int hg = e / D, dd = e % D;
    qs[e] = lde<T>(p.q, b * p.q_sb + i * p.q_st + (g * p.G + hg) * p.q_sh + dd) * sl2;
  }
  const T* kc = static_cast<const T*>(p.kc);
  const T* vc = static_cast<const T*>(p.vc);
  const int64_t kvbase = b * p.kv_sb + g * p.kv_sh;
  const bool vec = ((reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc)) & 15u) == 0 &&
                   ((p.kv_sb | p.kv_sl | p.kv_sh) * static_cast<int64_t>(sizeof(T))) % 16 == 0;
  // tile enumeration: kept block t, keys [pos0, pos0 + 64) of it
  auto tile_keys = [&](int t, int pos0) { return min(kSpTile, min((sel[t] + 1) * p.block_size, L) - pos0); };
  auto next_tile = [&](int& t, int& pos0) {
    pos0 += kSpTile;
    if (t < p.topk && sel[t] >= 0 && pos0 < min((sel[t] + 1) * p.block_size, L)) return;
    ++t;
    pos0 = (t < p.topk && sel[t] >= 0) ? sel[t] * p.block_size : 0;
  };
  auto valid_tile = [&](int t) { return t < p.topk && sel[t] >= 0; };
  auto load_tile = [&](int buf, int t, int pos0) {
    const int nk = tile_keys(t, pos0);
    uint8_t* kd = kv + buf * 2 * TL::kBytes;
    uint8_t* vd = kd + TL::kBytes;
    for (int e = tid; e < nk * TL::kNch; e += blockDim.x) {
      const int r = e / TL::kNch, c = e % TL::kNch;
      const uint32_t off = r * TL::kRowBytes + ((c ^ (r & TL::kSwz)) << 4);
      const int64_t src = kvbase + static_cast<int64_t>(pos0 + r) * p.kv_sl + c * (16 / sizeof(T));
      if (vec) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(kd + off))),
                     "l"(kc + src) : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(vd + off))),
                     "l"(vc + src) : "memory");
      } else {
        for (int u = 0; u < static_cast<int>(16 / sizeof(T)); ++u) {
          reinterpret_cast<T*>(kd + off)[u] = kc[src + u];
          reinterpret_cast<T*>(vd + off)[u] = vc[src + u];
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float m[HPW], l[HPW], acc[HPW][DL];
#pragma unroll
  for (int u = 0; u < HPW; ++u) {
    m[u] = -INFINITY;
    l[u] = 0.f;
#pragma unroll
    for (int q = 0; q < DL; ++q) acc[u][q] = 0.f;
  }
  int t = 0, pos0 = valid_tile(0) ? sel[0] * p.block_size : 0;
  if (valid_tile(0) && tile_keys(0, pos0) <= 0) next_tile(t, pos0);
  int buf = 0;
  if (valid_tile(t)) load_tile(0, t, pos0);
  while (valid_tile(t)) {
    int tn = t, pn = pos0;
    next_tile(tn, pn);
    if (valid_tile(tn)) load_tile(buf ^ 1, tn, pn);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const int nk = tile_keys(t, pos0);
    const uint8_t* kd = kv + buf * 2 * TL::kBytes;
    const uint8_t* vd = kd + TL::kBytes;
#pragma unroll
    for (int u = 0; u < HPW; ++u) {
      const int hg = warp + u * nwarps;
      if (hg >= p.G) break;
      const float* qh = qs + hg * D;
      // scores of keys lane and lane + 32
      float sc[2];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int r = lane + 32 * kk;
        float sdot = 0.f;
        if (r < nk) {
#pragma unroll
          for (int c = 0; c < TL::kNch; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4*>(kd + r * TL::kRowBytes + ((c ^ (r & TL::kSwz)) << 4));
            constexpr int E = 16 / sizeof(T);
            const T* ev = reinterpret_cast<const T*>(&raw);
            const float4* q4 = reinterpret_cast<const float4*>(qh + c * E);
#pragma unroll
            for (int x4 = 0; x4 < E / 4; ++x4) {
              const float4 qq = q4[x4];
              sdot = fmaf(qq.x, to_f32(ev[4 * x4 + 0]), sdot);
              sdot = fmaf(qq.y, to_f32(ev[4 * x4 + 1]), sdot);
              sdot = fmaf(qq.z, to_f32(ev[4 * x4 + 2]), sdot);
              sdot = fmaf(qq.w, to_f32(ev[4 * x4 + 3]), sdot);
            }
          }
        }
        sc[kk] = (r < nk) ? sdot : -INFINITY;
      }
      const float tmax = warp_max(fmaxf(sc[0], sc[1]));
      const float mn = fmaxf(m[u], tmax);
      const float corr = (m[u] == -INFINITY) ? 0.f : ex2_approx_f(m[u] - mn);
      const float p0 = ex2_approx_f(sc[0] - mn), p1 = ex2_approx_f(sc[1] - mn);
      l[u] = l[u] * corr + warp_sumf(p0 + p1);
      m[u] = mn;
#pragma unroll
      for (int q = 0; q < DL; ++q) acc[u][q] *= corr;
      // P V: lane owns dimensions [lane DL, lane DL + DL)
      for (int r = 0; r < nk; ++r) {
        const float pr = __shfl_sync(0xffffffffu, r < 32 ? p0 : p1, r & 31);
        const int byte = lane * DL * static_cast<int>(sizeof(T));
        const int c = byte >> 4, o = byte & 15;
        const T* vr = reinterpret_cast<const T*>(vd + r * TL::kRowBytes + ((c ^ (r & TL::kSwz)) << 4) + o);
#pragma unroll
        for (int q = 0; q < DL; ++q) acc[u][q] = fmaf(pr, to_f32(vr[q]), acc[u][q]);
      }
    }
    __syncthreads();                 // the buffer is refilled two tiles on
    t = tn; pos0 = pn; buf ^= 1;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int u = 0; u < HPW; ++u) {
    const int hg = warp + u * nwarps;
    if (hg >= p.G) break;
    const int h = g * p.G + hg;
    const int64_t pr = part_row(p, 0, b, i, h);
    const float inv = l[u] > 0.f ? 1.f / l[u] : 0.f;
#pragma unroll
    for (int q = 0; q < DL; ++q) p.part_o[pr * D + lane * DL + q] = acc[u][q] * inv;
    if (lane == 0) p.part_lse[pr] = l[u] > 0.f ? (m[u] + __log2f(l[u])) * 0.6931471805599453f : -INFINITY;
  }
}

cudaError_t launch_block_means(const AttnParams& p, float* kbar, cudaStream_t s) {
  if (p.nblk_max == 0) return cudaSuccess;
  dim3 grid(p.nblk_max, p.B * p.Hkv);
  if (p.dtype == TV_BF16) block_means_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p, kbar);
  else block_means_kernel<float><<<grid, 256, 0, s>>>(p, kbar);
  return cudaGetLastError();
}

cudaError_t launch_block_select(const AttnParams& p, cudaStream_t s) {
  cudaError_t e;
  if (p.nblk_max > 0) {
    const size_t ssm = 2 * sizeof(float) * static_cast<size_t>(p.d) * kScPad;
    dim3 sgrid((p.nblk_max + kScTile - 1) / kScTile, p.B * p.Hkv, (p.T + kScTile - 1) / kScTile);
    if (p.dtype == TV_BF16) {
      e = cudaFuncSetAttribute(block_scores_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(ssm));
      if (e != cudaSuccess) return e;
      block_scores_kernel<__nv_bfloat16><<<sgrid, 256, ssm, s>>>(p);
    } else {
      e = cudaFuncSetAttribute(block_scores_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(ssm));
      if (e != cudaSuccess) return e;
      block_scores_kernel<float><<<sgrid, 256, ssm, s>>>(p);
    }
  }
  const size_t smem = sizeof(float) * static_cast<size_t>(p.nblk_max);
  dim3 grid(p.T, p.B * p.Hkv);
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

template <typename T, int D, int HPW>
static cudaError_t launch_sparse_dh(const AttnParams& p, cudaStream_t s) {
  const int nwarps = p.G < 4 ? 4 : (p.G > 16 ? 16 : p.G);
  const size_t smem = 4 * static_cast<size_t>(SpTile<T, D>::kBytes) + static_cast<size_t>(p.G) * D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_sparse_kernel<T, D, HPW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(p.T, p.B * p.Hkv);
  attn_sparse_kernel<T, D, HPW><<<grid, nwarps * 32, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_sparse_d(const AttnParams& p, cudaStream_t s) {
  // heads per warp: G <= 16 one, up to 32 two, up to 64 four
  if (p.G <= 16) return launch_sparse_dh<T, D, 1>(p, s);
  if (p.G <= 32) return launch_sparse_dh<T, D, 2>(p, s);
  return launch_sparse_dh<T, D, 4>(p, s);
}

template <typename T>
static cudaError_t launch_sparse_t(const AttnParams& p, cudaStream_t s) {
  switch (p.d) {
    case 32: return launch_sparse_d<T, 32>(p, s);
    case 64: return launch_sparse_d<T, 64>(p, s);
    case 128: return launch_sparse_d<T, 128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_sparse(const AttnParams& p, cudaStream_t s) {
  if (p.dtype == TV_BF16) return launch_sparse_t<__nv_bfloat16>(p, s);
  return launch_sparse_t<float>(p, s);
}

}  // namespace tv
