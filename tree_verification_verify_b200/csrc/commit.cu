// tree_commit_kv kernel: append each sequence's accepted path to its K/V
// cache and advance prefix_len.
//
// The tokens accepted by one verification iteration become prefix for the
// next one (SpecExec page, "Approach"; "Key results" count accepted tokens
// per target iteration).  Path row r (r = 0 the root, then the accepted
// nodes in path order) goes to cache row prefix_len + r, for K and V and
// every kv head; prefix_len grows by the path length.
//
// Layout of the copy.  One CTA per sequence.  The path's (row, kv head)
// vectors of d elements are taken in row-major order, in chunks that fill a
// 16 KB shared-memory buffer per tensor: every thread loads its words of the
// chunk, the block synchronises, then stores them.  A chunk's reads all come
// before its writes, and a later chunk only reads rows at or after those
// earlier chunks wrote (path nodes increase, so node r of the path is >= r):
// a tree kept in the cache itself at rows >= prefix_len is therefore
// compacted in place.  Words are 16, 4 or 2 bytes, the widest that every
// base, stride and vector length allows.
#include "tv_common.cuh"

namespace tv {

struct CommitParams {
  int B, T, Hkv, d, Lmax, esize;
  char* kc;
  char* vc;
  int64_t kv_sb, kv_sl, kv_sh;            // element strides
  int32_t* prefix_len;
  const char* kt;
  const char* vt;
  int64_t kt_sb, kt_st, kt_sh;
  const int32_t* n_acc;
  const int32_t* acc;
  int64_t acc_sb;
  uint32_t* status;
};

constexpr int kCommitThreads = 256;
constexpr int kCommitBufBytes = 16384;    // per tensor

template <typename W>
__global__ void __launch_bounds__(kCommitThreads) commit_kv_kernel(CommitParams p) {
  __shared__ __align__(16) unsigned char buf[2 * kCommitBufBytes];
  __shared__ int s_L, s_n, s_ok;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) {
    const int L = p.prefix_len[b];
    const int n = p.n_acc[b];
    const bool ok = n >= 0 && n <= p.T - 1 && L >= 0 && L <= p.Lmax &&
                    static_cast<int64_t>(L) + n + 1 <= p.Lmax;
    if (!ok) set_status(p.status, TV_DEV_BAD_LEN);
    s_L = L;
    s_n = n;
    s_ok = ok ? 1 : 0;
  }
  __syncthreads();
  if (!s_ok) return;
  const int L = s_L, n = s_n;
  const int32_t* acc = p.acc + static_cast<int64_t>(b) * p.acc_sb;
  // the path: nodes in [1, T), strictly increasing
  int bad = 0;
  for (int r = tid; r < n; r += blockDim.x) {
    const int x = acc[r];
    if (x < 1 || x >= p.T || (r > 0 && acc[r - 1] >= x)) bad = 1;
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) set_status(p.status, TV_DEV_BAD_ROW);
    return;
  }
  const int wpu = p.d * p.esize / static_cast<int>(sizeof(W));                // words per vector
  const int upc = kCommitBufBytes / static_cast<int>(sizeof(W)) / wpu;        // vectors per chunk
  const int total = (n + 1) * p.Hkv;
  W* bk = reinterpret_cast<W*>(buf);
  W* bv = reinterpret_cast<W*>(buf + kCommitBufBytes);
  const int64_t es = p.esize;
  for (int u0 = 0; u0 < total; u0 += upc) {
    const int cnt = min(upc, total - u0) * wpu;
    for (int i = tid; i < cnt; i += blockDim.x) {
      const int u = u0 + i / wpu, w = i % wpu;
      const int r = u / p.Hkv, g = u % p.Hkv;
      const int x = (r == 0) ? 0 : acc[r - 1];
      const int64_t off = (static_cast<int64_t>(b) * p.kt_sb + static_cast<int64_t>(x) * p.kt_st +
                           static_cast<int64_t>(g) * p.kt_sh) * es;
      bk[i] = reinterpret_cast<const W*>(p.kt + off)[w];
      bv[i] = reinterpret_cast<const W*>(p.vt + off)[w];
    }
    __syncthreads();
    for (int i = tid; i < cnt; i += blockDim.x) {
      const int u = u0 + i / wpu, w = i % wpu;
      const int r = u / p.Hkv, g = u % p.Hkv;
      const int64_t off = (static_cast<int64_t>(b) * p.kv_sb + static_cast<int64_t>(L + r) * p.kv_sl +
                           static_cast<int64_t>(g) * p.kv_sh) * es;
      reinterpret_cast<W*>(p.kc + off)[w] = bk[i];
      reinterpret_cast<W*>(p.vc + off)[w] = bv[i];
    }
    __syncthreads();
  }
  if (tid == 0) p.prefix_len[b] = L + n + 1;
}

namespace {
bool aligned_to(const tv_commit_args* a, int esize, int w) {
  const uintptr_t ptrs[4] = {reinterpret_cast<uintptr_t>(a->k_cache), reinterpret_cast<uintptr_t>(a->v_cache),
                             reinterpret_cast<uintptr_t>(a->k_tree), reinterpret_cast<uintptr_t>(a->v_tree)};
  for (uintptr_t x : ptrs)
    if (x % static_cast<uintptr_t>(w) != 0) return false;
  const int64_t strides[6] = {a->kv_sb, a->kv_sl, a->kv_sh, a->kt_sb, a->kt_st, a->kt_sh};
  for (int64_t s : strides)
    if ((s * esize) % w != 0) return false;
  return (static_cast<int64_t>(a->d) * esize) % w == 0;
}
}  // namespace

// Word size the copy uses for these arguments (16, 4 or 2 bytes).
int commit_word_bytes(const tv_commit_args* a) {
  const int esize = a->dtype == TV_BF16 ? 2 : 4;
  if (aligned_to(a, esize, 16)) return 16;
  if (aligned_to(a, esize, 4)) return 4;
  return 2;
}

cudaError_t launch_commit(const tv_commit_args* a, cudaStream_t stream) {
  CommitParams p;
  p.B = a->B; p.T = a->T; p.Hkv = a->Hkv; p.d = a->d; p.Lmax = a->Lmax;
  p.esize = a->dtype == TV_BF16 ? 2 : 4;
  p.kc = static_cast<char*>(a->k_cache);
  p.vc = static_cast<char*>(a->v_cache);
  p.kv_sb = a->kv_sb; p.kv_sl = a->kv_sl; p.kv_sh = a->kv_sh;
  p.prefix_len = a->prefix_len;
  p.kt = static_cast<const char*>(a->k_tree);
  p.vt = static_cast<const char*>(a->v_tree);
  p.kt_sb = a->kt_sb; p.kt_st = a->kt_st; p.kt_sh = a->kt_sh;
  p.n_acc = a->n_accepted;
  p.acc = a->accepted_nodes;
  p.acc_sb = a->acc_sb;
  p.status = a->dev_status;
  const dim3 grid(static_cast<unsigned>(a->B)), block(kCommitThreads);
  switch (commit_word_bytes(a)) {
    case 16: commit_kv_kernel<uint4><<<grid, block, 0, stream>>>(p); break;
    case 4: commit_kv_kernel<uint32_t><<<grid, block, 0, stream>>>(p); break;
    default: commit_kv_kernel<uint16_t><<<grid, block, 0, stream>>>(p); break;
  }
  return cudaGetLastError();
}

}  // namespace tv
