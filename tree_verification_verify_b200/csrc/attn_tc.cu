// tree_verify_attn, tensor-core kernel for sm_100a (tcgen05 + TMEM + TMA),
// bf16 with d = 128.
//
// Tree attention (SpecExec page, "Approach": the whole tree is verified in
// one target pass): node i attends to the shared prefix and to its root
// path.  The G query heads of one kv head are packed with the tree nodes
// into M = 128 query rows (row r = node r / G, head r % G); every K/V tile
// is loaded once for all nodes and heads of the tile (the "inter-draft-token
// reuse" of the sparse verification page, "Methodology" 4).
//
// One CTA owns (sequence, kv head, 128-row tile, prefix chunk).  Its key
// tiles are the chunk's prefix tiles of 128 keys and, in chunk 0, the tree
// tiles: the union U of the tile's nodes' root paths, gathered into K/V
// tiles and masked per row by an ancestor bitmask built in shared memory
// from parent[] (slot of node a in U = number of marked nodes below a in a
// node bitmap).  All tiles share one online softmax.  With a single chunk
// the CTA writes the final output; otherwise every chunk writes a partial
// (O, lse) and a merge kernel (one warp per output row) combines them.
//
// Warp roles (192 threads):
//   warps 0-3  softmax / correction / epilogue: thread t owns query row t,
//              which is TMEM lane t (tcgen05.ld 32x32b);
//   warp 4     producer: Q once, prefix K/V tiles by TMA into a two-stage
//              ring (128B-swizzled; K-major for K, MN-major for V), the
//              tree bookkeeping, and the gathered tree tiles (cp.async);
//   warp 5     TMEM allocator and MMA issuer (one thread): S = Q K^T into one
//              of two TMEM S buffers, O += P V into the TMEM O accumulator.
// Online softmax in base 2 with a lazily updated row maximum: O and the row
// sum are rescaled only when the maximum grows by more than 2^8, which keeps
// P <= 256 (exact in the final O / l).  P goes to shared memory as bf16 in
// the 128B-swizzled K-major layout the PV MMA reads.
//
// Every mbarrier wait is bounded: on expiry the CTA records TV_DEV_TIMEOUT,
// stops issuing work, drains what it issued and frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn.cuh"

namespace tv {

namespace tc {

constexpr int kThreads = 192;
constexpr int kRows = 128;          // M
constexpr int kKeys = 128;          // keys per tile (N of QK, K of PV)
constexpr int kD = 128;
constexpr int kStages = 2;
constexpr int kMaxT = 4096;         // tree nodes handled by this kernel
constexpr uint32_t kHalfBytes = kRows * 128;            // 128 rows x 128 B
constexpr uint32_t kTileBytes = 2 * kHalfBytes;         // 32 KB (d = 128 bf16)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemKV = kSmemQ + kTileBytes;       // stage s: K at +s*64K, V at +32K
constexpr uint32_t kSmemP = kSmemKV + kStages * 2 * kTileBytes;
constexpr uint32_t kSmemU = kSmemP + kTileBytes;        // U list (int32, kMaxT)
constexpr uint32_t kSmemBytes = kSmemU + kMaxT * 4;     // 208 KB
constexpr uint32_t kTmemCols = 512;                     // S0, S1, O (128 each)
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr uint32_t kWaitLimit = 1u << 22;

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t tree_info;
  uint32_t tmem_base;
  int abort;
  int nU;                           // nodes in the union of root paths
  int last;                         // this CTA merges the group
  uint32_t bm[kMaxT / 32];          // node bitmap of U
  int pre[kMaxT / 32];              // marked nodes below each bitmap word
  int node_ok[kRows];               // root path of the tile's node is well formed
};


__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
// Bounded wait on phase `parity`; false when the CTA aborted or the limit
// expired (then the abort flag is raised).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort) {
  const uint32_t a = smem_u32(b);
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((it & 255u) == 255u && *abort) return false;
  }
  *abort = 1;
  return false;
}

__device__ __forceinline__ void tma_load_4d(const CUtensorMap* map, uint32_t dst, uint64_t* bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor: 128B swizzle, version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, M x N.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Slot of node a in U: the number of marked nodes below a.
__device__ __forceinline__ int u_slot(const Bars& bars, int a) {
  return bars.pre[a >> 5] + __popc(bars.bm[a >> 5] & ((1u << (a & 31)) - 1u));
}

// Ancestor bitmask of node i (whose root path is well formed) over tree
// tile tt, i.e. the slots [128 tt, 128 tt + 128) of U.
__device__ __forceinline__ void tree_mask(const int32_t* par, int i, int tt, const Bars& bars, uint32_t* mk) {
  mk[0] = mk[1] = mk[2] = mk[3] = 0u;
  int j = i;
  for (int step = 0; step <= i; ++step) {
    const int sl = u_slot(bars, j);
    if ((sl >> 7) == tt) mk[(sl >> 5) & 3] |= 1u << (sl & 31);
    if (j == 0) break;
    j = par[j];
  }
}

// Whether node i's root path reaches node 0 through parent[j] in [0, j).
__device__ __forceinline__ bool path_ok(const int32_t* par, int i) {
  if (par[0] != -1) return false;
  int j = i;
  for (int step = 0; step <= i && j != 0; ++step) {
    const int pj = par[j];
    if (pj < 0 || pj >= j) return false;
    j = pj;
  }
  return true;
}

}  // namespace tc

using namespace tc;

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v, AttnParams p) {
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ Bars bars;
  const int chunk = blockIdx.x;
  const int tile = blockIdx.y;
  const int b = blockIdx.z / p.Hkv, g = blockIdx.z % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) {
    if (chunk == 0 && tile == 0 && g == 0 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
    return;
  }
  const int i0 = tile * (kRows / G);
  if (i0 >= n) return;
  const int32_t* par = p.parent + b * p.par_sb;
  const int Lraw = p.prefix_len[b];
  const bool bad_len = (Lraw < 0 || Lraw > p.Lmax);
  const int L = bad_len ? 0 : Lraw;
  const int k0 = chunk * p.chunk_len;
  const int k1 = min(k0 + p.chunk_len, L);
  const int nprefix = (k1 > k0) ? (k1 - k0 + kKeys - 1) / kKeys : 0;
  const int nodes_here = min(kRows / G, n - i0);
  // this thread's query row (softmax warps)
  const int row_node = i0 + tid / G;
  const int row_head = g * G + tid % G;
  const bool row_valid = tid < kRows && (tid / G) < nodes_here;

  // 1024-aligned dynamic shared memory (128B swizzle atoms are 1 KB)
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem_raw + (base - raw);
  int* ulist = reinterpret_cast<int*>(gbase + kSmemU);
  volatile int* abort = &bars.abort;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 1); }
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&bars.s_full[s], 1); mbar_init(&bars.s_free[s], 4); }
    mbar_init(&bars.p_full, 4);
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.tree_info, 1);
    bars.abort = 0;
    bars.nU = 0;
    bars.last = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars.tmem_base;
  const bool has_tree = (chunk == 0);

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    const int first = min(nprefix, kStages);
    if (lane == 0) {
      const uint32_t sq = base + kSmemQ;
      mbar_expect_tx(&bars.q_full, kTileBytes);
      tma_load_4d(&tmap_q, sq, &bars.q_full, 0, g * G, i0, b);
      tma_load_4d(&tmap_q, sq + kHalfBytes, &bars.q_full, 64, g * G, i0, b);
      for (int j = 0; j < first; ++j) {
        const uint32_t sk = base + kSmemKV + j * 2 * kTileBytes;
        const int kb = k0 + j * kKeys;
        mbar_expect_tx(&bars.full[j], 2 * kTileBytes);
        tma_load_4d(&tmap_k, sk, &bars.full[j], 0, g, kb, b);
        tma_load_4d(&tmap_k, sk + kHalfBytes, &bars.full[j], 64, g, kb, b);
        tma_load_4d(&tmap_v, sk + kTileBytes, &bars.full[j], 0, g, kb, b);
        tma_load_4d(&tmap_v, sk + kTileBytes + kHalfBytes, &bars.full[j], 64, g, kb, b);
      }
    }
    int ntree = 0;
    if (has_tree) {
      // union U of the root paths of this tile's nodes, as a node bitmap
      const int nw = (n + 31) >> 5;
      for (int w = lane; w < nw; w += 32) bars.bm[w] = 0u;
      __syncwarp();
      for (int r = lane; r < nodes_here; r += 32) {
        const int i = i0 + r;
        int ok = (par[0] == -1) ? 1 : 0;
        int j = i;
        for (int step = 0; step <= i; ++step) {
          atomicOr(&bars.bm[j >> 5], 1u << (j & 31));
          if (j == 0) break;
          const int pj = par[j];
          if (pj < 0 || pj >= j) { ok = 0; break; }
          j = pj;
        }
        bars.node_ok[r] = ok;
      }
      __syncwarp();
      // prefix counts per bitmap word, then the U list in node order
      const int per = (nw + 31) / 32;
      const int lo = min(lane * per, nw), hi = min(lo + per, nw);
      int cnt = 0;
      for (int w = lo; w < hi; ++w) cnt += __popc(bars.bm[w]);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int run = incl - cnt;
      for (int w = lo; w < hi; ++w) {
        bars.pre[w] = run;
        uint32_t m = bars.bm[w];
        while (m) {
          const int bit = __ffs(m) - 1;
          ulist[run++] = w * 32 + bit;
          m &= m - 1u;
        }
      }
      if (lane == 31) bars.nU = incl;
      __syncwarp();
      ntree = (bars.nU + kKeys - 1) / kKeys;
      if (lane == 0) mbar_arrive(&bars.tree_info);
    }
    const int ntot = nprefix + ntree;
    int issued = first;
    for (int j = first; j < ntot; ++j) {
      const int s = j % kStages;
      bool ok = true;
      if (j >= kStages) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&bars.empty[s], ((j / kStages) - 1) & 1, abort);
        ok = __all_sync(0xffffffffu, w);
      }
      if (!ok) break;
      const uint32_t sk = base + kSmemKV + s * 2 * kTileBytes;
      if (j < nprefix) {
        if (lane == 0) {
          const int kb = k0 + j * kKeys;
          mbar_expect_tx(&bars.full[s], 2 * kTileBytes);
          tma_load_4d(&tmap_k, sk, &bars.full[s], 0, g, kb, b);
          tma_load_4d(&tmap_k, sk + kHalfBytes, &bars.full[s], 64, g, kb, b);
          tma_load_4d(&tmap_v, sk + kTileBytes, &bars.full[s], 0, g, kb, b);
          tma_load_4d(&tmap_v, sk + kTileBytes + kHalfBytes, &bars.full[s], 64, g, kb, b);
        }
      } else {
        // gathered tree tile: rows = U[128 tt ..], 128B-swizzled like TMA writes
        const int tt = j - nprefix;
        const int nU = bars.nU;
        const __nv_bfloat16* kt = static_cast<const __nv_bfloat16*>(p.kt);
        const __nv_bfloat16* vt = static_cast<const __nv_bfloat16*>(p.vt);
        for (int e = lane; e < kRows * 16; e += 32) {
          const int r = e >> 4, c = e & 15;
          const int slot = tt * kKeys + r;
          const uint32_t off = static_cast<uint32_t>(c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
          if (slot < nU) {
            const int a = ulist[slot];
            const int64_t src = b * p.kt_sb + static_cast<int64_t>(a) * p.kt_st + g * p.kt_sh + c * 8;
            cp_async16(sk + off, kt + src);
            cp_async16(sk + kTileBytes + off, vt + src);
          } else {
            *reinterpret_cast<uint4*>(gbase + (sk - base) + off) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(gbase + (sk - base) + kTileBytes + off) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        cp_async_wait_all();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.full[s]);
      }
      ++issued;
    }
    // drain: every issued load must land before the CTA can exit
    if (lane == 0) {
      mbar_wait(&bars.q_full, 0, abort);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j) {
        uint32_t it = 0;
        while (!mbar_wait(&bars.full[j % kStages], (j / kStages) & 1, abort) && ++it < 4) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      // the tree tiles follow the prefix tiles; their count is known once the
      // producer has built the union of root paths
      int ntot = nprefix;
      if (has_tree && nprefix == 0) {
        ok = mbar_wait(&bars.tree_info, 0, abort);
        ntot += (bars.nU + kKeys - 1) / kKeys;
      }
      const uint32_t idesc_qk = instr_desc(kRows, kKeys, 0, 0);
      const uint32_t idesc_pv = instr_desc(kRows, kD, 0, 1);
      const uint32_t sq = base + kSmemQ, sp = base + kSmemP;
      if (ok && ntot > 0) ok = mbar_wait(&bars.q_full, 0, abort);
      if (ok && ntot > 0) ok = mbar_wait(&bars.full[0], 0, abort);
      if (ok && ntot > 0) {
        fence_after();
        const uint32_t sk = base + kSmemKV;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_bf16(tmem + kColS0, smem_desc(sq + off, 16, 1024), smem_desc(sk + off, 16, 1024), idesc_qk,
                   kk > 0);
        }
        mma_commit(&bars.s_full[0]);
      }
      bool tree_known = !has_tree || nprefix == 0;
      for (int j = 0; j < ntot && ok; ++j) {
        if (!tree_known && j + 1 == ntot) {
          ok = mbar_wait(&bars.tree_info, 0, abort);
          if (!ok) break;
          ntot += (bars.nU + kKeys - 1) / kKeys;
          tree_known = true;
        }
        if (j + 1 < ntot) {
          const int s1 = (j + 1) % kStages;
          ok = mbar_wait(&bars.full[s1], ((j + 1) / kStages) & 1, abort);
          if (ok && j >= 1) ok = mbar_wait(&bars.s_free[(j + 1) & 1], ((j - 1) >> 1) & 1, abort);
          if (!ok) break;
          fence_after();
          const uint32_t sk = base + kSmemKV + s1 * 2 * kTileBytes;
          const uint32_t dcol = ((j + 1) & 1) ? kColS1 : kColS0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_bf16(tmem + dcol, smem_desc(sq + off, 16, 1024), smem_desc(sk + off, 16, 1024), idesc_qk,
                     kk > 0);
          }
          mma_commit(&bars.s_full[(j + 1) & 1]);
        }
        ok = mbar_wait(&bars.p_full, j & 1, abort);
        if (!ok) break;
        fence_after();
        const uint32_t sv = base + kSmemKV + (j % kStages) * 2 * kTileBytes + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_bf16(tmem + kColO, smem_desc(sp + aoff, 16, 1024), smem_desc(sv + kk * 2048, kHalfBytes, 1024),
                   idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars.pv_done);
        mma_commit(&bars.empty[j % kStages]);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const float sl2 = p.scale * 1.4426950408889634f;   // scores in log2 units
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int ntot = nprefix;
    bool my_ok = true;
    bool tree_known = !has_tree;
    for (int j = 0; ok; ++j) {
      if (!tree_known && j == nprefix) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.tree_info, 0, abort));
        if (!ok) break;
        ntot += (bars.nU + kKeys - 1) / kKeys;
        my_ok = row_valid && bars.node_ok[tid / G] != 0;
        tree_known = true;
      }
      if (j >= ntot) break;
      const bool tree_tile = j >= nprefix;
      const int nk = tree_tile ? 0 : min(kKeys, k1 - (k0 + j * kKeys));
      uint32_t mk[4] = {0u, 0u, 0u, 0u};
      if (tree_tile && my_ok) tree_mask(par, row_node, j - nprefix, bars, mk);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[j & 1], (j >> 1) & 1, abort));
      if (!ok) break;
      fence_after();
      float s[kKeys];
      const uint32_t scol = (j & 1) ? kColS1 : kColS0;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(trow + scol + c * 32, s + c * 32);
      tmem_wait_ld();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[j & 1]);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const bool keep = tree_tile ? ((mk[c >> 5] >> (c & 31)) & 1u) != 0u : c < nk;
        s[c] = keep ? s[c] * sl2 : -INFINITY;
        mt = fmaxf(mt, s[c]);
      }
      const float m_new = fmaxf(m_run, mt);
      const bool first = (j == 0);
      const bool grow = !first && (m_new > m_run + 8.0f);
      float factor = 1.f;
      if (first) {
        m_run = m_new;
      } else if (grow) {
        factor = ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      const float mu = (m_run == -INFINITY) ? 0.f : m_run;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        s[c] = ex2_approx(s[c] - mu);
        rs += s[c];
      }
      l_run = l_run * factor + rs;
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (j - 1) & 1, abort));
        if (!ok) break;
        fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(trow + kColO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= factor;
            tmem_st32(trow + kColO + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      if (!tree_tile && nk < kKeys) {
        // ragged prefix tile: V rows past the prefix end may hold anything
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.full[j % kStages], (j / kStages) & 1, abort));
        if (!ok) break;
        if (tid >= nk) {
          uint8_t* sv = gbase + kSmemKV + (j % kStages) * 2 * kTileBytes + kTileBytes;
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(sv + tid * 128 + c * 16) = z;
            *reinterpret_cast<uint4*>(sv + kHalfBytes + tid * 128 + c * 16) = z;
          }
        }
      }
      uint8_t* prow = gbase + kSmemP + tid * 128;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint4 v;
        v.x = pack_bf16(s[8 * c + 0], s[8 * c + 1]);
        v.y = pack_bf16(s[8 * c + 2], s[8 * c + 3]);
        v.z = pack_bf16(s[8 * c + 4], s[8 * c + 5]);
        v.w = pack_bf16(s[8 * c + 6], s[8 * c + 7]);
        const int half = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(prow + half * kHalfBytes + ((cc ^ (tid & 7)) << 4)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full);
    }
    // epilogue
    if (ok && ntot > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (ntot - 1) & 1, abort));
    if (ok) {
      fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      if (p.nchunk == 1) {
        // single chunk: this CTA holds the whole result
        const bool good = my_ok && !bad_len;
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + row_node * p.o_st + row_head * p.o_sh;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(trow + kColO + c * 32, v);
          tmem_wait_ld();
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 w;
              if (good) {
                w.x = pack_bf16(v[e] * inv, v[e + 1] * inv);
                w.y = pack_bf16(v[e + 2] * inv, v[e + 3] * inv);
                w.z = pack_bf16(v[e + 4] * inv, v[e + 5] * inv);
                w.w = pack_bf16(v[e + 6] * inv, v[e + 7] * inv);
              } else {
                w.x = w.y = w.z = w.w = pack_bf16(NAN, NAN);
              }
              *reinterpret_cast<uint4*>(o + c * 32 + e) = w;
            }
          }
        }
        if (row_valid) {
          if (p.lse) p.lse[(static_cast<int64_t>(b) * p.T + row_node) * p.Hq + row_head] = good ? lse : NAN;
          if (!my_ok) set_status(p.status, TV_DEV_BAD_PARENT);
          if (bad_len && row_node == 0 && row_head == 0) set_status(p.status, TV_DEV_BAD_LEN);
        }
      } else {
        float* po = row_valid ? p.part_o + part_row(p, chunk, b, row_node, row_head) * kD : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(trow + kColO + c * 32, v);
          tmem_wait_ld();
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(po + c * 32 + e) =
                  (l_run > 0.f) ? make_float4(v[e] * inv, v[e + 1] * inv, v[e + 2] * inv, v[e + 3] * inv)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        if (row_valid) {
          // invalid rows carry NaN into the merge
          const bool good = my_ok && !bad_len;
          p.part_lse[part_row(p, chunk, b, row_node, row_head)] = good ? lse : NAN;
          if (has_tree && !my_ok) set_status(p.status, TV_DEV_BAD_PARENT);
          if (bad_len && chunk == 0 && row_node == 0 && row_head == 0) set_status(p.status, TV_DEV_BAD_LEN);
        }
      }
    }
  }
  // ------------------------------------------------------------------ teardown
  fence_before();
  __syncthreads();
  if (*abort) {
    if (tid == 0) set_status(p.status, TV_DEV_TIMEOUT);
    if (row_valid) {
      if (p.nchunk == 1) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + row_node * p.o_st + row_head * p.o_sh;
        for (int c = 0; c < kD; ++c) o[c] = __float2bfloat16(NAN);
      } else {
        p.part_lse[part_row(p, chunk, b, row_node, row_head)] = NAN;
      }
    }
  }
  if (warp == 5) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// Log-sum-exp merge of the chunk partials of the tensor-core kernel: one
// warp per (sequence, node, query head); lane c holds chunk c's lse, lane l
// accumulates dimensions 4l .. 4l+3 with every chunk's load in flight.  The
// partials of rows that are invalid (malformed parent chain, prefix length
// out of range) carry lse = NaN and the merged row is NaN.
__global__ void __launch_bounds__(256) attn_tc_merge_kernel(AttnParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<int64_t>(p.B) * p.T * p.Hq) return;
  const int h = static_cast<int>(row % p.Hq);
  const int i = static_cast<int>((row / p.Hq) % p.T);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.Hq) * p.T));
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T || i >= n) return;
  // a NaN partial lse marks a row the tensor-core kernel found invalid
  const int np = p.nchunk;
  float lc = -INFINITY;
  if (lane < np) lc = __ldcg(&p.part_lse[part_row(p, lane, b, i, h)]);
  const bool good = !__any_sync(0xffffffffu, lc != lc);
  if (!good) lc = -INFINITY;
  const float M = warp_max(lc);
  const float wl = (lane < np && lc > -INFINITY) ? __expf(lc - M) : 0.f;
  const float den = warp_sumf(wl);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < np; c0 += 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = (c0 + u < np) ? __ldcg(reinterpret_cast<const float4*>(p.part_o + part_row(p, c0 + u, b, i, h) * kD) + lane)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float w = __shfl_sync(0xffffffffu, wl, (c0 + u) & 31);
      if (c0 + u < np) {
        acc.x = fmaf(w, v[u].x, acc.x); acc.y = fmaf(w, v[u].y, acc.y);
        acc.z = fmaf(w, v[u].z, acc.z); acc.w = fmaf(w, v[u].w, acc.w);
      }
    }
  }
  const bool ok = good && den > 0.f;
  const float inv = ok ? 1.f / den : 0.f;
  uint2 wv;
  if (ok) {
    wv.x = pack_bf16(acc.x * inv, acc.y * inv);
    wv.y = pack_bf16(acc.z * inv, acc.w * inv);
  } else {
    wv.x = wv.y = pack_bf16(NAN, NAN);
  }
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + i * p.o_st + h * p.o_sh;
  *reinterpret_cast<uint2*>(o + lane * 4) = wv;
  if (lane == 0 && p.lse) p.lse[row] = ok ? M + __logf(den) : NAN;
}

// ------------------------------------------------------------------ host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
              int64_t s1, int64_t s2, int64_t s3, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(s1) * 2, static_cast<cuuint64_t>(s2) * 2,
                                 static_cast<cuuint64_t>(s3) * 2};
  const cuuint32_t box[4] = {64, b1, b2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool stride_ok(int64_t s) { return s > 0 && (s * 2) % 16 == 0 && s * 2 < (1ll << 40); }

}  // namespace

bool attn_tc_supported(const tv_attn_args* a) {
  if (a->dtype != TV_BF16 || a->d != 128 || a->sparse_topk != 0) return false;
  if (a->B == 0 || a->T == 0 || a->Lmax == 0) return false;
  if (a->T > kMaxT) return false;
  const int G = a->Hq / a->Hkv;
  if (G > 128 || 128 % G != 0) return false;
  if (a->Lmax > (1 << 30)) return false;
  if (!stride_ok(a->q_sh) || !stride_ok(a->q_st) || !stride_ok(a->q_sb)) return false;
  if (!stride_ok(a->kv_sh) || !stride_ok(a->kv_sl) || !stride_ok(a->kv_sb)) return false;
  if (!stride_ok(a->kt_sh) || !stride_ok(a->kt_st) || !stride_ok(a->kt_sb)) return false;
  if (!stride_ok(a->o_sh) || !stride_ok(a->o_st) || !stride_ok(a->o_sb)) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->k_cache) |
                       reinterpret_cast<uintptr_t>(a->v_cache) | reinterpret_cast<uintptr_t>(a->k_tree) |
                       reinterpret_cast<uintptr_t>(a->v_tree) | reinterpret_cast<uintptr_t>(a->out);
  if (al & 15u) return false;
  if (!encode_fn()) return false;
  {
    CUtensorMap m;
    if (!make_map(&m, a->q, a->d, a->Hq, a->T, a->B, a->q_sh, a->q_st, a->q_sb, G, kRows / G) ||
        !make_map(&m, a->k_cache, a->d, a->Hkv, a->Lmax, a->B, a->kv_sh, a->kv_sl, a->kv_sb, 1, kKeys) ||
        !make_map(&m, a->v_cache, a->d, a->Hkv, a->Lmax, a->B, a->kv_sh, a->kv_sl, a->kv_sb, 1, kKeys))
      return false;
  }
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const int G = p.G;
  if (!make_map(&mq, p.q, p.d, p.Hq, p.T, p.B, p.q_sh, p.q_st, p.q_sb, G, kRows / G) ||
      !make_map(&mk, p.kc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys) ||
      !make_map(&mv, p.vc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = kSmemBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + p.node_tile - 1) / p.node_tile;
  dim3 grid(p.nchunk, ntiles, p.B * p.Hkv);
  attn_tc_kernel<<<grid, kThreads, smem, stream>>>(mq, mk, mv, p);
  if (p.nchunk > 1) {
    const int64_t rows = static_cast<int64_t>(p.B) * p.T * p.Hq;
    attn_tc_merge_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace tv
