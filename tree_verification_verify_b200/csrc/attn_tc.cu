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
// One CTA owns (sequence, kv head, 128-row tile, prefix chunk); the chunks
// of one row tile form a thread-block cluster.  A CTA's key tiles are its
// chunk's prefix tiles of 128 keys and, in the last chunk, the tree tiles: the
// union U of the tile's nodes' root paths, gathered into K/V tiles and
// masked per row by the row's ancestors in U.  All tiles share one online
// softmax.  At the end every CTA pushes its normalised O rows and their
// log-sum-exp over distributed shared memory to the CTA of the cluster that
// merges them; each CTA merges a share of the rows and writes the output.
//
// Warp roles (256 threads):
//   warps 0-3  softmax / correction / epilogue: thread t owns query row t,
//              which is TMEM lane t (tcgen05.ld 32x32b);
//   warp 4     Q and the K tiles: TMA into a three-stage ring (128B swizzle,
//              K-major) or, for tree tiles, a cp.async gather;
//   warp 5     TMEM allocator and MMA issuer (one thread): S = Q K^T into
//              one of two TMEM S buffers, O += P V with P read from TMEM;
//   warp 6     the V tiles, a two-stage ring (MN-major), like warp 4;
//   warp 7     tree bookkeeping (last chunk): parent[] into shared memory,
//              the node bitmap of U, the slot of every node of U and the
//              slot of its parent.
// A K stage is released when its S = Q K^T completes, a V stage when its
// P V completes, so the loads of later tiles start while earlier tiles are
// in the softmax.  Online softmax in base 2 with a lazily updated row
// maximum: O and the row sum are rescaled only when the maximum grows by
// more than 2^8, which keeps P <= 256 (exact in the final O / l).  P is
// written as bf16 over the first 64 columns of its S buffer.
//
// Every mbarrier wait is bounded: on expiry the CTA records TV_DEV_TIMEOUT,
// stops issuing work, drains what it issued, frees its TMEM, and its rows
// come out as NaN.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cooperative_groups.h>

#include "attn.cuh"

namespace cg = cooperative_groups;

namespace tv {

namespace tc {

constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;  // two threads per query row
constexpr int kWarpK = 8, kWarpMma = 9, kWarpV = 10, kWarpTree = 11;
constexpr int kRows = 128;          // M
constexpr int kKeys = 128;          // keys per tile (N of QK, K of PV)
constexpr int kD = 128;
constexpr int kKS = 3;              // K ring stages
constexpr int kVS = 2;              // V ring stages
constexpr int kMaxT = 2048;         // tree nodes handled by this kernel
constexpr int kMaxUnion = 1024;     // block top-k: kept blocks in the union of a row tile
constexpr int kMaxTopk = 64;        // block top-k: kept blocks per (node, kv head)
constexpr int kMaxSpNodes = 32;     // block top-k: nodes per row tile (G >= 4)
constexpr int kMaxBlk = 4096;       // block top-k: 64-key prefix blocks
constexpr int kMaxCluster = 8;      // chunks per row tile
constexpr uint32_t kHalfBytes = kRows * 128;            // 128 rows x 128 B
constexpr uint32_t kTileBytes = 2 * kHalfBytes;         // 32 KB (d = 128 bf16)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kKS * kTileBytes;
constexpr uint32_t kSmemPar = kSmemV + kVS * kTileBytes;  // parent[] (u16)
constexpr uint32_t kSmemUL = kSmemPar + kMaxT * 2;        // U: slot -> node (u16)
constexpr uint32_t kSmemUP = kSmemUL + kMaxT * 2;         // U: slot -> parent's slot (u16)
constexpr uint32_t kSmemUB = kSmemUP + kMaxT * 2;         // block top-k: union blocks (u16)
constexpr uint32_t kSmemNL = kSmemUB + kMaxUnion * 2;     // block top-k: kept lists per node (u16)
constexpr uint32_t kSmemUBM = kSmemNL + kMaxSpNodes * kMaxTopk * 2;   // block top-k: union bitmap
constexpr uint32_t kSmemBytes = kSmemUBM + kMaxBlk / 8;   // 211 KB
constexpr uint32_t kSmemInbox = kSmemK;                   // merge: fp32 O rows copied in by the cluster
constexpr uint32_t kSmemStage = kSmemV;                   // merge: this CTA's fp32 O rows (idle V ring)
constexpr int kMaxInboxRows = 144;                        // max over C of C * per (per = 4 * ceil(128 / 4C))
constexpr uint32_t kTmemCols = 512;                       // S0, S1, O (128 each)
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t kDrainLimit = 1u << 20;
constexpr uint16_t kRootMark = 0xFFFEu;   // parent[] entry of a well-formed root
constexpr uint16_t kBadMark = 0xFFFFu;    // malformed parent (or no parent slot)

static_assert(kSmemInbox + kMaxInboxRows * kD * 4 <= kSmemK + kKS * kTileBytes,
              "the merge inbox fits the K ring");
static_assert(kSmemStage + kRows * kD * 4 <= kSmemV + kVS * kTileBytes, "the merge stage fits the V ring");

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKS], k_empty[kKS];
  uint64_t v_full[kVS], v_empty[kVS];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done;
  uint64_t tree_info;
  uint64_t sparse_info;             // block top-k: the union of kept blocks is listed
  uint32_t tmem_base;
  int abort;
  int nU;                           // nodes in the union of root paths
  int nUB;                          // block top-k: blocks in the union of the tile's kept blocks
  uint32_t bm[kMaxT / 32];          // node bitmap of U
  int pre[kMaxT / 32];              // marked nodes below each bitmap word
  int node_ok[kRows];               // root path of the tile's node is well formed
  uint64_t inbox_full;              // the cluster's copies into this CTA's inbox have landed
  alignas(16) float st_lse[kRows];  // this CTA's rows: log2-sum-exp (NaN: invalid)
  uint64_t max_ready[2];            // both halves of every row have posted their tile maximum
  uint64_t sum_ready;               // both halves have posted their row sums
  float red_max[2][2][kRows];       // [tile parity][half][row] partial maxima
  float red_l[2][kRows];            // [half][row] partial row sums
  alignas(16) float in_lse[kMaxInboxRows];  // merge inbox: log2-sum-exp of row (chunk, row)
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

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// D (TMEM) (+)= A (TMEM, K-major: row m in lane m, two bf16 per column) x B
// (shared memory descriptor).
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Wait used while draining after an abort: bounded, ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const uint32_t a = smem_u32(b);
  for (uint32_t it = 0; it < kDrainLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return;
  }
}

// Slot of node a in U: the number of marked nodes below a.
__device__ __forceinline__ int u_slot(const Bars& bars, int a) {
  return bars.pre[a >> 5] + __popc(bars.bm[a >> 5] & ((1u << (a & 31)) - 1u));
}

__device__ __forceinline__ uint32_t s_col(int j) { return (j & 1) ? kColS1 : kColS0; }

// Shared-memory address `a` of this CTA mapped to CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t a, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}

// Bulk copy of `bytes` (a multiple of 16) from this CTA's shared memory to
// a cluster peer's, completing on the peer's mbarrier `bar`.
__device__ __forceinline__ void bulk_s2c(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "r"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Bytes a merging CTA receives from one chunk for `rows` rows: the fp32 O
// rows and their log-sum-exp (padded to 16 bytes).
__host__ __device__ constexpr uint32_t merge_bytes(int rows) {
  return rows > 0 ? static_cast<uint32_t>(rows) * kD * 4 + static_cast<uint32_t>((rows + 3) & ~3) * 4 : 0u;
}

// Bounded wait (cluster-scope acquire) on phase `parity`; false on expiry.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* b, uint32_t parity) {
  const uint32_t a = smem_u32(b);
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

}  // namespace tc

using namespace tc;

// SPARSE: block top-k verification attention.  The prefix tiles are then the
// union of the 64-key blocks that the tile's nodes keep (two blocks per key
// tile, loaded with 64-key boxes tmap_k64 / tmap_v64), and a row keeps a
// block only when its node selected it; one chunk per row tile.
template <bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_k64,
               const __grid_constant__ CUtensorMap tmap_v64, AttnParams p) {
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ Bars bars;
  cg::cluster_group cl = cg::this_cluster();
  const int chunk = blockIdx.x;            // = rank in the cluster (the cluster spans the chunks)
  const int C = static_cast<int>(gridDim.x);
  const int tile = blockIdx.y;
  const int b = blockIdx.z / p.Hkv, g = blockIdx.z % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  // the early exits depend on (sequence, row tile) only: a cluster leaves whole
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) {
    if (chunk == C - 1 && tile == 0 && g == 0 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
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
  // key tiles of the prefix: known here (dense), or once the union of the
  // kept blocks is listed (block top-k)
  int nprefix = SPARSE ? 0 : ((k1 > k0) ? (k1 - k0 + kKeys - 1) / kKeys : 0);
  const int nodes_here = min(kRows / G, n - i0);
  const bool has_tree = (chunk == C - 1);   // the last chunk is the shortest
  // this thread's query row (softmax warps)
  // softmax threads: query row tid % 128 (TMEM lane), column half tid / 128
  const int row = tid & (kRows - 1);
  const int half = tid >> 7;
  const int row_node = i0 + row / G;
  const bool row_valid = tid < kSoftmaxThreads && (row / G) < nodes_here;
  // rows [c * merge_per, (c + 1) * merge_per) of the tile are merged by CTA c
  const int merge_per = 4 * ((nodes_here * G + 4 * C - 1) / (4 * C));

  // 1024-aligned dynamic shared memory (128B swizzle atoms are 1 KB)
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem_raw + (base - raw);
  uint16_t* spar = reinterpret_cast<uint16_t*>(gbase + kSmemPar);
  uint16_t* ulist = reinterpret_cast<uint16_t*>(gbase + kSmemUL);
  uint16_t* uparent = reinterpret_cast<uint16_t*>(gbase + kSmemUP);
  uint16_t* ublk = reinterpret_cast<uint16_t*>(gbase + kSmemUB);
  uint16_t* nlist = reinterpret_cast<uint16_t*>(gbase + kSmemNL);
  uint32_t* ubm = reinterpret_cast<uint32_t*>(gbase + kSmemUBM);
  volatile int* abort = &bars.abort;
  // block top-k: blocks 2 jt and 2 jt + 1 of the union form key tile jt
  auto blk_of = [&](int slot) -> int { return slot < bars.nUB ? static_cast<int>(ublk[slot]) : -1; };
  auto blk_keys = [&](int blk) -> int { return blk < 0 ? 0 : min(64, L - 64 * blk); };

  if (tid == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kKS; ++s) { mbar_init(&bars.k_full[s], 1); mbar_init(&bars.k_empty[s], 1); }
    for (int s = 0; s < kVS; ++s) { mbar_init(&bars.v_full[s], 1); mbar_init(&bars.v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], kSoftmaxThreads / 32);
      mbar_init(&bars.max_ready[s], kSoftmaxThreads / 32);
    }
    mbar_init(&bars.sum_ready, kSoftmaxThreads / 32);
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.tree_info, 1);
    mbar_init(&bars.sparse_info, 1);
    mbar_init(&bars.inbox_full, 1);
    bars.abort = 0;
    bars.nU = 0;
    bars.nUB = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // the bytes the cluster will copy into this CTA's inbox
    const int own = max(0, min(merge_per, nodes_here * G - chunk * merge_per));
    mbar_expect_tx(&bars.inbox_full, static_cast<uint32_t>(C) * merge_bytes(own));
  }
  if (warp == kWarpMma) {
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

  if (warp == kWarpTree) {
    // ------------------------------------------------------------ tree bookkeeping
    if (SPARSE) {
      // the kept blocks of every node of the tile (ascending, 0xFFFF past
      // the end) and their union, listed in ascending block order
      const int nblk = (L + 63) / 64;
      const int nbw = (nblk + 31) >> 5;
      for (int w = lane; w < nbw; w += 32) ubm[w] = 0u;
      __syncwarp();
      const int32_t* sel = p.sel + (static_cast<int64_t>(b) * p.T + i0) * p.Hkv * p.topk + g * p.topk;
      for (int e = lane; e < nodes_here * p.topk; e += 32) {
        const int r = e / p.topk, t = e % p.topk;
        const int j = sel[static_cast<int64_t>(r) * p.Hkv * p.topk + t];
        const bool kept = j >= 0 && j < nblk;
        nlist[r * kMaxTopk + t] = kept ? static_cast<uint16_t>(j) : 0xFFFFu;
        if (kept) atomicOr(&ubm[j >> 5], 1u << (j & 31));
      }
      __syncwarp();
      const int per = (nbw + 31) / 32;
      const int lo = min(lane * per, nbw), hi = min(lo + per, nbw);
      int cnt = 0;
      for (int w = lo; w < hi; ++w) cnt += __popc(ubm[w]);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int run = incl - cnt;
      for (int w = lo; w < hi; ++w) {
        uint32_t m = ubm[w];
        while (m) {
          const int bit = __ffs(m) - 1;
          ublk[run++] = static_cast<uint16_t>(w * 32 + bit);
          m &= m - 1u;
        }
      }
      const int nUB = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) bars.nUB = nUB;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sparse_info);
    }
    if (has_tree) {
      for (int j = lane; j < n; j += 32) {
        const int pj = par[j];
        spar[j] = (j == 0) ? (pj == -1 ? kRootMark : kBadMark)
                           : ((pj >= 0 && pj < j) ? static_cast<uint16_t>(pj) : kBadMark);
      }
      const int nw = (n + 31) >> 5;
      for (int w = lane; w < nw; w += 32) bars.bm[w] = 0u;
      __syncwarp();
      // mark the root path of every node of the tile (parents strictly
      // decrease, so a walk takes at most i + 1 steps)
      for (int r = lane; r < nodes_here; r += 32) {
        int j = i0 + r;
        int ok = 1;
        for (int step = 0; step <= i0 + r; ++step) {
          atomicOr(&bars.bm[j >> 5], 1u << (j & 31));
          const uint16_t pj = spar[j];
          if (pj == kRootMark) break;
          if (pj == kBadMark) { ok = 0; break; }
          j = pj;
        }
        bars.node_ok[r] = ok;
      }
      __syncwarp();
      // prefix counts per bitmap word, then U in node order
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
          ulist[run++] = static_cast<uint16_t>(w * 32 + bit);
          m &= m - 1u;
        }
      }
      const int nU = __shfl_sync(0xffffffffu, incl, 31);
      __syncwarp();
      // the parent of a node of U is in U (or the node is the root / malformed)
      for (int sl = lane; sl < nU; sl += 32) {
        const uint16_t pa = spar[ulist[sl]];
        uparent[sl] = (pa < kRootMark) ? static_cast<uint16_t>(u_slot(bars, pa)) : kBadMark;
      }
      if (lane == 0) bars.nU = nU;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.tree_info);
    }
  } else if (warp == kWarpK || warp == kWarpV) {
    // ------------------------------------------------------------ producers
    const bool isk = (warp == kWarpK);
    const int NS = isk ? kKS : kVS;
    uint64_t* full = isk ? bars.k_full : bars.v_full;
    uint64_t* empty = isk ? bars.k_empty : bars.v_empty;
    const CUtensorMap* map = isk ? &tmap_k : &tmap_v;
    const uint32_t ring = base + (isk ? kSmemK : kSmemV);
    const __nv_bfloat16* src_tree = static_cast<const __nv_bfloat16*>(isk ? p.kt : p.vt);
    if (isk && lane == 0) {
      const uint32_t sq = base + kSmemQ;
      mbar_expect_tx(&bars.q_full, kTileBytes);
      tma_load_4d(&tmap_q, sq, &bars.q_full, 0, g * G, i0, b);
      tma_load_4d(&tmap_q, sq + kHalfBytes, &bars.q_full, 64, g * G, i0, b);
    }
    bool sparse_ok = true;
    if (SPARSE) {
      bool w = true;
      if (lane == 0) w = mbar_wait(&bars.sparse_info, 0, abort);
      sparse_ok = __all_sync(0xffffffffu, w);
      nprefix = sparse_ok ? (bars.nUB + 1) / 2 : 0;
    }
    int ntot = nprefix, ntree = 0;
    bool tree_known = !has_tree;
    int issued = 0;
    for (int j = 0; sparse_ok; ++j) {
      if (!tree_known && j == nprefix) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&bars.tree_info, 0, abort);
        if (!__all_sync(0xffffffffu, w)) break;
        ntree = (bars.nU + kKeys - 1) / kKeys;
        ntot += ntree;
        tree_known = true;
      }
      if (j >= ntot) break;
      const int s = j % NS;
      if (j >= NS) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&empty[s], ((j / NS) - 1) & 1, abort);
        if (!__all_sync(0xffffffffu, w)) break;
      }
      const uint32_t dst = ring + s * kTileBytes;
      if (SPARSE && j < nprefix) {
        // kept blocks 2 j and 2 j + 1 of the union, 64 keys each, as rows
        // 0-63 and 64-127 of the tile
        if (lane == 0) {
          const CUtensorMap* map64 = isk ? &tmap_k64 : &tmap_v64;
          const int ja = blk_of(2 * j), jb = blk_of(2 * j + 1);
          mbar_expect_tx(&full[s], (jb >= 0 ? 2u : 1u) * (kTileBytes / 2));
          tma_load_4d(map64, dst, &full[s], 0, g, 64 * ja, b);
          tma_load_4d(map64, dst + kHalfBytes, &full[s], 64, g, 64 * ja, b);
          if (jb >= 0) {
            tma_load_4d(map64, dst + 64 * 128, &full[s], 0, g, 64 * jb, b);
            tma_load_4d(map64, dst + kHalfBytes + 64 * 128, &full[s], 64, g, 64 * jb, b);
          }
        }
      } else if (j < nprefix) {
        if (lane == 0) {
          const int kb = k0 + j * kKeys;
          mbar_expect_tx(&full[s], kTileBytes);
          tma_load_4d(map, dst, &full[s], 0, g, kb, b);
          tma_load_4d(map, dst + kHalfBytes, &full[s], 64, g, kb, b);
        }
      } else {
        // gathered tree tile (tree tiles run from the last slots down):
        // rows = U[128 tt ..], 128B-swizzled as TMA writes them
        const int tt = ntree - 1 - (j - nprefix);
        const int nU = bars.nU;
        uint8_t* gdst = gbase + (dst - base);
        for (int e = lane; e < kRows * 16; e += 32) {
          const int r = e >> 4, c = e & 15;
          const int slot = tt * kKeys + r;
          const uint32_t off = static_cast<uint32_t>(c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
          if (slot < nU) {
            const int a = ulist[slot];
            cp_async16(dst + off, src_tree + b * p.kt_sb + static_cast<int64_t>(a) * p.kt_st + g * p.kt_sh + c * 8);
          } else {
            *reinterpret_cast<uint4*>(gdst + off) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        cp_async_wait_all();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
      ++issued;
    }
    // drain: every issued load lands before the CTA can exit
    if (lane == 0) {
      if (isk) mbar_drain(&bars.q_full, 0);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j) mbar_drain(&full[j % NS], (j / NS) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (SPARSE) {
        ok = mbar_wait(&bars.sparse_info, 0, abort);
        nprefix = ok ? (bars.nUB + 1) / 2 : 0;
      }
      int ntot = nprefix;
      bool tree_known = !has_tree;
      // the tree tiles follow the prefix tiles; their count is known once
      // the tree warp has built U
      auto know = [&](int upto) -> bool {
        if (!tree_known && upto >= nprefix) {
          if (!mbar_wait(&bars.tree_info, 0, abort)) return false;
          ntot += (bars.nU + kKeys - 1) / kKeys;
          tree_known = true;
        }
        return true;
      };
      const uint32_t idesc_qk = instr_desc(kRows, kKeys, 0, 0);
      const uint32_t idesc_pv = instr_desc(kRows, kD, 0, 1);
      const uint32_t sq = base + kSmemQ;
      int s_issued = 0, pv_issued = 0;
      auto issue_s = [&](int j) {
        const uint32_t sk = base + kSmemK + (j % kKS) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_bf16(tmem + s_col(j), smem_desc(sq + off, 16, 1024), smem_desc(sk + off, 16, 1024), idesc_qk,
                   kk > 0);
        }
        mma_commit(&bars.k_empty[j % kKS]);
        mma_commit(&bars.s_full[j & 1]);
        ++s_issued;
      };
      ok = ok && know(0);
      if (ok && ntot > 0) ok = mbar_wait(&bars.q_full, 0, abort);
      for (int j = 0; j < 2 && ok; ++j) {
        ok = know(j);
        if (!ok || j >= ntot) break;
        ok = mbar_wait(&bars.k_full[j % kKS], (j / kKS) & 1, abort);
        if (!ok) break;
        fence_after();
        issue_s(j);
      }
      for (int j = 0; ok; ++j) {
        ok = know(j);
        if (!ok || j >= ntot) break;
        ok = mbar_wait(&bars.p_full[j & 1], (j >> 1) & 1, abort);
        if (ok) ok = mbar_wait(&bars.v_full[j % kVS], (j / kVS) & 1, abort);
        if (!ok) break;
        fence_after();
        const uint32_t sv = base + kSmemV + (j % kVS) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + kColO, tmem + s_col(j) + kk * 8, smem_desc(sv + kk * 2048, kHalfBytes, 1024),
                      idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars.v_empty[j % kVS]);
        mma_commit(&bars.pv_done);
        ++pv_issued;
        const int jn = j + 2;
        ok = know(jn);
        if (!ok) break;
        if (jn < ntot) {
          ok = mbar_wait(&bars.k_full[jn % kKS], (jn / kKS) & 1, abort);
          // S(jn) overwrites the buffer P(j) is read from
          if (ok) ok = mbar_wait(&bars.pv_done, j & 1, abort);
          if (!ok) break;
          fence_after();
          issue_s(jn);
        }
      }
      if (!ok) {
        // the issued MMAs complete before the TMEM is freed
        if (s_issued > 1) mbar_drain(&bars.s_full[(s_issued - 2) & 1], ((s_issued - 2) >> 1) & 1);
        if (s_issued > 0) mbar_drain(&bars.s_full[(s_issued - 1) & 1], ((s_issued - 1) >> 1) & 1);
        if (pv_issued > 1) mbar_drain(&bars.pv_done, (pv_issued - 2) & 1);
        if (pv_issued > 0) mbar_drain(&bars.pv_done, (pv_issued - 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    // Row r is TMEM lane r: warps w and w + 4 share lanes 32 (w % 4) ..; warp
    // w < 4 takes key columns 0-63 of every tile, warp w + 4 columns 64-127.
    // The two halves exchange their tile maxima (shared memory + mbarrier),
    // keep their own row sums, and add them at the end.
    const float sl2 = p.scale * 1.4426950408889634f;   // scores in log2 units
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t hcol = 64u * static_cast<uint32_t>(half);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    if (SPARSE) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.sparse_info, 0, abort));
      nprefix = ok ? (bars.nUB + 1) / 2 : 0;
    }
    int ntot = nprefix, ntree = 0;
    bool my_ok = true;
    bool tree_known = !has_tree;
    int cur = -1;                 // walk position (slot) on this row's root path
    int lcur = 0;                 // block top-k: cursor into this row's node's kept list
    const uint16_t* mylist = nlist + (row / G) * kMaxTopk;
    for (int j = 0; ok; ++j) {
      if (!tree_known && j == nprefix) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.tree_info, 0, abort));
        if (!ok) break;
        ntree = (bars.nU + kKeys - 1) / kKeys;
        ntot += ntree;
        my_ok = row_valid && bars.node_ok[row / G] != 0;
        cur = my_ok ? u_slot(bars, row_node) : -1;
        tree_known = true;
      }
      if (j >= ntot) break;
      const bool tree_tile = j >= nprefix;
      const int nk = (tree_tile || SPARSE) ? 0 : min(kKeys, k1 - (k0 + j * kKeys));
      // key mask of this half's 64 columns: two words, kept in registers
      uint32_t mkA = 0u, mkB = 0u;
      if (tree_tile) {
        // ancestors of this row's node in slots [128 tt + 64 half, + 64);
        // the tiles run downwards and slots decrease along the path, so the
        // walk continues where the previous tile left it
        const int lo = (ntree - 1 - (j - nprefix)) * kKeys;
        while (cur >= lo) {
          const int w = (cur - lo) >> 5;           // 0..3 in the tile
          if (cur < lo + kKeys && (w >> 1) == half) {
            const uint32_t bit = 1u << (cur & 31);
            mkA |= (w & 1) == 0 ? bit : 0u;
            mkB |= (w & 1) == 1 ? bit : 0u;
          }
          const uint16_t up = uparent[cur];
          cur = (up == kBadMark) ? -1 : static_cast<int>(up);
        }
      } else if (SPARSE) {
        // this half's block (slot 2 j + half of the union): kept by this
        // row's node?  Both the kept list and the union ascend, so the
        // cursor only moves forward.
        const int blk = blk_of(2 * j + half);
        bool member = false;
        if (row_valid && blk >= 0) {
          while (lcur < p.topk && mylist[lcur] < blk) ++lcur;
          member = lcur < p.topk && mylist[lcur] == blk;
        }
        const int nh = member ? blk_keys(blk) : 0;
        mkA = nh >= 32 ? 0xffffffffu : (nh <= 0 ? 0u : ((1u << nh) - 1u));
        mkB = nh >= 64 ? 0xffffffffu : (nh <= 32 ? 0u : ((1u << (nh - 32)) - 1u));
      } else {
        const int nh = nk - 64 * half;              // valid keys in this half
        mkA = nh >= 32 ? 0xffffffffu : (nh <= 0 ? 0u : ((1u << nh) - 1u));
        mkB = nh >= 64 ? 0xffffffffu : (nh <= 32 ? 0u : ((1u << (nh - 32)) - 1u));
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[j & 1], (j >> 1) & 1, abort));
      if (!ok) break;
      fence_after();
      float s[64];
      const uint32_t scol = s_col(j);
      tmem_ld32(trow + scol + hcol, s);
      tmem_ld32(trow + scol + hcol + 32, s + 32);
      tmem_wait_ld();
      // masked scores in log2 units; this half's maximum over four
      // interleaved partial maxima (the maximum does not depend on order)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const uint32_t mw = (c < 32) ? mkA : mkB;
        s[c] = ((mw >> (c & 31)) & 1u) ? s[c] * sl2 : -INFINITY;
        mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      }
      const float mh = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      bars.red_max[j & 1][half][row] = mh;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.max_ready[j & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.max_ready[j & 1], (j >> 1) & 1, abort));
      if (!ok) break;
      const float mt = fmaxf(mh, bars.red_max[j & 1][half ^ 1][row]);
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
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        s[c] = ex2_approx(s[c] - mu);
        ps[c & 3] += s[c];
      }
      l_run = l_run * factor + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      if (__any_sync(0xffffffffu, grow)) {
        // O holds the tiles up to j - 1: wait for their P V, then rescale
        // this half's 64 columns of O
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (j - 1) & 1, abort));
        if (!ok) break;
        fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(trow + kColO + hcol + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= factor;
          tmem_st32(trow + kColO + hcol + c * 32, o);
        }
      }
      // P as bf16 pairs over the first 64 columns of the S buffer: this
      // half's keys 64 half .. 64 half + 63 are columns 32 half .. + 31
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(s[2 * e], s[2 * e + 1]);
        tmem_st32u(trow + scol + 32u * static_cast<uint32_t>(half), pk);
      }
      tmem_wait_st();
      // V rows that are not keys of this tile (past the prefix end, or an
      // absent second block) may hold anything: zero them
      int vka = 64, vkb = 64;
      if (SPARSE && !tree_tile) { vka = blk_keys(blk_of(2 * j)); vkb = blk_keys(blk_of(2 * j + 1)); }
      const bool ragged = SPARSE ? (!tree_tile && (vka < 64 || vkb < 64)) : (!tree_tile && nk < kKeys);
      if (ragged) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.v_full[j % kVS], (j / kVS) & 1, abort));
        if (!ok) break;
        const bool dead_row = SPARSE ? (row < 64 ? row >= vka : row - 64 >= vkb) : row >= nk;
        if (half == 0 && dead_row) {
          uint8_t* sv = gbase + kSmemV + (j % kVS) * kTileBytes;
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(sv + row * 128 + c * 16) = z;
            *reinterpret_cast<uint4*>(sv + kHalfBytes + row * 128 + c * 16) = z;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[j & 1]);
    }
    // ------------------------------------------------------------ epilogue
    // The last P V is pv_done's phase ntot - 1.  S(ntot - 1) having landed
    // only proves P V up to ntot - 3, and a parity wait cannot tell phase
    // ntot - 1 from ntot - 3: wait for phase ntot - 2 first, then ntot - 1.
    if (ok && ntot > 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (ntot - 2) & 1, abort));
    if (ok && ntot > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (ntot - 1) & 1, abort));
    fence_after();
    // the row sum is the two halves' sums
    bars.red_l[half][row] = l_run;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.sum_ready);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars.sum_ready, 0, abort));
    const float l_row = ok ? l_run + bars.red_l[half ^ 1][row] : 0.f;
    const bool have = ok && l_row > 0.f;
    const float inv = have ? 1.f / l_row : 0.f;
    // this half of the row's normalised O into the stage (the idle V ring;
    // fp32, float4 q of row t at q ^ (t & 7)) and the row's log2-sum-exp
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    float* stage = reinterpret_cast<float*>(gbase + kSmemStage) + row * kD;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v[32];
      tmem_ld32(trow + kColO + hcol + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int qq = 16 * half + c * 8 + q;
        *reinterpret_cast<float4*>(stage + ((qq ^ (row & 7)) * 4)) =
            have ? make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const bool good = !(has_tree && !my_ok) && !bad_len && ok;
    if (half == 0) bars.st_lse[row] = !good ? NAN : (l_row > 0.f ? m_run + __log2f(l_row) : -INFINITY);
    // the stage is read by bulk copies (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (half == 0 && row_valid && has_tree && !my_ok) set_status(p.status, TV_DEV_BAD_PARENT);
    if (bad_len && has_tree && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
  }

  // ------------------------------------------------------------ cluster merge
  // Row t of the tile is merged by CTA t / merge_per.  Once every CTA is
  // past its main loop (the inboxes are the idle K rings), each CTA copies
  // its staged rows and their log-sum-exp to the owners with bulk copies
  // over distributed shared memory, completing on the owner's mbarrier;
  // each owner then merges its rows from local shared memory.
  const int rows_here = nodes_here * G;
  fence_before();
  cl.sync();                  // every CTA is past its main loop
  fence_after();
  if (warp == kWarpMma) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
  if (tid == 0) {
    for (int o = 0; o < C; ++o) {
      const int r0 = o * merge_per;
      const int nr = max(0, min(merge_per, rows_here - r0));
      if (nr == 0) continue;
      const uint32_t dst_rows = cluster_addr(base + kSmemInbox + (chunk * merge_per) * kD * 4, o);
      const uint32_t dst_lse = cluster_addr(smem_u32(&bars.in_lse[chunk * merge_per]), o);
      const uint32_t bar = cluster_addr(smem_u32(&bars.inbox_full), o);
      bulk_s2c(dst_rows, base + kSmemStage + r0 * kD * 4, static_cast<uint32_t>(nr) * kD * 4, bar);
      bulk_s2c(dst_lse, smem_u32(&bars.st_lse[r0]), static_cast<uint32_t>((nr + 3) & ~3) * 4, bar);
    }
  }
  // all copies into this CTA have landed
  const bool inbox_ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bars.inbox_full, 0));
  if (!inbox_ok) bars.abort = 1;
  // peers may leave once every CTA has received its rows (so every copy
  // that reads this CTA's stage is complete); the wait is at the very end
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (*abort && tid == 0) set_status(p.status, TV_DEV_TIMEOUT);
  {
    const float* inbox = reinterpret_cast<const float*>(gbase + kSmemInbox);
    const int r0 = chunk * merge_per;
    const bool bad_all = !inbox_ok;
    for (int lt = warp; lt < merge_per && r0 + lt < rows_here; lt += kThreads / 32) {
      const int t = r0 + lt;
      // every lane reads the chunks' log-sum-exp (shared-memory broadcast)
      float lc[kMaxCluster];
      float M = -INFINITY;
      bool bad = bad_all;
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c) {
        lc[c] = (c < C) ? bars.in_lse[c * merge_per + lt] : -INFINITY;
        bad |= (lc[c] != lc[c]);
        M = fmaxf(M, lc[c]);
      }
      float den = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const int phys = lane ^ (t & 7);
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c) {
        const float w = (c < C && lc[c] > -INFINITY) ? ex2_approx(lc[c] - M) : 0.f;
        den += w;
        if (w != 0.f) {
          const float4 v = *reinterpret_cast<const float4*>(inbox + (c * merge_per + lt) * kD + phys * 4);
          acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
          acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
        }
      }
      const bool okr = !bad && den > 0.f;
      const float iv = okr ? 1.f / den : 0.f;
      uint2 wv;
      if (okr) {
        wv.x = pack_bf16(acc.x * iv, acc.y * iv);
        wv.y = pack_bf16(acc.z * iv, acc.w * iv);
      } else {
        wv.x = wv.y = pack_bf16(NAN, NAN);
      }
      const int node = i0 + t / G, head = g * G + t % G;
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + node * p.o_st + head * p.o_sh;
      *reinterpret_cast<uint2*>(o + lane * 4) = wv;
      if (lane == 0 && p.lse)
        p.lse[(static_cast<int64_t>(b) * p.T + node) * p.Hq + head] =
            okr ? (M + __log2f(den)) * 0.6931471805599453f : NAN;
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
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

bool attn_tc_sparse_supported(const tv_attn_args* a) {
  if (a->sparse_topk <= 0 || a->block_size != 64 || a->sparse_topk > kMaxTopk) return false;
  if (a->Hq % a->Hkv != 0) return false;
  const int G = a->Hq / a->Hkv;
  if (G < 4 || 128 % G != 0) return false;                  // at most 32 nodes per row tile
  if ((kRows / G) * a->sparse_topk > kMaxUnion) return false;
  if ((a->Lmax + 63) / 64 > kMaxBlk) return false;
  tv_attn_args dense = *a;
  dense.sparse_topk = 0;
  return attn_tc_supported(&dense);
}

int attn_tc_active_clusters(int c) {
  // clusters of c chunk CTAs that can be resident at once (cached per device)
  static int cached[64][kMaxCluster + 1];
  static bool done[64][kMaxCluster + 1];
  int dev = 0;
  if (c < 1 || c > kMaxCluster) return 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (done[dev][c]) return cached[dev][c];
  int n = 0;
  const size_t smem = kSmemBytes + 1024;
  if (cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<false>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev][c] = n;
  done[dev][c] = true;
  return n;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mk64, mv64;
  const int G = p.G;
  if (p.nchunk < 1 || p.nchunk > kMaxCluster) return cudaErrorInvalidValue;
  if (p.tc_sparse && p.nchunk != 1) return cudaErrorInvalidValue;
  if (!make_map(&mq, p.q, p.d, p.Hq, p.T, p.B, p.q_sh, p.q_st, p.q_sb, G, kRows / G) ||
      !make_map(&mk, p.kc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys) ||
      !make_map(&mv, p.vc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys))
    return cudaErrorInvalidValue;
  if (p.tc_sparse) {
    if (!make_map(&mk64, p.kc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, 64) ||
        !make_map(&mv64, p.vc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, 64))
      return cudaErrorInvalidValue;
  } else {
    mk64 = mk;
    mv64 = mv;
  }
  auto kernel = p.tc_sparse ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  const size_t smem = kSmemBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + p.node_tile - 1) / p.node_tile;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nchunk, ntiles, p.B * p.Hkv);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.nchunk;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, mk64, mv64, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tv
