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
// Warp roles (384 threads):
//   warps 0-7  softmax / correction / epilogue: warps w and w + 4 own TMEM
//              lanes 32 (w % 4) .. (query rows), warp w < 4 key columns
//              0-63 of every tile, warp w + 4 columns 64-127 (tcgen05.ld
//              32x32b).  The two column halves of a row keep independent
//              online-softmax states, each with its own O accumulator, and
//              combine them once at the end;
//   warp 8     Q and the K tiles: TMA into a three-stage ring (128B swizzle,
//              K-major) or, for tree tiles, a cp.async gather;
//   warp 9     TMEM allocator and MMA issuer (one thread): S = Q K^T into
//              one of two TMEM S buffers, O_h += P_h V_h per column half h
//              with P_h read from TMEM;
//   warp 10    the V tiles, a two-stage ring (MN-major), like warp 8;
//   warp 11    tree bookkeeping (last chunk): parent[] into shared memory,
//              the node bitmap of U, the slot of every node of U and the
//              slot of its parent.
// A K stage is released when its S = Q K^T completes, a V stage when its
// P V completes, so the loads of later tiles start while earlier tiles are
// in the softmax.  S(j+2) reuses the TMEM buffer that P(j) is read from; it
// is issued right behind P(j) V (MMAs of one thread execute in issue order).  Online softmax in base 2 with a lazily updated maximum
// per row half: O_h and its row sum are rescaled only when the half's
// maximum grows by more than 2^8, which keeps P <= 256 (exact in the final
// O / l).  P_h is written as bf16 over the first 32 columns of the half's
// own 64 S columns, so neither half writes where the other still reads.
// Every mbarrier wait is bounded: on expiry the CTA records TV_DEV_TIMEOUT,
// stops issuing work, drains what it issued, frees its TMEM, and its rows
// come out as NaN.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cooperative_groups.h>

#include "attn.cuh"
#include "tc_prims.cuh"

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
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;  // O_h: column half h
constexpr uint16_t kRootMark = 0xFFFEu;   // parent[] entry of a well-formed root
constexpr uint16_t kBadMark = 0xFFFFu;    // malformed parent (or no parent slot)

static_assert(kSmemInbox + kMaxInboxRows * kD * 4 <= kSmemK + kKS * kTileBytes,
              "the merge inbox fits the K ring");
static_assert(kSmemStage + kRows * kD * 4 <= kSmemV + kVS * kTileBytes, "the merge stage fits the V ring");

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKS], k_empty[kKS];
  uint64_t v_full[kVS], v_empty[kVS];
  uint64_t s_full[2], p_full[2][2];   // p_full[S buffer][column half]
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
  uint64_t sum_ready;               // both halves have posted their final maximum and row sum
  float red_m[2][kRows];            // [half][row] the half's running maximum (log2 units)
  float red_l[2][kRows];            // [half][row] the half's row sum
  alignas(16) float in_lse[kMaxInboxRows];  // merge inbox: log2-sum-exp of row (chunk, row)
};


// Slot of node a in U: the number of marked nodes below a.
__device__ __forceinline__ int u_slot(const Bars& bars, int a) {
  return bars.pre[a >> 5] + __popc(bars.bm[a >> 5] & ((1u << (a & 31)) - 1u));
}

__device__ __forceinline__ uint32_t s_col(int j) { return (j & 1) ? kColS1 : kColS0; }

// Bytes a merging CTA receives from one chunk for `rows` rows: the fp32 O
// rows and their log-sum-exp (padded to 16 bytes).
__host__ __device__ constexpr uint32_t merge_bytes(int rows) {
  return rows > 0 ? static_cast<uint32_t>(rows) * kD * 4 + static_cast<uint32_t>((rows + 3) & ~3) * 4 : 0u;
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
  // the last chunk (the shortest) also runs the tree tiles, unless the call
  // is a prefix-only partial
  const bool has_tree = (chunk == C - 1) && !p.prefix_only;
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
      mbar_init(&bars.p_full[s][0], kSoftmaxThreads / 64);
      mbar_init(&bars.p_full[s][1], kSoftmaxThreads / 64);
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
        // V(j) and the first half's P(j) in one wait
        ok = mbar_wait3(&bars.v_full[j % kVS], (j / kVS) & 1, &bars.p_full[j & 1][0], (j >> 1) & 1, nullptr, 0u,
                        abort);
        const uint32_t sv = base + kSmemV + (j % kVS) * kTileBytes;
        // O_h += P_h V_h: P_h (128 rows x 64 keys, bf16 pairs) sits in the
        // first 32 columns of the half's own S columns 64 h ..; V_h is rows
        // 64 h .. 64 h + 63 of the V tile (16 keys = 2 KB per K step).  Once
        // any of it is issued, its completion is committed (V stage, pv_done)
        // even when the second half never comes.
        bool any = false;
        for (int h = 0; h < 2 && ok; ++h) {
          if (h > 0) ok = mbar_wait(&bars.p_full[j & 1][h], (j >> 1) & 1, abort);
          if (!ok) break;
          fence_after();
          const uint32_t od = tmem + (h ? kColO1 : kColO0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(od, tmem + s_col(j) + 64 * h + kk * 8,
                        smem_desc(sv + (4 * h + kk) * 2048, kHalfBytes, 1024), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          any = true;
        }
        if (any) {
          mma_commit(&bars.v_empty[j % kVS]);
          mma_commit(&bars.pv_done);
          ++pv_issued;
        }
        if (!ok) break;
        const int jn = j + 2;
        ok = know(jn);
        if (!ok) break;
        if (jn < ntot) {
          ok = mbar_wait(&bars.k_full[jn % kKS], (jn / kKS) & 1, abort);
          if (!ok) break;
          fence_after();
          // S(jn) overwrites the buffer P(j) is read from: MMAs of this
          // thread execute in issue order, so it is queued right behind P(j) V
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
    // Each half runs its own online softmax (maximum, row sum, O_h); the two
    // are combined once, in the epilogue.
    const float sl2 = p.scale * 1.4426950408889634f;   // scores in log2 units
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t hcol = 64u * static_cast<uint32_t>(half);
    const uint32_t ocol = half ? kColO1 : kColO0;
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
      // a full prefix tile needs no mask (the common case)
      const bool full = !tree_tile && !SPARSE && nk == kKeys;
      // key mask of this half's 64 columns: two words, kept in registers
      uint32_t mkA = 0xffffffffu, mkB = 0xffffffffu;
      if (tree_tile) {
        // ancestors of this row's node in slots [128 tt + 64 half, + 64);
        // the tiles run downwards and slots decrease along the path, so the
        // walk continues where the previous tile left it
        mkA = mkB = 0u;
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
      } else if (!full) {
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
      // the half's tile maximum of the raw scores (scale > 0 keeps the
      // order), over four interleaved partial maxima
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint32_t mw = (c < 32) ? mkA : mkB;
          s[c] = ((mw >> (c & 31)) & 1u) ? s[c] : -INFINITY;
          mx[c & 3] = fmaxf(mx[c & 3], s[c]);
        }
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
      const float m_new = fmaxf(m_run, mt);
      const bool grow = m_new > m_run + 8.0f;       // also the first finite maximum
      float factor = 1.f;
      if (grow) {
        factor = ex2_approx(m_run - m_new);         // 0 when m_run = -inf
        m_run = m_new;
      }
      const float nmu = (m_run == -INFINITY) ? 0.f : -m_run;
      // p = 2^(s sl2 - m): one FFMA and one ex2 per score (masked scores are
      // -inf and give 0)
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        s[c] = ex2_approx(fmaf(s[c], sl2, nmu));
        ps[c & 3] += s[c];
      }
      l_run = l_run * factor + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      if (__any_sync(0xffffffffu, grow) && j > 0) {
        // O_h holds the tiles up to j - 1: wait for their P V, then rescale
        // this half's accumulator (all 128 columns)
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (j - 1) & 1, abort));
        if (!ok) break;
        fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(trow + ocol + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= factor;
          tmem_st32(trow + ocol + c * 32, o);
        }
      }
      // P_h as bf16 pairs over the first 32 of the half's own 64 S columns
      // (this thread has read them all already)
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(s[2 * e], s[2 * e + 1]);
        tmem_st32u(trow + scol + hcol, pk);
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
        // the V rows a half multiplies are its own keys' rows: each half
        // zeroes the dead rows among its 64
        const int vr = 64 * half + (row & 63);
        const bool dead_row = SPARSE ? (half == 0 ? (row & 63) >= vka : (row & 63) >= vkb) : vr >= nk;
        if (row < 64 && dead_row) {
          uint8_t* sv = gbase + kSmemV + (j % kVS) * kTileBytes;
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(sv + vr * 128 + c * 16) = z;
            *reinterpret_cast<uint4*>(sv + kHalfBytes + vr * 128 + c * 16) = z;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[j & 1][half]);
    }
    // ------------------------------------------------------------ epilogue
    // The last P V is pv_done's phase ntot - 1.  S(ntot - 1) having landed
    // only proves P V up to ntot - 3, and a parity wait cannot tell phase
    // ntot - 1 from ntot - 3: wait for phase ntot - 2 first, then ntot - 1.
    if (ok && ntot > 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (ntot - 2) & 1, abort));
    if (ok && ntot > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (ntot - 1) & 1, abort));
    fence_after();
    // combine the halves: M = max(m_0, m_1), c_h = 2^(m_h - M),
    // O = (c_0 O_0 + c_1 O_1) / (c_0 l_0 + c_1 l_1); half h writes d columns
    // 64 h .. 64 h + 63
    bars.red_m[half][row] = m_run;
    bars.red_l[half][row] = l_run;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.sum_ready);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars.sum_ready, 0, abort));
    const float m_o = ok ? bars.red_m[half ^ 1][row] : -INFINITY;
    const float l_o = ok ? bars.red_l[half ^ 1][row] : 0.f;
    const float m_0 = half ? m_o : m_run, m_1 = half ? m_run : m_o;
    const float l_0 = half ? l_o : l_run, l_1 = half ? l_run : l_o;
    const float M = fmaxf(m_0, m_1);
    const float c_0 = (m_0 == -INFINITY) ? 0.f : ex2_approx(m_0 - M);
    const float c_1 = (m_1 == -INFINITY) ? 0.f : ex2_approx(m_1 - M);
    const float l_row = c_0 * l_0 + c_1 * l_1;
    const bool have = ok && l_row > 0.f;
    const float inv = have ? 1.f / l_row : 0.f;
    const float w0 = c_0 * inv, w1 = c_1 * inv;
    // this half's columns of the row's normalised O into the stage (the idle
    // V ring; fp32, float4 q of row t at q ^ (t & 7)) and the row's
    // log2-sum-exp
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    float* stage = reinterpret_cast<float*>(gbase + kSmemStage) + row * kD;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v0[32], v1[32];
      tmem_ld32(trow + kColO0 + hcol + c * 32, v0);
      tmem_ld32(trow + kColO1 + hcol + c * 32, v1);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int qq = 16 * half + c * 8 + q;
        float4 o;
        o.x = fmaf(w0, v0[4 * q], w1 * v1[4 * q]);
        o.y = fmaf(w0, v0[4 * q + 1], w1 * v1[4 * q + 1]);
        o.z = fmaf(w0, v0[4 * q + 2], w1 * v1[4 * q + 2]);
        o.w = fmaf(w0, v0[4 * q + 3], w1 * v1[4 * q + 3]);
        *reinterpret_cast<float4*>(stage + ((qq ^ (row & 7)) * 4)) = have ? o : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const bool good = !(has_tree && !my_ok) && !bad_len && ok;
    if (half == 0) bars.st_lse[row] = !good ? NAN : (l_row > 0.f ? M + __log2f(l_row) : -INFINITY);
    // the stage is read by bulk copies (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (half == 0 && row_valid && has_tree && !my_ok) set_status(p.status, TV_DEV_BAD_PARENT);
    if (bad_len && chunk == C - 1 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
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
      // no keys at all (an empty slice of a prefix-only partial): O = 0,
      // lse = -inf
      const bool empty = !bad && den == 0.f;
      const bool okr = !bad && den > 0.f;
      const float iv = okr ? 1.f / den : 0.f;
      uint2 wv;
      if (okr) {
        wv.x = pack_bf16(acc.x * iv, acc.y * iv);
        wv.y = pack_bf16(acc.z * iv, acc.w * iv);
      } else {
        wv.x = wv.y = empty ? 0u : pack_bf16(NAN, NAN);
      }
      const int node = i0 + t / G, head = g * G + t % G;
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + node * p.o_st + head * p.o_sh;
      *reinterpret_cast<uint2*>(o + lane * 4) = wv;
      if (lane == 0 && p.lse)
        p.lse[(static_cast<int64_t>(b) * p.T + node) * p.Hq + head] =
            okr ? (M + __log2f(den)) * 0.6931471805599453f : (empty ? -INFINITY : NAN);
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ host side

using tcmap::encode_fn;
using tcmap::make_map;

namespace {

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
