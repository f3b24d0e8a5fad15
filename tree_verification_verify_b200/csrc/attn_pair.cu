// tree_verify_attn, tensor-core kernel for long prefixes (sm_100a: tcgen05 +
// TMEM + TMA), bf16 with d = 128: two 128-row query tiles per CTA.
//
// Same computation as attn_tc.cu (SpecExec page, "Approach": the whole tree
// is verified in one target pass; node i attends to the shared prefix and to
// its root path), organised for throughput when the prefix is long.  The G
// query heads of one kv head are packed with the tree nodes into 128-row
// tiles A and B (row r = node r / G, head r % G), and every K/V tile a CTA
// loads serves both: half the K/V traffic per FLOP of a one-tile CTA.  The two
// tiles' chains interleave on the tensor pipe,
//
//     ... PV_A(j)  S_A(j+1)  PV_B(j)  S_B(j+1)  PV_A(j+1) ...
//
// so the softmax of one tile runs while the other tile's MMAs execute.
// TMEM (512 columns): S_A, S_B, O_A, O_B (128 each); P_t is written as bf16
// pairs over the first 64 columns of S_t.
//
// One CTA owns (sequence, kv head, tile pair, prefix chunk); the chunks of a
// pair form a thread-block cluster.  The last chunk also runs the tree tiles:
// the union U of the root paths of both tiles' nodes, gathered into K/V
// tiles and masked per row by the row's ancestors in U.  At the end the
// chunks' normalised O rows and log-sum-exps are merged over distributed
// shared memory, tile A then tile B; or, when the planner splits a pair into
// more chunks than a cluster holds at once, through the workspace: every
// chunk writes its normalised fp32 rows and log-sum-exps to its slot, and
// the last chunk of the pair to finish (a ticket) merges them.
//
// Warp roles (384 threads):
//   warps 0-3  softmax / correction / epilogue of tile A: thread t owns row
//              t (TMEM lane t) and all 128 key columns of every S tile;
//   warps 4-7  the same for tile B;
//   warp 8     Q (both tiles) and the K tiles: TMA into a two-stage ring
//              (128B swizzle, K-major) or, for tree tiles, a cp.async gather;
//   warp 9     TMEM allocator and MMA issuer (one thread, both tiles);
//   warp 10    the V tiles, a two-stage ring (MN-major), like warp 8;
//   warp 11    tree bookkeeping (last chunk): parent[] into shared memory,
//              the node bitmap of U, the slot of every node of U and the
//              slot of its parent.
// A K stage is released when the last S of its tile completes, a V stage
// when the last P V completes.  S_t(j+1) overwrites P_t(j): it is issued
// right behind P_t(j) V (MMAs of one thread execute in issue order).  Online softmax in base 2 with a lazily
// updated maximum: O_t and its row sum are rescaled only when the maximum
// grows by more than 2^8, which keeps P <= 256 (exact in the final O / l).
//
// Every mbarrier wait is bounded: on expiry the CTA records TV_DEV_TIMEOUT,
// stops issuing work, drains what it issued, frees its TMEM, and its rows
// come out as NaN.
#include <cooperative_groups.h>

#include "attn.cuh"
#include "tc_prims.cuh"

namespace cg = cooperative_groups;

namespace tv {

namespace tcp {

using namespace tc;

constexpr int kThreads = 384;
constexpr int kWarpK = 8, kWarpMma = 9, kWarpV = 10, kWarpTree = 11;
constexpr int kRows = 128;          // M of one query tile
constexpr int kKeys = 128;          // keys per K/V tile
constexpr int kD = 128;
constexpr int kKS = 2;              // K ring stages
constexpr int kVS = 2;              // V ring stages
constexpr int kMaxT = 2048;         // tree nodes handled by this kernel
constexpr int kMaxCluster = 8;      // chunks per tile pair merged over distributed shared memory
constexpr int kMaxChunksGlobal = 16;  // chunks per tile pair merged through the workspace
constexpr uint32_t kHalfBytes = kRows * 128;            // 128 rows x 128 B
constexpr uint32_t kTileBytes = 2 * kHalfBytes;         // 32 KB (d = 128 bf16)
constexpr uint32_t kSmemQ = 0;                            // Q_A, Q_B
constexpr uint32_t kSmemK = kSmemQ + 2 * kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kKS * kTileBytes;
constexpr uint32_t kSmemPar = kSmemV + kVS * kTileBytes;  // parent[] (u16)
constexpr uint32_t kSmemUL = kSmemPar + kMaxT * 2;        // U: slot -> node (u16)
constexpr uint32_t kSmemUP = kSmemUL + kMaxT * 2;         // U: slot -> parent's slot (u16)
constexpr uint32_t kSmemBytes = kSmemUP + kMaxT * 2;      // 204 KB
constexpr uint32_t kSmemInbox = kSmemQ;                   // merge: Q region and K ring (idle)
constexpr uint32_t kSmemStage = kSmemV;                   // merge: the idle V ring
constexpr int kMaxInboxRows = 144;                        // max over C of C * per (per = 4 * ceil(128 / 4C))
constexpr uint32_t kTmemCols = 512;
constexpr uint16_t kRootMark = 0xFFFEu;   // parent[] entry of a well-formed root
constexpr uint16_t kBadMark = 0xFFFFu;    // malformed parent (or no parent slot)

static_assert(kSmemInbox + kMaxInboxRows * kD * 4 + kMaxInboxRows * 4 <= kSmemStage,
              "the merge inbox fits below the stage");
static_assert(kSmemStage + kRows * kD * 4 <= kSmemV + kVS * kTileBytes, "the merge stage fits the V ring");

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int t) { return t ? 384u : 256u; }

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKS], k_empty[kKS];
  uint64_t v_full[kVS], v_empty[kVS];
  uint64_t s_full[2];               // per query tile: S_t(j) landed
  uint64_t p_full[2];               // per query tile: P_t(j) written (4 warps)
  uint64_t pv_done[2];              // per query tile: P_t(j) V completed
  uint64_t tree_info;
  uint64_t inbox_full;              // merge round r: phase r
  uint32_t tmem_base;
  int abort;
  int last;                         // workspace merge: this CTA merges the pair's chunks
  int nU;                           // nodes in the union of root paths
  uint32_t bm[kMaxT / 32];          // node bitmap of U
  int pre[kMaxT / 32];              // marked nodes below each bitmap word
  int node_ok[2 * kRows];           // root path of the pair's node is well formed
  alignas(16) float st_lse[kRows];  // this CTA's rows of the round's tile: log2-sum-exp (NaN: invalid)
  alignas(16) float in_lse[kMaxInboxRows];  // merge inbox: log2-sum-exp of row (chunk, row)
};

// Slot of node a in U: the number of marked nodes below a.
__device__ __forceinline__ int u_slot(const Bars& bars, int a) {
  return bars.pre[a >> 5] + __popc(bars.bm[a >> 5] & ((1u << (a & 31)) - 1u));
}

// Bytes a merging CTA receives from one chunk for `rows` rows: the fp32 O
// rows and their log-sum-exp (padded to 16 bytes).
__host__ __device__ constexpr uint32_t merge_bytes(int rows) {
  return rows > 0 ? static_cast<uint32_t>(rows) * kD * 4 + static_cast<uint32_t>((rows + 3) & ~3) * 4 : 0u;
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

}  // namespace tcp

using namespace tcp;

__global__ void __launch_bounds__(kThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, AttnParams p) {
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ Bars bars;
  cg::cluster_group cl = cg::this_cluster();
  const int chunk = blockIdx.x;            // = rank in the cluster (the cluster spans the chunks)
  const int C = static_cast<int>(gridDim.x);
  const int pair = blockIdx.y;
  const int b = blockIdx.z / p.Hkv, g = blockIdx.z % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int NT = kRows / G;                // nodes per query tile
  // the early exits depend on (sequence, pair) only: a cluster leaves whole
  const int n = p.n_nodes ? p.n_nodes[b] : p.T;
  if (n < 0 || n > p.T) {
    if (chunk == C - 1 && pair == 0 && g == 0 && tid == 0) set_status(p.status, TV_DEV_BAD_LEN);
    return;
  }
  const int i0 = pair * 2 * NT;
  if (i0 >= n) return;
  const int32_t* par = p.parent + b * p.par_sb;
  const int Lraw = p.prefix_len[b];
  const bool bad_len = (Lraw < 0 || Lraw > p.Lmax);
  const int L = bad_len ? 0 : Lraw;
  const int k0 = chunk * p.chunk_len;
  const int k1 = min(k0 + p.chunk_len, L);
  const int nprefix = (k1 > k0) ? (k1 - k0 + kKeys - 1) / kKeys : 0;
  const int nodes_a = min(NT, n - i0);
  const int nodes_b = max(0, min(NT, n - i0 - NT));
  const int nq = nodes_b > 0 ? 2 : 1;      // query tiles with rows
  const int nodes_here = nodes_a + nodes_b;
  // the last chunk (the shortest) also runs the tree tiles, unless the call
  // is a prefix-only partial
  const bool has_tree = (chunk == C - 1) && !p.prefix_only;
  // softmax threads: tile qt = warp / 4, row = TMEM lane = tid % 128
  const int qt = (warp >> 2) & 1;
  const int row = tid & (kRows - 1);
  const int row_node = i0 + qt * NT + row / G;
  const int nodes_qt = qt ? nodes_b : nodes_a;
  const bool row_valid = warp < 8 && qt < nq && (row / G) < nodes_qt;

  // 1024-aligned dynamic shared memory (128B swizzle atoms are 1 KB)
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem_raw + (base - raw);
  uint16_t* spar = reinterpret_cast<uint16_t*>(gbase + kSmemPar);
  uint16_t* ulist = reinterpret_cast<uint16_t*>(gbase + kSmemUL);
  uint16_t* uparent = reinterpret_cast<uint16_t*>(gbase + kSmemUP);
  volatile int* abort = &bars.abort;

  // rows [c * per, (c + 1) * per) of a tile are merged by CTA c
  auto merge_per = [&](int t) -> int {
    const int rows = (t ? nodes_b : nodes_a) * G;
    return 4 * ((rows + 4 * C - 1) / (4 * C));
  };
  auto own_rows = [&](int t) -> int {
    const int rows = (t ? nodes_b : nodes_a) * G;
    const int per = merge_per(t);
    return max(0, min(per, rows - chunk * per));
  };

  if (tid == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kKS; ++s) { mbar_init(&bars.k_full[s], 1); mbar_init(&bars.k_empty[s], nq); }
    for (int s = 0; s < kVS; ++s) { mbar_init(&bars.v_full[s], 1); mbar_init(&bars.v_empty[s], nq); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], 4);
      mbar_init(&bars.pv_done[t], 1);
    }
    mbar_init(&bars.tree_info, 1);
    mbar_init(&bars.inbox_full, 1);
    bars.abort = 0;
    bars.nU = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // the bytes the cluster will copy into this CTA's inbox in round 0
    if (!p.gmerge) mbar_expect_tx(&bars.inbox_full, static_cast<uint32_t>(C) * merge_bytes(own_rows(0)));
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
  // a softmax thread's row after its main loop: log2-sum-exp (NaN: invalid)
  // and 1 / row sum (0: no keys), staged in the tile's merge round
  float ep_lse2 = NAN, ep_inv = 0.f;

  // ------------------------------------------------------------ MMA issuer
  // One thread issues both tiles' chains: S_t(0), then per key tile j and
  // tile t, P_t(j) V and S_t(j + 1), which overwrites P_t(j) in TMEM.  MMAs
  // issued by one thread execute in issue order, so S_t(j + 1) queued behind
  // P_t(j) V writes S_t only after that MMA has read P_t(j): both go to the
  // tensor pipe back to back.  Issuing tile A's pair, then tile B's, keeps
  // the two softmaxes a half period apart (each runs while the other tile's
  // MMAs execute); one issuer per tile lets them drift into step and fight
  // for the same schedulers.  A K or V stage is released when both tiles'
  // MMAs that read it have completed (the empty barriers count one commit
  // per tile).
  auto run_issuer = [&]() {
    bool ok = true;
    int ntot = nprefix;
    bool tree_known = !has_tree;
    // the tree tiles follow the prefix tiles; their count is known once the
    // tree warp has built U
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
    int s_issued[2] = {0, 0}, pv_issued[2] = {0, 0};
    // S_t(j) = Q_t K_j^T into S_t
    auto issue_s = [&](int t, int j) {
      const uint32_t sq = base + kSmemQ + t * kTileBytes;
      const uint32_t sk = base + kSmemK + (j % kKS) * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_bf16(tmem + col_s(t), smem_desc(sq + off, 16, 1024), smem_desc(sk + off, 16, 1024), idesc_qk,
                 kk > 0);
      }
      mma_commit(&bars.s_full[t]);
      mma_commit(&bars.k_empty[j % kKS]);
      ++s_issued[t];
    };
    // O_t += P_t(j) V_j, P_t read from the first 64 columns of S_t
    auto issue_pv = [&](int t, int j) {
      const uint32_t sv = base + kSmemV + (j % kVS) * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, smem_desc(sv + kk * 2048, kHalfBytes, 1024),
                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars.pv_done[t]);
      mma_commit(&bars.v_empty[j % kVS]);
      ++pv_issued[t];
    };
    ok = know(0);
    if (ok && ntot > 0) ok = mbar_wait3(&bars.q_full, 0, &bars.k_full[0], 0, nullptr, 0u, abort);
    if (ok && ntot > 0) {
      fence_after();
      for (int t = 0; t < nq; ++t) issue_s(t, 0);
    }
    for (int j = 0; ok; ++j) {
      ok = know(j);
      if (!ok || j >= ntot) break;
      ok = know(j + 1);
      if (!ok) break;
      const bool next = j + 1 < ntot;
      for (int t = 0; t < nq && ok; ++t) {
        // P_t(j), V(j) and, for S_t(j + 1), K(j + 1): one wait
        ok = mbar_wait3(&bars.p_full[t], j & 1, &bars.v_full[j % kVS], (j / kVS) & 1,
                        next ? &bars.k_full[(j + 1) % kKS] : nullptr, ((j + 1) / kKS) & 1, abort);
        if (!ok) break;
        fence_after();
        issue_pv(t, j);
        if (next) issue_s(t, j + 1);
      }
    }
    if (!ok) {
      // the issued MMAs complete before the TMEM is freed: they execute in
      // issue order, and a tile's next P V waits for its softmax, which
      // waits for its S, so each barrier has at most its last phase open
      for (int t = 0; t < 2; ++t) {
        if (s_issued[t] > 0) mbar_drain(&bars.s_full[t], (s_issued[t] - 1) & 1);
        if (pv_issued[t] > 0) mbar_drain(&bars.pv_done[t], (pv_issued[t] - 1) & 1);
      }
    }
  };

  if (warp == kWarpTree) {
    // ------------------------------------------------------------ tree bookkeeping
    if (has_tree) {
      for (int j = lane; j < n; j += 32) {
        const int pj = par[j];
        spar[j] = (j == 0) ? (pj == -1 ? kRootMark : kBadMark)
                           : ((pj >= 0 && pj < j) ? static_cast<uint16_t>(pj) : kBadMark);
      }
      const int nw = (n + 31) >> 5;
      for (int w = lane; w < nw; w += 32) bars.bm[w] = 0u;
      __syncwarp();
      // mark the root path of every node of the pair (parents strictly
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
  } else if (warp == kWarpMma) {
    if (lane == 0) run_issuer();
    __syncwarp();
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
      mbar_expect_tx(&bars.q_full, static_cast<uint32_t>(nq) * kTileBytes);
      for (int t = 0; t < nq; ++t) {
        tma_load_4d(&tmap_q, sq + t * kTileBytes, &bars.q_full, 0, g * G, i0 + t * NT, b);
        tma_load_4d(&tmap_q, sq + t * kTileBytes + kHalfBytes, &bars.q_full, 64, g * G, i0 + t * NT, b);
      }
    }
    int ntot = nprefix, ntree = 0;
    bool tree_known = !has_tree;
    int issued = 0;
    for (int j = 0;; ++j) {
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
      if (j < nprefix) {
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
  } else if (qt < nq) {
    // ------------------------------------------------------------ softmax warps of tile qt
    const float sl2 = p.scale * 1.4426950408889634f;   // scores in log2 units
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t scol = col_s(qt), ocol = col_o(qt);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int ntot = nprefix, ntree = 0;
    bool my_ok = true;
    bool tree_known = !has_tree;
    int cur = -1;                 // walk position (slot) on this row's root path
    for (int j = 0; ok; ++j) {
      if (!tree_known && j == nprefix) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.tree_info, 0, abort));
        if (!ok) break;
        ntree = (bars.nU + kKeys - 1) / kKeys;
        ntot += ntree;
        my_ok = row_valid && bars.node_ok[qt * NT + row / G] != 0;
        cur = my_ok ? u_slot(bars, row_node) : -1;
        tree_known = true;
      }
      if (j >= ntot) break;
      const bool tree_tile = j >= nprefix;
      const int nk = tree_tile ? 0 : min(kKeys, k1 - (k0 + j * kKeys));
      const bool full = !tree_tile && nk == kKeys;
      // key mask of the tile's 128 columns, four words
      uint32_t mk[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (tree_tile) {
        // ancestors of this row's node in slots [128 tt, + 128); the tiles
        // run downwards and slots decrease along the path, so the walk
        // continues where the previous tile left it
        mk[0] = mk[1] = mk[2] = mk[3] = 0u;
        const int lo = (ntree - 1 - (j - nprefix)) * kKeys;
        while (cur >= lo) {
          if (cur < lo + kKeys) {
            const int w = (cur - lo) >> 5;
            const uint32_t bit = 1u << (cur & 31);
            mk[0] |= w == 0 ? bit : 0u;
            mk[1] |= w == 1 ? bit : 0u;
            mk[2] |= w == 2 ? bit : 0u;
            mk[3] |= w == 3 ? bit : 0u;
          }
          const uint16_t up = uparent[cur];
          cur = (up == kBadMark) ? -1 : static_cast<int>(up);
        }
      } else if (!full) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int nh = nk - 32 * w;
          mk[w] = nh >= 32 ? 0xffffffffu : (nh <= 0 ? 0u : ((1u << nh) - 1u));
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[qt], j & 1, abort));
      if (!ok) break;
      fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(trow + scol + 32 * c, s + 32 * c);
      tmem_wait_ld();
      // the tile maximum of the raw scores (scale > 0 keeps the order)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          s[c] = ((mk[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
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
      // p = 2^(s sl2 - m) (masked scores are -inf and give 0), written as
      // bf16 pairs: keys 32 c .. 32 c + 31 into columns 16 c .. 16 c + 15,
      // which this thread has read already
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a0 = ex2_approx(fmaf(s[32 * c + 2 * e], sl2, nmu));
          const float a1 = ex2_approx(fmaf(s[32 * c + 2 * e + 1], sl2, nmu));
          ps[(2 * e) & 3] += a0;
          ps[(2 * e + 1) & 3] += a1;
          pk[e] = pack_bf16(a0, a1);
        }
        tmem_st16u(trow + scol + 16 * c, pk);
      }
      l_run = l_run * factor + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      if (__any_sync(0xffffffffu, grow) && j > 0) {
        // O_t holds the tiles up to j - 1: wait for their P V, then rescale
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done[qt], (j - 1) & 1, abort));
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
      tmem_wait_st();
      // V rows that are not keys of this tile (past the prefix end) may hold
      // anything: tile A's warps zero them before the first P V reads the
      // tile (tile B's P V is issued after tile A's)
      if (qt == 0 && !tree_tile && nk < kKeys) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.v_full[j % kVS], (j / kVS) & 1, abort));
        if (!ok) break;
        if (row >= nk) {
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
      if (lane == 0) mbar_arrive(&bars.p_full[qt]);
    }
    // ------------------------------------------------------------ epilogue
    // S_t(ntot - 1) executed after P_t(ntot - 2) V (issue order), so phase
    // ntot - 1 of pv_done is the next one to complete
    if (ok && ntot > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done[qt], (ntot - 1) & 1, abort));
    fence_after();
    const bool have = ok && l_run > 0.f;
    const float inv = have ? 1.f / l_run : 0.f;
    const bool good = !(has_tree && !my_ok) && !bad_len && ok;
    const float lse2 = !good ? NAN : (l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY);
    ep_lse2 = lse2;
    ep_inv = inv;
    if (row_valid && has_tree && !my_ok) set_status(p.status, TV_DEV_BAD_PARENT);
    if (bad_len && chunk == C - 1 && qt == 0 && row == 0) set_status(p.status, TV_DEV_BAD_LEN);
  }

  if (p.gmerge) {
    // ---------------------------------------------------------- workspace merge
    // Slot (unit, chunk) holds the chunk's normalised fp32 O rows of both
    // tiles and their log2-sum-exp; the last chunk to finish merges.
    const int unit = static_cast<int>(blockIdx.z) * static_cast<int>(gridDim.y) + pair;
    fence_before();
    __syncthreads();
    fence_after();
    if (warp < 8 && qt < nq) {
      const float inv = ep_inv;
      const bool have = inv > 0.f;
      float* dst = p.part_o + ((static_cast<int64_t>(unit) * C + chunk) * 2 + qt) * kRows * kD +
                   static_cast<int64_t>(row) * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + col_o(qt) + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          __stcg(reinterpret_cast<float4*>(dst + c * 32 + 4 * q),
                 have ? make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv)
                      : make_float4(0.f, 0.f, 0.f, 0.f));
      }
      __stcg(p.part_lse + ((static_cast<int64_t>(unit) * C + chunk) * 2 + qt) * kRows + row, ep_lse2);
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int t = atomicAdd(&p.tickets[unit], 1);
      bars.last = (t == C - 1) ? 1 : 0;
      if (bars.last) {
        __threadfence();
        p.tickets[unit] = 0;                   // ready for the next call
      }
    }
    __syncthreads();
    if (bars.last) {
      for (int r = 0; r < nq; ++r) {
        const int rows_r = (r ? nodes_b : nodes_a) * G;
        for (int t = warp; t < rows_r; t += kThreads / 32) {
          const float* ls = p.part_lse + static_cast<int64_t>(unit) * C * 2 * kRows + r * kRows + t;
          float M = -INFINITY;
          bool bad = false;
          for (int c = 0; c < C; ++c) {
            const float lc = __ldcg(ls + c * 2 * kRows);
            bad |= (lc != lc);
            M = fmaxf(M, lc);
          }
          float den = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int c = 0; c < C; ++c) {
            const float lc = __ldcg(ls + c * 2 * kRows);
            const float w = (lc > -INFINITY) ? ex2_approx(lc - M) : 0.f;
            den += w;
            if (w != 0.f) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(
                  p.part_o + ((static_cast<int64_t>(unit) * C + c) * 2 + r) * kRows * kD +
                  static_cast<int64_t>(t) * kD + lane * 4));
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
          const int node = i0 + r * NT + t / G, head = g * G + t % G;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + node * p.o_st + head * p.o_sh;
          *reinterpret_cast<uint2*>(o + lane * 4) = wv;
          if (lane == 0 && p.lse)
            p.lse[(static_cast<int64_t>(b) * p.T + node) * p.Hq + head] =
                okr ? (M + __log2f(den)) * 0.6931471805599453f : (empty ? -INFINITY : NAN);
        }
      }
    }
  } else {
  // ------------------------------------------------------------ cluster merge
  // One round per query tile.  Each CTA stages its normalised fp32 O rows of
  // the tile (the idle V ring) and their log2-sum-exp; once every CTA has
  // staged (cluster barrier), each copies its rows to their owners with bulk
  // copies over distributed shared memory, completing on the owner's
  // mbarrier; each owner merges its share from local shared memory.  A
  // second cluster barrier ends the round: every copy out of every stage has
  // landed, so the stage and inbox can be reused.
  for (int r = 0; r < nq; ++r) {
    const int rows_r = (r ? nodes_b : nodes_a) * G;
    const int per = merge_per(r);
    // every warp is past its main loop: the last P V of each tile has
    // completed (the softmax warps waited for it), so no MMA reads the V
    // ring any more and it can hold the stage
    fence_before();
    __syncthreads();
    fence_after();
    if (warp < 8 && qt == r) {
      const float lse2 = ep_lse2, inv = ep_inv;
      const bool have = inv > 0.f;
      float* stage = reinterpret_cast<float*>(gbase + kSmemStage) + row * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + col_o(r) + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int qq = c * 8 + q;
          *reinterpret_cast<float4*>(stage + ((qq ^ (row & 7)) * 4)) =
              have ? make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      bars.st_lse[row] = lse2;
      // the stage is read by bulk copies (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    fence_before();
    cl.sync();                  // every CTA has staged; every inbox is idle
    fence_after();
    if (tid == 0) {
      for (int o = 0; o < C; ++o) {
        const int r0 = o * per;
        const int nr = max(0, min(per, rows_r - r0));
        if (nr == 0) continue;
        const uint32_t dst_rows = cluster_addr(base + kSmemInbox + (chunk * per) * kD * 4, o);
        const uint32_t dst_lse = cluster_addr(smem_u32(&bars.in_lse[chunk * per]), o);
        const uint32_t bar = cluster_addr(smem_u32(&bars.inbox_full), o);
        bulk_s2c(dst_rows, base + kSmemStage + r0 * kD * 4, static_cast<uint32_t>(nr) * kD * 4, bar);
        bulk_s2c(dst_lse, smem_u32(&bars.st_lse[r0]), static_cast<uint32_t>((nr + 3) & ~3) * 4, bar);
      }
    }
    // all copies into this CTA have landed
    const bool inbox_ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bars.inbox_full, r & 1));
    if (!inbox_ok) bars.abort = 1;
    __syncthreads();
    // the next round's bytes (peers copy them only after the next barrier)
    if (tid == 0 && r + 1 < nq)
      mbar_expect_tx(&bars.inbox_full, static_cast<uint32_t>(C) * merge_bytes(own_rows(r + 1)));
    {
      const float* inbox = reinterpret_cast<const float*>(gbase + kSmemInbox);
      const int r0 = chunk * per;
      const bool bad_all = !inbox_ok;
      for (int lt = warp; lt < per && r0 + lt < rows_r; lt += kThreads / 32) {
        const int t = r0 + lt;
        // every lane reads the chunks' log-sum-exp (shared-memory broadcast)
        float lc[kMaxCluster];
        float M = -INFINITY;
        bool bad = bad_all;
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c) {
          lc[c] = (c < C) ? bars.in_lse[c * per + lt] : -INFINITY;
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
            const float4 v = *reinterpret_cast<const float4*>(inbox + (c * per + lt) * kD + phys * 4);
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
        const int node = i0 + r * NT + t / G, head = g * G + t % G;
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + b * p.o_sb + node * p.o_st + head * p.o_sh;
        *reinterpret_cast<uint2*>(o + lane * 4) = wv;
        if (lane == 0 && p.lse)
          p.lse[(static_cast<int64_t>(b) * p.T + node) * p.Hq + head] =
              okr ? (M + __log2f(den)) * 0.6931471805599453f : (empty ? -INFINITY : NAN);
      }
    }
    fence_before();
    cl.sync();                  // every copy out of every stage has landed; inboxes consumed
    fence_after();
  }
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
  if (*abort && tid == 0) set_status(p.status, TV_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ host side

int attn_pair_active_clusters(int c) {
  // clusters of c chunk CTAs that can be resident at once (cached per device)
  static int cached[64][kMaxCluster + 1];
  static bool done[64][kMaxCluster + 1];
  int dev = 0;
  if (c < 1 || c > kMaxCluster) return 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (done[dev][c]) return cached[dev][c];
  int n = 0;
  const size_t smem = kSmemBytes + 1024;
  if (cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev][c] = n;
  done[dev][c] = true;
  return n;
}

cudaError_t launch_attn_pair(const AttnParams& p, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const int G = p.G;
  if (p.nchunk < 1 || p.nchunk > (p.gmerge ? kMaxChunksGlobal : kMaxCluster) || p.T > kMaxT || p.d != kD)
    return cudaErrorInvalidValue;
  if (!tcmap::make_map(&mq, p.q, p.d, p.Hq, p.T, p.B, p.q_sh, p.q_st, p.q_sb, G, kRows / G) ||
      !tcmap::make_map(&mk, p.kc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys) ||
      !tcmap::make_map(&mv, p.vc, p.d, p.Hkv, p.Lmax, p.B, p.kv_sh, p.kv_sl, p.kv_sb, 1, kKeys))
    return cudaErrorInvalidValue;
  const size_t smem = kSmemBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + kRows / G - 1) / (kRows / G);
  const int npairs = (ntiles + 1) / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nchunk, npairs, p.B * p.Hkv);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.nchunk;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.gmerge ? 0 : 1;         // chunks merged through the workspace need no cluster
  e = cudaLaunchKernelEx(&cfg, attn_pair_kernel, mq, mk, mv, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tv
