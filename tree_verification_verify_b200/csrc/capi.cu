// The C ABI of libtreeverify.so: host-side argument checks, the split-KV
// plan and workspace layout, and dispatch to the kernels.  Declared in
// include/tree_verify.h.
#include <cmath>
#include <cstring>

#include "attn.cuh"

namespace tv {
size_t accept_workspace_bytes(int B, int T);
constexpr int kAcceptMaxB = 16384;
cudaError_t launch_accept(const tv_accept_args* a, int mode, void* ws, cudaStream_t stream);
size_t expand_pool_bytes(int budget, int V);
cudaError_t launch_expand_init(const tv_expand_args* a, int root_token, cudaStream_t stream);
cudaError_t launch_expand(const tv_expand_args* a, cudaStream_t stream);
cudaError_t launch_expand_exp(const double* t, double* out, int n, cudaStream_t stream);
cudaError_t expand_set_wait_limit(uint32_t polls);
bool attn_tc_supported(const tv_attn_args* a);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream);
int attn_tc_active_clusters(int c);
cudaError_t launch_attn_pair(const AttnParams& p, cudaStream_t stream);
int attn_pair_active_clusters(int c);
bool attn_tc_sparse_supported(const tv_attn_args* a);
cudaError_t launch_block_means(const AttnParams& p, float* kbar, cudaStream_t stream);
cudaError_t launch_block_select(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_sparse(const AttnParams& p, cudaStream_t stream);
int num_sms();
cudaError_t launch_commit(const tv_commit_args* a, cudaStream_t stream);
cudaError_t launch_attn_partial_merge(const tv_attn_merge_args* a, cudaStream_t stream);
}  // namespace tv

using namespace tv;

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

tv_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TV_OK : TV_ERR_CUDA; }

bool ws_ok(const void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return true;
  return ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0;
}

// ------------------------------------------------------------ attention plan

struct AttnPlan {
  bool tc;            // tensor-core prefix kernel
  bool pair;          // ... in its two-query-tile form (attn_pair.cu)
  bool gmerge;        // ... with its chunks merged through the workspace
  bool sparse;
  bool tc_sparse;     // block top-k on the tensor-core kernel
  int nchunk, chunk_len, node_tile, nblk_max;
  size_t off_o, off_lse, off_ok, off_kbar, off_sel, off_scores, total;
};

tv_status check_attn(const tv_attn_args* a) {
  if (!a) return TV_ERR_INVALID_ARG;
  if (a->dtype != TV_FP32 && a->dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Lmax < 0) return TV_ERR_INVALID_ARG;
  if (a->Hq % a->Hkv != 0) return TV_ERR_INVALID_ARG;
  if (!(a->scale >= 0.f) || !std::isfinite(a->scale)) return TV_ERR_INVALID_ARG;
  if (a->sparse_topk < 0) return TV_ERR_INVALID_ARG;
  if (a->sparse_topk > 0 && a->block_size <= 0) return TV_ERR_INVALID_ARG;
  if (a->prefix_only != 0 && a->prefix_only != 1) return TV_ERR_INVALID_ARG;
  if (a->prefix_only && a->sparse_topk > 0) return TV_ERR_UNSUPPORTED;
  if (a->d != 32 && a->d != 64 && a->d != 128) return TV_ERR_UNSUPPORTED;
  if (a->Hq / a->Hkv > 64) return TV_ERR_UNSUPPORTED;
  if (a->B > 0 && a->T > 0) {
    if (!a->q || !a->prefix_len || !a->k_tree || !a->v_tree || !a->parent || !a->out)
      return TV_ERR_INVALID_ARG;
    if (a->Lmax > 0 && (!a->k_cache || !a->v_cache)) return TV_ERR_INVALID_ARG;
  }
  return TV_OK;
}

// Time of one 128-key tile in a two-tile CTA (both row tiles), in units of
// the same tile in a one-tile CTA, and the two-tile CTA's fixed cost (start,
// first loads, a two-round merge) in the same unit; measured on B200 with the
// long-context and Llama-3-8B-shaped workloads.
constexpr double kPairTile = 1.5;
constexpr double kPairFixed = 6.0;
// The two-tile CTA whose chunks merge through the workspace: no cluster (so
// any number of chunks up to 16 and no co-scheduling of a pair's chunks),
// for a fixed cost 1.5 tiles higher (its rows written out and, by the last
// chunk, read back).
constexpr double kPairGlobalFixed = 7.5;
constexpr int kPairGlobalMaxChunks = 16;

AttnPlan plan_attn(const tv_attn_args* a) {
  AttnPlan pl;
  std::memset(&pl, 0, sizeof(pl));
  const int G = a->Hq / a->Hkv;
  pl.sparse = a->sparse_topk > 0;
  pl.tc = !pl.sparse && attn_tc_supported(a);
  pl.tc_sparse = pl.sparse && attn_tc_sparse_supported(a);
  pl.node_tile = G >= 64 ? 1 : 64 / G;
  if (pl.tc || pl.tc_sparse) pl.node_tile = 128 / G > 0 ? 128 / G : 1;
  const int64_t ntiles = (a->T + pl.node_tile - 1) / pl.node_tile;
  const int64_t units = static_cast<int64_t>(a->B) * a->Hkv * (ntiles > 0 ? ntiles : 1);
  if (a->Lmax == 0 || pl.sparse) {
    pl.nchunk = pl.sparse ? 1 : 0;
    pl.chunk_len = 128;
  } else {
    // about four waves of CTAs (balance across ragged prefixes); the
    // tensor-core kernel takes at least four 128-key tiles per chunk (its
    // pipeline is amortised over the chunk) and at most one cluster of
    // chunks per row tile (it merges them over distributed shared memory);
    // the CUDA-core path takes at most 31 chunks so that its merge reads
    // every partial of a row with one warp
    const int64_t target = 4LL * num_sms();
    int64_t want = (target + units - 1) / units;
    int64_t maxc = (a->Lmax + 127) / 128;
    if (maxc > 31) maxc = 31;
    if (want < 1) want = 1;
    if (want > maxc) want = maxc;
    int64_t len = (a->Lmax + want - 1) / want;
    len = (len + 127) / 128 * 128;
    if (pl.tc) {
      // tensor-core kernels: c chunks of a row tile (or of a pair of row
      // tiles) form one cluster.  Cost model in the time of one 128-key
      // tile of a one-tile CTA: each CTA pays about three tiles of latency
      // (start-up, first loads, merge) plus its chunk's tiles, a two-tile
      // CTA kPairTile per key tile for both of its row tiles, and the
      // clusters run in waves of what the device holds at once.
      const int64_t tiles = (a->Lmax + 127) / 128;
      const int64_t units_pair = static_cast<int64_t>(a->B) * a->Hkv * ((ntiles + 1) / 2);
      const bool pair_ok = a->T <= 2048;
      double best = 1e300;
      int64_t best_len = tiles;
      // forms: 0 one tile per CTA, 1 a tile pair (chunks in a cluster), 2 a
      // tile pair with its chunks merged through the workspace (2..16
      // chunks, as many CTAs as the device holds at once)
      const bool global_ok = pair_ok && units_pair <= kMaxTickets;
      for (int form = 0; form < (pair_ok ? (global_ok ? 3 : 2) : 1); ++form) {
        for (int c = (form == 2 ? 2 : 1); c <= (form == 2 ? kPairGlobalMaxChunks : 8); ++c) {
          const int64_t lt = (tiles + c - 1) / c;
          if (c > 1 && lt < 4) break;                       // at least four tiles per chunk
          if ((tiles + lt - 1) / lt != c) continue;          // c chunks not realisable
          const int act = form == 2 ? attn_pair_active_clusters(1)
                                    : (form ? attn_pair_active_clusters(c) : attn_tc_active_clusters(c));
          if (act <= 0) continue;
          const int64_t u = form == 2 ? units_pair * c : (form ? units_pair : units);
          const double waves = static_cast<double>((u + act - 1) / act);
          const double fixed = form == 2 ? kPairGlobalFixed : (form ? kPairFixed : 3.0);
          const double cost = waves * (fixed + static_cast<double>(lt) * (form ? kPairTile : 1.0));
          if (cost < best) { best = cost; best_len = lt; pl.pair = form >= 1; pl.gmerge = form == 2; }
        }
      }
      len = best_len * 128;
    }
    pl.chunk_len = static_cast<int>(len);
    pl.nchunk = static_cast<int>((a->Lmax + len - 1) / len);
  }
  if (pl.tc && pl.nchunk == 0) { pl.nchunk = 1; pl.chunk_len = 128; }
  const size_t rows = static_cast<size_t>(a->B) * a->T * a->Hq;
  // the tensor-core path merges its chunks on chip; the other paths merge
  // partials (prefix chunks + the tree-path partial) through the workspace
  const size_t nparts = (pl.tc || pl.tc_sparse) ? 0 : static_cast<size_t>(pl.nchunk) + 1;
  size_t off = kTicketBytes;
  if (pl.gmerge) {
    // the two-tile kernel's workspace merge: per (pair, chunk) both tiles'
    // 128 rows of d fp32 values and their log-sum-exps
    const int64_t ntiles2 = (a->T + pl.node_tile - 1) / pl.node_tile;
    const size_t slots = static_cast<size_t>(a->B) * a->Hkv * ((ntiles2 + 1) / 2) * pl.nchunk * 2 * 128;
    pl.off_o = off;  off = align256(off + slots * a->d * sizeof(float));
    pl.off_lse = off; off = align256(off + slots * sizeof(float));
  } else {
    pl.off_o = off;  off = align256(off + nparts * rows * a->d * sizeof(float));
    pl.off_lse = off; off = align256(off + nparts * rows * sizeof(float));
  }
  pl.off_ok = off;  off = align256(off + static_cast<size_t>(a->B) * a->T * sizeof(int32_t));
  if (pl.sparse) {
    pl.nblk_max = (a->Lmax + a->block_size - 1) / a->block_size;
    pl.off_kbar = off;
    if (!a->k_block_mean)
      off = align256(off + static_cast<size_t>(a->B) * pl.nblk_max * a->Hkv * a->d * sizeof(float));
    pl.off_sel = off;
    off = align256(off + static_cast<size_t>(a->B) * a->T * a->Hkv * a->sparse_topk * sizeof(int32_t));
    pl.off_scores = off;
    off = align256(off + static_cast<size_t>(a->B) * a->T * a->Hkv * pl.nblk_max * sizeof(float));
  }
  pl.total = off;
  return pl;
}

}  // namespace

// ------------------------------------------------------------ attention

extern "C" size_t tree_verify_attn_workspace_size(const tv_attn_args* a) {
  if (check_attn(a) != TV_OK) return 0;
  return plan_attn(a).total;
}

extern "C" int32_t tv_attn_path(const tv_attn_args* a) {
  if (check_attn(a) != TV_OK) return -1;
  const AttnPlan pl = plan_attn(a);
  return pl.sparse ? (pl.tc_sparse ? 3 : 2) : (pl.tc ? (pl.pair ? (pl.gmerge ? 5 : 4) : 1) : 0);
}

extern "C" int32_t tv_attn_launches(const tv_attn_args* a) {
  if (check_attn(a) != TV_OK) return -1;
  if (a->B == 0 || a->T == 0) return 0;
  const AttnPlan pl = plan_attn(a);
  if (pl.sparse) return (a->k_block_mean ? 0 : 1) + 2 + (pl.tc_sparse ? 1 : 3);
  if (pl.tc) return 1;
  return 3;
}

extern "C" tv_status tree_verify_attn(const tv_attn_args* a, void* ws, size_t ws_bytes,
                                      tv_stream_t stream) {
  const tv_status st = check_attn(a);
  if (st != TV_OK) return st;
  if (a->B == 0 || a->T == 0) return TV_OK;
  const AttnPlan pl = plan_attn(a);
  if (!ws_ok(ws, ws_bytes, pl.total)) return TV_ERR_WORKSPACE;
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.dtype = a->dtype;
  p.B = a->B; p.T = a->T; p.Hq = a->Hq; p.Hkv = a->Hkv; p.d = a->d; p.Lmax = a->Lmax;
  p.G = a->Hq / a->Hkv;
  p.q = a->q; p.q_sb = a->q_sb; p.q_st = a->q_st; p.q_sh = a->q_sh;
  p.kc = a->k_cache; p.vc = a->v_cache; p.kv_sb = a->kv_sb; p.kv_sl = a->kv_sl; p.kv_sh = a->kv_sh;
  p.prefix_len = a->prefix_len;
  p.kt = a->k_tree; p.vt = a->v_tree; p.kt_sb = a->kt_sb; p.kt_st = a->kt_st; p.kt_sh = a->kt_sh;
  p.parent = a->parent; p.par_sb = a->parent_sb;
  p.n_nodes = a->n_nodes;
  p.scale = a->scale > 0.f ? a->scale : 1.0f / std::sqrt(static_cast<float>(a->d));
  p.out = a->out; p.o_sb = a->o_sb; p.o_st = a->o_st; p.o_sh = a->o_sh;
  p.lse = a->lse;
  p.status = a->dev_status;
  p.prefix_only = a->prefix_only;
  p.gmerge = pl.gmerge ? 1 : 0;
  p.nchunk = pl.nchunk; p.chunk_len = pl.chunk_len; p.node_tile = pl.node_tile;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.part_o = reinterpret_cast<float*>(w + pl.off_o);
  p.part_lse = reinterpret_cast<float*>(w + pl.off_lse);
  p.node_ok = reinterpret_cast<int32_t*>(w + pl.off_ok);
  p.tickets = reinterpret_cast<int32_t*>(w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (pl.sparse) {
    p.topk = a->sparse_topk; p.block_size = a->block_size; p.nblk_max = pl.nblk_max;
    p.kbar = a->k_block_mean ? a->k_block_mean : reinterpret_cast<float*>(w + pl.off_kbar);
    p.sel = reinterpret_cast<int32_t*>(w + pl.off_sel);
    p.scores = reinterpret_cast<float*>(w + pl.off_scores);
    p.sel_out = a->sel_blocks;
    if (!a->k_block_mean) {
      e = launch_block_means(p, reinterpret_cast<float*>(w + pl.off_kbar), s);
      if (e != cudaSuccess) return from_cuda(e);
    }
    e = launch_block_select(p, s);
    if (e != cudaSuccess) return from_cuda(e);
    if (pl.tc_sparse) {
      // the kept blocks' union as key tiles of the tensor-core kernel
      p.tc_sparse = 1;
      return from_cuda(launch_attn_tc(p, s));
    }
    e = launch_attn_sparse(p, s);
  } else if (pl.tc) {
    // one kernel: prefix tiles, tree tiles and the cluster merge of the chunks
    return from_cuda(pl.pair ? launch_attn_pair(p, s) : launch_attn_tc(p, s));
  } else {
    e = launch_attn_simt(p, s);
  }
  if (e != cudaSuccess) return from_cuda(e);
  e = launch_attn_tree(p, s);
  if (e != cudaSuccess) return from_cuda(e);
  e = launch_attn_merge(p, s);
  return from_cuda(e);
}

extern "C" tv_status tree_verify_attn_merge(const tv_attn_merge_args* a, tv_stream_t stream) {
  if (!a) return TV_ERR_INVALID_ARG;
  if (a->dtype != TV_FP32 && a->dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (a->N < 1 || a->B < 0 || a->T < 0 || a->Hq < 0) return TV_ERR_INVALID_ARG;
  if (a->N > 64) return TV_ERR_UNSUPPORTED;
  if (a->d != 32 && a->d != 64 && a->d != 128) return TV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(a->B) * a->T * a->Hq == 0) return TV_OK;
  if (!a->o_parts || !a->lse_parts || !a->out) return TV_ERR_INVALID_ARG;
  return from_cuda(launch_attn_partial_merge(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ acceptance

namespace tv {
int resolve_mode(const tv_accept_args* a) {
  if (a->temperature == 0.f) return TV_ACCEPT_GREEDY;
  if (a->mode == TV_ACCEPT_AUTO) return TV_ACCEPT_SPECSAMPLE;
  return a->mode;
}

tv_status check_accept(const tv_accept_args* a) {
  if (!a) return TV_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->V < 1) return TV_ERR_INVALID_ARG;
  if (a->B > kAcceptMaxB) return TV_ERR_UNSUPPORTED;
  if (a->mode < TV_ACCEPT_AUTO || a->mode > TV_ACCEPT_SPECEXEC) return TV_ERR_INVALID_ARG;
  if (!(a->temperature >= 0.f) || !std::isfinite(a->temperature)) return TV_ERR_INVALID_ARG;
  if (a->B > 0) {
    if (!a->n_accepted || !a->accepted_nodes && a->T > 0 || !a->out_tokens) return TV_ERR_INVALID_ARG;
    if (a->T > 0) {
      if (!a->target_logits || !a->draft_tokens || !a->parent) return TV_ERR_INVALID_ARG;
      if (a->T > 1 && a->tl_st < a->V) return TV_ERR_INVALID_ARG;
      if (resolve_mode(a) == TV_ACCEPT_SPECSAMPLE) {
        if (!a->draft_probs) return TV_ERR_INVALID_ARG;
        if (a->T > 1 && a->dp_st < a->V) return TV_ERR_INVALID_ARG;
      }
    }
  }
  return TV_OK;
}
}  // namespace tv

extern "C" size_t tree_accept_workspace_size(const tv_accept_args* a) {
  if (tv::check_accept(a) != TV_OK) return 0;
  return align256(accept_workspace_bytes(a->B, a->T));
}

extern "C" tv_status tree_accept(const tv_accept_args* a, void* ws, size_t ws_bytes,
                                 tv_stream_t stream) {
  const tv_status st = tv::check_accept(a);
  if (st != TV_OK) return st;
  if (a->B == 0) return TV_OK;
  if (!ws_ok(ws, ws_bytes, accept_workspace_bytes(a->B, a->T))) return TV_ERR_WORKSPACE;
  return from_cuda(launch_accept(a, tv::resolve_mode(a), ws, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ expansion

namespace {
tv_status check_expand(const tv_expand_args* a, bool need_rows) {
  if (!a) return TV_ERR_INVALID_ARG;
  if (a->V < 1 || a->budget < 1 || a->Bsel < 1 || a->R < 0) return TV_ERR_INVALID_ARG;
  if (a->V > 262144 || a->budget > 8192) return TV_ERR_UNSUPPORTED;
  if (!(a->draft_temperature > 0.f) || !std::isfinite(a->draft_temperature)) return TV_ERR_INVALID_ARG;
  if (a->mode != TV_EXPAND_BESTFIRST && a->mode != TV_EXPAND_BEAM) return TV_ERR_INVALID_ARG;
  if (!a->n_nodes || !a->parent || !a->token || !a->logp || !a->pool) return TV_ERR_INVALID_ARG;
  if (a->pool_bytes < tv::expand_pool_bytes(a->budget, a->V)) return TV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(a->pool) & 255u) != 0) return TV_ERR_WORKSPACE;
  if (need_rows) {
    if (!a->frontier || !a->n_appended) return TV_ERR_INVALID_ARG;
    if (a->R > 0 && (!a->draft_logits || !a->row_node || a->ld_logits < a->V)) return TV_ERR_INVALID_ARG;
  }
  return TV_OK;
}
}  // namespace

extern "C" size_t tree_expand_pool_bytes(int32_t budget, int32_t V) {
  if (budget < 1 || V < 1) return 0;
  return tv::expand_pool_bytes(budget, V);
}

extern "C" size_t tree_expand_workspace_size(const tv_expand_args*) { return 0; }

extern "C" tv_status tree_expand_init(const tv_expand_args* a, int32_t root_token, tv_stream_t stream) {
  const tv_status st = check_expand(a, false);
  if (st != TV_OK) return st;
  return from_cuda(launch_expand_init(a, root_token, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" tv_status tree_expand_topb(const tv_expand_args* a, void*, size_t, tv_stream_t stream) {
  const tv_status st = check_expand(a, true);
  if (st != TV_OK) return st;
  return from_cuda(launch_expand(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ KV commit

namespace {
tv_status check_commit(const tv_commit_args* a) {
  if (!a) return TV_ERR_INVALID_ARG;
  if (a->dtype != TV_FP32 && a->dtype != TV_BF16) return TV_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->Hkv <= 0 || a->Lmax < 0 || a->d < 1) return TV_ERR_INVALID_ARG;
  if (a->d > 1024) return TV_ERR_UNSUPPORTED;
  if (a->B > 0) {
    if (a->T < 1) return TV_ERR_INVALID_ARG;
    if (!a->k_cache || !a->v_cache || !a->prefix_len || !a->k_tree || !a->v_tree || !a->n_accepted)
      return TV_ERR_INVALID_ARG;
    if (a->T > 1 && !a->accepted_nodes) return TV_ERR_INVALID_ARG;
    const uintptr_t es = a->dtype == TV_BF16 ? 2u : 4u;
    const uintptr_t ptrs[4] = {reinterpret_cast<uintptr_t>(a->k_cache), reinterpret_cast<uintptr_t>(a->v_cache),
                               reinterpret_cast<uintptr_t>(a->k_tree), reinterpret_cast<uintptr_t>(a->v_tree)};
    for (uintptr_t x : ptrs)
      if (x % es != 0) return TV_ERR_INVALID_ARG;
  }
  return TV_OK;
}
}  // namespace

extern "C" tv_status tree_commit_kv(const tv_commit_args* a, tv_stream_t stream) {
  const tv_status st = check_commit(a);
  if (st != TV_OK) return st;
  if (a->B == 0) return TV_OK;
  return from_cuda(launch_commit(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ utilities

namespace tv {
__global__ void philox_uniforms_kernel(uint64_t seed, uint64_t step, const int32_t* b,
                                       const int32_t* node, const int32_t* draw,
                                       const int32_t* tag, double* out, int n) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < n) out[k] = accept_uniform(seed, step, b[k], node[k], draw[k], tag[k]);
}

int num_sms() {
  static int cached = 0;
  if (cached == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      cached = v;
    else
      cached = 148;
  }
  return cached;
}
}  // namespace tv

extern "C" tv_status tv_philox_uniforms(uint64_t seed, uint64_t step, const int32_t* b,
                                        const int32_t* node, const int32_t* draw,
                                        const int32_t* tag, double* out, int32_t n,
                                        tv_stream_t stream) {
  if (n < 0) return TV_ERR_INVALID_ARG;
  if (n == 0) return TV_OK;
  if (!b || !node || !draw || !tag || !out) return TV_ERR_INVALID_ARG;
  philox_uniforms_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      seed, step, b, node, draw, tag, out, n);
  return from_cuda(cudaGetLastError());
}

extern "C" tv_status tv_expand_set_wait_limit(uint32_t polls) {
  return from_cuda(tv::expand_set_wait_limit(polls));
}

extern "C" tv_status tv_expand_exp(const double* t, double* out, int32_t n, tv_stream_t stream) {
  if (n < 0) return TV_ERR_INVALID_ARG;
  if (n == 0) return TV_OK;
  if (!t || !out) return TV_ERR_INVALID_ARG;
  return from_cuda(tv::launch_expand_exp(t, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" const char* tree_verify_version(void) { return "treeverify 0.1.0 sm_100a"; }

extern "C" const char* tv_status_string(tv_status s) {
  switch (s) {
    case TV_OK: return "ok";
    case TV_ERR_INVALID_ARG: return "invalid argument";
    case TV_ERR_UNSUPPORTED: return "unsupported configuration";
    case TV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TV_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}
