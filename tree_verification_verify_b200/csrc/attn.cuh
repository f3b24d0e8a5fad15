// Shared declarations of the tree_verify_attn kernels.
#pragma once

#include "tv_common.cuh"

namespace tv {

// Parameters of one tree_verify_attn call plus the split-KV plan.
struct AttnParams {
  int dtype;
  int B, T, Hq, Hkv, d, Lmax, G;
  const void* q;  int64_t q_sb, q_st, q_sh;
  const void* kc; const void* vc; int64_t kv_sb, kv_sl, kv_sh;
  const int32_t* prefix_len;
  const void* kt; const void* vt; int64_t kt_sb, kt_st, kt_sh;
  const int32_t* parent; int64_t par_sb;
  const int32_t* n_nodes;
  float scale;                 // resolved (> 0)
  void* out; int64_t o_sb, o_st, o_sh;
  float* lse;
  uint32_t* status;
  int prefix_only;             // partial over the prefix keys alone (no tree keys)
  int gmerge;                  // two-tile kernel: chunks merged through the workspace
                               // (part_o [unit][chunk][2][128][d], part_lse [unit][chunk][2][128])
  // block top-k
  int topk, block_size, nblk_max;
  const float* kbar;           // [B][nblk_max][Hkv][d] (caller's or workspace)
  int32_t* sel;                // [B][T][Hkv][topk] kept blocks (workspace)
  float* scores;               // [B][T][Hkv][nblk_max] cheap block scores (workspace)
  int tc_sparse;               // the tensor-core kernel runs the block top-k variant
  int32_t* sel_out;            // caller's copy or NULL
  // split-KV plan and workspace
  int nchunk;                  // prefix chunks (the tree part is chunk nchunk)
  int chunk_len;               // prefix positions per chunk (multiple of 128)
  int node_tile;               // nodes per CTA of the CUDA-core kernel
  float* part_o;               // [nchunk+1][B][T][Hq][d]
  float* part_lse;             // [nchunk+1][B][T][Hq]
  int32_t* node_ok;            // [B][T]
  int32_t* tickets;            // per-group counters, zero between calls
};

// The first kTicketBytes of every workspace hold ticket counters that each
// call returns to zero (so calls of any shape may share one workspace).
constexpr size_t kTicketBytes = 64 * 1024;
constexpr int kMaxTickets = static_cast<int>(kTicketBytes / sizeof(int32_t));

__host__ __device__ inline int64_t part_row(const AttnParams& p, int chunk, int b, int i, int h) {
  return ((static_cast<int64_t>(chunk) * p.B + b) * p.T + i) * p.Hq + h;
}

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_tree(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_merge(const AttnParams& p, cudaStream_t stream);

}  // namespace tv
