"""Tree-masked attention, fp64 oracle.

What is computed (plain definition; the method reaches exactly this up to
rounding order):

The SpecExec page ("Approach") verifies the whole draft tree in one target
pass; the EasySpec page ("Experimental setup", baseline "+tree") names tree
attention.  Neither spells out the mask; the plain reading used here is the
standard one: draft node i of sequence b attends to

    K(i) = { prefix positions 0 .. L_b - 1 }  u  { tree nodes on the path
           root .. i, node i included }

with contiguous GQA groups (query head h reads kv head h // (Hq / Hkv)),

    s_j = scale * <q_{i,h}, k_{j,g}>,   o_{i,h} = sum_j softmax(s)_j v_{j,g},
    lse_{i,h} = log sum_j exp(s_j)   (natural log),

computed two-pass (row max, then sum) in float64.  Queries and keys arrive
post-RoPE; scale = 0 means 1/sqrt(d).

Block top-k variant (sparse verification page, "Methodology" 3, attention
sparsity: keep only the top-k keys/values per query, in structured blocks,
chosen by a cheap relevance score).  Reading: the cheap score of prefix block
j (block_size consecutive positions) for node i and kv head g is

    sigma(i, g, j) = sum_{h in group g} <q_{i,h}, kbar_{j,g}>,

kbar_{j,g} the mean of the block's valid keys (a partial last block averages
its valid keys only).  The top-k blocks by (score desc, block index asc) are
kept for all heads of the group; with at most k blocks all are kept.  The
node then attends to the kept blocks' keys plus its tree path, exactly as
above.

Prefix-only partial (for splitting a long prefix across GPUs, the long
contexts the sparse verification page is about): with prefix_only the node
attends to the prefix keys alone, K(i) = {0 .. L_b - 1}
(parent[] is not read); a row with no keys has out = 0 and lse = -inf.
Partials over disjoint key sets of the same rows combine by their
log-sum-exp (merge_partials): with M = max_r lse_r and w_r = exp(lse_r - M),
out = sum_r w_r out_r / sum_r w_r and lse = M + log sum_r w_r, which is the
softmax over the union of the key sets.

Malformed input (reported as bits of a status word, outputs defined):
  BAD_PARENT (1): parent[0] != -1, or a node whose parent chain does not
      reach the root through parent[j] in [0, j): its outputs are NaN.
  BAD_LEN   (16): n_nodes[b] outside [0, T] (nothing written for b) or
      prefix_len[b] outside [0, Lmax] (the rows of b are NaN).
Rows i >= n_nodes[b] are not written.
"""

from __future__ import annotations

import numpy as np

ST_BAD_PARENT = 1
ST_BAD_TOKEN = 2
ST_NONFINITE = 4
ST_BAD_ROW = 8
ST_BAD_LEN = 16


def _f64(x):
    """Widen a torch tensor (fp32 / bf16) or array to a float64 ndarray."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


def ancestor_path(parent_row, i):
    """Nodes on the path root .. i (i included), or None when the chain of
    parent pointers from i does not reach node 0 through parent[j] in [0, j)
    or parent[0] != -1."""
    if parent_row[0] != -1:
        return None
    path = [i]
    j = i
    while j != 0:
        p = parent_row[j]
        if p < 0 or p >= j:
            return None
        path.append(p)
        j = p
    return path[::-1]


def block_means(k_cache, prefix_len, block_size):
    """kbar[b][j][g][:] = mean of the valid keys of prefix block j."""
    K = _f64(k_cache)
    L = _i64(prefix_len)
    B, Lmax, Hkv, d = K.shape
    nbmax = (Lmax + block_size - 1) // block_size
    kbar = np.zeros((B, nbmax, Hkv, d))
    for b in range(B):
        Lb = int(L[b])
        for j in range((Lb + block_size - 1) // block_size):
            lo, hi = j * block_size, min((j + 1) * block_size, Lb)
            kbar[b, j] = K[b, lo:hi].mean(axis=0)
    return kbar


def select_blocks(qi_group, kbar_bg, nblk, topk):
    """Block top-k for one (node, kv head): qi_group [G][d], kbar_bg
    [nblk][d].  Returns (kept block ids ascending, score gap between rank k
    and rank k+1 relative to max |score| (inf when all blocks are kept),
    scores)."""
    # [nblk][G] dot products, summed over the group's heads
    scores = np.sum(kbar_bg[:nblk] @ qi_group.T, axis=1)
    order = sorted(range(nblk), key=lambda j: (-scores[j], j))
    if nblk <= topk:
        return sorted(order), float("inf"), scores
    kept = sorted(order[:topk])
    gap = scores[order[topk - 1]] - scores[order[topk]]
    scale = max(1e-300, float(np.max(np.abs(scores))))
    return kept, gap / scale, scores


def tree_verify_attn(q, k_cache, v_cache, prefix_len, k_tree, v_tree, parent,
                     n_nodes=None, scale=0.0, sparse_topk=0, block_size=64,
                     k_block_mean=None, rows=None, forced_sel=None, prefix_only=False):
    """Oracle for tree_verify_attn.

    Shapes: q [B][T][Hq][d], k_cache/v_cache [B][Lmax][Hkv][d],
    prefix_len [B], k_tree/v_tree [B][T][Hkv][d], parent [B][T],
    n_nodes [B] or None, k_block_mean [B][nblk][Hkv][d] or None.

    Returns a dict: out [B][T][Hq][d] and lse [B][T][Hq] (float64, NaN
    where not written or invalid), written [B][T] bool, valid [B][T] bool,
    sel [B][T][Hkv][topk] kept block ids (-1 padded; sparse only),
    sel_gap [B][T][Hkv] relative rank-k/k+1 score gap (sparse only),
    status (int bit set).  `rows`, a set of (b, i) pairs, restricts the
    computation to those nodes (sampled checks of large cases); the status
    word is still computed over every node.  `forced_sel` [B][T][Hkv][k]
    (block ids, -1 ignored), sparse only: the node attends to these blocks
    instead of its own top-k (sel and sel_gap still report the top-k); this
    checks an output whose selection was taken elsewhere at a near-tie of
    the k-th and (k+1)-th block scores.
    """
    Q = _f64(q)
    K = _f64(k_cache)
    Vc = _f64(v_cache)
    KT = _f64(k_tree)
    VT = _f64(v_tree)
    L = _i64(prefix_len)
    P = _i64(parent)
    B, T, Hq, d = Q.shape
    Lmax, Hkv = K.shape[1], K.shape[2]
    G = Hq // Hkv
    sc = float(scale) if scale and scale > 0 else 1.0 / np.sqrt(d)
    nn = _i64(n_nodes) if n_nodes is not None else np.full(B, T, dtype=np.int64)

    out = np.full((B, T, Hq, d), np.nan)
    lse = np.full((B, T, Hq), np.nan)
    written = np.zeros((B, T), dtype=bool)
    valid = np.zeros((B, T), dtype=bool)
    topk = int(sparse_topk)
    sel = np.full((B, T, Hkv, max(topk, 1)), -1, dtype=np.int64)
    sel_gap = np.full((B, T, Hkv), np.inf)
    status = 0

    kbar = None
    if topk > 0:
        kbar = _f64(k_block_mean) if k_block_mean is not None else block_means(k_cache, prefix_len, block_size)

    for b in range(B):
        n = int(nn[b])
        if n < 0 or n > T:
            status |= ST_BAD_LEN
            continue
        Lb = int(L[b])
        bad_len = Lb < 0 or Lb > Lmax
        if bad_len:
            status |= ST_BAD_LEN
        if not prefix_only:
            if n > 0 and P[b, 0] != -1:
                status |= ST_BAD_PARENT
            for i in range(1, n):
                if P[b, i] < 0 or P[b, i] >= i:
                    status |= ST_BAD_PARENT
        nblk = (Lb + block_size - 1) // block_size if not bad_len else 0
        for i in range(n):
            if rows is not None and (b, i) not in rows:
                continue
            written[b, i] = True
            path = [] if prefix_only else ancestor_path(P[b], i)
            if path is None or bad_len:
                if path is None:
                    status |= ST_BAD_PARENT
                continue
            valid[b, i] = True
            for g in range(Hkv):
                if topk > 0:
                    kept, gap, _ = select_blocks(Q[b, i, g * G:(g + 1) * G], kbar[b, :nblk, g], nblk, topk)
                    sel[b, i, g, :len(kept)] = kept
                    sel_gap[b, i, g] = gap
                    if forced_sel is not None:
                        kept = sorted(int(j) for j in np.asarray(forced_sel[b][i][g]) if 0 <= j < nblk)
                    pos = [p for j in kept for p in range(j * block_size, min((j + 1) * block_size, Lb))]
                    kp = K[b, pos, g]
                    vp = Vc[b, pos, g]
                else:
                    kp = K[b, :Lb, g]
                    vp = Vc[b, :Lb, g]
                keys = np.concatenate([kp, KT[b, path, g]], axis=0)
                vals = np.concatenate([vp, VT[b, path, g]], axis=0)
                if len(keys) == 0:
                    out[b, i, g * G:(g + 1) * G] = 0.0
                    lse[b, i, g * G:(g + 1) * G] = -np.inf
                    continue
                # the G query heads of group g, one row each: [G][|K(i)|]
                s = (Q[b, i, g * G:(g + 1) * G] @ keys.T) * sc
                m = np.max(s, axis=1, keepdims=True)
                e = np.exp(s - m)
                l = np.sum(e, axis=1, keepdims=True)
                out[b, i, g * G:(g + 1) * G] = (e @ vals) / l
                lse[b, i, g * G:(g + 1) * G] = (m + np.log(l))[:, 0]
    return dict(out=out, lse=lse, written=written, valid=valid,
                sel=(sel if topk > 0 else None), sel_gap=(sel_gap if topk > 0 else None),
                status=status)


def merge_partials(outs, lses):
    """Log-sum-exp merge of attention partials over disjoint key sets of the
    same rows: outs [N][...][d], lses [N][...] (natural log).  Rows whose
    partials all have lse = -inf get out = 0 and lse = -inf; a NaN lse
    makes the row NaN."""
    O = np.asarray(outs, dtype=np.float64)
    Lz = np.asarray(lses, dtype=np.float64)
    bad = np.any(np.isnan(Lz), axis=0)
    M = np.max(np.where(np.isnan(Lz), -np.inf, Lz), axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(Lz), np.exp(np.where(np.isfinite(Lz), Lz, 0.0) - Ms[None]), 0.0)
    den = np.sum(w, axis=0)
    num = np.sum(w[..., None] * np.nan_to_num(O), axis=0)
    out = np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
    lse = np.where(den > 0, Ms + np.log(np.where(den > 0, den, 1.0)), -np.inf)
    out[bad] = np.nan
    lse[bad] = np.nan
    return out, lse
