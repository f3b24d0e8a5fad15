"""KV commit of the accepted path, fp64 oracle -- TEST INFRASTRUCTURE ONLY.

What is computed (plain definition):

The SpecExec page runs verification in iterations ("Approach"; "Key
results" and "Experimental setup" count the accepted tokens per target
iteration): the tokens accepted by one iteration become prefix for the next
one, whose draft tree attends to them.  The pages do not spell out the cache
update.  The plain reading used here: for sequence b with L = prefix_len[b],
n = n_accepted[b] and the path rows = (0, a_0, ..., a_{n-1}) -- the root
(the last committed token, tree node 0), then the accepted nodes in path
order as the acceptance walk returns them --

    cache[b][L + r][g] = tree[b][rows[r]][g]     r = 0 .. n, every kv head g,
                                                 for K and for V
    prefix_len[b] <- L + n + 1

with every row read before any row is written, so a tree whose K/V sit in
the cache itself at rows >= L of the same sequence is compacted in place.
The bonus token emitted by the walk has no K/V yet; it is the next tree's
root.

Malformed input (bits of the status word; the sequence is left untouched):
  BAD_ROW (8):  a path node outside [1, T), or a path that is not strictly
                increasing (a path from the root only visits larger indices);
  BAD_LEN (16): n outside [0, T - 1], L outside [0, Lmax], or
                L + n + 1 > Lmax.
"""

from __future__ import annotations

import numpy as np

from .attention import _f64, _i64

ST_BAD_ROW = 8
ST_BAD_LEN = 16


def tree_commit_kv(k_cache, v_cache, prefix_len, k_tree, v_tree, n_accepted, accepted_nodes,
                   tree_in_cache_at=None):
    """Oracle for tree_commit_kv.

    Shapes: k_cache/v_cache [B][Lmax][Hkv][d], prefix_len [B], k_tree/v_tree
    [B][T][Hkv][d] (or None with tree_in_cache_at), n_accepted [B],
    accepted_nodes [B][>= n] (the acceptance walk's path, root excluded).
    tree_in_cache_at: None, or per-sequence row offsets off[b]: the tree K/V
    of sequence b are then the cache rows off[b] .. off[b] + T - 1 (T taken
    from accepted_nodes' width).

    Returns a dict: k_cache, v_cache (float64 copies after the commit),
    prefix_len (int64), status (int bit set).
    """
    K = _f64(k_cache)
    Vc = _f64(v_cache)
    Kout = K.copy()
    Vout = Vc.copy()
    L = _i64(prefix_len).copy()
    n_acc = _i64(n_accepted)
    acc = _i64(accepted_nodes)
    B, Lmax = K.shape[0], K.shape[1]
    if tree_in_cache_at is None:
        KT = _f64(k_tree)
        VT = _f64(v_tree)
        T = KT.shape[1]
    else:
        off = _i64(tree_in_cache_at)
        T = acc.shape[1]
    status = 0
    for b in range(B):
        n = int(n_acc[b])
        Lb = int(L[b])
        if n < 0 or n > T - 1 or Lb < 0 or Lb > Lmax or Lb + n + 1 > Lmax:
            status |= ST_BAD_LEN
            continue
        rows = [0] + [int(acc[b, r]) for r in range(n)]
        bad = any(x < 1 or x >= T for x in rows[1:]) or any(rows[r] <= rows[r - 1] for r in range(1, n + 1))
        if bad:
            status |= ST_BAD_ROW
            continue
        # every source row is read (copied) before any destination is written
        if tree_in_cache_at is None:
            src_k = np.stack([KT[b, x] for x in rows])
            src_v = np.stack([VT[b, x] for x in rows])
        else:
            o = int(off[b])
            src_k = np.stack([K[b, o + x] for x in rows])
            src_v = np.stack([Vc[b, o + x] for x in rows])
        Kout[b, Lb:Lb + n + 1] = src_k
        Vout[b, Lb:Lb + n + 1] = src_v
        L[b] = Lb + n + 1
    return dict(k_cache=Kout, v_cache=Vout, prefix_len=L, status=status)
