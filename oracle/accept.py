"""The acceptance walk over a verified draft tree, fp64 oracle.

Node 0 is the root (the last committed token): its target row predicts the
first new token and it is never itself "accepted".  Children of a node are
taken in ascending node index; a child j counts only if parent[j] is in
[0, j).  Row c of the target logits is the target's prediction after node c;
row c of the draft distribution q is the distribution the node's children
were drawn from.

GREEDY (temperature 0; plain definition: the longest draft path that matches
the target's argmax).  At node c let a = argmax_t z_c[t] (lowest index on
ties).  If a child of c carries token a, accept the lowest-index such child
and continue from it; otherwise stop and emit a as the bonus token.

SPECSAMPLE (temperature > 0; multi-draft speculative sampling with residual
resampling, the rule the SpecExec page lists under "Builds on: speculative
sampling, SpecInfer").  At node c, p = softmax(z_c / tau).  For the children
c_1 < c_2 < ... with tokens x_j: draw u_j; accept c_j when
u_j < p(x_j) / q_c(x_j) (q_c(x_j) = 0: accept iff p(x_j) > 0) and continue
from c_j with that node's own p.  Otherwise replace p by the residual
(p - q_c)^+ / sum (p - q_c)^+ (kept unchanged when that sum is 0) and try
the next child.  When every child is rejected, or c is a leaf, draw u and
emit the inverse-CDF sample of p: the smallest t with
sum_{s<=t} p_s > u * sum_s p_s (token order 0 .. V-1).

SPECEXEC (deterministic trees, SpecExec page, "Approach": the sampling
procedure stays equivalent to sequential sampling from the target, so it
works with deterministic trees).  At node c draw x from softmax(z_c / tau) by
the same inverse CDF; if a child of c carries token x, descend to the
lowest-index such child, otherwise emit x and stop.  At a leaf emit x.

At temperature 0 every mode is GREEDY.  Uniforms come from philox.uniform
with tags 1 (child test j), 2 (residual sample) and 3 (deterministic-tree
sample).

Malformed input (status bits; outputs stay defined):
  BAD_PARENT (1): parent[0] != -1 or parent[j] outside [0, j) for some
      1 <= j < n (such nodes are nobody's child).
  BAD_TOKEN  (2): a draft token outside [0, V) on a node 1 <= j < n; that
      child is skipped (its draw index is still consumed).
  NONFINITE  (4): a visited target row with NaN (greedy) or any non-finite
      value (sampling), or a visited draft row with a negative or non-finite
      value: the walk stops there with bonus token -1.
  BAD_LEN   (16): n_nodes[b] outside [0, T]; nothing is accepted.

Near-threshold decisions: every accept test records |u - ratio| and every
inverse-CDF sample records min(cum_t - u*S, u*S - cum_{t-1}) / S at its
chosen index t; `min_margin` is the smallest along the walk (inf when the
walk made no such decision).
"""

from __future__ import annotations

import numpy as np

from .philox import uniform, TAG_CHILD, TAG_RESIDUAL, TAG_SPECEXEC
from .attention import _f64, _i64, ST_BAD_PARENT, ST_BAD_TOKEN, ST_NONFINITE, ST_BAD_LEN

GREEDY = "greedy"
SPECSAMPLE = "specsample"
SPECEXEC = "specexec"
AUTO = "auto"


def softmax_t(z, tau):
    """p = softmax(z / tau) in float64, two-pass."""
    x = np.asarray(z, dtype=np.float64) / float(tau)
    m = np.max(x)
    e = np.exp(x - m)
    return e / np.sum(e)


def inverse_cdf(p, u):
    """Smallest t with cumsum(p)[t] > u * sum(p).  Returns (t, margin)."""
    cum = np.cumsum(p)
    total = cum[-1]
    target = u * total
    t = int(np.searchsorted(cum, target, side="right"))
    if t >= len(p):                        # u*total rounded up to total
        t = int(np.nonzero(p > 0)[0][-1])
    prev = cum[t - 1] if t > 0 else 0.0
    margin = min(cum[t] - target, target - prev) / total
    return t, float(margin)


def _children(par_row, tok_row, n, V):
    kids = {}
    bad_parent = n > 0 and par_row[0] != -1
    bad_token = False
    for j in range(1, n):
        p = int(par_row[j])
        if p < 0 or p >= j:
            bad_parent = True
            continue
        t = int(tok_row[j])
        if t < 0 or t >= V:
            bad_token = True
        kids.setdefault(p, []).append(j)
    return kids, bad_parent, bad_token


def tree_accept(target_logits, draft_probs, draft_tokens, parent, n_nodes=None,
                mode=AUTO, temperature=0.0, seed=0, step=0, uniform_fn=None):
    """Oracle for tree_accept.  Returns a dict with n_accepted [B],
    accepted_nodes [B][T] (-1 padded), out_tokens [B][T+1] (accepted draft
    tokens, then the bonus token, -1 padded), min_margin [B], status, and
    trace (per sequence, the list of decisions taken).

    uniform_fn(b, node, draw, tag), when given, replaces the Philox stream
    (exact-enumeration tests drive the walk with chosen uniforms)."""
    if uniform_fn is None:
        def uniform_fn(b, node, draw, tag):
            return uniform(seed, step, b, node, draw, tag)
    Z = target_logits
    Zshape = tuple(Z.shape)
    B, T, V = Zshape
    Q = draft_probs
    tok = _i64(draft_tokens)
    par = _i64(parent)
    nn = _i64(n_nodes) if n_nodes is not None else np.full(B, T, dtype=np.int64)
    tau = float(np.float32(temperature))     # the call takes an fp32 temperature
    if tau <= 0.0:
        mode = GREEDY
    elif mode == AUTO:
        mode = SPECSAMPLE

    n_acc = np.zeros(B, dtype=np.int64)
    acc_nodes = np.full((B, T), -1, dtype=np.int64)
    out_tok = np.full((B, T + 1), -1, dtype=np.int64)
    min_margin = np.full(B, np.inf)
    status = 0
    traces = []

    def zrow(b, c):
        return _f64(Z[b, c])

    def qrow(b, c):
        return _f64(Q[b, c])

    for b in range(B):
        n = int(nn[b])
        trace = []
        traces.append(trace)
        if n < 0 or n > T:
            status |= ST_BAD_LEN
            continue
        if n == 0:
            continue
        kids, bad_parent, bad_token = _children(par[b], tok[b], n, V)
        if bad_parent:
            status |= ST_BAD_PARENT
        if bad_token:
            status |= ST_BAD_TOKEN
        path = []
        c = 0
        bonus = -1
        while True:
            z = zrow(b, c)
            ch = kids.get(c, [])
            nxt = None
            if mode == GREEDY:
                if np.any(np.isnan(z)):
                    status |= ST_NONFINITE
                    trace.append(("nonfinite", c))
                    break
                a = int(np.argmax(z))           # first maximum
                trace.append(("argmax", c, a))
                for j in ch:
                    if int(tok[b, j]) == a:
                        nxt = j
                        break
                if nxt is None:
                    bonus = a
            elif mode == SPECEXEC:
                if not np.all(np.isfinite(z)):
                    status |= ST_NONFINITE
                    trace.append(("nonfinite", c))
                    break
                p = softmax_t(z, tau)
                u = uniform_fn(b, c, 0, TAG_SPECEXEC)
                x, mg = inverse_cdf(p, u)
                min_margin[b] = min(min_margin[b], mg)
                trace.append(("sample", c, x, u, mg))
                for j in ch:
                    if int(tok[b, j]) == x:
                        nxt = j
                        break
                if nxt is None:
                    bonus = x
            elif mode == SPECSAMPLE:
                if not np.all(np.isfinite(z)):
                    status |= ST_NONFINITE
                    trace.append(("nonfinite", c))
                    break
                p = softmax_t(z, tau)
                if ch:
                    qc = qrow(b, c)
                    if not np.all(np.isfinite(qc)) or np.any(qc < 0):
                        status |= ST_NONFINITE
                        trace.append(("nonfinite_q", c))
                        break
                    for k, j in enumerate(ch):
                        x = int(tok[b, j])
                        if x < 0 or x >= V:
                            trace.append(("skip", c, j))
                            continue
                        px, qx = p[x], qc[x]
                        if qx > 0:
                            ratio = px / qx
                        else:
                            ratio = np.inf if px > 0 else 0.0
                        u = uniform_fn(b, c, k, TAG_CHILD)
                        if np.isfinite(ratio):
                            min_margin[b] = min(min_margin[b], abs(u - ratio))
                        ok = u < ratio
                        trace.append(("test", c, j, k, u, float(ratio), ok))
                        if ok:
                            nxt = j
                            break
                        r = np.maximum(p - qc, 0.0)
                        zs = np.sum(r)
                        if zs > 0:
                            p = r / zs
                if nxt is None:
                    u = uniform_fn(b, c, 0, TAG_RESIDUAL)
                    x, mg = inverse_cdf(p, u)
                    min_margin[b] = min(min_margin[b], mg)
                    trace.append(("residual", c, x, u, mg))
                    bonus = x
            else:
                raise ValueError(mode)
            if nxt is None:
                break
            path.append(nxt)
            c = nxt
        n_acc[b] = len(path)
        acc_nodes[b, :len(path)] = path
        out_tok[b, :len(path)] = [int(tok[b, j]) for j in path]
        out_tok[b, len(path)] = bonus
    return dict(n_accepted=n_acc, accepted_nodes=acc_nodes, out_tokens=out_tok,
                min_margin=min_margin, status=status, trace=traces, mode=mode)
