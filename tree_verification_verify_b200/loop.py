"""One speculative-decoding iteration on the GPU, with random-weight
stand-in models, for timing the path as a loop and checking that its calls
compose: the tree is built, verified and accepted and the cache committed
without a host round trip, so the whole iteration can be captured and
replayed as one CUDA graph."""

from __future__ import annotations

import torch


class Iteration:
    """One speculative-decoding iteration as a single CUDA graph (the
    SpecExec page's loop: build a draft tree, verify it in one target pass,
    accept, continue from the accepted tokens), with random-weight stand-ins
    for the two models:
      drafter   a bigram model: the logits after a node are
                emb_d[token] @ W_d (V = 32000);
      target    one attention layer: q, k, v = emb_t[token] @ (Wq, Wk, Wv)
                (32 query / 8 kv heads, d = 128, bf16), tree_verify_attn
                over the prefix cache and the tree, logits = the drafter's
                logits + out @ W_lm (a target that agrees with the drafter
                in part, so that some draft tokens are accepted).
    Per iteration: tree_expand_init, `rounds` tree_expand_topb rounds of
    Bsel (each after the drafter's rows for the frontier), the layer and
    tree_verify_attn, the target logits, tree_accept (SpecExec at
    temperature 0.6), tree_commit_kv of the accepted path; the bonus token is
    the next iteration's root (device to device, no host round trip).  The
    weights are random, so the accepted lengths carry no quality meaning."""

    def __init__(self, dev, prefix=4096, budget=64, Bsel=16, V=32000, hidden=1024, iters_room=256, seed=0,
                 temperature=0.6, lm_scale=64.0):
        import tree_verification_verify_b200 as tv
        self.tv, self.dev = tv, dev
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        self.V, self.budget, self.Bsel = V, budget, Bsel
        self.rounds = (budget - 1 + Bsel - 1) // Bsel
        Hq, Hkv, d = 32, 8, 128
        self.Hq, self.Hkv, self.d = Hq, Hkv, d
        bf = torch.bfloat16
        r = lambda *shape, s=1.0: (torch.randn(*shape, generator=g, device=dev) * s)
        # the drafter computes in fp32 (bf16 logits tie often; exact ties are
        # ordered by token on every side, but fp32 keeps the ranking generic)
        self.emb_d = r(V, 256, s=1.0)
        self.W_d = r(256, V, s=4.0 / 16.0)                     # logits ~ N(0, 4^2)
        self.emb_t = r(V, hidden).to(bf)
        self.Wq = r(hidden, Hq * d, s=hidden ** -0.5).to(bf)
        self.Wk = r(hidden, Hkv * d, s=hidden ** -0.5).to(bf)
        self.Wv = r(hidden, Hkv * d, s=hidden ** -0.5).to(bf)
        self.W_lm = r(Hq * d, V, s=lm_scale / (Hq * d) ** 0.5).to(bf)
        Lmax = prefix + iters_room * (budget + 1)
        self.kc = r(1, Lmax, Hkv, d).to(bf)
        self.vc = r(1, Lmax, Hkv, d).to(bf)
        self.prefix0 = prefix
        self.prefix_len = torch.full((1,), prefix, dtype=torch.int32, device=dev)
        self.st = tv.tree_expand_init(budget, V, Bsel, device=dev)
        self.root = torch.zeros(1, dtype=torch.int32, device=dev)      # the next root token
        self.root_row = torch.zeros(1, dtype=torch.int32, device=dev)  # row node 0
        self.rows = torch.empty(Bsel, dtype=torch.int32, device=dev)   # the frontier a round expands
        self.temperature = temperature
        self.record = None     # set to a list to keep each round's rows and logits (tests)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.acc_out = dict(n_accepted=torch.empty(1, dtype=torch.int32, device=dev),
                            accepted_nodes=torch.empty(1, budget, dtype=torch.int32, device=dev),
                            out_tokens=torch.empty(1, budget + 1, dtype=torch.int32, device=dev),
                            min_margin=torch.empty(1, dtype=torch.float64, device=dev))
        self.emitted = torch.zeros(1, dtype=torch.int64, device=dev)   # tokens emitted over the run

    def drafter_rows(self, nodes):
        tok = self.st.token[nodes.clamp(min=0).long()]
        return self.emb_d[tok.long()] @ self.W_d

    def step(self):
        tv, st = self.tv, self.st
        tv.tree_expand_init(self.budget, self.V, self.Bsel, state=st)
        st.token[0:1].copy_(self.root)
        for k in range(self.rounds):
            if k == 0:
                rows = self.root_row
            else:
                self.rows.copy_(st.frontier)
                rows = self.rows
            z = self.drafter_rows(rows)
            if self.record is not None:
                self.record.append((rows.clone(), z.clone()))
            tv.tree_expand_topb(st, z, rows, dev_status=self.status)
        T = self.budget
        tok = st.token[:T].long()
        x = self.emb_t[tok]
        q = (x @ self.Wq).view(1, T, self.Hq, self.d)
        kt = (x @ self.Wk).view(1, T, self.Hkv, self.d)
        vt = (x @ self.Wv).view(1, T, self.Hkv, self.d)
        par = st.parent[:T].view(1, T)
        out, _, _ = tv.tree_verify_attn(q, self.kc, self.vc, self.prefix_len, kt, vt, par,
                                        n_nodes=st.n_nodes, want_lse=False, dev_status=self.status)
        z = self.emb_d[tok] @ self.W_d + (out.view(T, self.Hq * self.d) @ self.W_lm).float()
        z = z.view(1, T, self.V)
        self.target_logits = z
        self.kt, self.vt, self.q = kt, vt, q
        o = tv.tree_accept(z, st.token[:T].view(1, T), par, n_nodes=st.n_nodes, mode="specexec",
                           temperature=self.temperature, seed=1234, step=0, dev_status=self.status,
                           outputs=self.acc_out)
        tv.tree_commit_kv(self.kc, self.vc, self.prefix_len, kt, vt, o["n_accepted"], o["accepted_nodes"],
                          dev_status=self.status)
        n = o["n_accepted"].long()
        self.root.copy_(o["out_tokens"][0].gather(0, n))
        self.emitted += n + 1

    def launches_per_step(self):
        return 1 + self.rounds + self.tv.last_attn_launches + 1 + 1
