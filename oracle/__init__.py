"""fp64 CPU oracle for tree verification -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct restatement of what the tree-verification
path computes, written from the method's definitions:

* philox.py    -- Philox4x32-10 counter-based uniforms (Salmon, Moraes, Dror,
                  Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11).
* attention.py -- tree-masked attention: every draft node attends to the
                  shared prefix plus its own ancestors and itself (SpecExec
                  page, "Approach": the whole tree is verified in one target
                  pass), with the optional block top-k sparse variant (sparse
                  verification page, "Methodology" 3, attention sparsity).
* accept.py    -- the acceptance walk: greedy longest match at temperature 0,
                  multi-draft speculative sampling with residual resampling
                  (SpecExec page, "Experimental setup": builds on speculative
                  sampling / SpecInfer), and SpecExec's sample-and-descend rule
                  for deterministic trees (SpecExec page, "Approach").
* commit.py    -- appending the accepted path's K/V to the cache, the step
                  that makes the accepted tokens prefix for the next
                  iteration (SpecExec page, "Approach" / "Key results":
                  accepted tokens per target iteration).
* expand.py    -- SpecExec's batched best-first (Dijkstra-style) expansion
                  that keeps the highest cumulative-probability continuations
                  (SpecExec page, "Approach"; "Builds on": Dijkstra's
                  algorithm), plus an independent heap-based simulation and a
                  beam-search constructor used only as pins.

Only the tests, the package's smoke entry and the bench's CPU-baseline leg
may import this package.  It shares no code with the CUDA library: it reads
the raw input arrays, widens them to float64 and computes from scratch.
"""
