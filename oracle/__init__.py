"""CPU fp64 oracle of one parent-conditioned draft-tree decode round.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The product path (the C-ABI library and its Python binding)
never imports, links or calls anything here, and this package shares no code,
table or constant generator with the CUDA sources.

Modules
-------
philox       Philox4x32-10 and the uniform / counter conventions.
markov_tree  parent-conditioned node distributions and the best-first
             budget-N tree (PCTree summary "k=4, N=32 / k=1 gives the greedy
             chain" paragraph; TreeSpark article "core idea" section).
accept       greedy and recursive-residual acceptance walk (TreeSpark article,
             "lossless decoding" section; PCTree summary "setup").
verify_attn  tree-masked GQA attention over prefix + root + ancestors.
treeflash    SwiGLU AR-approximator round (TreeFlash explainer, method
             sections 1 and 2).
variants     the baseline trees of the PCTree summary's mechanism isolation
             (chain, marginal-ranked, Shared-Markov) and acceptance length.
load_policy  survival-ordered allocation of a round's verification capacity
             over a batch (TreeSpark article, load-adaptive serving policy).
calibration  logged (depth, log-probability, accepted) triples and the
             per-depth maximum-likelihood fit of the calibration.

Every floating quantity is fp64; inputs are the exact stored values.
"""
