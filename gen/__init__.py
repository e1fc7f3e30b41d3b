"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This package only draws random arrays with the shapes, value distributions and
structure of the workloads the source pages measure on (Qwen3-shaped drafter
blocks, Markov heads, KV prefixes, target logits).  It contains none of the
draft-tree method's arithmetic: no softmax, no top-k, no tree selection, no
attention, no acceptance rule.
"""
from .workloads import *  # noqa: F401,F403
