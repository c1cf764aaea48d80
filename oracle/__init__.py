"""Plain float64 CPU oracle for the tree-verify step.  TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
shares no code with the CUDA path: it reads the same seeded inputs (bf16 bit
patterns as uint16 arrays, int32 trees) and computes, slowly and in the most
direct form, what the verify step is defined to produce.

Sources (page title, section):
  * "The Architecture of Pragmatic Ambition" -- "The Knowledge Architecture"
    (DDTree: target attention over the draft tree under a visibility mask; greedy
    walk to the longest prefix matching the target's predictions) and "The
    Thinking Process" (MLA absorb form: q_nope . (W_UK c_kv) rewritten as
    (q_nope W_UK) . c_kv).
  * "The Architectural Keystone: Writing the Model Header ..." -- "The Reasoning
    That Preceded the Header" (budget+1 nodes, root re-processed at the next free
    slot, accepted latents gathered into contiguous slots, cache length advanced
    by the accepted count, budget 0 = plain decode) and "Mistakes and Iterative
    Refinement" (compaction must read all kept rows before writing any).

Every function is pinned by the CPU tests in tests/test_oracle.py (special
cases that reduce to a library routine, closed forms, brute force, invariants).
"""
from .tree import check_parents, ancestors, depths, visibility_words, n_words
from .attention import tree_verify_attention, bf16_to_f64
from .accept import tree_accept
from .cache import kv_compact, kv_write_nodes
from .step import verify_step

__all__ = [
    "check_parents", "ancestors", "depths", "visibility_words", "n_words",
    "tree_verify_attention", "bf16_to_f64", "tree_accept", "kv_compact",
    "kv_write_nodes", "verify_step",
]
