"""fp64 CPU oracle for the Windowed-MTP decode-attention path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg are the only users.  The CUDA library and its Python binding never import it.
"""
from .oracle import (  # noqa: F401
    MODE_CAUSAL, MODE_TREE, MODE_WINDOW, accept_greedy, accept_stochastic, attention, attention_kv8,
    e4m3_decode, e4m3_value, key_visible, max_threads, ring_kv_append, ring_slot, tree_visible,
    window_member,
)
