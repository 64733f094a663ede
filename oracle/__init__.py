"""CPU fp64 oracle for the context-parallel attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code
with the CUDA library (no kernels, headers, helpers or constant tables);
the two meet only at the seeded input generators, which hold none of the
method's arithmetic.

Everything here is the plain definition, written out in float64 NumPy:

* ``attention``          one-shot scaled-dot-product softmax attention over
                         the whole key sequence, returning the output and
                         the natural-log log-sum-exp per query row;
* ``attention_partial``  the same restricted to one K/V chunk (one ring step);
* ``lse_merge``          the fp32-style merge of two (out, lse) partials;
* ``ring_attention``     the literal ring walk: partial per chunk + merge;
* ``ulysses_permute``    the sequence-shard <-> head-shard all-to-all index map;
* ``usp_attention``      the unified (Ulysses x Ring) composition;
* ``ulysses_anything_*``  the all-to-all and attention with uneven sequence
                         and head splits (Ulysses Anything).

Pins: every function is checked in ``tests/test_oracle.py`` against facts
that do not come from the oracle itself (closed forms, brute force loops on
tiny inputs, torch's own CPU attention, permutation invariants and the
worked examples in ``tests/golden/``).  No function is left parity-unpinned.
"""
from .attention import (attention, attention_partial, attention_bruteforce,
                        lse_merge, ring_attention, ring_chunk_offsets)
from .ulysses import (ulysses_permute, ulysses_permute_bruteforce, usp_attention,
                      uneven_offsets, ulysses_anything_permute, ulysses_anything_attention)

__all__ = [
    "attention", "attention_partial", "attention_bruteforce", "lse_merge",
    "ring_attention", "ring_chunk_offsets", "ulysses_permute",
    "ulysses_permute_bruteforce", "usp_attention", "uneven_offsets",
    "ulysses_anything_permute", "ulysses_anything_attention",
]
