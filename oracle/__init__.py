"""Plain, slow, obviously-correct CPU oracle for exact softmax attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it. It shares no code with the CUDA path.

Everything is computed in float64 with NumPy, materialising the score matrix
S and the probability matrix P exactly as the plain definition states
(see ``oracle.attention`` for the citations).
"""

from .attention import (  # noqa: F401
    allowed_mask,
    oracle_attention,
    oracle_attention_backward,
    oracle_attention_rows,
    oracle_attention_varlen,
    oracle_decode,
    oracle_decode_paged,
    oracle_probabilities,
    paged_to_contiguous,
    key_chunk_attention,
    online_softmax,
    merge_partials,
    brute_force_attention,
)
