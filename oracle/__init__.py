"""CPU oracle of the KVzip hot path.  Test infrastructure only: imported by
the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg,
never by the product path."""
from .kvz_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    compact,
    keep_count,
    row_lse,
    row_logits,
    score,
    select,
    visible_pairs,
)
