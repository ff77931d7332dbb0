"""CPU oracle (fp64 numpy) for the Spava / APB-V approximate-attention prefill.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  The library under
``sequence_approximate_attention_b200`` never imports, links or runs anything here,
and nothing here imports the library: the two share no code, only the seeded
input generator in ``workloads/``.
"""

from .spava_oracle import (  # noqa: F401
    approx_attention,
    attention_rows,
    bf16_bits_to_f64,
    contiguous_owners,
    dense_causal,
    host_costs,
    host_of_row,
    host_offsets,
    key_set,
    longest_first_owners,
    lse_merge,
    prefill,
    probe_scores,
    select_passing,
    sharded_attention,
    zigzag_owners,
)
