"""B200-native MLA decode over a paged latent KV cache.

The compute path lives in ``libmla_b200.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/mla_b200.h``).  ``binding`` marshals torch tensors
into that ABI; ``longrow`` is the host side of one row split across GPUs
(shard rule, per-rank block tables, the (out, lse) exchange); ``inputs`` builds
seeded synthetic workloads.  Importing this package loads nothing: the library
is opened on first use by ``binding``.
"""

__all__ = ["binding", "inputs", "longrow"]
