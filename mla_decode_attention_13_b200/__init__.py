"""B200-native MLA decode over a paged latent KV cache.

The compute path lives in ``libmla_b200.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/mla_b200.h``).  ``binding`` marshals torch tensors
into that ABI; ``inputs`` builds seeded synthetic workloads.  Importing this
package loads nothing: the library is opened on first use by ``binding``.
"""

__all__ = ["binding", "inputs"]
