"""CPU oracle for the Kimi-K3 MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
leg of ``bench.py`` (plus ``bench.py --impl reference``) use it.

It is a plain, slow, fp64 NumPy restatement of what the layer computes, written
from the source pages (cited per function) and the OCP microscaling formats.
It shares no code with the CUDA path.  It applies no blocking, fusion or
reordering beyond what the definitions state.

Modules:
  mx       E2M1 / E4M3 / E8M0 decode tables, the MX block quantiser, nibble packing
  router   sigmoid router logits, top-k selection, renormalised weights
  permute  token -> expert histogram, exclusive scan, stable permutation
  layer    routed expert GLU MLP, MXFP8 requantisation, shared expert, combine

Parity status: every function here is pinned by ``tests/test_oracle_*.py``.
SiTU has no published formula and is not implemented.  The latent option
(``layer.latent_moe_layer``, reading R22) is implemented; where its projections
sit is a reading, not something the pages fix, and it is pinned against a
torch restatement of that same reading.  The Quantile Balancing update rule is
unpublished: ``router.routing_margins`` and ``router.margin_quantiles`` compute
the margins and quantiles such a rule would read (pinned), while the rule itself
is the caller's and is "parity unpinned".
"""
