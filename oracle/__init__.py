"""CPU fp64 oracle for the equivariant graph attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` (plus ``bench.py --impl reference``) may use it.  It shares
no code, table or helper with the CUDA library; the only thing both sides
consume is the seeded input generator (``equivariant_graph_attention_b200.synth``),
and this package does not import even that.

It computes the plain definitions, slowly and in float64:

* ``so3``: complex Clebsch–Gordan coefficients by the Racah formula, the
  complex-to-real spherical-harmonic basis change, real coupling tensors,
  real spherical and solid harmonics, real Wigner-D matrices (solved from
  their defining property) and the alignment rotation.
* ``graph``: brute-force O(N^2) radius graph in exact integer arithmetic with
  K-nearest truncation.
* ``attention``: dense tensor-product source coupling, invariant logits,
  two-pass softmax over each atom's neighbours, aggregation, dense target
  coupling, and the composed forward pass.
* ``projection``: the invariant query/key projection (a linear map of the
  degree-0 channels).
* ``storage``: bfloat16 rounding, where a test models the bf16 storage the
  workloads specify.
* ``escn``: the edge-centric eSCN convolution (rotate each neighbour's
  features into its edge frame, SO(2) linear layer, rotate back, sum), the
  comparison workload.

Citations name the pages by title:

* [EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" (explainer page)
* [TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
  Memory" (technical-summary page; its Dutch and Italian versions carry the
  same sections)

Parity status: every function here is pinned by tests under ``tests/`` marked
``not gpu`` (library routines, closed forms, invariants and brute force); the
absolute end-to-end values have no printed worked example on the pages, so the
composed forward is pinned through those component pins and its symmetry
properties (rotation and permutation equivariance, the ℓ_max = 0 reduction to
masked scaled-dot-product attention).
"""
from . import so3, graph, attention, projection, storage, escn  # noqa: F401
