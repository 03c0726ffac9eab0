"""Plain, slow, fp64 CPU oracle of the on-the-fly equivariant attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call,
link or execute anything in this package; only the tests, the smoke check
and the benchmark's CPU-baseline / reference legs do.  It shares no code,
header, table or constant with the CUDA library under
``atomistic_mlip_b200/csrc``: the only thing both sides share is the seeded
input generator ``atomistic_mlip_b200.workloads``, which holds none of the
method's arithmetic.

Modules
-------
sh          real spherical harmonics and Wigner-D matrices, built two
            independent ways (least-squares fit and Euler / Wigner small-d)
neighbors   brute-force all-pairs radius graph with the exact fp32 predicate
            (NumPy, plus a plain-C all-pairs loop for large N)
attention   the operator itself, edge by edge in fp64
attention_grad
            the same operator restated in PyTorch CPU ops (fp64), whose
            autograd gives the gradients of a scalar of the outputs with
            respect to positions, features and weights
block       the E2Former-V2 block around the attention (merged RMS norm,
            scalar-gated FFN, residuals)
cg          Clebsch-Gordan coefficients (Racah formula) and the dense
            x (x) Y(rhat) convolution in the global frame, the reference for
            the re-indexed (edge-frame) CG convolution

Sources (web pages on E2Former-V2, EquiformerV3 and DPA4):
  * "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
    Memory" (gist.science technical summary), §2.1 "Axis-aligned equivariant
    sparsification (EAAS)" and §2.2 "On-the-fly equivariant attention".
  * "EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-
    Equivariant Graph Attention Transformers", §2B.3 "Smooth radius cutoff
    attention" (envelope inside the softmax denominator).
  * "DPA4: ... EMFA SO(2) Convolution", §2.1 A3 "Envelope-gated attention".

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_*.py`` (closed forms, invariants, special cases, brute
force).  The readings of what the pages leave open (the exact form of the
invariant projections, what the SO(2) blocks mix, where the radial scale
applies, the RBF details, weight fan-in) are conventions fixed by the
workload description; they cannot be checked against the authors' model,
which is not available.
"""
