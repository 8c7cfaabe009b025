"""Oracle: plain, slow, fp64 CPU restatement of the SO(2)-equivariant (eSCN) edge layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (``equivariant_gnn_electronic_b200``) and neither
imports the other; both take their inputs from the seeded generators in
``synth``.

Modules
  sh      real spherical harmonics, edge frames, Wigner-D by projection
  graph   periodic neighbour list (brute force and cell list) -> destination CSR
  layer   one eSCN message-passing layer (rotate, gated SO(2) linear, attention,
          rotate back, per-atom softmax aggregation)
  cg      real Clebsch-Gordan coefficients by null space
  head    Hamiltonian off-diagonal block head (labels -> blocks, Eq. (1))

Sources: "MALOQ: Massively Accelerated Learning of Operators for Quantum
Transport" (arXiv 2606.28911) Sections II-B1, III, III-B1 (Eq. 1), III-C1 and
Fig. 3; the review page of "Distributed Equivariant Graph Neural Networks for
Large-Scale Electronic Structure Prediction" (arXiv 2507.03840), "What carries
the argument" (incoming-edge layout) and "free parameters".  Where the pages
leave a step open the plainest reading is taken; each such reading is stated
in the function that takes it.

Parity status: every function here is pinned by tests/test_oracle_*.py
against closed forms, library routines, brute force or exact invariants.
"""
