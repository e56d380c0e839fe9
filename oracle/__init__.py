"""Float64 CPU oracle for the equivariant edge tensor-product convolution.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the
CUDA library (``equivariant_mlip_tensor_edge_b200``); the only module both
sides use is ``workloads`` (seeded input generation, none of the method's
arithmetic).

What it computes (plain definitions, no blocking, fusion or reordering):

* ``cg``     -- Clebsch-Gordan coefficients from Racah's closed form, exact in
               rational arithmetic, moved to the real spherical-harmonic basis
               (for l1 + l2 + l3 odd: the imaginary part of the moved tensor).
* ``sh``     -- real spherical harmonics, component normalisation, as solid
               harmonic polynomials, with their analytic gradient.
* ``wigner`` -- Wigner D matrices from Wigner's small-d formula (used by the
               equivariance pins).
* ``radial`` -- Bessel radial basis times the polynomial cutoff envelope.
* ``graph``  -- brute-force neighbour list and canonical receiver-sorted CSR.
* ``conv``   -- irreps/path enumeration (any multiplicities and parities), the
               forward edge convolution and its analytic vector-Jacobian product.
* ``product``-- the node-local path-reduced product and product ladder.

Sources. The pages behind this build ("Fast and Accurate Foundation Models for
Equivariant MLIPs", section VII Methods; "FlashCart", Fig. 3 caption, Table C1,
Fig. D1) name the operation -- a Clebsch-Gordan tensor product of sender
features with spherical harmonics of the edge direction, weighted per path and
channel by a learned projection of a radial basis and summed into the receiver
-- but do not print its formulas. The formulas below are the textbook
definitions, with the conventions listed in the repository's design notes.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against something other than itself (library routines, closed forms,
invariants, the Table C1 operation counts, finite differences, complex-step
derivatives). No function is parity-unpinned.
"""
