"""CPU oracle for the E(3)-equivariant message-passing convolution.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
anything under ``oracle/``; only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may.  The oracle shares no code, tables or
constants with the CUDA library: it computes the Clebsch-Gordan coefficients
with its own Racah-formula implementation (exact rationals), the spherical
harmonics with its own Legendre construction, and the convolution with plain
loops (C, fp64 accumulation) or plain NumPy.

What it computes follows the pages:

* e3j: an Efficient and Open-Source Backend for Euclidean Equivariant
  Operations on GPU and TPU (arXiv 2609.35099), abstract and Table 1: the
  message-passing convolution of MACE-style potentials, forward and backward.
* FlashCart: Fast Cartesian Tensor Products for Equivariant Interatomic
  Potentials (arXiv 2610.06409), App. B (direction tensors of degree l are the
  real spherical tensors; admissible paths obey the triangle rule and the
  coupling is unique up to normalisation; natural-parity outputs), §4 / App. D
  (receiver sums, channel-diagonal products, feature rows ordered rank block ->
  component -> channel) and §2 (forces are gradients of the energy).

Where the pages leave a convention open (SH normalisation, CG phase, output
irreps) the readings are listed in the module docstrings below.

Modules
-------
irreps   parse irreps strings, enumerate coupling paths, block offsets
cg       complex CG by the Racah formula, complex->real change of basis
sh       real spherical harmonics and their gradient w.r.t. the edge vector
csr      receiver/sender CSR offsets and stable permutations
conv     the convolution: NumPy brute force (per-edge messages) and the C
         loop implementation in ``conv_ref.c`` (fp64 accumulation); output
         variants (both parities, per-path blocks)
dbl      the double backward (VJP of the backward), NumPy brute force
nodeprod the node-local channel-diagonal product, forward and backward
radial   Bessel basis, polynomial envelope and radial MLP with their VJP
build    compiles ``conv_ref.c`` with gcc
"""
