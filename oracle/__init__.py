"""CPU oracle of gated delta-rule decode over a slot or paged state pool.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
The CUDA library never calls it and shares no code with it: the two meet
only through the seeded input generators in ``workloads``.

The oracle computes in float64 (the fp8 tile codec and the int8_hadamard32
codec in binary32, so that codes and scales are exactly reproducible) and follows the pages' literal
step order; see ``oracle.gdn`` for the sources and for every reading of a
point the pages leave open.

Parity status of each function:

* ``gated_delta_step`` and the pool drivers: pinned by closed forms
  (alpha=1/beta=0 keeps S; alpha=0/beta=1 gives k v^T; unit-norm key with
  beta=1 overwrites; beta=0 gives the product of decays), an independent
  transition-matrix formulation, exact rational arithmetic on tiny inputs,
  sequential == repeated single steps, and the paged and slot pool rules.
* ``step_unit`` (the storage of bf16, fp8 and int8_hadamard32 states between
  tokens, and the ``readout`` flag): pinned by the token write events of
  the ModelOpt decode reference (a T-token call equals T one-token calls
  that pass the state through the pool, bit for bit, on the slot, paged and
  KDA drivers, and differs from encoding once at the end) and by the
  stored readout equalling q^ times the decoded stored state, while the
  working readout equals the fp32 step of the decoded state.
* ``formats``: pinned by the OCP E4M3 format's defined points, by library
  conversions (torch bf16 and float8_e4m3fn casts) and by grid properties.
  The int8_hadamard32 codec: its rotation by scipy's Sylvester Hadamard
  matrix and by closed forms (constant and unit vectors, R R = I), its
  rounding by ties-to-even points, its grouping by the page's statement (one
  scale per key channel and 32 values) and its error by the bound that an
  orthonormal rotation carries over from the rotated domain.
* conventions the pages do not fix (parity unpinned): the L2-norm epsilon,
  the GQA head map ``hv // (HV // H)``, the KDA gate's use of the GDN form
  per key channel, the tile codec's scale formula, and for int8_hadamard32
  the Hadamard order and normalisation and the scale formula amax / 127.
"""

from . import formats, gdn  # noqa: F401
