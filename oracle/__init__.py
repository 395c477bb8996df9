"""CPU oracle for the microscaled (NVFP4 / MXFP8) linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``fp8_gemm_diffusion_b200``) never imports it and never falls
back to it; the two share no code.  The only shared module is ``workloads``,
which draws the seeded synthetic inputs and holds none of the method's
arithmetic.

Plain numpy, written to be checked by eye against the definitions:

* ``formats``  - E2M1 / E4M3 / E8M0 codecs (table search, RNE, saturating).
* ``quant``    - NVFP4 and MXFP8 quantisation, scale-factor layout.
* ``gemm``     - float64 reference of the quantised linear and its tolerance.
* ``dispatch`` - the selective-quantisation rule.
* ``producer`` - a linear layer with the GELU activation fused into its
  epilogue, and that epilogue's error scale.
* ``attention`` - 8-bit (MXFP8) attention with per-token scales: softmax in
  float64 on the dequantised operands, and its error bound.

Every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` to facts other than itself (code tables, tie cases,
exact blocks, closed forms, brute force on tiny shapes, an independent library
cast, byte offsets of the scale-factor layout worked by hand from its
published description).
"""

from . import formats, quant, gemm, dispatch, producer, attention  # noqa: F401
from .formats import *  # noqa: F401,F403
from .quant import *  # noqa: F401,F403
from .gemm import *  # noqa: F401,F403
from .dispatch import *  # noqa: F401,F403
