"""Plain fp64 CPU oracle for the dequantize-in-prologue quantized Linear.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run it.  It shares no
code with the CUDA library (``weight_only_quantized_prologue_b200``) and the
library never calls back into it.

Modules
-------
formats   number formats: E2M1, E4M3 ("fn"), E8M0, BF16, FP32 rounding.
quant     the weight quantizers and the nibble packer of the five formats.
linear    dequantization, the fp64 GEMM reference, static-FP8 activation
          quantization and calibration, SQNR, and the FP4 x FP4 reference
          (dynamic MX / NVFP4 activation quantization).

Parity status of every function is stated in its docstring; functions whose
result is not pinned by an independent check say "parity unpinned".
"""

from . import formats, quant, linear  # noqa: F401
