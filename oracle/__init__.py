"""CPU oracle of the FP8 E4M3 quantization path.

TEST INFRASTRUCTURE ONLY.  The test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only code allowed to import it; the
product library never does, and this package never imports the product.

``core`` wraps the plain C oracle (``fp8q_oracle.c``: E4M3 encoding, group
quantization, absmax, reshape_and_cache_fp8, freeze scale) and restates the
K-major scale layout with zeroed phantom rows on top of it.  ``calibration``
restates the calibration window (staging, freeze, chronological replay) on
the host on top of it.

Pins (tests/test_oracle_*.py) tie every function to something other than
itself: torch's E4M3 conversion as a library routine, exact rational
arithmetic, hand-worked groups, closed forms and brute force.
"""
from . import core, calibration  # noqa: F401
from .core import (GROUP, absmax, bf16_to_f32, build, e4m3_encode, freeze_scale,  # noqa: F401
                   group_quant, group_quant_kmajor, group_quant_strided, group_scale,
                   kv_write)
