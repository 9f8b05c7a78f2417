"""fp64 CPU oracle for the canvas denoise path -- TEST INFRASTRUCTURE ONLY.

Only tests/, the package's smoke() check in __graft_entry__.py and bench.py's
CPU-baseline / reference leg may import or call this package. The product path
(the C-ABI library and its Python binding) never touches it and fails loudly
when its CUDA library is missing.

Contents:
  philox.py   -- Philox-4x64-10 from Salmon et al. (SC'11), plus the canvas draw.
  numerics.py -- storage-format rounding (bf16 round-to-nearest-even, f32).
  model.py    -- the step and decode, in fp64, following the pages step by step.

Parity pins live in tests/test_oracle_pins.py. Functions with no pin other than
their own definition are marked "parity unpinned" in their docstrings (none at
present beyond the trained-model averages, which are not computed here).
"""
from . import model, numerics, philox  # noqa: F401
