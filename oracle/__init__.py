"""CPU oracle for NF4 + double quantization and the QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain, obviously-correct
restatement of the method that the CUDA path is checked against.  Only the test
suite (``tests/``), ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import it.  It imports nothing from the CUDA path and
the CUDA path imports nothing from it: they share no kernels, tables, constants
or helpers.  Everything here is numpy on the host, float64 unless a step of the
method fixes a narrower rounding (fp32 / bf16 / e4m3), in which case that single
rounding is applied exactly as stated.

Sources, cited by page title and section:

* "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and
  Paged Optimizers" (fullstackaihub teardown) -- section 2 (codebook), section 3
  (blockwise quantization and double quantization), section 4 (forward pass and
  dequantization helper, backward statement).
* "QLoRA, explained." (vibeengines) -- the numbered method steps 1-5 and the
  notation list.
* "QLoRA Explained: What Actually Trains in 4 Bits? | Part 2/6" (video
  description) -- the Appendix-E lookup example and the storage arithmetic.

Pin status of every function is listed in the module docstrings of
``oracle.nf4``, ``oracle.linear``, ``oracle.variants`` (the FP4-E2M1 and INT4 code books,
single-level quantization without double quantization, adapter merge + re-quantization) and
``oracle.adamw`` (the AdamW step of the paged optimizer).  No function is "parity unpinned": each has
at least one check against the pages or the mathematics in ``tests/``.
"""

from . import nf4, linear, variants, adamw  # noqa: F401
