"""Plain, slow CPU oracle for blockwise NF4 quantisation, double quantisation
and the QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
constant, table or helper with the CUDA library; the two meet only through
the seeded input generator in ``qlora_linear_layers_b200.synth``.

Every function cites the web page passage it follows, by page title and
section.  The pages used:

* "QLoRA Explained: A 4-Bit Base, NF4, and What It Really Costs"
  (skillsuites.com) -- the technical core: the scale-and-round worked
  example, blocks of 64, the quantile table, double quantisation, the
  dequantise-before-matmul steps.
* "LoRA vs QLoRA: Efficient Fine-Tuning Explained" (masterainow.com) --
  the LoRA product W' = W + (alpha/r) * B @ A.
* "What is QLoRA, and how does it enable fine-tuning on consumer hardware?"
  (studyaidesign.com) -- the N*b/8 memory formula and 2rd adapter count.
* zenaique.com QLoRA multiselect quiz -- the ~0.37 bits/param saving and
  bf16 adapters.

Where the pages are silent or disagree, the reading taken is stated in the
docstring of the function that depends on it.

Parity status: every function here is pinned by ``tests/test_oracle.py``
against something other than itself (brute force, the pages' worked
example, closed forms, library routines, autograd, invariants).
"""

from .nf4 import (  # noqa: F401
    BLOCKSIZE,
    DQ_BLOCKSIZE,
    nf4_table,
    uniform_table,
    fp4_table,
    distinct_values,
    thresholds,
    block_absmax,
    normalise,
    nearest_code,
    quantize,
    pack,
    unpack,
    dq_mean,
    double_quantize,
    dq_absmax,
    e4m3_values,
    e4m3_encode,
    e4m3_decode,
    dequantize,
    round_bf16,
    stored_bits_per_param,
)
from . import dropout  # noqa: F401
from .linear import linear_fwd, linear_bwd, linear_bwd_adapters, merge, round_bf16_f64  # noqa: F401
