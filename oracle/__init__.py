"""CPU oracle for the NF4 + double-quantized QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the QLoRA pages define, written in NumPy (fp32 where the
format fixes fp32, fp64 for the linear algebra).  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The CUDA library never imports, links or
calls anything here, and nothing here imports the CUDA library: the two share
no code, tables or constant generators.

Sources (web pages, cited by title and section):

* [P1] "QLoRA > Summary" (mbrenndoerfer.com)
* [P2] "QLoRA" (techbytebybyte.com tutorial)
* [P3] "QLoRA and Quantized Training" (fanout lesson)
* [P4] "QLoRA Explained: 4-bit NF4, Double Quantization and Paged Optimizers"
* [P5] "A 65B fine-tune on the GPU you already have" (attention.sh)

Modules:

* ``nf4``     -- the 16 NormalFloat levels and the decision midpoints.
* ``quant``   -- blockwise absmax quantization, packing, double quantization,
                 dequantization, bf16 rounding.
* ``linear``  -- forward / backward of Y = X.dequant(W)^T + s.(X.A^T).B^T.
* ``memory``  -- bytes-per-parameter arithmetic of the storage format.
* ``codebooks`` -- the FP4 and INT4 baselines beside NF4.
* ``merge``   -- folding the adapter into the dequantized base (export).
* ``dropout`` -- LoRA dropout on the adapter input (Philox4x64-10 mask).
* ``dq_fp8``  -- the mean-subtracted 8-bit-float (E4M3) double quantization.

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle.py``
against invariants, closed forms, brute force or a library routine; none is
"parity unpinned".
"""

from . import nf4, quant, linear, memory  # noqa: F401
