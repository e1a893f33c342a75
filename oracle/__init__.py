"""Float64 CPU oracle for the QLoRA adapted linear layer.

THIS PACKAGE IS TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (``quantized_rank_fine_b200`` and ``libqlora.so``) never imports,
links or calls anything here, and nothing here imports the product path: the two
share no code. The only module both sides use is ``synth`` (seeded input
generators, which contain none of the method's arithmetic).

The oracle is plain, slow and written to be checked by eye against the pages it
restates. Sources (cited by page title and section throughout):

* "QLoRA (low-rank adapters on a quantized model)" (herodthegreater.github.io,
  pigeon guide): sections "How it works", "What QLoRA adds over LoRA",
  "The code, line by line", "Source code".
* "LLMs · QLoRA" (blog.sahaj.si): the hand-built NF4-style vs uniform 4-bit
  blockwise quantiser and its printed output.
* "LoRA & QLoRA" (codewithdark-git.github.io): "Mathematical Formulation",
  "4-bit NormalFloat (NF4)" and its value table, "Double Quantization".
* "LoRA and QLoRA: Efficient Fine-Tuning Explained" (glorytecks.com): the
  parameter-count arithmetic of "A real run".

Modules:

* ``oracle.nf4``    -- codebook, blockwise absmax, nearest-level encode, E4M3
  double quantisation, dequantisation, bf16 rounding, the blog's experiment.
* ``oracle.linear`` -- forward, backward (adapter scale, dropout), merge and
  parameter counts.
* ``oracle.adam``   -- the Adam / AdamW step on the adapters.
* ``oracle.loftq``  -- merge -> re-quantise round trip and the SVD initialisation.
* ``oracle.intq``   -- the symmetric uniform INT quantiser with one scale per 16
  weights (2-bit ternary, 3 and 4 bits).

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_*.py``
against something other than itself (printed values, closed forms, brute force,
library routines). No function here is "parity unpinned".
"""

from . import nf4, linear  # noqa: F401
