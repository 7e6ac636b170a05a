"""CPU oracle for the fused attention forward pass -- TEST INFRASTRUCTURE ONLY.

This package is the slow, obviously-correct fp64 statement of what the CUDA
path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import it.  The product path
(``io_aware_attention_02_b200``) never imports, links or executes anything
here, and nothing here imports the product package: the two share no code.
The only module both sides use is the seeded input generator
(``io_aware_attention_02_b200.inputs``), which holds none of the method's
arithmetic.

Sources (page title, section):

* "FlashAttention-3: como exprimir H100 al limite con atencion IO-aware"
  (dibro.site), sections "Arquitectura y metodo" (tiling, m/l statistics) and
  "Contribuciones clave" (causal attention, masked blocks skipped).
* "FlashAttention-3" explainer (droidorbit.com), opening definition
  Softmax(Q K^T / sqrt(d)) V and section "Mathematical Formulation: The Online
  Softmax Rescaling Trick"; FAQ "linear attention approximations" (the method
  is exact).
* Quantum-bit repost "H100 utilisation 75% ... FlashAttention-3" (m.ruangu.net),
  third technical upgrade (FP8, block-wise quantisation, incoherent
  processing) and the FP8 accuracy experiment.
* "FlashAttention-3 (HE)" (systems-analysis.info), section "Technical
  innovations", item 3 (incoherent processing with a Hadamard matrix).

Modules:

* ``attention`` -- exact attention (the definition), probabilities, LSE.
* ``fp8``       -- e4m3 rounding from the format's definition, Sylvester
  Hadamard matrix, per-block quantisation as the pages describe it.
* ``backward``  -- gradients (dQ, dK, dV) of exact attention, the chain rule
  written out.
* ``baselines`` -- the per-tensor FP8 and standard FP16 attentions of the
  pages' accuracy experiment.
* ``decode``    -- fewer queries than keys (decode causal alignment) and the
  split-KV merge of partial results.

Parity status: every function here is pinned by ``tests/test_oracle.py``
against closed forms, invariants, a hand-computed two-token example, a
pure-Python brute force and library routines (``torch`` SDPA in float64,
``torch.float8_e4m3fn`` casting).  The relative FP8 error ratios the pages
print (2.6x, 1.7x) are NOT pinned: "parity unpinned" for those ratios.
"""

from . import attention, backward, baselines, decode, fp8  # noqa: F401
