"""Oracle: a plain, slow, fp64 CPU statement of what the Delta-CoMe serving path computes.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library, its Python binding) may
import, call, link or execute anything in this package.  Only ``tests/``, the smoke check in
``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` use it.  It shares no code with
the CUDA path: the only thing both sides consume is the seeded input module
``tenant_mixed_precision_b200.synth``, which draws numbers and holds none of the method's
arithmetic.

Sources (web pages; cited by title and section):

* [P1] "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法" (paooo.com news article),
  sections "Delta-CoMe的技术原理" (technical principles) and "Delta-CoMe的应用场景" (uses).
* [P2] "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
  Models" (atlas.scime.ai summary), sections "Problem", "Approach", "Key results",
  "Limitations", "Experimental setup".
* [P4] "Enhancing Delta Compression in LLMs via SVD-based Quantization Error Minimization"
  (gist.science explanation of PrinMix), section 2.1 (eq. 5) and 2.3, for the orientation
  W = U Sigma V and the order "quantize V, then U".

Parity status of each function is stated in its docstring; every function here is pinned by
``tests/test_oracle_pins.py`` against closed forms, invariants, brute force or hand-derived
fixtures under ``tests/golden/``.
"""
from .delta_come import (  # noqa: F401
    Artefact,
    QuantVector,
    activation_error,
    allocate_ranks,
    budget_bits,
    brute_force_linear,
    code_bits_used,
    compress_delta,
    compress_factors,
    delta_only,
    delta_linear,
    delta_weights,
    dequantize_vector,
    dequantized_factors,
    eckart_young_tail,
    route_tokens,
    rtn_quantize_group,
    rtn_quantize_vector,
    svd_factors,
    GROUP,
)
