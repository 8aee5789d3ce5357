"""CPU float64 oracle of the LatentMoE layer forward pass.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py; never by the product path (the CUDA library and
its Python binding), with which it shares no code.

  lmoe   -- router, segments, latent-space experts, shared expert, layer output
  nvfp4  -- E2M1 / E4M3 codes and the NVFP4 quantise-dequantise image

Pins (tests/test_oracle_*.py, run with -m "not gpu") tie every function here to
the pages and to mathematics that does not depend on this code: brute-force
top-K, a loop-only dense-masked restatement of the layer, closed-form special
cases, the pages' eq.(1) example and layer tables (tests/golden/), exhaustive
E2M1 codes and torch's E4M3 conversion.
"""
from . import lmoe, nvfp4  # noqa: F401
from .lmoe import (layer_forward, route, segments, token_forward,  # noqa: F401
                   scaling_relation, is_valid_topk, sigmoid, sqrelu)
