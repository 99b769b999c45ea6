"""CPU oracle for the NVFP4 W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product.

Every function is a plain, slow restatement of what the paper "Why Gated
DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a
Hybrid 27B LLM" says the layer computes, with the number-format arithmetic the
pages leave open filled in by the plainest reading (listed in the module
docstring of ``oracle.nvfp4``).

Pinning status (what each function is checked against in ``tests/``):
  e2m1_encode / e2m1_decode  -- ml_dtypes.float4_e2m1fn (dense exhaustive
                                sweep) + hand tie table (tests/golden)
  e4m3_encode / e4m3_decode  -- ml_dtypes.float8_e4m3fn and torch.float8_e4m3fn
                                on every rounding boundary + hand table
  quantize                   -- round trip on grid inputs, outlier locality,
                                hand-derived block (tests/golden)
  dequantize / linear64      -- exact Fraction brute force, all E2M1 pairs
  fused_linear64             -- closed-form mismatch ratio, per-segment
                                decomposition
  sigmoid64 / gdn_decay64    -- Lipschitz bounds, limits, closed values
  silu_mul_bf16              -- ml_dtypes bfloat16 RNE (random and exact ties),
                                closed values and limits of SiLU
  kv_quantize / kv_scale /
  kv_dequantize              -- ml_dtypes.float8_e4m3fn on every finite bf16
                                value, saturation and signed zeros by hand
  gdn_recurrence_seq         -- exact overwrite along the key, decay-only action
                                orthogonal to it, gradient step on the key-value
                                loss (finite differences)
  gdn_recurrence_chunked     -- equals gdn_recurrence_seq (ragged chunks)
  gdn_error_contraction /
  gdn_noise_plateau          -- simulated impulse decay and noise plateau
No function is "parity unpinned".
"""
from .nvfp4 import (  # noqa: F401
    E2M1_VALUES, GS_DIVISOR, e2m1_encode, e2m1_decode, e4m3_encode, e4m3_decode,
    global_scale, quantize, dequantize, pack_codes, linear64, fused_linear64,
    fused_linear64_shared_scale, sigmoid64, gdn_decay64, silu_mul_bf16,
)
from .kv import kv_scale, kv_quantize, kv_dequantize  # noqa: F401
from .gdn import (  # noqa: F401
    gdn_recurrence_seq, gdn_recurrence_chunked, gdn_error_contraction, gdn_noise_plateau,
    gdn_error_trace,
)
