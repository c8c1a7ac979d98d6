"""CPU oracle for the quantized-attention hot path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The CUDA library does not import it and it does not import the
CUDA library; the two share no code.  Inputs come from the separate ``synth``
generator module.

Modules:
* numerics    - BF16 / FP64->BF16 / E4M3 codecs (pinned against torch casts and
                exact rational rounding).
* sage_oracle - the method's steps: K/V column statistics, INT8 block quant,
                V FP8 per-channel quant, tiled online-softmax attention, plus an
                exact FP64 attention and a quantization-off run of the same tile
                loop used to pin it.
"""
from . import numerics, sage_oracle  # noqa: F401
