"""CPU oracle for group-32 4-bit weight-only quantization and the dequantize-fused
linear.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may use it. It is a plain, slow, obviously-correct NumPy restatement of what the
source pages define, shares no code, table or constant generator with the CUDA
library, and is itself pinned by the ``-m "not gpu"`` tests against hand-worked
examples, closed forms, invariants and brute force.

Functions whose parity has no independent pin say so in their docstring
("parity unpinned"): only ``quantize_asym_minmax``, which exists to shape
synthetic input data for the asymmetric variant.

``oracle.q4_0`` restates the GGUF Q4_0 block format (32 elements in 18 bytes: a
binary16 scale, then 16 bytes of 4-bit codes) and its linear, pinned in
``tests/test_q4_0_oracle.py``.
"""

from .w4_oracle import (  # noqa: F401
    FLOOR,
    GROUP,
    STATUS,
    bf16_bits_to_f32,
    check_linear,
    dequantize,
    dequantize_asym_gidx,
    f32_to_bf16_bits,
    linear,
    linear_backward_x,
    lora_merge,
    linear_asym_gidx,
    pack_nibbles,
    payload_bytes,
    quantize_asym_minmax,
    quantize_rtn,
    quantize_rtn_channel,
    expand_channel_scales,
    unpack_signed,
    unpack_unsigned,
    validate,
    validate_asym,
)
