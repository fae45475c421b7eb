"""CPU oracle for the QLoRA NF4 frozen linear layer with a LoRA adapter.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything from this package.  The
product path (the CUDA library and its Python binding) never imports, links or
runs it, and this package imports nothing from the product: the two share no
code, table or constant generator.  Inputs reach both sides from the seeded
generators in ``bit_nf4_quantized_27_b200.inputs``, which hold none of the
method's arithmetic.

Every function here is the plain definition of one step of the method, written
from the pages it cites.  No blocking, fusion or reordering beyond what the
definition states; matrix products use numpy's float64 ``@`` as a library
primitive.
"""

from .nf4_oracle import (  # noqa: F401
    BLOCK,
    GROUP,
    E4M3_MAX,
    E5M2_MAX,
    U8_MAX,
    SCALE_FORMATS,
    norm_ppf,
    nf4_levels,
    uniform4_levels,
    block_absmax,
    assign_codes,
    pack_codes,
    unpack_codes,
    e4m3_decode,
    e4m3_encode,
    e5m2_decode,
    e5m2_encode,
    u8_encode,
    scale_format_max,
    scale_decode,
    scale_encode,
    double_quantize,
    quantize,
    dequantize_scales,
    dequantize,
    bf16_round,
    bf16_bits,
    storage_bytes,
    lora_scale,
    linear_fwd,
    linear_bwd,
    linear_fwd_multi,
    unpack_keep,
    linear_fwd_dropout,
    linear_bwd_dropout,
    merged_weight,
    merge_export,
    adamw_step,
)
