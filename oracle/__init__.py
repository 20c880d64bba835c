"""CPU oracle for the ConvRot packed-INT4 quantized linear.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or call it. It shares no
code, tables or helpers with the CUDA library under
``bit_quantized_linear_rotate_b200/csrc``.

Every function is a plain, slow, obviously-correct restatement of what the
pages define, in float64 wherever the pages leave the precision open:

* the groupwise Hadamard rotation and rowwise symmetric quantization of
  comfy-kitchen PR #155 "[Feat][Ascend] Add fused RotateQuant backend"
  (sections "What this PR does" and "How was this patch tested?");
* the packed uint4 codec and the AWQ W4A16 dequantization formula of
  ``comfy_kitchen/tensor/awq_w4a16.py`` (module docstring and
  ``TensorCoreAWQW4A16Layout.dequantize``);
* the integer matmul with a rowwise-scale epilogue of comfy-kitchen
  PR #182 "HIP port of #176: W4A8 decode GEMV and fused GatedDeltaNet
  decode" (Description: shared codec and ``EpiRowwise`` epilogue) and of
  stable-diffusion.cpp PR #2276 "feat: support packed INT4 convrot models"
  (Summary: ``convrot_w4a4`` and ``asym_w4a8_int8``).

Parity status: every public function is pinned by ``tests/test_oracle.py``
against closed forms, invariants, brute force or hand-worked fixtures under
``tests/golden/``. The order of the fp32 epilogue products is a reading (the
pages do not fix it); it is pinned only through the 1e-2 output tolerance.
"""

from .convrot import (  # noqa: F401
    QMAX,
    awq_dequantize,
    bf16_bits_to_f64,
    epilogue_rowwise,
    gemv_awq_w4a16,
    gemv_w4a8,
    hadamard_closed_form,
    hadamard_sylvester,
    int_matmul,
    linear_w4a4,
    linear_w4a8,
    pack_nibbles,
    quantize_rowwise,
    rotate_groups,
    rotate_quant_rowwise,
    to_bf16_bits,
    unpack_nibbles,
)
