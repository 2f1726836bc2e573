"""Seeded synthetic inputs for the fused chunked KL-distillation loss.

This package is shared by the fp64 oracle (``oracle/``) and the CUDA path
(``chunked_kl_loss_ckl_b200``).  It draws random numbers and lays them out;
it holds none of the loss arithmetic (no softmax over the vocabulary, no KL,
no gradient).  See :mod:`ckl_synth.inputs`.
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_config,
    make_inputs,
    student_topk_numpy,
    student_topk_torch,
)
