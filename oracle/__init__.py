"""Oracle for the QLoRA NF4 + double-quantization codec and the QLoRA linear.

TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the CPU-baseline
leg of the benchmark may import this package.  The product library never calls
it and shares no code with it: the CUDA path and this oracle are written
independently and compared on the same seeded inputs.

Source: "QLoRA: Efficient Finetuning of Quantized LLMs"
(inquiringlines.com/papers/2305.14314), section "Method", and the LoRA
formula x_out = (W_q + BA) x_in of "QLoRA: Efficient Fine-Tuning of Quantized
Language Models" (mbrenndoerfer.com), section "Low-Rank Adaptation (LoRA)".

Modules
  codebook  NF-k data type from normal quantiles (paragraph "4-bit NormalFloat
            Quantization", steps (1)-(2) and the asymmetric construction).
  exact     exactly rounded helpers: binary32 rounding of a rational number,
            the exactly rounded mean used by double quantization.
  codec     quantize / double-quantize / dequantize (C loops in nf4_ref.c,
            driven from Python).
  linear    QLoRA linear forward and backward in float64 (numpy).
  optim     AdamW update of the adapters in float64 (the paged optimizer).
  block     one LLaMA-layout QLoRA transformer block, forward and backward, float64.

Parity status: every function has a pin in tests/test_oracle_*.py except the
individual NF4 codebook values beyond the structural invariants, and the
claim that every bin holds the same expected share of values, which the
pages make but never back with numbers ("parity unpinned" for those two).
"""

from . import codebook, exact, codec, linear, optim, block  # noqa: F401
