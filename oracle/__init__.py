"""Oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct CPU restatement (NumPy, float64 unless a
step fixes another precision) of what the GPU library computes:

* ``oracle.nf4``   -- the 4-bit NormalFloat codebook, blockwise absmax quantisation, nibble
  packing, the double-quantised absmax variant and dequantisation;
* ``oracle.qlora`` -- the LoRA-adapted linear forward ``h = X deq(W0)^T + (alpha/r) (X A^T) B^T``
  and its hand-derived backward, plus the SwiGLU glue used by the MLP workload.

Rules this package keeps:

* It shares no code with the CUDA path (``nf4_base_lora_blockwise_b200``) and neither side
  imports the other.  Only the seeded input generator module ``nf4_base_lora_blockwise_b200.synth``
  (which holds none of the method's arithmetic) feeds both.
* Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference
  legs may import it.  The product path never routes through it.

Citations name the web page and the section they follow:

* "Unsloth vs QLoRA vs Liger-Kernel" (mojostudio.in), section 1 "The Bottlenecks in Standard
  PyTorch Fine-Tuning" -- the LoRA forward formula; FAQ "What is the difference between LoRA
  and QLoRA?" -- base weights quantised to 4-bit NormalFloat (NF4); FAQ "Does Unsloth cause
  accuracy degradation?" -- gradients equal plain FP32 autograd up to rounding.
* "Speed up fine-tuning 2x" (adhdecode), section "4-bit quantisation" -- frozen 4-bit base.
* "FTDD-03" teaching script, decision 1/2 -- hand-derived backward of the linear layer.

Where the pages are silent (codebook values, block size, nibble order, double-quant format,
backward formulas) the readings are stated in each function's docstring.
"""
