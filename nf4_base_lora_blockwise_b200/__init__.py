"""QLoRA linear layer over a frozen NF4 (4-bit NormalFloat) base weight, for sm_100a (B200).

The compute lives in ``libqlora_nf4.so`` (C ABI, declared in ``include/qlora_nf4.h``);
``nf4_base_lora_blockwise_b200.abi`` is the thin ctypes binding over it and
``nf4_base_lora_blockwise_b200.linear`` the tensor-level API.  Importing the package does not
load the shared library; the first compute call does, and fails loudly if it is missing.
"""

__all__ = ["abi", "linear", "synth"]
