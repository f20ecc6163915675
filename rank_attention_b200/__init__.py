"""Flash-LoRA-Attention for B200 (sm_100a).

Submodules:
  lora_attn   -- ctypes binding of liblora_attn.so (the C ABI in include/lora_attn.h)
  workloads   -- seeded synthetic inputs shaped like the pages' workloads
  build_lib   -- nvcc build of the library
Importing ``rank_attention_b200.lora_attn`` raises if the library is not built.
"""
