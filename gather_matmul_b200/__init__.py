"""B200 (sm_100a) multi-LoRA shrink / expand: BGMV (per-token adapters, for
decode) and SGMV (segment-grouped, for prefill) behind the C ABI of
include/lora.h (liblora_b200.so), with a thin torch binding in ops.py.

Importing the package does not load the CUDA library; the first call in
ops.py does, and raises if it has not been built.
"""
__all__ = ["ops", "workloads", "build"]
