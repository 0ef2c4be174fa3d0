"""B200 (sm_100a) greedy decode step of a Qwen3-style decoder.

The compute lives in libdec.so (C ABI in include/dec.h); `capi` binds it with
ctypes and `decoder` wraps it for PyTorch callers.  `synth` draws the seeded
synthetic inputs and `roofline` counts the algorithmic bytes of a step.
"""
