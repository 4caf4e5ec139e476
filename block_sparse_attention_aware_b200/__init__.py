"""FVAttn block-sparse attention, single-GPU hot path, native to B200 (sm_100a).

The compute lives in `libfvattn.so` (CUDA kernels behind a C ABI declared in
include/fvattn.h).  `block_sparse_attention_aware_b200.fvattn` is the thin
ctypes binding; `synth` draws seeded synthetic inputs.  Importing the package
does not load the native library; the binding loads it on first use and
raises if it is missing.
"""
__all__ = ["fvattn", "synth"]
