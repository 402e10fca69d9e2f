"""Block-sparse 3D-RoPE video self-attention for B200 (sm_100a).

The compute lives in ``liblcbsa.so`` (C-ABI, declared in ``include/lc_bsa.h``);
this package only marshals arguments to it.  Import the bindings from
``block_sparse_attention_rope_b200.api``; importing the package itself does not
load the shared library.
"""
__all__ = ["api", "synthetic"]
