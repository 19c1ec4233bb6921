"""InfLLM-V2 dense-sparse switchable attention for one causal GQA layer, on B200.

The compute path is the C-ABI library libinfv2.so (hand-written sm_100a CUDA);
`trainable_block_sparse_mean_b200.infv2` is its thin Python binding.  Importing
this package loads nothing; the binding loads the library on first use and
raises if it is missing.
"""
__all__ = ["infv2", "synth"]
