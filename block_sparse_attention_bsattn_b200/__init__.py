"""bsattn: block-sparse attention forward (static block masks and the BLASST
softmax-threshold skip) for NVIDIA B200 (sm_100a).

The computation runs in the CUDA library ``libbsattn.so`` behind the C ABI of
``include/bsattn.h``; :mod:`.ops` is a thin ctypes binding with the same entry
point names (argument marshalling only).  ``import
block_sparse_attention_bsattn_b200.ops`` loads the library.
"""
