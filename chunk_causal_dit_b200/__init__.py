"""B200-native (sm_100a) wave-round chunk-causal attention for Wave Forcing.

The product is ``libwf.so`` (CUDA kernels behind a C ABI, see ``include/wf.h``);
``chunk_causal_dit_b200.wf`` is a thin ctypes binding with the same names.
Submodules are imported explicitly (``from chunk_causal_dit_b200 import wf``)
so that the seeded input generators (``chunk_causal_dit_b200.inputs``) import
on machines where the library has not been built.
"""
