"""libgnf4: grouped 4-bit (NF4 / MXFP4) MoE expert GEMM for one B200.

The compute lives in the C-ABI shared library ``libgnf4.so`` (CUDA, sm_100a).
``bit_grouped_moe_b200.gnf4`` is the thin ctypes binding; import it to use the
library.  ``bit_grouped_moe_b200.inputs`` draws seeded synthetic inputs.
"""
