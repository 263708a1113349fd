"""B200 (sm_100a) library for the single-GPU core of MoE token dispatch and
combine: dispatch layout (counts, scan, stable source-row map), permute into
a packed expert-major buffer (bf16, fused block FP8, fused NVFP4, the MX FP4
token format), the gate-weighted combine, the fused SwiGLU + requantisation
of the experts' gate/up rows, and the backward of dispatch and combine.

The compute lives in ``libmoedc.so`` (hand-written CUDA behind a C ABI,
declared in ``include/moe_dc.h``); :mod:`.binding` is a thin ctypes layer with
the same entry-point names.  Importing this package does not load the
library; the first call does, and it raises if the library is missing.
:mod:`.ep` moves the dispatch rows between the ranks of an expert-parallel
group (torch.distributed all-to-alls).
"""

__all__ = ["binding", "ep", "inputs"]
