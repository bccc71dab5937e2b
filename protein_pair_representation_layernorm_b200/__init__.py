"""B200 (sm_100a) triangle attention over protein pair representations.

The computation runs in the CUDA kernels of ``_lib/libtriattn.so`` behind the
C ABI declared in ``include/tri_attn.h``; ``binding`` is its thin Python
binding and ``workloads`` draws the seeded synthetic inputs.
"""
from . import binding, workloads  # noqa: F401
from .binding import TriangleAttention  # noqa: F401
