"""B200-native fused tiled attention (prefill + paged-KV decode).

The compute lives in libtiledattn.so (hand-written sm_100a CUDA, C ABI in
include/tiledattn.h).  `tiled_attention_17_b200.binding` marshals arguments to
it; `inputs` builds the seeded synthetic workloads; `accounting` turns shapes
into FLOP/byte counts.  Importing the package does not load the CUDA library;
the first call through `binding` does, and raises if it is missing.
"""
from . import accounting, inputs  # noqa: F401
