"""OCTOPUS KV-cache codec for NVIDIA B200 (sm_100a): encode and fused decode attention.

The compute path is the C ABI in ``include/octopus.h`` (library
``liboctopus_b200.so``, built by ``build.py``); :mod:`.api` is a thin
PyTorch binding of it. :mod:`.inputs` draws the seeded synthetic workloads.
"""

from .api import (ROUND_JOINT, ROUND_SCALAR, Cache, DeviceTables, Layout, Workspace, codebook_build,  # noqa: F401
                  decode_attn, decode_attn_workspace_bytes, encode, qjl_build, rotation_build)
