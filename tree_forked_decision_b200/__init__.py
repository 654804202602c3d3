"""ForkAttention hot path (tree-forked decision inference) for one B200.

The CUDA library ``libflide.so`` (sources in ``csrc/``, C ABI in
``include/flide.h``) does all the work; ``flide`` is a ctypes binding that only
marshals arguments, and ``inputs`` draws the seeded synthetic workloads.
"""
from .flide import (DeviceTree, FlideError, TreeIndex, fork_attn, fork_gdn, load,  # noqa: F401
                    state_resume, state_save, tree_build)
