"""ForkAttention hot path (tree-forked decision inference) for one B200.

The CUDA library ``libflide.so`` (sources in ``csrc/``, C ABI in
``include/flide.h``) does all the work; ``flide`` is a ctypes binding that only
marshals arguments, ``history`` and ``schedule`` drive the library's calls for
multi-step histories and memory-bounded GDN scans, and ``inputs`` draws the
seeded synthetic workloads.

One decision step (a request = a shared prefix and its option branches in one
flattened token stream; parent ids are request-local, -1 for the root):

    import math, torch
    from tree_forked_decision_b200 import flide

    rp, parent, seg, past = [0, 3], [-1, 0, 0], [2048, 32, 32], [0]   # root + 2 options
    dt = flide.DeviceTree(rp, parent, seg, past, max_depth=1)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
    flide.tree_build(dt, idx)                         # tree -> GPU indices

    T = sum(seg)                                      # q [T,Hq,128], k/v [T,Hkv,128] bf16
    q = torch.randn(T, 16, 128, device="cuda", dtype=torch.bfloat16)
    k = torch.randn(T, 4, 128, device="cuda", dtype=torch.bfloat16)
    v = torch.randn_like(k)
    o = flide.fork_attn(q, k, v, idx, 1 / math.sqrt(128))   # every branch as if isolated

    # Gated DeltaNet layer: q, k, v [T,H,128] bf16, g = log(alpha), beta [T,H] fp32;
    # node_state holds the roots' and inner nodes' end states
    node_state = torch.empty(flide.state_slots(dt), 16, 128, 128, device="cuda")
    go = flide.fork_gdn(gq, gk, gv, g, beta, idx, node_state)

    flide.state_save(...)   # the prefix becomes checkpointed history for the next step
    torch.cuda.synchronize(); assert idx.status() == 0   # device-detected errors

Further calls: ``fork_attn_fp8`` and
``fork_gdn_fp8`` with ``amax`` / ``quantize_e4m3`` (e4m3 inputs), ``fork_attn_paged`` and
``history.HistoryStore`` (growing histories in a block pool),
``branch_logprob`` / ``option_probs`` (decision probabilities over the
options), ``schedule.BoundedGdn`` (GDN under a node-state memory budget) and
``graphs.GraphBuckets`` (captured CUDA graphs per shape bucket).
"""
from .flide import (DeviceTree, FlideError, TreeIndex, amax, branch_logprob,  # noqa: F401
                    fork_attn, fork_attn_fp8, fork_attn_paged, fork_gdn, fork_gdn_fp8, load,
                    option_probs,
                    quantize_e4m3, state_resume, state_save, state_slots, tree_build)
