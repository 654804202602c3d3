"""Paged past rows (flide_fork_attn_paged): each request's past K/V scattered
into random blocks of a pool and read in place through the block table must
give, bit for bit, what the same kernel gives over the packed past rows (same
key tiles in the same order), for bf16 and e4m3 inputs and block sizes of one
and two key tiles; the bf16 case also against the oracle; a missing block or
a bad slot is reported in the status word."""
import math

import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, build, oracle_attn

pytestmark = pytest.mark.gpu

TREES = {
    "fanout_past300": lambda rng: inputs.fanout_tree(3, 150, 6, 13, past=300),
    "leveled_resume": lambda rng: inputs.leveled_tree(rng, 4, depth_range=(1, 3), options_range=(3, 20),
                                                      prefix_range=(100, 600), n_resume=3,
                                                      resume_delta=(4, 40)),
    "random_past": lambda rng: inputs.random_tree(rng, R=5, max_nodes=9, prefix_range=(0, 90),
                                                  branch_range=(1, 40), past_range=(0, 700)),
}


def _scatter(pasts, past_len, block_rows, rng, spare_blocks=3, spare_slots=2):
    """Pools (one per tensor in `pasts`, same layout), block table and request
    slots holding the packed rows (request r's past_len[r] rows in order) in
    random blocks."""
    R = len(past_len)
    need = [-(-int(n) // block_rows) for n in past_len]
    n_blocks = sum(need) + spare_blocks
    max_blocks = max(max(need), 1)
    n_slots = R + spare_slots
    slots = rng.permutation(n_slots)[:R].astype(np.int32)
    free = list(rng.permutation(n_blocks))
    table = np.full((n_slots, max_blocks), -1, np.int32)
    pools = [torch.zeros((n_blocks * block_rows,) + tuple(x.shape[1:]), dtype=x.dtype) for x in pasts]
    p0 = 0
    for r in range(R):
        for b in range(need[r]):
            blk = int(free.pop())
            table[slots[r], b] = blk
            n = min(block_rows, int(past_len[r]) - b * block_rows)
            for pool, x in zip(pools, pasts):
                pool[blk * block_rows: blk * block_rows + n] = x[p0 + b * block_rows: p0 + b * block_rows + n]
        p0 += int(past_len[r])
    return pools, torch.from_numpy(table.ravel()), torch.from_numpy(slots), max_blocks


def _run_both(tree, a, block_rows, rng, e4m3=False):
    _, idx = build(tree)
    scale = 1.0 / math.sqrt(128)
    dev = {k_: v_.cuda() for k_, v_ in a.items()}
    if e4m3:
        packed = flide.fork_attn_fp8(dev["q"], dev["k"], dev["v"], idx, scale, dev["descale"],
                                     past_k=dev["past_k"], past_v=dev["past_v"])
    else:
        packed = flide.fork_attn(dev["q"], dev["k"], dev["v"], idx, scale, past_k=dev["past_k"],
                                 past_v=dev["past_v"])
    (pk, pv), table, slots, mb = _scatter([a["past_k"], a["past_v"]], tree.past_len, block_rows, rng)
    paged = flide.fork_attn_paged(dev["q"], dev["k"], dev["v"], idx, scale, pk.cuda(), pv.cuda(),
                                  table.cuda(), slots.cuda(), block_rows, mb,
                                  descale=dev["descale"] if e4m3 else None)
    torch.cuda.synchronize()
    assert idx.status() == 0, idx.status()
    return packed, paged, scale


@pytest.mark.parametrize("block_rows", [128, 256])
@pytest.mark.parametrize("case", sorted(TREES))
def test_paged_equals_packed_bf16(case, block_rows):
    rng = np.random.default_rng(len(case) * 7 + block_rows)
    tree = TREES[case](rng)
    assert tree.P_past > 0
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    packed, paged, scale = _run_both(tree, a, block_rows, rng)
    assert torch.equal(packed, paged)
    if case == "fanout_past300":
        assert_close(paged.float().cpu().numpy(), oracle_attn(tree, a, scale), torch.bfloat16)


@pytest.mark.parametrize("block_rows", [128, 384])
def test_paged_equals_packed_e4m3(block_rows):
    rng = np.random.default_rng(block_rows)
    tree = TREES["random_past"](rng)
    a = inputs.fp8_attn_inputs(tree, 8, 2, 128, rng)
    packed, paged, _ = _run_both(tree, a, block_rows, rng, e4m3=True)
    assert torch.equal(packed, paged)


def test_paged_missing_block_and_bad_slot_are_reported():
    rng = np.random.default_rng(3)
    tree = inputs.fanout_tree(2, 40, 3, 5, past=200)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    (pk,), table, slots, mb = _scatter([a["past_k"]], tree.past_len, 128, rng)
    dev = {k_: v_.cuda() for k_, v_ in a.items()}
    scale = 1.0 / math.sqrt(128)
    # request 1's second block missing from its table
    bad = table.clone().view(-1, mb)
    bad[int(slots[1]), 1] = -1
    _, idx = build(tree)
    flide.fork_attn_paged(dev["q"], dev["k"], dev["v"], idx, scale, pk.cuda(), pk.cuda(),
                          bad.view(-1).cuda(), slots.cuda(), 128, mb)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_INVALID
    # a slot outside the table
    _, idx = build(tree)
    oob = slots.clone()
    oob[0] = table.numel() // mb
    flide.fork_attn_paged(dev["q"], dev["k"], dev["v"], idx, scale, pk.cuda(), pk.cuda(),
                          table.cuda(), oob.cuda(), 128, mb)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_INVALID
    # blocks that are not a multiple of the key tile are refused on the host
    with pytest.raises(flide.FlideError):
        flide.fork_attn_paged(dev["q"], dev["k"], dev["v"], idx, scale, pk.cuda(), pk.cuda(),
                              table.cuda(), slots.cuda(), 100, mb)
