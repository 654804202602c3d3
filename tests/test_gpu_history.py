"""A multi-step agent episode through the block-paged history store: at every
decision step each request resumes from its history in the pool, adds a new
observation (its root) and scores new options; afterwards the observation and
the root's end state are appended.  Every step's outputs (attention and GDN,
observation and option rows) must equal the oracle run from scratch over the
whole history (resume equals scratch, step after step).  One request ends its
episode after step 1 and starts a new one in the same slot.  With blocks of
128 rows the attention also runs with the past read in place from the blocks
(flide_fork_attn_paged) and must equal the gathered-past result bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
from tree_forked_decision_b200 import flide, inputs
from tree_forked_decision_b200.history import HistoryStore

from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

Hq, Hkv, d, H, dk, dv = 8, 2, 128, 2, 128, 128


def _chunk(rng, L):
    """Attention and GDN inputs for L consecutive tokens."""
    t = inputs.fanout_tree(1, L, 0, 0)
    a = inputs.attn_inputs(t, Hq, Hkv, d, torch.bfloat16, rng)
    g = inputs.gdn_inputs(t, H, dk, dv, torch.bfloat16, rng, gate_scale=0.1)
    return {"q": a["q"], "k": a["k"], "v": a["v"], "gq": g["q"], "gk": g["k"], "gv": g["v"],
            "gg": g["g"], "gb": g["beta"]}


def _cat(chunks):
    return {key: torch.cat([c[key] for c in chunks]) for key in chunks[0]}


@pytest.mark.parametrize("block_rows", [16, 128])
def test_agent_episode_through_paged_history(block_rows):
    rng = np.random.default_rng(21)
    R, steps = 3, 3
    n_blocks = 64 if block_rows == 16 else 12
    store = HistoryStore(n_blocks=n_blocks, block_rows=block_rows, max_requests=4,
                         max_blocks=16 if block_rows == 16 else 4, Hkv=Hkv, d=d, H=H, dk=dk, dv=dv)
    slots = [0, 1, 2]
    history = [[] for _ in range(R)]  # observation chunks of the current episode
    for step in range(steps):
        fresh = [step == 0 or (r == 2 and step == 1) for r in range(R)]
        if step == 1:
            store.release(2)  # request 2's episode ends; its slot starts over
            history[2] = []
        obs = [_chunk(rng, int(rng.integers(20, 80))) for _ in range(R)]
        opts = [[_chunk(rng, int(rng.integers(3, 10))) for _ in range(int(rng.integers(2, 6)))]
                for _ in range(R)]
        # the GPU step: past = history in the pool, root = new observation
        past_len, pk, pv, state_in = store.resume([-1 if f else s for f, s in zip(fresh, slots)])
        hist_len = [sum(c["k"].shape[0] for c in history[r]) for r in range(R)]
        tree = inputs._tree([(hist_len[r], [(-1, obs[r]["k"].shape[0])]
                              + [(0, o["k"].shape[0]) for o in opts[r]]) for r in range(R)], 1)
        data = _cat([c for r in range(R) for c in [obs[r]] + opts[r]])
        dt = flide.DeviceTree(tree.req_node_ptr, tree.parent, tree.seg_len, tree.past_len, max_depth=1)
        dt.past_len = past_len  # the lengths the store wrote on the device
        idx = flide.TreeIndex(dt.R, dt.N, dt.T, 1)
        flide.tree_build(dt, idx)
        dev = {k_: v_.cuda() for k_, v_ in data.items()}
        has_past = sum(hist_len) > 0
        o = flide.fork_attn(dev["q"], dev["k"], dev["v"], idx, 1 / math.sqrt(d),
                            past_k=pk if has_past else None, past_v=pv if has_past else None)
        if block_rows % 128 == 0:
            # same lengths without the packed copy, past rows read in place
            plen2, state2 = store.resume_lengths([-1 if f else s for f, s in zip(fresh, slots)])
            o_paged = store.fork_attn_paged(dev["q"], dev["k"], dev["v"], idx, 1 / math.sqrt(d),
                                            [-1 if f else s for f, s in zip(fresh, slots)])
            torch.cuda.synchronize()
            assert torch.equal(plen2, past_len) and torch.equal(state2, state_in)
            assert torch.equal(o_paged, o)
        node_state = torch.zeros((max(flide.state_slots(tree), 1), H, dv, dk), device="cuda")
        go = flide.fork_gdn(dev["gq"], dev["gk"], dev["gv"], dev["gg"], dev["gb"], idx, node_state,
                            state_in=state_in if has_past else None)
        store.commit(slots, tree, idx, dev["k"], dev["v"], node_state)
        torch.cuda.synchronize()
        assert idx.status() == 0 and int(store.status.item()) == 0
        assert past_len.cpu().tolist() == hist_len
        for r in range(R):
            history[r].append(obs[r])
            assert store.length(slots[r]) == sum(c["k"].shape[0] for c in history[r])
        # the oracle from scratch: root = the whole episode's observations
        scratch = inputs._tree([(0, [(-1, sum(c["k"].shape[0] for c in history[r]))]
                                 + [(0, o_["k"].shape[0]) for o_ in opts[r]]) for r in range(R)], 1)
        sdata = _cat([c for r in range(R) for c in history[r] + opts[r]])
        # rows of this step's stream inside the scratch stream
        rows, s0 = [], 0
        for r in range(R):
            old = sum(c["k"].shape[0] for c in history[r][:-1])
            new = history[r][-1]["k"].shape[0] + sum(o_["k"].shape[0] for o_ in opts[r])
            rows += list(range(s0 + old, s0 + old + new))
            s0 += old + new
        rows = np.asarray(rows)
        f = lambda t: t.float().numpy()
        want_a = oracle.attention_all(scratch.arrays(), f(sdata["q"]), f(sdata["k"]), f(sdata["v"]),
                                      np.zeros((0, Hkv, d)), np.zeros((0, Hkv, d)), 1 / math.sqrt(d))
        want_g = oracle.gdn(scratch.arrays(), f(sdata["gq"]), f(sdata["gk"]), f(sdata["gv"]),
                            f(sdata["gg"]), f(sdata["gb"]))
        assert_close(o.float().cpu().numpy(), want_a[rows], torch.bfloat16)
        assert_close(go.float().cpu().numpy(), want_g[rows], torch.bfloat16)
    assert store.free_blocks() == n_blocks - sum(-(-store.length(s) // block_rows) for s in slots)
