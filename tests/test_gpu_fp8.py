"""GPU parity of the e4m3 path through the C ABI.

Quantisation (flide_amax, flide_quantize_e4m3): codes, amax and descale
bit-exact against the oracle's float32 scaling steps.

Fork attention over e4m3 inputs (flide_fork_attn_fp8): against the fp64
oracle over the decoded inputs.  Q K^T of e4m3 values is exact in fp32, so the
one rounding the kernel adds is that of the softmax weights to e4m3 before
they multiply v: a weight p (its row's largest is 1..4, stored times 2^6)
moves by at most 2^-4 p in the normal range and 2^-16 below it; one weight in
eight comes from a cubic with relative error < 2^-13 instead of the hardware
exp2; the row sum l (>= 1) uses the unrounded weights.  Per output element
this bounds the error by
    (2^-4 + 2^-13) sv sum_j w_j |V_j| + 2^-16 n sv mean_j |V_j| + 2^-8 |o| + 1e-5
(w the exact softmax weights, n the number of visible keys, V the decoded v
codes; 2^-8 |o| covers the bf16 output and fp32 arithmetic).  Both sums come
from the oracle: attention of |v| with the real and with all-zero queries.
The rounding's relative rms error is about 0.026 for a uniform mantissa, so
with random v the outputs' relative L2 error sits near that; the test asks
for <= 0.04."""
import ctypes
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as ofp8
from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, build

pytestmark = pytest.mark.gpu

FP8_REL_L2 = 0.04


# ---------------------------------------------------------------------------
# quantisation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 7, 8, 1003, 4099, (1 << 20) + 5])
def test_quantize_bit_exact(dtype, n):
    rng = np.random.default_rng(n)
    x = torch.from_numpy(inputs.normals(rng, (n,)) * np.float32(3.0)).to(dtype)
    xd = x.cuda()
    am = flide.amax(xd)
    codes, ds = flide.quantize_e4m3(xd, am)
    torch.cuda.synchronize()
    xf = x.float().numpy()
    want, wds = ofp8.quantize_e4m3(xf)
    assert am.item() == np.abs(xf).max()
    assert np.float32(ds.item()) == wds
    assert np.array_equal(codes.cpu().numpy(), want)


def test_quantize_shared_amax_and_saturation():
    rng = np.random.default_rng(4)
    a = torch.from_numpy(inputs.normals(rng, (5000,)))
    b = torch.from_numpy(inputs.normals(rng, (777,)) * np.float32(4.0))
    am = flide.amax(a.cuda())
    flide.amax(b.cuda(), out=am, accumulate=True)
    ca, _ = flide.quantize_e4m3(a.cuda(), am)
    cb, ds = flide.quantize_e4m3(b.cuda(), am)
    shared = max(np.abs(a.numpy()).max(), np.abs(b.numpy()).max())
    assert am.item() == shared
    assert np.array_equal(ca.cpu().numpy(), ofp8.quantize_e4m3(a.numpy(), shared)[0])
    assert np.array_equal(cb.cpu().numpy(), ofp8.quantize_e4m3(b.numpy(), shared)[0])
    # an amax below the data's saturates to +-448
    small = torch.tensor([0.5], device="cuda")
    cs, _ = flide.quantize_e4m3(b.cuda(), small)
    want, _ = ofp8.quantize_e4m3(b.numpy(), 0.5)
    assert np.array_equal(cs.cpu().numpy(), want)
    assert (want[np.abs(b.numpy()) > 0.5] & 0x7F == 0x7E).all()


def test_quantize_zero_tensor():
    z = torch.zeros(100, device="cuda")
    codes, ds = flide.quantize_e4m3(z)
    torch.cuda.synchronize()
    assert (codes.cpu().numpy() == 0).all() and ds.item() == 1.0


# ---------------------------------------------------------------------------
# fork attention over e4m3 inputs
# ---------------------------------------------------------------------------

FP8_CASES = {
    # name: (tree builder, Hq, Hkv)
    "fanout_g4_ragged": (lambda rng: inputs.fanout_tree(2, 300, 6, 13), 8, 2),
    "fanout_g4_past": (lambda rng: inputs.fanout_tree(2, 170, 5, 29, past=77), 8, 2),
    "fanout_g1": (lambda rng: inputs.fanout_tree(1, 260, 3, 50), 2, 2),
    "fanout_g8": (lambda rng: inputs.fanout_tree(2, 140, 9, 5), 16, 2),
    "leveled_depth3_resume": (lambda rng: inputs.leveled_tree(rng, 3, depth_range=(2, 3),
                                                              options_range=(5, 40),
                                                              prefix_range=(100, 400),
                                                              n_resume=2), 8, 2),
    "random_irregular": (lambda rng: inputs.random_tree(rng, R=4, max_nodes=12,
                                                        prefix_range=(0, 200),
                                                        branch_range=(1, 70),
                                                        past_range=(0, 90)), 4, 1),
    "depth8_chain": (lambda rng: inputs._tree([(3, [(-1, 17)] + [(i, 5 + i) for i in range(8)])],
                                              8), 8, 2),
    "zero_token_root_with_past": (lambda rng: inputs._tree([(50, [(-1, 0), (0, 5), (0, 7)]),
                                                            (0, [(-1, 20), (0, 3)])], 1), 8, 2),
    "long_prefix_2k": (lambda rng: inputs.fanout_tree(1, 2048, 16, 32), 16, 4),
}


def _run_fp8(tree, a, idx):
    dev = {k: v.cuda() for k, v in a.items()}
    has_past = a["past_k"].shape[0] > 0
    scale = 1.0 / math.sqrt(a["q"].shape[2])
    out = flide.fork_attn_fp8(dev["q"], dev["k"], dev["v"], idx, scale, dev["descale"],
                              past_k=dev["past_k"] if has_past else None,
                              past_v=dev["past_v"] if has_past else None)
    torch.cuda.synchronize()
    assert idx.status() == 0, idx.status()
    return out.float().cpu().numpy(), scale


def _oracle_and_bound(tree, a, scale, rows=None):
    n = lambda t: t.numpy()
    ds = a["descale"].numpy()
    args = (n(a["q"]), n(a["k"]), n(a["v"]), n(a["past_k"]), n(a["past_v"]))
    want = ofp8.attention_fp8(tree.arrays(), *args, ds, scale, rows)
    absv, abspv = n(a["v"]) & 0x7F, n(a["past_v"]) & 0x7F  # |V| by clearing the sign bit
    wabs = ofp8.attention_fp8(tree.arrays(), args[0], args[1], absv, args[3], abspv, ds, scale,
                              rows)
    zq = np.zeros_like(args[0])
    mabs = ofp8.attention_fp8(tree.arrays(), zq, args[1], absv, args[3], abspv, ds, scale, rows)
    pos = oracle.tree_index(*tree.arrays())["token_pos"]
    nvis = (pos + 1).astype(np.float64)
    nvis = nvis[rows[:, 0]][:, None] if rows is not None else nvis[:, None, None]
    tol = (2.0 ** -4 + 2.0 ** -13) * wabs + 2.0 ** -16 * nvis * mabs + 2.0 ** -8 * np.abs(want) + 1e-5
    return want, tol


def _assert_within(got, want, tol):
    assert np.all(np.isfinite(got))
    err = np.abs(got - want)
    bad = err > tol
    assert not bad.any(), (int(bad.sum()), float(err.max()), float((err / tol).max()))
    rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    assert rel <= FP8_REL_L2, rel
    return float(err.max()), rel


@pytest.mark.parametrize("case", sorted(FP8_CASES))
def test_fork_attn_fp8_vs_oracle(case):
    rng = np.random.default_rng(zlib.crc32(case.encode()) % 1000)
    build_tree, Hq, Hkv = FP8_CASES[case]
    tree = build_tree(rng)
    a = inputs.fp8_attn_inputs(tree, Hq, Hkv, 128, rng)
    _, idx = build(tree)
    got, scale = _run_fp8(tree, a, idx)
    want, tol = _oracle_and_bound(tree, a, scale)
    _assert_within(got, want, tol)


def test_fork_attn_fp8_one_hot_rows_exact():
    """A key far above the others gets weight 2^6 (exact) and the rest
    underflow to zero, so each output row is exactly sv V of that key."""
    tree = inputs.fanout_tree(1, 40, 2, 4)
    rng = np.random.default_rng(0)
    a = inputs.fp8_attn_inputs(tree, 4, 1, 128, rng)
    q = np.zeros((tree.T, 4, 128), np.uint8)
    q[:, :, 0] = 0x7E                       # 448 in dim 0 for every query
    k = np.zeros((tree.T, 1, 128), np.uint8)
    k[0, 0, 0] = 0x7E                       # only key 0 has a score
    a["q"], a["k"] = torch.from_numpy(q), torch.from_numpy(k)
    a["descale"] = torch.tensor([1.0, 1.0, 1.0 / 64])
    _, idx = build(tree)
    got, _ = _run_fp8(tree, a, idx)
    # every token sees key 0 (the root's first token) with logit 448^2/sqrt(128)
    v0 = ofp8.decode_e4m3(a["v"].numpy()[0, 0]) / 64
    want = np.broadcast_to(v0, got.shape).copy()
    want[0] = v0                            # token 0 sees only itself
    bf = torch.from_numpy(want).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got, bf)


def test_fork_attn_fp8_rejects_unsupported():
    tree = inputs.fanout_tree(1, 10, 2, 3)
    a = inputs.fp8_attn_inputs(tree, 4, 2, 64, np.random.default_rng(1))
    _, idx = build(tree)
    with pytest.raises(flide.FlideError):
        flide.fork_attn_fp8(a["q"].cuda(), a["k"].cuda(), a["v"].cuda(), idx, 0.125,
                            a["descale"].cuda())
    # the bf16/fp32 entry point refuses e4m3 (it has no descale factors)
    a = inputs.fp8_attn_inputs(tree, 4, 2, 128, np.random.default_rng(1))
    q, k, v = a["q"].cuda(), a["k"].cuda(), a["v"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    lib = flide.load()
    assert lib.flide_fork_attn(flide._ptr(q), flide._ptr(k), flide._ptr(v), None, None, 0,
                               ctypes.byref(idx.c), 4, 2, 128, flide.E4M3, 1.0, flide._ptr(out),
                               0, flide._stream()) == flide.ERR_SHAPE


@pytest.mark.parametrize("name", ["attn_fanout_bf16", "mixed_hybrid_bf16", "large_fanout_bf16"])
def test_fullsize_fork_attn_fp8_sampled(name):
    """The benched workloads' trees and head counts with e4m3 inputs, checked
    on the full-size test's row sample (first and last root rows, every
    branch row of query head 0, random rows) under the same bound."""
    from test_gpu_fullsize import _rows
    tree, spec, _, _, rng = inputs.workload(name)
    a = inputs.fp8_attn_inputs(tree, spec["Hq"], spec["Hkv"], spec["d"], rng)
    _, idx = build(tree)
    got, scale = _run_fp8(tree, a, idx)
    rows = _rows(tree, spec["Hq"], spec["Hkv"], 1500, np.random.default_rng(1))
    want, tol = _oracle_and_bound(tree, a, scale, rows)
    _assert_within(got[rows[:, 0], rows[:, 1]], want, tol)


# ---------------------------------------------------------------------------
# Gated DeltaNet fork scan over e4m3 inputs
# ---------------------------------------------------------------------------

GDN8_CASES = {
    "leveled_resume": lambda rng: inputs.leveled_tree(rng, 3, depth_range=(1, 3), options_range=(3, 30),
                                                      prefix_range=(60, 300), branch_range=(2, 40),
                                                      n_resume=2),
    "fanout_long_prefix": lambda rng: inputs.fanout_tree(2, 700, 9, 13, past=5),
    "deep_chain": lambda rng: inputs._tree([(3, [(-1, 17)] + [(i, 5 + i) for i in range(8)])], 8),
    "zero_token_root_with_past": lambda rng: inputs._tree([(50, [(-1, 0), (0, 5), (0, 70)]),
                                                           (0, [(-1, 20), (0, 3)])], 1),
}


def _run_gdn8(tree, g8, H):
    _, idx = build(tree)
    dev = {k_: v_.cuda() for k_, v_ in g8.items() if isinstance(v_, torch.Tensor)}
    has_state = bool(np.any(tree.past_len > 0))
    node_state = torch.zeros((max(flide.state_slots(tree), 1), H, 128, 128), device="cuda")
    out = flide.fork_gdn_fp8(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], idx, node_state,
                             dev["descale"], state_in=dev["state_in"] if has_state else None)
    torch.cuda.synchronize()
    assert idx.status() == 0, idx.status()
    return out, node_state, idx, dev, has_state


@pytest.mark.parametrize("case", sorted(GDN8_CASES))
def test_fork_gdn_fp8_vs_oracle_and_bf16(case):
    """Against the oracle over the decoded inputs (bf16 bar), and bit for bit
    against flide_fork_gdn on bf16 inputs holding the same values: e4m3 codes
    convert exactly, and with power-of-two descale factors folding them into
    the scan's products changes no rounding."""
    rng = np.random.default_rng(zlib.crc32(case.encode()) % 1000)
    tree = GDN8_CASES[case](rng)
    H = 2
    g8 = inputs.fp8_gdn_inputs(tree, H, 128, 128, rng, gate_scale=0.1)
    out, node_state, idx, dev, has_state = _run_gdn8(tree, g8, H)
    n = lambda t: t.numpy()
    want = ofp8.gdn_fp8(tree.arrays(), n(g8["q"]), n(g8["k"]), n(g8["v"]), n(g8["g"]), n(g8["beta"]),
                        n(g8["descale"]), state_in=n(g8["state_in"]) if has_state else None)
    assert_close(out.float().cpu().numpy(), want, torch.bfloat16)
    # the bf16 kernel on the decoded values (exact in bf16)
    ds = g8["descale"].tolist()
    deq = lambda c, s: (torch.from_numpy(ofp8.decode_e4m3(n(c)) * s).to(torch.bfloat16)).cuda()
    ns2 = torch.zeros_like(node_state)
    ref = flide.fork_gdn(deq(g8["q"], ds[0]), deq(g8["k"], ds[1]), deq(g8["v"], ds[2]), dev["g"],
                         dev["beta"], idx, ns2, state_in=dev["state_in"] if has_state else None)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(node_state, ns2)


@pytest.mark.parametrize("name,n_pairs", [("gdn_fanout_bf16", 6), ("large_fanout_bf16", 4)])
def test_fullsize_fork_gdn_fp8_sampled(name, n_pairs):
    """The GDN workloads' trees and head counts with e4m3 inputs; every token of
    sampled (request, head) pairs against the oracle."""
    tree, _, spec, _, rng = inputs.workload(name)
    H = spec["H"]
    g8 = inputs.fp8_gdn_inputs(tree, H, 128, 128, rng, gate_scale=spec["gate_scale"])
    out, _, _, _, has_state = _run_gdn8(tree, g8, H)
    got = out.float().cpu().numpy()
    prng = np.random.default_rng(2)
    sel = prng.choice(tree.R * H, size=n_pairs, replace=False)
    heads = sorted({int(i % H) for i in sel})
    pairs = [(int(i // H), heads.index(int(i % H))) for i in sel]
    hs = lambda t: np.ascontiguousarray(t.numpy()[:, heads])
    want = ofp8.gdn_fp8(tree.arrays(), hs(g8["q"]), hs(g8["k"]), hs(g8["v"]), hs(g8["g"]),
                        hs(g8["beta"]), g8["descale"].numpy(),
                        state_in=hs(g8["state_in"]) if has_state else None, pairs=pairs)
    starts = np.concatenate([[0], np.cumsum(tree.seg_len)])
    rp = tree.req_node_ptr
    for (r, hi) in pairs:
        toks = np.arange(starts[rp[r]], starts[rp[r + 1]])
        assert_close(got[toks, heads[hi]], want[toks, hi], torch.bfloat16)
