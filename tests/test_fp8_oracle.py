"""Pins of the e4m3 oracle (oracle/fp8.py) against things other than itself:
the format's defining values (OCP 8-bit floating point specification, e4m3),
PyTorch's own float8_e4m3fn conversion (a library routine) over every code and
over random in-range values, round-half-to-even ties, saturation, the
per-tensor scaling steps, and brute-force fp64 attention and token-by-token
delta rule on tiny trees."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.decode_e4m3(codes)
    assert np.array_equal(got, want, equal_nan=True)


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x39, 1.125), (0x40, 2.0), (0x7E, 448.0), (0xB8, -1.0), (0xFE, -448.0),
])
def test_decode_defining_values(code, value):
    assert fp8.decode_e4m3(np.array([code], np.uint8))[0] == value


def test_nan_codes():
    v = fp8.decode_e4m3(np.array([0x7F, 0xFF], np.uint8))
    assert np.isnan(v).all()
    assert fp8.encode_e4m3(np.array([np.nan]))[0] & 0x7F == 0x7F


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    assert np.array_equal(fp8.encode_e4m3(fp8.decode_e4m3(codes)), codes)


def test_encode_matches_torch_on_random_in_range_values():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 120.0)])
    x = x[np.abs(x) < 440].astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode_e4m3(x), want)


def test_ties_round_to_even_and_saturation():
    enc = lambda v: int(fp8.encode_e4m3(np.array([v]))[0])
    assert enc(1.0625) == 0x38      # halfway 1.0 / 1.125 -> even mantissa 0
    assert enc(1.1875) == 0x3A      # halfway 1.125 / 1.25 -> even mantissa 2
    assert enc(2.0 ** -10) == 0x00  # halfway 0 / 2^-9 -> 0
    assert enc(3 * 2.0 ** -10) == 0x02
    assert enc(15 * 2.0 ** -10) == 0x08  # halfway 7*2^-9 / 2^-6 -> 2^-6 (even)
    assert enc(1.96875) == 0x40     # halfway 1.875 / 2.0 -> carry into the exponent
    for v in (448.0, 460.0, 470.0, 1e9):
        assert enc(v) == 0x7E and enc(-v) == 0xFE
    assert enc(-0.0) == 0x80 and enc(-2.0 ** -12) == 0x80


def test_quantize_scaling_steps():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(4096).astype(np.float32)
    codes, ds = fp8.quantize_e4m3(x)
    amax = np.abs(x).max()
    assert ds == np.float32(amax / np.float32(448.0))
    i = int(np.argmax(np.abs(x)))
    assert codes[i] in (0x7E, 0xFE)                         # amax -> +-448
    # error bound of round-to-nearest: half a step of the code's binade
    y = x.astype(np.float64) * float(np.float32(448.0) / np.float32(amax))
    err = np.abs(fp8.decode_e4m3(codes) - y)
    assert (err <= np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)).all()
    # a shared amax larger than the tensor's own
    codes2, ds2 = fp8.quantize_e4m3(x, amax=2 * amax)
    assert ds2 == np.float32(np.float32(2 * amax) / np.float32(448.0))
    assert np.abs(fp8.decode_e4m3(codes2)).max() <= 224.0 + 16
    z, dz = fp8.quantize_e4m3(np.zeros(7, np.float32))
    assert (z == 0).all() and dz == 1.0


def _brute_attention(parent, seg, past, q, k, v, pk, pv, scale):
    """Each node's isolated sequence written out by walking parents (one
    request), then plain softmax attention per (token, head) in fp64."""
    starts = np.concatenate([[0], np.cumsum(seg)])
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros((T, Hq, d))
    for n in range(len(seg)):
        chain = []
        a = n
        while a >= 0:
            chain.append(a)
            a = parent[a]
        chain.reverse()
        for t in range(starts[n], starts[n + 1]):
            keys = [("p", i) for i in range(past)]
            for a in chain:
                hi = starts[a + 1] if a != n else t + 1
                keys += [("s", j) for j in range(starts[a], hi)]
            for h in range(Hq):
                kv = h // G
                kk = np.array([(pk if s == "p" else k)[j, kv] for s, j in keys])
                vv = np.array([(pv if s == "p" else v)[j, kv] for s, j in keys])
                s = kk @ q[t, h] * scale
                w = np.exp(s - s.max())
                out[t, h] = w @ vv / w.sum()
    return out


def test_attention_fp8_equals_brute_force_on_dequantized_inputs():
    rng = np.random.default_rng(9)
    parent, seg, past = [-1, 0, 0, 1], [5, 3, 2, 4], 3
    T, Hq, Hkv, d = sum(seg), 4, 2, 8
    raw = {n: rng.standard_normal(s).astype(np.float32) * m for n, s, m in [
        ("q", (T, Hq, d), 1.0), ("k", (T, Hkv, d), 2.0), ("v", (T, Hkv, d), 0.5),
        ("pk", (past, Hkv, d), 2.0), ("pv", (past, Hkv, d), 0.5)]}
    q8, sq = fp8.quantize_e4m3(raw["q"])
    ak = max(np.abs(raw["k"]).max(), np.abs(raw["pk"]).max())
    av = max(np.abs(raw["v"]).max(), np.abs(raw["pv"]).max())
    k8, sk = fp8.quantize_e4m3(raw["k"], ak)
    pk8, _ = fp8.quantize_e4m3(raw["pk"], ak)
    v8, sv = fp8.quantize_e4m3(raw["v"], av)
    pv8, _ = fp8.quantize_e4m3(raw["pv"], av)
    deq = lambda c, s: fp8.decode_e4m3(c) * float(s)
    scale = 1 / math.sqrt(d)
    want = _brute_attention(parent, seg, past, deq(q8, sq), deq(k8, sk), deq(v8, sv),
                            deq(pk8, sk), deq(pv8, sv), scale)
    tree = ([0, 4], parent, seg, [past])
    got = fp8.attention_fp8(tree, q8, k8, v8, pk8, pv8, (sq, sk, sv), scale)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)
    # the (token, head) form agrees with the full form
    rows = np.array([[0, 0], [T - 1, 3], [6, 1]])
    part = fp8.attention_fp8(tree, q8, k8, v8, pk8, pv8, (sq, sk, sv), scale, rows)
    np.testing.assert_allclose(part, got[rows[:, 0], rows[:, 1]], rtol=0, atol=0)


def _brute_gdn(parent, seg, q, k, v, g, beta, s0):
    """Token-by-token delta rule along each node's isolated path (one request,
    fp64): S <- alpha (S - beta (S k) k^T) + beta v k^T, o = S q."""
    starts = np.concatenate([[0], np.cumsum(seg)])
    T, H, dk = q.shape
    out = np.zeros((T, H, v.shape[2]))
    for n in range(len(seg)):
        chain = []
        a = n
        while a >= 0:
            chain.append(a)
            a = parent[a]
        toks = [t for a in reversed(chain) for t in range(starts[a], starts[a + 1])]
        for h in range(H):
            S = s0[h].copy()
            for t in toks:
                al = np.exp(g[t, h])
                u = S @ k[t, h]
                S = al * (S - beta[t, h] * np.outer(u, k[t, h])) + beta[t, h] * np.outer(v[t, h], k[t, h])
                if starts[n] <= t < starts[n + 1]:
                    out[t, h] = S @ q[t, h]
    return out


def test_gdn_fp8_equals_brute_force_on_dequantized_inputs():
    rng = np.random.default_rng(13)
    parent, seg = [-1, 0, 0, 1], [6, 3, 4, 2]
    T, H, dk = sum(seg), 2, 8
    tree = ([0, 4], parent, seg, [1])
    codes = lambda x, amp: torch.from_numpy((x * amp).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q8 = codes(unit(rng.standard_normal((T, H, dk))), 256.0)
    k8 = codes(unit(rng.standard_normal((T, H, dk))), 256.0)
    v8 = codes(rng.standard_normal((T, H, dk)), 64.0)
    g = -np.logaddexp(0.0, rng.standard_normal((T, H))).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((T, H))))).astype(np.float32)
    s0 = (rng.standard_normal((1, H, dk, dk)) * 0.1).astype(np.float32)
    ds = (1 / 256, 1 / 256, 1 / 64)
    dec = lambda c, s: fp8.decode_e4m3(c) * s
    want = _brute_gdn(parent, seg, dec(q8, ds[0]), dec(k8, ds[1]), dec(v8, ds[2]),
                      g.astype(np.float64), beta.astype(np.float64), s0[0].astype(np.float64))
    got = fp8.gdn_fp8(tree, q8, k8, v8, g, beta, ds, state_in=s0)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)


def test_fp8_input_generators_emit_no_nan_codes():
    """The seeded e4m3 generators clamp before casting, so no code is NaN even
    for values beyond the format's range; shapes follow the tree."""
    from tree_forked_decision_b200 import inputs
    tree = inputs.fanout_tree(2, 40, 3, 5, past=7)
    a = inputs.fp8_attn_inputs(tree, 4, 2, 16, np.random.default_rng(0), amp=400.0)
    g = inputs.fp8_gdn_inputs(tree, 2, 16, 16, np.random.default_rng(1), amp_v=400.0)
    for t in (a["q"], a["k"], a["v"], a["past_k"], a["past_v"], g["q"], g["k"], g["v"]):
        c = t.numpy()
        assert c.dtype == np.uint8 and not np.any((c & 0x7F) == 0x7F)
    assert a["q"].shape == (tree.T, 4, 16) and a["past_k"].shape == (tree.P_past, 2, 16)
    assert np.isclose(a["descale"].numpy(), 1 / 400.0).all()


def test_every_midpoint_rounds_like_torch():
    """Each halfway point between neighbouring finite magnitudes (and the
    points just either side of it) encodes as torch's float8_e4m3fn
    conversion does: ties go to the even mantissa."""
    mags = np.unique(np.abs(fp8.decode_e4m3(np.arange(0x7F, dtype=np.uint8))))
    mid = (mags[:-1] + mags[1:]) / 2
    pts = np.concatenate([mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)])
    pts = np.concatenate([pts, -pts]).astype(np.float32)
    pts = pts[np.abs(pts) < 448]
    want = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode_e4m3(pts), want)


def test_dequantised_values_round_trip_within_half_a_step():
    """decode(code) * descale returns x to within half a code step of the
    scaled value (relative 2^-4 for normals, 2^-10 absolute below), and a
    value past the tensor's amax saturates to +-448 times descale."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(3000) * 3.0).astype(np.float32)
    codes, ds = fp8.quantize_e4m3(x)
    back = fp8.decode_e4m3(codes) * float(ds)
    scale = float(ds)
    tol = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale) * (1 + 1e-6)
    assert (np.abs(back - x) <= tol).all()
    codes2, ds2 = fp8.quantize_e4m3(x * 4, amax=np.abs(x).max())
    over = np.abs(x * 4) > np.abs(x).max() * (1 + 2.0 ** -3)
    assert over.any() and np.allclose(np.abs(fp8.decode_e4m3(codes2[over])), 448.0)


def test_encode_saturates_and_never_makes_nan():
    big = np.array([448.0, 449.0, 464.0, 480.0, 1000.0, 3.0e38, np.inf], np.float64)
    for v in (big, -big):
        c = fp8.encode_e4m3(v)
        assert ((c & 0x7F) == 0x7E).all()
        assert np.array_equal(fp8.decode_e4m3(c), np.sign(v) * 448.0)


def test_attention_fp8_two_keys_closed_form():
    """One request, a root of two tokens: the second query attends to both
    keys with weights softmax(c sq sk <Q, K_j>) and returns sv times the
    weighted decoded values -- the descale factors of q, k and v each enter
    once."""
    d = 4
    q8 = fp8.encode_e4m3(np.array([[[1.0, 0.5, 0.0, -1.0]]] * 2))
    k8 = fp8.encode_e4m3(np.array([[[2.0, 0.0, 1.0, 0.0]], [[0.0, 1.0, -1.0, 2.0]]]))
    v8 = fp8.encode_e4m3(np.array([[[1.0, 2.0, 3.0, 4.0]], [[-1.0, 0.0, 0.5, 8.0]]]))
    sq, sk, sv, scale = 0.5, 0.25, 2.0, 1.0 / math.sqrt(d)
    tree = ([0, 1], [-1], [2], [0])
    got = fp8.attention_fp8(tree, q8, k8, v8, None, None, (sq, sk, sv), scale)
    Q, K, V = (fp8.decode_e4m3(a) for a in (q8, k8, v8))
    s = scale * (sq * Q[1, 0]) @ (sk * K[:, 0]).T
    w = np.exp(s - s.max())
    w /= w.sum()
    np.testing.assert_allclose(got[1, 0], w @ (sv * V[:, 0]), rtol=1e-12)
    np.testing.assert_allclose(got[0, 0], sv * V[0, 0], rtol=1e-12)   # first token: its own key only
