"""Host-side argument checks of every device entry point, run on the CPU: each
case below is refused before the call touches the device (no launch, no CUDA
runtime call), so the pointers are fake, aligned addresses that nothing
dereferences.  The status codes are the ones include/flide.h documents.

Without a device, any CUDA runtime call or launch a case reached would fail
with FLIDE_ERR_CUDA, so a passing run also shows that every refusal comes
before the first device call.  Where a device exists the module is skipped: a
check moved behind a launch would then launch on the fake addresses."""
import ctypes

import pytest
import torch

from tree_forked_decision_b200 import flide

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device addresses: runs only where no device exists")

A = 1 << 20          # a fake, 256-byte aligned device address (never dereferenced)
B = A + (1 << 16)
NUL = None
S, C, I = flide.ERR_SHAPE, flide.ERR_CAPACITY, flide.ERR_INVALID


@pytest.fixture(scope="module")
def lib():
    return flide.load()


def _idx(R=2, N=5, T=64, max_depth=2, work_len=1 << 12):
    x = flide.TreeIndexC()
    x.R, x.N, x.T, x.max_depth = R, N, T, max_depth
    for i, name in enumerate(flide.INDEX_ARRAYS):
        setattr(x, name, A + 256 * i)
    x.work_len = work_len
    return ctypes.byref(x)


def _attn(lib, **kw):
    a = dict(q=A, k=A, v=A, pk=NUL, pv=NUL, past_rows=0, idx=_idx(), Hq=16, Hkv=4, d=128,
             dtype=flide.BF16, scale=0.1, out=B, flags=0)
    a.update(kw)
    return lib.flide_fork_attn(a["q"], a["k"], a["v"], a["pk"], a["pv"], a["past_rows"], a["idx"],
                               a["Hq"], a["Hkv"], a["d"], a["dtype"], a["scale"], a["out"],
                               a["flags"], NUL)


@pytest.mark.parametrize("kw,code", [
    (dict(idx=NUL), S), (dict(q=NUL), S), (dict(out=NUL), S),
    (dict(Hq=0), S), (dict(Hkv=0), S), (dict(Hq=12, Hkv=8), S),
    (dict(past_rows=-1), S), (dict(pk=A), S), (dict(pv=A), S),
    (dict(dtype=flide.E4M3), S),          # e4m3 needs descale factors: the fp8 entry point
])
@pytest.mark.parametrize("entry", ["flide_fork_attn", "flide_fork_attn_noalloc"])
def test_fork_attn_refusals(lib, kw, code, entry):
    if entry == "flide_fork_attn":
        assert _attn(lib, **kw) == code
    else:
        a = dict(q=A, k=A, v=A, pk=NUL, pv=NUL, past_rows=0, idx=_idx(), Hq=16, Hkv=4, d=128,
                 dtype=flide.BF16, scale=0.1, out=B, flags=0)
        a.update(kw)
        assert lib.flide_fork_attn_noalloc(*a.values(), NUL) == code


def test_fork_attn_noalloc_request_cap(lib):
    a = [A, A, A, NUL, NUL, 0, _idx(R=16385), 16, 4, 128, flide.BF16, 0.1, B, 0, NUL]
    assert lib.flide_fork_attn_noalloc(*a) == C


@pytest.mark.parametrize("kw,code", [
    (dict(descale=NUL), S), (dict(idx=NUL), S), (dict(pk=A), S),
    (dict(d=64), S),                      # the e4m3 path is the d = 128 tensor-core kernel
    (dict(Hq=12, Hkv=8), S), (dict(Hq=256, Hkv=1), S),   # group wider than a 128-row half
    (dict(idx=_idx(max_depth=1 << 20)), S),
])
def test_fork_attn_fp8_refusals(lib, kw, code):
    a = dict(q=A, k=A, v=A, pk=NUL, pv=NUL, past_rows=0, idx=_idx(), Hq=16, Hkv=4, d=128,
             descale=A, scale=0.1, out=B)
    a.update(kw)
    assert lib.flide_fork_attn_fp8(*a.values(), NUL) == code


@pytest.mark.parametrize("kw,code", [
    (dict(block_rows=64), S), (dict(block_rows=0), S), (dict(n_blocks=0), S),
    (dict(max_blocks=0), S), (dict(n_slots=0), S), (dict(table=NUL), S), (dict(req_slot=NUL), S),
    (dict(pool_k=NUL), S), (dict(n_blocks=1 << 24, block_rows=256), C),
    (dict(dtype=flide.E4M3, descale=NUL), S), (dict(dtype=flide.F32), S), (dict(d=64), S),
])
def test_fork_attn_paged_refusals(lib, kw, code):
    a = dict(q=A, k=A, v=A, pool_k=A, pool_v=A, n_blocks=8, block_rows=128, table=A, max_blocks=4,
             req_slot=A, n_slots=2, idx=_idx(), Hq=16, Hkv=4, d=128, dtype=flide.BF16,
             descale=NUL, scale=0.1, out=B)
    a.update(kw)
    assert lib.flide_fork_attn_paged(*a.values(), NUL) == code


@pytest.mark.parametrize("kw,code", [
    (dict(idx=NUL), S), (dict(g=NUL), S), (dict(beta=NUL), S), (dict(node_state=NUL), S),
    (dict(H=0), S), (dict(slots=0), S), (dict(dtype=flide.E4M3), S),
])
def test_fork_gdn_refusals(lib, kw, code):
    a = dict(q=A, k=A, v=A, g=A, beta=A, state_in=NUL, idx=_idx(), H=4, dk=128, dv=128,
             dtype=flide.BF16, out=B, node_state=B, slots=4, flags=0)
    a.update(kw)
    assert lib.flide_fork_gdn(*a.values(), NUL) == code


@pytest.mark.parametrize("kw,code", [
    (dict(descale=NUL), S), (dict(node_state=NUL), S), (dict(H=0), S), (dict(slots=0), S),
    (dict(dk=64), S), (dict(dv=64), S),   # the e4m3 scan is the 128 x 128 tensor-core kernel
])
def test_fork_gdn_fp8_refusals(lib, kw, code):
    a = dict(q=A, k=A, v=A, descale=A, g=A, beta=A, state_in=NUL, idx=_idx(), H=4, dk=128,
             dv=128, out=B, node_state=B, slots=4)
    a.update(kw)
    assert lib.flide_fork_gdn_fp8(*a.values(), NUL) == code


def test_amax_and_quantize_refusals(lib):
    assert lib.flide_amax(A, 16, flide.E4M3, B, 0, NUL) == S        # input dtype f32 / bf16
    assert lib.flide_amax(A, -1, flide.F32, B, 0, NUL) == S
    assert lib.flide_amax(A, 16, flide.F32, NUL, 0, NUL) == S
    assert lib.flide_amax(NUL, 16, flide.F32, B, 0, NUL) == S
    assert lib.flide_amax(A + 4, 16, flide.F32, B, 0, NUL) == S     # 16-byte aligned input
    assert lib.flide_amax(A, 16, flide.F32, B + 2, 0, NUL) == S
    q = lambda x=A, n=16, dt=flide.BF16, amax=B, out=B + 256, ds=B + 512: \
        lib.flide_quantize_e4m3(x, n, dt, amax, out, ds, NUL)
    assert q(dt=flide.E4M3) == S
    assert q(amax=NUL) == S
    assert q(out=NUL) == S
    assert q(x=A + 8) == S
    assert q(out=B + 260) == S                                       # 8-byte aligned output
    assert q(n=-5) == S


@pytest.mark.parametrize("kw,code", [
    (dict(idx=NUL), S), (dict(h=NUL), S), (dict(workspace=NUL), S), (dict(dtype=flide.F32), S),
    (dict(D=0), S), (dict(D=96), S), (dict(V=100), S), (dict(idx=_idx(R=-1)), S),
    (dict(idx=_idx(R=100, work_len=150)), C),      # the row-tile table needs 2 (R + 1) entries
])
def test_branch_logprob_refusals(lib, kw, code):
    a = dict(h=A, w=A, targets=A, idx=_idx(), D=128, V=256, dtype=flide.BF16, logp=B,
             workspace=B, ws_bytes=1 << 20)
    a.update(kw)
    assert lib.flide_branch_logprob(*a.values(), NUL) == code


def test_option_probs_refusals_and_empty(lib):
    assert lib.flide_option_probs(NUL, A, A, A, NUL) == S
    assert lib.flide_option_probs(_idx(), A, NUL, A, NUL) == S
    assert lib.flide_option_probs(_idx(R=0), A, A, A, NUL) == flide.OK   # nothing to launch


def test_tree_build_refusals(lib):
    desc = flide.TreeDesc(2, 5, 64, 2, A, A, A, A)
    assert lib.flide_tree_build(NUL, _idx(), NUL) == S
    assert lib.flide_tree_build(ctypes.byref(desc), NUL, NUL) == S
    for cap in (dict(R=1), dict(N=4), dict(T=63), dict(max_depth=1)):  # index built for less
        assert lib.flide_tree_build(ctypes.byref(desc), _idx(**cap), NUL) == C
    bad = flide.TreeDesc(2, 5, 64, 2, A, NUL, A, A)                    # N > 0 needs parents
    assert lib.flide_tree_build(ctypes.byref(bad), _idx(), NUL) == S
    neg = flide.TreeDesc(-1, 5, 64, 2, A, A, A, A)
    assert lib.flide_tree_build(ctypes.byref(neg), _idx(), NUL) == S
    x = flide.TreeIndexC()
    x.R, x.N, x.T, x.max_depth = 2, 5, 64, 2                             # status array unset
    assert lib.flide_tree_build(ctypes.byref(desc), ctypes.byref(x), NUL) == S


@pytest.mark.parametrize("kw", [
    dict(dtype=flide.E4M3), dict(idx=NUL),
    dict(Hkv=1, d=4),                    # 8-byte K/V rows: rows are copied in 16-byte words
    dict(k=NUL), dict(ck=NUL),
    # the state half is refused before the K/V half launches anything
    dict(cS=NUL), dict(node_state=NUL), dict(dk=0), dict(dk=3, dv=3),
])
def test_state_save_refusals(lib, kw):
    a = dict(idx=_idx(), k=A, v=A, pk=NUL, pv=NUL, Hkv=4, d=128, dtype=flide.BF16,
             node_state=A, H=4, dk=128, dv=128, ck=B, cv=B, cS=B, ckpt_rows=64)
    a.update(kw)
    assert lib.flide_state_save(*a.values(), NUL) == S


@pytest.mark.parametrize("kw", [
    dict(dtype=flide.E4M3), dict(R=-1), dict(R=4097), dict(src_req=NUL), dict(status=NUL),
    dict(past_len=NUL), dict(Hkv=0), dict(Hkv=1, d=4), dict(pk=NUL),
    dict(state_in=A, sS=NUL), dict(state_in=A, sS=A, H=0), dict(state_in=A, sS=A, dk=3, dv=3),
])
def test_state_resume_refusals(lib, kw):
    a = dict(R=2, src_req=A, src_R=2, src_start=A, sk=A, sv=A, sS=NUL, Hkv=4, d=128,
             dtype=flide.BF16, H=4, dk=128, dv=128, past_len=B, pk=B, pv=B, past_rows=64,
             state_in=NUL, status=B)
    a.update(kw)
    want = C if kw == dict(R=4097) else S          # past the kernel's 4096-request table
    assert lib.flide_state_resume(*a.values(), NUL) == want


@pytest.mark.parametrize("kw,code", [
    (dict(idx=NUL), S), (dict(table=NUL), S), (dict(pool_k=NUL), S), (dict(max_blocks=0), S),
    (dict(block_rows=0), S), (dict(dtype=7), S), (dict(Hkv=1, d=4), S),
    (dict(pool_S=B), S),                 # node states and the state pool come together
    (dict(node_state=A, pool_S=B, H=0), S), (dict(node_state=A, pool_S=B, H=1, dk=3, dv=3), S),   # 9 floats a state
    (dict(idx=_idx(R=0)), flide.OK),     # empty batch: nothing to launch
])
def test_history_append_refusals(lib, kw, code):
    a = dict(idx=_idx(), req_slot=A, start=A, table=A, max_blocks=4, block_rows=128, k=A, v=A,
             pool_k=B, pool_v=B, Hkv=4, d=128, dtype=flide.BF16, node_state=NUL, H=4, dk=128,
             dv=128, pool_S=NUL)
    a.update(kw)
    assert lib.flide_history_append(*a.values(), NUL) == code


@pytest.mark.parametrize("kw,code", [
    (dict(R=4097), C), (dict(R=-1), C), (dict(status=NUL), S), (dict(hist_len=NUL), S),
    (dict(max_requests=0), S), (dict(past_rows=-1), S), (dict(pk=NUL, pv=NUL), S),
    (dict(pv=NUL), S), (dict(dtype=7), S), (dict(Hkv=1, d=4), S),
    (dict(state_in=A, H=0), S),
    (dict(R=0), flide.OK),               # empty batch: nothing to launch
    (dict(R=0, past_rows=0, pk=NUL, pv=NUL), flide.OK),   # lengths only, nothing to launch
])
def test_history_gather_refusals(lib, kw, code):
    a = dict(R=2, req_slot=A, max_requests=4, hist_len=A, table=A, max_blocks=4, block_rows=128,
             pool_k=A, pool_v=A, Hkv=4, d=128, dtype=flide.BF16, pool_S=NUL, H=4, dk=128,
             dv=128, past_len=B, pk=B, pv=B, past_rows=64, state_in=NUL, status=B)
    a.update(kw)
    assert lib.flide_history_gather(*a.values(), NUL) == code


def test_copy_rows_refusals(lib):
    assert lib.flide_copy_rows(A, B, NUL, NUL, -1, 16, NUL) == S
    assert lib.flide_copy_rows(A, B, NUL, NUL, 4, 0, NUL) == S
    assert lib.flide_copy_rows(A, B, NUL, NUL, 4, 6, NUL) == S      # rows of whole 4-byte words
    assert lib.flide_copy_rows(NUL, B, NUL, NUL, 4, 16, NUL) == S
    assert lib.flide_copy_rows(A + 2, B, NUL, NUL, 4, 16, NUL) == S
    assert lib.flide_copy_rows(A, B, NUL, NUL, 0, 16, NUL) == flide.OK  # nothing to copy


def test_selftest_wait_refusals(lib):
    assert lib.flide_selftest_wait_timeout(NUL, 1000, 1, NUL) == S
    assert lib.flide_selftest_wait_timeout(A, 0, 1, NUL) == S
    assert lib.flide_selftest_wait_timeout(A, 10000001, 1, NUL) == S  # waits are bounded at 10 s


def test_binding_refuses_host_and_strided_tensors():
    """The binding hands only dense device arrays to the library: a strided
    view or a host tensor raises before any call."""
    x = torch.zeros(8, 4, 16)
    with pytest.raises(ValueError, match="contiguous"):
        flide._ptr(x.transpose(0, 1))
    with pytest.raises(ValueError, match="CUDA"):
        flide._ptr(x)
    assert flide._ptr(None) is None
    idx = object.__new__(flide.TreeIndex)
    with pytest.raises(ValueError, match="CUDA"):
        flide.fork_attn(torch.zeros(8, 4, 16, dtype=torch.bfloat16),
                        torch.zeros(8, 2, 16, dtype=torch.bfloat16),
                        torch.zeros(8, 2, 16, dtype=torch.bfloat16), idx, 0.25,
                        out=torch.zeros(8, 4, 16, dtype=torch.bfloat16))


def test_binding_checks_element_types_and_shapes():
    """The library reads every tensor of a call as q's element type, so the
    binding refuses mixed types and inconsistent shapes before any call."""
    idx = object.__new__(flide.TreeIndex)
    bf, f32 = torch.bfloat16, torch.float32
    q, k = torch.zeros(8, 4, 16, dtype=bf), torch.zeros(8, 2, 16, dtype=bf)
    for fn in (flide.fork_attn, flide.fork_attn_noalloc):
        with pytest.raises(TypeError, match="k is"):
            fn(q, k.float(), k, idx, 0.25)
        with pytest.raises(TypeError, match="out is"):
            fn(q, k, k, idx, 0.25, out=torch.zeros(8, 4, 16))
        with pytest.raises(ValueError):
            fn(q, k, torch.zeros(8, 2, 8, dtype=bf), idx, 0.25)          # v shape
        with pytest.raises(ValueError):
            fn(q, torch.zeros(7, 2, 16, dtype=bf), torch.zeros(7, 2, 16, dtype=bf), idx, 0.25)
        with pytest.raises(ValueError):
            fn(q, k, k, idx, 0.25, past_k=torch.zeros(3, 1, 16, dtype=bf),
               past_v=torch.zeros(3, 1, 16, dtype=bf))                   # past heads
        with pytest.raises(TypeError, match="past_k is"):
            fn(q, k, k, idx, 0.25, past_k=torch.zeros(3, 2, 16), past_v=torch.zeros(3, 2, 16))
    gq, gv = torch.zeros(8, 2, 16, dtype=bf), torch.zeros(8, 2, 32, dtype=bf)
    g = torch.zeros(8, 2, dtype=f32)
    ns = torch.zeros(3, 2, 32, 16, dtype=f32)
    with pytest.raises(TypeError, match="g must"):
        flide.fork_gdn(gq, gq, gv, g.double(), g, idx, ns)
    with pytest.raises(TypeError, match="node_state"):
        flide.fork_gdn(gq, gq, gv, g, g, idx, torch.zeros(3, 2, 16, 32, dtype=f32))   # [dv, dk] swapped
    with pytest.raises(TypeError, match="state_in"):
        flide.fork_gdn(gq, gq, gv, g, g, idx, ns, state_in=torch.zeros(1, 2, 32, 16, dtype=bf))
    with pytest.raises(TypeError, match="v is"):
        flide.fork_gdn(gq, gq, gv.float(), g, g, idx, ns)
    with pytest.raises(ValueError):
        flide.fork_gdn(gq, gq, torch.zeros(7, 2, 32, dtype=bf), g, g, idx, ns)
    # consistent arguments get as far as the device check
    with pytest.raises(ValueError, match="CUDA"):
        flide.fork_gdn(gq, gq, gv, g, g, idx, ns, state_in=torch.zeros(1, 2, 32, 16, dtype=f32))


def test_binding_checks_paged_and_e4m3_arguments():
    idx = object.__new__(flide.TreeIndex)
    bf, u8 = torch.bfloat16, torch.uint8
    q, k = torch.zeros(8, 4, 128, dtype=bf), torch.zeros(8, 2, 128, dtype=bf)
    pool = torch.zeros(256, 2, 128, dtype=bf)
    tab, slot = torch.zeros(4, dtype=torch.int32), torch.zeros(1, dtype=torch.int32)
    paged = lambda **kw: flide.fork_attn_paged(*[kw.get(n, dflt) for n, dflt in (
        ("q", q), ("k", k), ("v", k), ("index", idx), ("scale", 0.1), ("pool_k", pool),
        ("pool_v", pool), ("block_table", tab), ("req_slot", slot), ("block_rows", 128),
        ("max_blocks", 2))], out=kw.get("out"))
    with pytest.raises(TypeError, match="pool_k is"):
        paged(pool_k=pool.float())
    with pytest.raises(ValueError, match="pools"):
        paged(pool_v=torch.zeros(256, 1, 128, dtype=bf))
    with pytest.raises(TypeError, match="block_table"):
        paged(block_table=tab.long())
    with pytest.raises(TypeError, match="out must be bfloat16"):
        paged(out=torch.zeros(8, 4, 128))
    with pytest.raises(ValueError, match="CUDA"):           # consistent: up to the device check
        paged()
    q8, k8 = torch.zeros(8, 4, 128, dtype=u8), torch.zeros(8, 2, 128, dtype=u8)
    ds = torch.ones(3)
    with pytest.raises(TypeError, match="out must be bfloat16"):
        flide.fork_attn_fp8(q8, k8, k8, idx, 0.1, ds, out=torch.zeros(8, 4, 128))
    g8, g = torch.zeros(8, 2, 128, dtype=u8), torch.zeros(8, 2)
    ns = torch.zeros(2, 2, 128, 128)
    with pytest.raises(TypeError, match="beta must"):
        flide.fork_gdn_fp8(g8, g8, g8, g, g[:, :1].contiguous(), idx, ns, ds)
    with pytest.raises(TypeError, match="node_state"):
        flide.fork_gdn_fp8(g8, g8, g8, g, g, idx, torch.zeros(2, 2, 128, 64), ds)


def test_binding_checks_checkpoint_arguments():
    idx = object.__new__(flide.TreeIndex)
    bf, i32 = torch.bfloat16, torch.int32
    k = torch.zeros(8, 2, 16, dtype=bf)
    ns, cS = torch.zeros(3, 2, 4, 8), torch.zeros(1, 2, 4, 8)
    with pytest.raises(TypeError, match="ckpt_k"):
        flide.state_save(idx, k, k, torch.zeros(9, 2, 16), torch.zeros(9, 2, 16, dtype=bf), None)
    with pytest.raises(TypeError, match="past_v"):
        flide.state_save(idx, k, k, torch.zeros(9, 2, 16, dtype=bf), torch.zeros(9, 2, 16, dtype=bf),
                         None, past_k=torch.zeros(1, 2, 16, dtype=bf), past_v=torch.zeros(1, 1, 16, dtype=bf))
    with pytest.raises(TypeError, match="ckpt_S"):
        flide.state_save(idx, None, None, None, None, torch.zeros(1, 2, 8, 4), node_state=ns)
    z = lambda n: torch.zeros(n, dtype=i32)
    with pytest.raises(TypeError, match="src_req"):
        flide.state_resume(torch.zeros(1, dtype=torch.int64), z(2), k, k, None, z(1), k, k, None, z(1))
    with pytest.raises(TypeError, match="past_k"):
        flide.state_resume(z(1), z(2), k, k, None, z(1), torch.zeros(8, 2, 16), k, None, z(1))
    with pytest.raises(TypeError, match="src_S"):
        flide.state_resume(z(1), z(2), k, k, torch.zeros(1, 2, 4, 8, dtype=bf), z(1), k, k, cS, z(1))


def test_binding_checks_decision_arguments():
    idx = flide.TreeIndex.__new__(flide.TreeIndex)
    idx.R, idx.N, idx.T = 1, 3, 8
    bf = torch.bfloat16
    h, w = torch.zeros(8, 64, dtype=bf), torch.zeros(128, 64, dtype=bf)
    y, lp, ws = torch.zeros(8, dtype=torch.int32), torch.zeros(8), torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError, match="w_lm"):
        flide.branch_logprob(h, w.float(), y, idx, logp=lp, workspace=ws)
    with pytest.raises(TypeError, match="w_lm"):
        flide.branch_logprob(h, torch.zeros(128, 32, dtype=bf), y, idx, logp=lp, workspace=ws)
    with pytest.raises(TypeError, match="targets"):
        flide.branch_logprob(h, w, y.long(), idx, logp=lp, workspace=ws)
    with pytest.raises(ValueError, match="entries"):
        flide.branch_logprob(h, w, y[:5], idx, logp=lp, workspace=ws)
    with pytest.raises(TypeError, match="logp must"):
        flide.option_probs(idx, lp.double(), path_logp=torch.zeros(3), prob=torch.zeros(3))
    with pytest.raises(ValueError, match="entries"):
        flide.option_probs(idx, lp, path_logp=torch.zeros(2), prob=torch.zeros(3))
