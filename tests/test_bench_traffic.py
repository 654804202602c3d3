"""The bench line's `traffic` figures come from the committed DRAM capture
(profiles/traffic.json) only while the kernel source is the captured one:
attention per launch, the GDN per layer (its tree-level launches together),
null as soon as the source's hash differs.  Host only."""
import hashlib
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(root):
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.ROOT = str(root)
    return mod


def _tree(tmp_path, entries, sources):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "tree_forked_decision_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in sources.items():
        (csrc / name).write_text(text)
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entries))


def _sha(text):
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def test_traffic_per_unit_and_source_pinning(tmp_path):
    src_a, src_g = "// attention\n", "// gdn\n"
    _tree(tmp_path,
          {"attn_tc_kernel": {"bytes_per_launch": 1000, "source_sha": _sha(src_a)},
           "gdn_ws_kernel": {"bytes_per_layer": 3000, "bytes_per_launch": 7, "source_sha": _sha(src_g)}},
          {"attn_tc.cu": src_a, "gdn_tc.cu": src_g})
    b = _bench(tmp_path)
    assert b.traffic_for("attn_tc_kernel", "attn_tc.cu") == 1000
    assert b.traffic_for("gdn_ws_kernel", "gdn_tc.cu") == 3000  # the layer, not one launch
    assert b.traffic_for("missing_kernel", "attn_tc.cu") is None
    # the source changes after the capture: no figure
    (tmp_path / "tree_forked_decision_b200" / "csrc" / "gdn_tc.cu").write_text("// gdn, edited\n")
    assert b.traffic_for("gdn_ws_kernel", "gdn_tc.cu") is None
    assert b.traffic_for("attn_tc_kernel", "attn_tc.cu") == 1000


def test_committed_capture_names_the_bench_kernels():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for k in ("attn_tc_kernel", "gdn_ws_kernel"):
        assert k in rec and len(rec[k]["source_sha"]) == 16
    assert rec["attn_tc_kernel"]["bytes_per_launch"] > 0
    assert rec["gdn_ws_kernel"]["bytes_per_layer"] > 0
    # the roofline objects of the bench line look these names up
    text = open(os.path.join(ROOT, "bench.py")).read()
    assert 'traffic_for("attn_tc_kernel", "attn_tc.cu")' in text
    assert 'traffic_for("gdn_ws_kernel", "gdn_tc.cu")' in text
