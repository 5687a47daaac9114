"""CPU: the bench's bookkeeping that turns a run into a report line.

The recorded ncu traffic is reported only for the call and the kernel code it was
captured on (a comment edit keeps it, a code edit drops it), and the algorithmic
bytes follow the formula stated for a decode call."""

import json

import numpy as np

import bench


def test_traffic_record_holds_only_for_the_captured_code(monkeypatch, tmp_path):
    rec = {"gqa": {"call": "pa_decode_append", "kernel_hash": "abc", "dram_bytes_per_launch": 7}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "decode_kernel_hash", lambda: "abc")
    assert bench.recorded_traffic("gqa", "pa_decode_append") == 7
    assert bench.recorded_traffic("gqa", "pa_decode") is None      # another call
    assert bench.recorded_traffic("long", "pa_decode_append") is None
    monkeypatch.setattr(bench, "decode_kernel_hash", lambda: "def")
    assert bench.recorded_traffic("gqa", "pa_decode_append") is None  # the kernels changed


def test_code_hash_ignores_comments_and_blank_lines():
    a = "int f() {  // the first\n\n  return 1; /* a\n block */\n}\n"
    b = "int f() {\n  return 1;\n}\n"
    c = "int f() {\n  return 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(b) != bench._code_only(c)


def test_committed_traffic_record_matches_the_sources_it_names():
    """profiles/traffic.json is keyed by the hash of the kernel sources it was captured on;
    each entry names the call it covers and gives bytes near the algorithmic figure."""
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for name, e in rec.items():
        if name.startswith("_"):
            continue
        assert e["call"] in ("pa_decode_append", "pa_decode")
        assert 0.9 < e["dram_bytes_per_launch"] / e["alg_bytes_per_launch"] < 1.2


def test_decode_bytes_formula():
    # sum_b 2 L_b Hkv D e + 2 B Hq D e + sum_b ceil(L_b / bs) 4 + 4 B
    lens = np.array([10, 7, 0])
    B, Hq, Hkv, D, bs, e = 3, 8, 2, 64, 4, 2
    kv = sum(2 * int(L) * Hkv * D * e for L in lens)
    expect = kv + 2 * B * Hq * D * e + sum(-(-int(L) // bs) * 4 for L in lens) + 4 * B
    total, kv_only = bench.decode_bytes(lens, B, Hq, Hkv, D, bs, e)
    assert (total, kv_only) == (expect, kv)
