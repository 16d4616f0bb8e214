"""The benchmark's reference arm (the float64 oracle timed on the host cores) prints the
JSON line the benchmark contract asks for.  Run on the tiny geometry so that it takes
seconds; the r2 / r3 workloads differ only in sizes."""
import argparse
import json
import os
import sys

import kva_inputs as KI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "geometry", lambda name: KI.TINY)
    args = argparse.Namespace(workload="r3", steps=2, warmup=1)
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["higher_is_better"] is True and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks(capsys):
    sys.path.insert(0, ROOT)
    import bench
    bench.run_reference(argparse.Namespace(workload="r3", steps=1, warmup=0), 1, 2)
    assert capsys.readouterr().out == ""


def test_algorithmic_work_from_the_parameter_counts():
    """The roofline's FLOPs and bytes per 1024-token ubatch, recomputed from the printed
    parameter counts: 2 T per linear parameter, causal attention over the unmasked pairs of
    every projector block, 4 d_k d_v per token and value head for the recurrence; bytes are
    the 16-bit weights once, the residual in, the states read and written, the KV rows and
    the drafter outputs written."""
    sys.path.insert(0, ROOT)
    import bench
    T = 1024
    for g in (KI.R3, KI.R2):
        params = g.param_counts()["total"]
        w = g.window or T
        pairs = sum(min(i % w, i) + 1 for i in range(T))          # unmasked (query, key) pairs
        attn = g.n_blocks * g.n_heads * pairs * 4 * g.head_dim
        scan = g.n_gdn * g.gdn_n_v * T * 4 * g.gdn_d_k * g.gdn_d_v
        flops = 2 * T * params + attn + scan
        state = g.n_gdn * g.gdn_n_v * g.gdn_d_k * g.gdn_d_v * 4
        kv = 2 * g.n_attn * T * g.attn_n_kv * g.attn_d_h * 2
        approx_bytes = 2 * params + T * g.hidden * 2 + 2 * state + kv + T * g.n_draft * g.hidden * 2
        got_f, got_b = bench.algorithmic(g)
        assert abs(got_f - flops) / flops < 1e-3, (g.name, got_f, flops)
        # the conv tails and the fp32 gains are the only terms left out here (< 0.5 %)
        assert 0 <= got_b - approx_bytes < 5e-3 * approx_bytes, (g.name, got_b, approx_bytes)
    f3, b3 = bench.algorithmic(KI.R3)
    assert round(f3 / 1e12, 3) == 2.632 and round(b3 / 1e9, 2) == 2.72


def test_traffic_gate_hash_ignores_comments_only(tmp_path):
    """The heads GEMM's DRAM traffic is reported only while the GEMM's code matches the code
    it was captured on: an edit of comments or blank lines keeps the hash, an edit of code
    changes it."""
    sys.path.insert(0, ROOT)
    import bench
    base = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text(base)
    b.write_text("/* header\n   lines */\n" + base.replace("// add one", "// a different note") + "\n\n")
    c.write_text(base.replace("x + 1", "x + 2"))
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


def test_state_workload_and_last_token_accounting():
    """The HBM rooflines of the state-only workload and of the last-token pass rest on these
    byte counts; each is checked against its r3 value worked out from the model card's shapes
    (24 gated-DeltaNet layers of 48 value heads, 128 x 128 fp32 states, 10 240 conv channels,
    8 attention layers of 4 KV heads of 256, mixer rows of 264 448 16-bit values)."""
    sys.path.insert(0, ROOT)
    import bench
    g = KI.R3
    # 8 sequences x 1024 tokens
    mixer = 8 * 1024 * 264448 * 2
    states = 8 * 24 * 48 * 128 * 128 * 4 * 2        # read and written
    tails = 8 * 24 * 3 * 10240 * 2 * 2              # read and written
    kv = 8 * 1024 * 8 * 2 * 4 * 256 * 2             # K and V rows written
    flops, nbytes, parts = bench.state_algorithmic(g, 8, 1024)
    assert nbytes == mixer + states + tails + kv
    assert abs(nbytes / 1e9 - 5.83) < 0.01         # 5.83 GB per call
    assert flops == 8 * 1024 * 24 * 48 * 4 * 128 * 128
    assert parts["kv_written"] == kv and parts["state_rw"] == states
    # last token at position 32767: all 32768 rows of K and V of every attention layer
    attn, rest = bench.last_token_bytes(g, 32767)
    assert attn == 8 * 2 * 4 * 256 * 2 * 32768 == 2 ** 30
    assert rest >= 24 * 48 * 128 * 128 * 4 * 2     # at least the states read and written
