"""Host logic of bench.py that needs no GPU: the source hash that ties a
committed ncu traffic figure to the kernel it was captured on, and the
lookup that drops the figure once the sources change."""
import os

import bench


def test_code_hash_ignores_comments_and_blank_lines(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) {\n  return x + 1;\n}\n")
    b.write_text("// a comment\nint f(int x) {  // trailing note\n\n  return x + 1;\n}\n")
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


def test_captured_traffic_needs_matching_sources(tmp_path, monkeypatch):
    root = tmp_path
    csrc = root / "kv_cache_attention_flash_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, body in (("step_bf16.cu", "int a;\n"), ("ptx.cuh", "int b;\n"), ("api.cu", "int c;\n")):
        (csrc / name).write_text(body)
    hashes = [bench.code_hash(str(csrc / n)) for n in ("step_bf16.cu", "ptx.cuh", "api.cu")]
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setattr(bench, "CAPTURED_TRAFFIC",
                        {"demo": {"bytes": 12345.0, "sources": hashes, "source": "test"}})
    assert bench.captured_traffic("demo") == 12345.0
    (csrc / "api.cu").write_text("int c;  // same code, new comment\n")
    assert bench.captured_traffic("demo") == 12345.0
    (csrc / "api.cu").write_text("int c2;\n")
    assert bench.captured_traffic("demo") is None
    assert bench.captured_traffic("missing") is None


def test_reference_arm_times_whole_sampled_steps(capsys):
    """The reference arm's ms_per_step is the measured time of its sampled
    steps, so ms_per_step x steps fits the run."""
    import json
    import time
    t0 = time.time()
    assert bench.main(["--impl", "reference", "--workload", "tiny_f32", "--steps", "3",
                       "--warmup", "3"]) == 0
    wall = time.time() - t0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["ms_per_step"] * line["steps"] / 1000.0 <= wall
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_layers_option_changes_the_layer_count_for_one_run(capsys):
    """--layers runs a layer workload with another layer count (the same
    per-layer shapes) and leaves the workload table as it was."""
    import json

    import pytest

    from kv_cache_attention_flash_b200 import workloads as W
    before = W.WORKLOADS["tiny_f32"]
    assert bench.main(["--impl", "reference", "--workload", "tiny_f32", "--layers", "2",
                       "--steps", "3", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"]["layers"] == 2
    assert line["config"]["hidden"] == before.shape.hidden
    assert W.WORKLOADS["tiny_f32"] is before
    with pytest.raises(SystemExit):
        bench.main(["--workload", "tiny_f32", "--layers", "0"])
    with pytest.raises(SystemExit):
        bench.main(["--workload", "verify_b8", "--layers", "1"])
