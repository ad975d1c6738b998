"""Host-side bookkeeping of bench.py (CPU, no GPU).

`roofline.traffic` comes from a committed ncu capture and may only be reported
while the kernel's own sources are unchanged since that capture; these tests
pin that rule with a copy of the source tree.  The reference arm's JSON line
(with its oracle sampler stubbed), its rank rule and the warm-up minimum are
checked too, and every bench command recorded in profiles/ must still parse.
"""

import importlib.util
import json
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench(root):
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(root, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _tree(tmp_path):
    """bench.py, the CUDA sources and profiles/ncu_traffic.json in a scratch root."""
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "exact_memory_efficient_b200", "csrc"),
                    root / "exact_memory_efficient_b200" / "csrc")
    (root / "profiles").mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "bench.py"), root / "bench.py")
    return root


def test_traffic_reported_only_for_matching_sources(tmp_path):
    root = _tree(tmp_path)
    b = _load_bench(str(root))
    b.ROOT = str(root)
    b.CSRC = str(root / "exact_memory_efficient_b200" / "csrc")
    sha = b.source_sha(b.KERNEL_SOURCES["bwd_main_kernel"])
    (root / "profiles" / "ncu_traffic.json").write_text(json.dumps(
        {"bwd_main_kernel<128>": {"src_sha": sha, "dram_bytes_per_launch": 123}}))
    assert b.ncu_traffic("bwd_main_kernel<128>") == 123
    assert b.ncu_traffic("fwd_bf16_kernel<128>") is None          # no entry
    assert b.ncu_traffic("unknown_kernel<1>") is None
    # a change to a file the kernel does not compile leaves the figure valid
    (root / "exact_memory_efficient_b200" / "csrc" / "decode.cu").write_text("// changed\n")
    assert b.ncu_traffic("bwd_main_kernel<128>") == 123
    # a change to the kernel's own source voids it
    with open(root / "exact_memory_efficient_b200" / "csrc" / "bwd_bf16.cu", "a") as f:
        f.write("\n// changed\n")
    assert b.ncu_traffic("bwd_main_kernel<128>") is None


def test_committed_traffic_names_known_kernels():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        d = json.load(f)
    b = _load_bench(ROOT)
    for name, e in d.items():
        assert name.split("<")[0] in b.KERNEL_SOURCES, name
        assert e["dram_bytes_per_launch"] == int(e["dram_read"] + e["dram_write"]), name


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """`--impl reference` prints one JSON line with the keys of the bench
    contract; the oracle sampler is replaced by a stub so no oracle work runs."""
    import argparse
    bench = _load_bench(ROOT)
    calls = []

    def fake_sample(w, seed):
        calls.append(seed)
        return 0.02 + 0.001 * len(calls), 1.5, 8, "stub sample"

    monkeypatch.setattr(bench, "cpu_oracle_sample", fake_sample)
    monkeypatch.delenv("RANK", raising=False)
    assert bench.run_reference(argparse.Namespace(gpus=1, steps=2, warmup=3)) == 0
    assert len(calls) == 5                        # warm-up samples run too, and are discarded
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] == round((0.024 + 0.025) / 2, 6)   # median of the two timed samples
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 8
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import argparse
    bench = _load_bench(ROOT)
    monkeypatch.setattr(bench, "cpu_oracle_sample", lambda w, seed: (_ for _ in ()).throw(AssertionError))
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(argparse.Namespace(gpus=2, steps=2, warmup=3)) == 0
    assert capsys.readouterr().out == ""


def test_fewer_than_three_warmup_steps_is_refused(monkeypatch):
    import pytest
    bench = _load_bench(ROOT)
    monkeypatch.setattr("sys.argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert e.value.code == 2


def test_profile_commands_parse_with_the_current_bench():
    """Every `python bench.py ...` command recorded in profiles/*.md is accepted
    by the current argument parser, and names a known workload."""
    import glob
    import re
    import shlex
    from synthetic_inputs import WORKLOADS
    bench = _load_bench(ROOT)
    found = 0
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(path, encoding="utf-8"):
            m = re.search(r"python bench\.py((?:\s+--?[\w-]+(?:\s+[\w.]+)?)*)", line)
            if not m:
                continue
            args = bench.build_parser().parse_args(shlex.split(m.group(1)))
            assert args.warmup >= 3, (path, line)
            for name in (args.workload, args.profile):
                assert name is None or name in WORKLOADS, (path, name)
            found += 1
    assert found >= 4
