"""Host-side bookkeeping of bench.py (CPU, no GPU).

`roofline.traffic` comes from a committed ncu capture and may only be reported
while the kernel's own sources are unchanged since that capture; these tests
pin that rule with a copy of the source tree.
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
