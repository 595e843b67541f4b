"""bench.py's measurement bookkeeping on the CPU: the algorithmic byte count of
a token, and the ncu traffic record -- written from an ncu CSV, read back only
while the kernel sources hash the same and the workload matches."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_token_bytes_llama3_8b(bench):
    # x + kept rows of both INT4 proxies + two fp16 scale rows per group +
    # k channel records (gate and up) + k W_down rows + out
    d, f, k, n_x = 4096, 14336, 4301, 2048
    want = 4 * d + n_x * f + 4 * f * (d // 128) + 4 * k * d + 2 * k * d + 4 * d
    assert bench.token_bytes(d, f, k, n_x) == want
    assert abs(want / 1e6 - 136.9) < 0.1


def _csv(path, rows):
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
            '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
            '"Metric Value"')
    with open(path, "w") as fh:
        fh.write("==PROF== preamble line that is not CSV\n")
        fh.write(head + "\n")
        for rid, kern, name, unit, val in rows:
            fh.write(f'"{rid}","1","python","h","{kern}","1","7","(544, 1, 1)","(148, 1, 1)",'
                     f'"0","10.0","Command line profiler metrics","{name}","{unit}","{val}"\n')


def test_traffic_record_roundtrip(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "token_traffic.json"))
    csv_path = tmp_path / "dram.csv"
    kern = "void prox::<unnamed>::token_kernel<4, 4>(prox::TokenArgs)"
    _csv(csv_path, [
        (0, kern, "dram__bytes_read.sum", "byte", "137,000,000"),
        (0, kern, "dram__bytes_write.sum", "byte", "100,000"),
        (1, "other_kernel", "dram__bytes_read.sum", "byte", "5"),
        (1, "other_kernel", "dram__bytes_write.sum", "byte", "5"),
        (2, kern, "dram__bytes_read.sum", "Mbyte", "136.5"),
        (2, kern, "dram__bytes_write.sum", "Kbyte", "50"),
        (3, kern, "dram__bytes_read.sum", "byte", "136800000"),
        (3, kern, "dram__bytes_write.sum", "byte", "0"),
    ])
    wl = "llama3_8b ffn layer d_model=4096 d_ff=14336 s1=50% s2=70% k=4301"
    rec = bench.record_traffic(str(csv_path), wl, 136.9e6, "ncu ... bench.py")
    assert rec["launches"] == 3
    assert rec["dram_bytes_per_launch"] == 136_800_000  # median of 137.1, 136.55, 136.8 MB
    assert rec["source_hash"] == bench.kernel_source_hash()
    got = bench.profiled_traffic(wl)
    assert got is not None and got["dram_bytes_per_launch"] == 136_800_000
    assert bench.profiled_traffic(wl.replace("k=4301", "k=5734")) is None
    # a record taken on other kernel sources is not reported
    with open(bench.PROFILE_TRAFFIC) as fh:
        doc = json.load(fh)
    doc["source_hash"] = "0" * 16
    with open(bench.PROFILE_TRAFFIC, "w") as fh:
        json.dump(doc, fh)
    assert bench.profiled_traffic(wl) is None


def test_kernel_source_hash_covers_every_token_kernel_source(bench, tmp_path, monkeypatch):
    # the traffic record is tied to the token kernel's code: editing the code
    # of any of its sources changes the hash; editing only comments, or
    # another source, does not
    src = tmp_path / "csrc"
    src.mkdir()
    for name in bench.TOKEN_KERNEL_SOURCES + ("batch.cu",):
        (src / name).write_text("// " + name + "\nint v = 0;\n")
    monkeypatch.setattr(bench, "CSRC", str(src))
    h0 = bench.kernel_source_hash()
    for name in bench.TOKEN_KERNEL_SOURCES:
        (src / name).write_text("/* reworded\n comment */ // " + name + "\n\nint v = 0;  // same code\n")
        assert bench.kernel_source_hash() == h0
        (src / name).write_text("// " + name + "\nint v = 1;\n")
        h1 = bench.kernel_source_hash()
        assert h1 != h0
        h0 = h1
    (src / "batch.cu").write_text("int w = 2;\n")
    assert bench.kernel_source_hash() == h0
