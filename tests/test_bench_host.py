"""Host-side figures of the benchmark, on CPU.

* profiled_traffic: the DRAM traffic reported beside the roofline comes from a
  committed ncu summary, and only while the kernel source it was captured from
  is unchanged (its sha256 is recorded in the summary).
* transposable_int_ops: the integer-op count behind the transposable mask's
  roofline rests on the comparator count of Batcher's odd-even merge sort,
  which is tabulated (Knuth, TAOCP vol. 3, 5.3.4: 19, 63, 191, 543 comparators
  for 8, 16, 32, 64 keys).
"""
import hashlib
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fields(path):
    out = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                out[k.strip()] = v.strip()
    return out


def test_traffic_is_read_from_the_summary_while_the_source_matches():
    for (workload, kernel), rel in bench.TRAFFIC_PROFILES.items():
        f = _fields(os.path.join(ROOT, rel))
        with open(os.path.join(ROOT, f["source_file"]), "rb") as fh:
            src = fh.read()
        got = bench.profiled_traffic(workload, kernel)
        if hashlib.sha256(src).hexdigest() == f["source_sha256"]:
            assert got == int(f["traffic_bytes_per_launch"])
        else:
            assert got is None
    assert bench.profiled_traffic("linear_4096", "nm_mask") is None
    assert bench.profiled_traffic("mlp_pair", "nm_mask_up") is None


def test_traffic_is_dropped_when_the_kernel_changes(tmp_path, monkeypatch):
    rel = bench.TRAFFIC_PROFILES[("linear_4096", "nm_spmm")]
    f = _fields(os.path.join(ROOT, rel))
    for r in (rel, f["source_file"]):
        os.makedirs(tmp_path / os.path.dirname(r), exist_ok=True)
        shutil.copy(os.path.join(ROOT, r), tmp_path / r)
    src = tmp_path / f["source_file"]
    # a summary that matches this copy of the source reports its figure ...
    summary = (tmp_path / rel).read_text().replace(f["source_sha256"], hashlib.sha256(src.read_bytes()).hexdigest())
    (tmp_path / rel).write_text(summary)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("linear_4096", "nm_spmm") == int(f["traffic_bytes_per_launch"])
    # ... and none once the kernel source is edited
    src.write_bytes(src.read_bytes() + b"\n// edited\n")
    assert bench.profiled_traffic("linear_4096", "nm_spmm") is None
    # a summary without the figure reports none
    src.write_bytes(src.read_bytes()[: -len(b"\n// edited\n")])
    assert bench.profiled_traffic("linear_4096", "nm_spmm") is not None
    (tmp_path / rel).write_text("\n".join(l for l in summary.splitlines() if not l.startswith("traffic_bytes_per_launch")))
    assert bench.profiled_traffic("linear_4096", "nm_spmm") is None


def test_transposable_int_ops_uses_batchers_comparator_counts():
    # per M x M block: 2 per comparator on the padded key count, 7 per greedy step, 2 per key
    assert bench.transposable_int_ops(2) == 2 * 5 + 9 * 4          # 4 keys: 5 comparators
    assert bench.transposable_int_ops(4) == 2 * 63 + 9 * 16        # 16 keys
    assert bench.transposable_int_ops(8) == 2 * 543 + 9 * 64       # 64 keys
    assert bench.transposable_int_ops(3) == 2 * 63 + 9 * 9         # 9 keys padded to 16
    assert bench.transposable_int_ops(5) == 2 * 191 + 9 * 25       # 25 keys padded to 32
