"""bench.py reports a roofline `traffic` figure only when the committed ncu capture matches the kernel source
and the inputs it is reported for (CPU; no GPU work)."""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path):
    """A copy of the kernel sources and an empty profiles/ folder under a temporary root."""
    for rel in set(bench.KERNEL_SRC.values()) | {"attention_ikbo_b200/csrc/sm100.cuh"}:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_traffic_requires_matching_source_and_inputs(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    part = bench.make_parts("dca")[0]
    entry = {"src_sha": bench.kernel_sha(part.kernel), "inputs": bench.part_signature(part),
             "dram_bytes_per_unit": 10.0, "units_per_launch": part.units}
    table = root / "profiles" / "ncu_traffic.json"
    table.write_text(json.dumps({part.name: entry}))
    assert bench.ncu_traffic(part) == 10.0 * part.units
    # another input recipe under the same part name: no figure
    other = bench.make_parts("dca_short")[0]
    assert other.name == part.name and bench.ncu_traffic(other) is None
    # an entry keyed by name and inputs serves that input set alongside the plain one
    entry2 = dict(entry, inputs=bench.part_signature(other), dram_bytes_per_unit=20.0)
    table.write_text(json.dumps({part.name: entry, f"{other.name}@{bench.part_signature(other)}": entry2}))
    assert bench.ncu_traffic(other) == 20.0 * other.units
    assert bench.ncu_traffic(part) == 10.0 * part.units
    # the kernel source changes: both go stale
    src = root / bench.KERNEL_SRC[part.kernel]
    src.write_text(src.read_text() + "\n// edited\n")
    assert bench.ncu_traffic(part) is None and bench.ncu_traffic(other) is None

