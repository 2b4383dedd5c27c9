"""Host logic of bench.py that needs no GPU: the ncu traffic figures are
reported only for the workload and the kernel sources they were captured on,
and the roofline labels name the weight format of the workload."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _entries():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    return {k: v for k, v in d.items() if not k.startswith("_")}


def test_traffic_entries_name_workload_and_sources():
    for name, e in _entries().items():
        assert e["workload"] in ("decode", "verify", "prefill", "stack", "tiny"), name
        assert len(e["source_hash"]) == 16, name
        assert e["dram_bytes_per_launch"] > 0, name


def test_traffic_only_for_its_workload(monkeypatch):
    ents = _entries()
    monkeypatch.setattr(bench, "source_hash", lambda: ents["gate_up"]["source_hash"])
    assert bench.traffic_for("gate_up", "decode") == ents["gate_up"]["dram_bytes_per_launch"]
    # another workload runs the same kernel on other shapes: no figure for it
    assert bench.traffic_for("gate_up", "verify") is None
    assert bench.traffic_for("gate_up", "stack") is None
    assert bench.traffic_for("no_such_kernel", "decode") is None


def test_traffic_null_once_sources_change(monkeypatch):
    monkeypatch.setattr(bench, "source_hash", lambda: "0" * 16)
    for name, e in _entries().items():
        assert bench.traffic_for(name, e["workload"]) is None


def test_gemv_label_names_the_format():
    from quantized_latent_moe_b200 import synth
    for wname in ("decode", "verify"):
        wl = synth.WORKLOADS[wname]
        label = bench.KERNEL_NAMES["gate_up"][5].format(fmt=wl.fmt.upper())
        assert ("Q4_0" in label) == (wl.fmt == "q4_0"), label
        assert ("Q8_0" in label) == (wl.fmt == "q8_0"), label
