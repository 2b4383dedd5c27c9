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
        assert e["workload"] in ("decode", "verify", "prefill", "prefill_nvfp4", "stack", "tiny"), name
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
    for wname in ("decode", "verify", "decode_nvfp4"):
        wl = synth.WORKLOADS[wname]
        afmt = "NVFP4" if wl.expert_fmt == "nvfp4" else "Q8_1"
        label = bench.KERNEL_NAMES["gate_up"][5].format(fmt=wl.expert_fmt.upper(), afmt=afmt)
        assert ("Q4_0" in label) == (wl.expert_fmt == "q4_0"), label
        assert ("Q8_0" in label) == (wl.expert_fmt == "q8_0"), label
        assert label.count("NVFP4") == (2 if wl.expert_fmt == "nvfp4" else 0), label


class _FakeGraph:
    def replay(self):
        pass


def test_timed_run_replays_only_prepared_graphs(monkeypatch):
    """The driver's warm-up and step counts (5 and 20 with 64-step graphs):
    prepare() captures every graph the timed run() replays, so the timed
    region never captures one."""
    captured = []

    def fake_get(self, key):
        if key not in self.graphs:
            captured.append(key)
            self.graphs[key] = _FakeGraph()
        return self.graphs[key]

    monkeypatch.setattr(bench.GraphSet, "_get", fake_get)
    for G, period, warm, steps in ((64, 64, 5, 20), (64, 64, 64, 4096), (16, 16, 3, 37), (4, 16, 4, 64)):
        gs = bench.GraphSet(G, lambda i: None, period=period)
        pos = gs.run(warm)
        gs.prepare(steps, pos)
        before = list(captured)
        end = gs.run(steps, pos)
        assert captured == before, (G, warm, steps)
        assert end == warm + steps
        assert sum(n for n, _ in gs.keys(steps, pos)) == steps
        captured.clear()


def test_graph_keys_follow_the_step_phase():
    gs = bench.GraphSet(64, lambda i: None)
    assert gs.keys(20, 5) == [(20, 5)]
    assert gs.keys(130, 5) == [(64, 5), (64, 5), (2, 5)]
    gs = bench.GraphSet(4, lambda i: None, period=16)
    assert gs.keys(10, 14) == [(4, 14), (4, 2), (2, 6)]
