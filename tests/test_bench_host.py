"""Host-side bookkeeping of bench.py (no GPU): the algorithmic bytes and
FLOPs behind the roofline, the compute dtype per layer, and the guard that
drops stored DRAM traffic once the kernel source has changed."""
import json
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_top_routed_b200 import synth  # noqa: E402


def test_gate_up_bytes_of_the_decode_shape_by_hand():
    L = synth.make_layer("decode", T=8, d=256, E=4, k=2, I=128)
    touched = [0, 2]
    # INT4 g128: codes 2I x d / 2 bytes, bf16 scales 2I x d/128 x 2 bytes, per touched expert
    w = 2 * (2 * 128 * 256 // 2 + 2 * 128 * (256 // 128) * 2)
    x = 8 * 256 * 2
    h = 8 * 2 * 128 * 2
    assert bench.gate_up_bytes(L, touched) == w + x + h


def test_layer_flops_by_hand():
    L = synth.make_layer("fine", T=16, d=256, E=8, k=2, I=128, S=2)
    # router 2 T d E + gate/up 4 T (k+S) d I + down 2 T (k+S) d I
    assert bench.layer_flops(L) == 2 * 16 * 256 * 8 + 6 * 16 * 4 * 256 * 128
    assert bench.gate_up_flops(L) == 4 * 16 * 4 * 256 * 128


@pytest.mark.parametrize("name,kw,want", [
    ("prefill", dict(T=4, d=256, I=128, E=2, k=1), "f16"),       # all FP8: fp16 MMAs
    ("mixed", dict(T=4, d=256, I=128, E=4, k=1, fmt="mixed_fp8"), "bf16"),
    ("decode", dict(T=4, d=256, I=128, E=4, k=1), "bf16"),
])
def test_compute_dtype(name, kw, want):
    assert bench.compute_dtype(synth.make_layer(name, **kw)) == want


def test_traffic_is_dropped_when_the_kernel_source_changes(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "quantized_top_routed_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemm.cu").write_text("kernel v1")
    (csrc / "qmoe_internal.cuh").write_text("header v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1" + b"header v1").hexdigest()
    (prof / "traffic.json").write_text(json.dumps({"kernel_source_sha256": h,
                                                   "decode:T=256:gate_up": {"dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    L = types.SimpleNamespace(name="decode", T=256)
    assert bench.traffic_from_profiles(L, "gate_up") == 123
    assert bench.traffic_from_profiles(L, "down") is None
    (csrc / "gemm.cu").write_text("kernel v2")
    assert bench.traffic_from_profiles(L, "gate_up") is None


def test_down_bytes_of_the_fine_shape_by_hand():
    L = synth.make_layer("fine", T=8, d=256, E=4, k=2, I=128, S=1)
    touched = [1, 3]
    # INT4 g128 W2: codes d x I / 2 bytes, bf16 scales d x I/128 x 2 bytes; touched + shared experts
    w = 3 * (256 * 128 // 2 + 256 * (128 // 128) * 2)
    h = 8 * (2 + 1) * 128 * 2
    y = 8 * (2 + 1) * 256 * 2
    assert bench.down_bytes(L, touched) == w + h + y


def test_load_report_recovers_a_zipf_exponent():
    import numpy as np
    L = types.SimpleNamespace(name="fine")               # a Zipf(1.2)-biased workload
    counts = np.round(1e5 * np.arange(1, 65, dtype=np.float64) ** -1.2).astype(np.int64)
    rep = bench.load_report(L, np.random.default_rng(0).permutation(counts))
    assert rep["zipf_s_target"] == 1.2
    assert abs(rep["zipf_s_fit"] - 1.2) < 0.01
    assert rep["touched_experts"] == 64 and sum(rep["counts"]) == counts.sum()
    flat = bench.load_report(types.SimpleNamespace(name="decode"), np.full(8, 5))
    assert "zipf_s_fit" not in flat and flat["max_over_mean"] == 1.0


@pytest.mark.parametrize("name", ["fine", "mixed"])
def test_realised_zipf_load_of_the_skewed_workloads(name):
    """Realised per-expert load of the Zipf-biased workloads, routed by the fp64
    oracle on the seeded inputs ("OmniMoE" explainer, section 2.2: tasks grouped
    by expert).  The bias ranks the experts by the Zipf share, so the load must
    follow that ranking; top-k on the biased logits concentrates it beyond the
    nominal exponent.  The histogram and the fit printed here are what the
    bench reports under "load" for the same inputs."""
    import numpy as np
    import oracle.qmoe_oracle as O
    cfg = synth.CONFIGS[name]
    x, wr, b = synth.make_router_inputs(name)
    idx = O.topk(O.router_logits(x, wr, b), cfg["k"])
    counts = np.bincount(idx.ravel(), minlength=cfg["E"])
    rep = bench.load_report(types.SimpleNamespace(name=name), counts)
    order = np.argsort(-counts, kind="stable")
    print(f"{name}: fitted Zipf exponent {rep['zipf_s_fit']} (nominal {cfg['zipf']}), "
          f"max/mean {rep['max_over_mean']}, touched {rep['touched_experts']}/{cfg['E']}; "
          f"rows per expert, largest first: {counts[order].tolist()}")
    assert counts.sum() == cfg["T"] * cfg["k"]
    assert rep["zipf_s_fit"] > cfg["zipf"]
    # rank correlation of bias and load (Spearman, no ties in the bias)
    rb = np.argsort(np.argsort(-b)).astype(np.float64)
    rc = np.argsort(np.argsort(-counts, kind="stable")).astype(np.float64)
    assert np.corrcoef(rb, rc)[0, 1] > 0.9
