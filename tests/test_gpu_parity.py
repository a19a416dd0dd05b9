"""CUDA path (through the C ABI) against the fp64 oracle, on a B200.

Bars (stated by the layer's specification):
  * routing from supplied logits: expert indices, counts, offsets, the
    permutation (sorted_token, inv_pos) bit-exact; gates within 1e-6;
  * routing from x: indices exact on every token whose oracle k-th/(k+1)-th
    logit margin exceeds 1e-4 (the others are counted); the schedule is
    bit-exact against the oracle's schedule of the GPU's own indices;
  * layer output: relative L2 error <= 1e-2 and max abs error <= 3e-2 against
    the oracle evaluated on the GPU's expert choice (identical on all margin-
    safe tokens), with identical dequantised weights.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle.qmoe_oracle as O  # noqa: E402
from quantized_top_routed_b200 import qmoe, synth  # noqa: E402

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 3e-2
GATE_TOL = 1e-6      # gates from supplied logits: same fp32 inputs, softmax rounding only
# Gates from raw x inherit the fp32 rounding of the logits.  A d-term fp32
# dot product of x ~ N(0,1) with w ~ N(0,1/d) accumulates about
# 2^-24 * d / sqrt(2) * rms(x_i w_i) ~ 3e-6 of error at d = 4096 (one sigma);
# the renormalised softmax has |dg/dz| <= 1/2, so gates agree within 1e-5
# with a wide margin.  The same bound keeps every token with a logit margin
# above 1e-4 on the oracle's experts.
GATE_TOL_X = 1e-5
MARGIN = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qmoe.load()


def sub_layer(layer, T):
    return dataclasses.replace(layer, T=T, x=layer.x[:T])


def to_f64(t):
    return O.bf16_to_f64(t.cpu().numpy().view(np.uint16))


def run_forward(dl, T):
    out = torch.empty((T, dl.layer.d), dtype=torch.int16, device="cuda")
    qmoe.qmoe_forward(dl.handle, dl.x, T, out, torch.cuda.current_stream())
    torch.cuda.synchronize()
    qmoe.qmoe_check_error(dl.handle)
    return to_f64(out)


def run_route(dl, T, logits=None):
    L = dl.layer
    dev = "cuda"
    r = dict(idx=torch.empty((T, L.k), dtype=torch.int32, device=dev),
             gates=torch.empty((T, L.k), dtype=torch.float32, device=dev),
             counts=torch.empty(L.E, dtype=torch.int32, device=dev),
             offsets=torch.empty(L.E + 1, dtype=torch.int32, device=dev),
             sorted_token=torch.empty(T * L.k, dtype=torch.int32, device=dev),
             inv_pos=torch.empty((T, L.k), dtype=torch.int32, device=dev))
    lg = torch.from_numpy(logits).to(dev) if logits is not None else None
    qmoe.qmoe_route(dl.handle, None if lg is not None else dl.x, lg, T, r["idx"], r["gates"], r["counts"],
                    r["offsets"], r["sorted_token"], r["inv_pos"], torch.cuda.current_stream())
    torch.cuda.synchronize()
    return {k_: v.cpu().numpy() for k_, v in r.items()}


def assert_schedule_equal(got, ref):
    for key in ("counts", "offsets", "sorted_token", "inv_pos"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=key)


def check_route_from_x(dl, T):
    """Margin rule on indices, gates on safe tokens, exact schedule of the GPU's indices."""
    L = sub_layer(dl.layer, T)
    g = run_route(dl, T)
    ref = O.route(L)
    safe = O.margin_safe(ref["margin"], MARGIN)
    np.testing.assert_array_equal(g["idx"][safe], ref["idx"][safe])
    np.testing.assert_allclose(g["gates"][safe], ref["gates"][safe], rtol=0, atol=GATE_TOL_X)
    np.testing.assert_allclose(g["gates"].sum(axis=1), 1.0, rtol=0, atol=GATE_TOL)
    assert_schedule_equal(g, O.schedule(g["idx"], L.E))
    return g, int((~safe).sum())


def check_forward(dl, T, tokens=None):
    """Layer output against the oracle on the GPU's routing; returns (rel_l2, max_abs, unsafe).

    tokens: None (every token), an index array, or a callable that picks the
    tokens from the GPU's routing result."""
    L = sub_layer(dl.layer, T)
    g, unsafe = check_route_from_x(dl, T)
    out = run_forward(dl, T)
    if callable(tokens):
        tokens = tokens(g, L)
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = O.forward(L, tokens=tok, idx_override=g["idx"][tok])
    got = out[tok]
    rel = O.rel_l2(got, ref["out"])
    mx = float(np.abs(got - ref["out"]).max())
    assert np.all(np.isfinite(got))
    assert rel <= REL_L2, f"rel L2 {rel:.3e}"
    assert mx <= MAX_ABS, f"max abs {mx:.3e}"
    return rel, mx, unsafe


def sample_tokens(T, n=48, seed=0):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(T, size=min(n, T), replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(pick))


def covering_tokens(block=64, n_random=16):
    """Token picker for full-size layers: for every expert segment of the
    schedule (routed experts from the GPU's offsets, then the identity
    segments of the shared experts), the token of the first row of every
    `block`-row block and of the segment's last row, so every token block of
    the grouped GEMMs (token blocks are at most 128 rows and a multiple of 16)
    contributes a checked output, ragged last blocks included; plus a few
    random tokens."""
    def pick(g, L):
        tok = set(sample_tokens(L.T, n_random).tolist())
        st, off = g["sorted_token"], g["offsets"]
        for e in range(L.E):
            lo, hi = int(off[e]), int(off[e + 1])
            if hi > lo:
                tok.update(int(st[p]) for p in range(lo, hi, block))
                tok.add(int(st[hi - 1]))
        if L.S:
            tok.update(range(0, L.T, block))
            tok.add(L.T - 1)
        return np.array(sorted(tok))
    return pick


# ---------------------------------------------------------------------------
# routing from supplied logits: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("E,k,T", [(8, 2, 64), (128, 8, 256), (128, 8, 1), (8, 2, 8192), (64, 6, 4096),
                                   (64, 4, 16384), (5, 5, 33), (1, 1, 7), (256, 16, 300), (40, 3, 1000)])
def test_route_from_logits_bit_exact(E, k, T):
    L = synth.make_layer("tiny", T=T, d=128, I=128, E=E, k=k)
    dl = qmoe.DeviceLayer(L)
    rng = np.random.default_rng(E * 1000 + T)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[: T // 2] = np.round(logits[: T // 2] * 2) / 2      # exact ties
    g = run_route(dl, T, logits=logits)
    ref = O.route(L, logits=logits)
    np.testing.assert_array_equal(g["idx"], ref["idx"])
    np.testing.assert_allclose(g["gates"], ref["gates"], rtol=0, atol=GATE_TOL)
    np.testing.assert_allclose(g["gates"].sum(axis=1), 1.0, rtol=0, atol=GATE_TOL)
    assert_schedule_equal(g, ref)
    dl.close()


def test_route_worked_example_flip():
    """The routing-flip example of the DREAM-MoE news item, through the GPU router."""
    L = synth.make_layer("tiny", T=2, d=128, I=128, E=2, k=1)
    dl = qmoe.DeviceLayer(L)
    g = run_route(dl, 2, logits=np.array([[2.0, 1.9], [1.8, 1.9]], np.float32))
    assert g["idx"][:, 0].tolist() == [0, 1]
    assert np.all(g["gates"] == 1.0)
    dl.close()


# ---------------------------------------------------------------------------
# whole layer, the five workloads
# ---------------------------------------------------------------------------
def test_tiny_full():
    dl = qmoe.DeviceLayer(synth.make_layer("tiny"))
    check_forward(dl, 64)
    dl.close()


@pytest.fixture(scope="module")
def decode_layer():
    dl = qmoe.DeviceLayer(synth.make_layer("decode", T=256))
    yield dl
    dl.close()


@pytest.mark.parametrize("T", synth.DECODE_SWEEP)
def test_decode_sweep(decode_layer, T):
    check_forward(decode_layer, T)


def test_prefill_full_size_sampled():
    L = synth.make_layer("prefill")
    dl = qmoe.DeviceLayer(L)
    check_forward(dl, L.T, tokens=covering_tokens(64))
    dl.close()


def test_fine_shared_zipf_full_size_sampled():
    L = synth.make_layer("fine")
    dl = qmoe.DeviceLayer(L)
    check_forward(dl, L.T, tokens=covering_tokens(64))
    dl.close()


def test_mixed_precision_full_size_sampled():
    L = synth.make_layer("mixed")
    dl = qmoe.DeviceLayer(L)
    check_forward(dl, L.T, tokens=covering_tokens(128))
    dl.close()


# ---------------------------------------------------------------------------
# several tiles with ragged tails, every token checked
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kw", [
    dict(name="fine", T=300, d=256, I=256, E=16, k=3, S=2),                 # INT4 + shared, ragged
    dict(name="prefill", T=517, d=256, I=384, E=4, k=2),                   # FP8, >128 rows per expert
    dict(name="mixed", T=777, d=384, I=256, E=8, k=4, zipf=1.0),           # INT8 / INT4 mixed, skew
    dict(name="tiny", T=1000, d=256, I=512, E=8, k=2),                     # INT8, BN=128 tiles
    dict(name="decode", T=200, d=512, I=256, E=32, k=8),                   # INT4, BN=64
    dict(name="mixed", T=333, d=256, I=256, E=8, k=2, fmt="mixed_fp8"),    # FP8 beside INT4 (bf16 MMAs)
])
def test_multi_tile_ragged(kw):
    kw = dict(kw)
    name = kw.pop("name")
    L = synth.make_layer(name, **kw)
    dl = qmoe.DeviceLayer(L)
    check_forward(dl, L.T)
    dl.close()


# ---------------------------------------------------------------------------
# degenerate cases
# ---------------------------------------------------------------------------
def test_single_token():
    dl = qmoe.DeviceLayer(synth.make_layer("tiny", T=1))
    check_forward(dl, 1)
    dl.close()


def test_k_equals_E_uniform_router_is_mean_of_experts():
    L = synth.make_layer("tiny", T=40, E=4, k=4, I=256)
    L.router_w = np.zeros_like(L.router_w)
    dl = qmoe.DeviceLayer(L)
    g = run_route(dl, 40)
    assert np.all(g["idx"] == np.arange(4))
    np.testing.assert_allclose(g["gates"], 0.25, rtol=0, atol=GATE_TOL)
    out = run_forward(dl, 40)
    x = O.bf16_to_f64(L.x)
    mean = np.mean([O.expert_ffn(x, *O.dequantize_expert(ex, L.d, L.I), L.I) for ex in L.experts], axis=0)
    assert O.rel_l2(out, mean) <= REL_L2
    assert float(np.abs(out - mean).max()) <= MAX_ABS
    dl.close()


def test_one_expert_is_dense_ffn():
    L = synth.make_layer("tiny", T=50, E=1, k=1)
    dl = qmoe.DeviceLayer(L)
    check_forward(dl, 50)
    dl.close()


def test_many_empty_experts():
    L = synth.make_layer("tiny", T=3, E=256, k=1, d=128, I=128)
    dl = qmoe.DeviceLayer(L)
    g, _ = check_route_from_x(dl, 3)
    assert (g["counts"] == 0).sum() >= 253
    check_forward(dl, 3)
    dl.close()


def test_max_tokens_and_smaller_T_reuse_handle():
    L = synth.make_layer("tiny", T=96)
    dl = qmoe.DeviceLayer(L, max_tokens=96)
    for T in (96, 17, 96, 1):
        check_forward(dl, T)
    dl.close()


def test_forward_host_matches_device_call():
    L = synth.make_layer("tiny", T=64)
    dl = qmoe.DeviceLayer(L)
    dev_out = run_forward(dl, 64)
    x_host = torch.from_numpy(L.x.view(np.int16).copy()).pin_memory()
    out_host = torch.empty((64, L.d), dtype=torch.int16).pin_memory()
    qmoe.qmoe_forward_host(dl.handle, x_host, 64, out_host, torch.cuda.current_stream())
    np.testing.assert_array_equal(to_f64(out_host), dev_out)
    dl.close()


def test_deterministic_across_calls():
    dl = qmoe.DeviceLayer(synth.make_layer("fine", T=300, d=256, I=256, E=16, k=3, S=2))
    a = run_forward(dl, 300)
    b = run_forward(dl, 300)
    np.testing.assert_array_equal(a, b)
    dl.close()


# ---------------------------------------------------------------------------
# argument errors at the boundary (nothing is launched)
# ---------------------------------------------------------------------------
def test_boundary_errors():
    L = synth.make_layer("tiny", T=8)
    dl = qmoe.DeviceLayer(L)
    out = torch.empty((8, L.d), dtype=torch.int16, device="cuda")
    for T in (0, 9, -1):
        with pytest.raises(qmoe.QmoeError) as ei:
            qmoe.qmoe_forward(dl.handle, dl.x, T, out)
        assert ei.value.status == qmoe.QMOE_ERR_INVALID
    with pytest.raises(qmoe.QmoeError):
        qmoe.qmoe_forward(dl.handle, None, 8, out)
    with pytest.raises(qmoe.QmoeError):
        qmoe.qmoe_forward(dl.handle, int(dl.x.data_ptr()) + 2, 8, out)   # misaligned
    g = run_route(dl, 8)   # still usable
    assert g["counts"].sum() == 8 * L.k
    dl.close()
