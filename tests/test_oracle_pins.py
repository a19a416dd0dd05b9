"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against a value the pages print (a worked
example), a closed form, an invariant that characterises the result, a
library routine for a special case, or brute force on tiny inputs.  The
``test_mutation_*`` tests plant plausible mistakes in the oracle and check
that some pin catches each of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle.qmoe_oracle as O
from quantized_top_routed_b200 import synth


# ---------------------------------------------------------------------------
# helpers to build tiny layers by hand
# ---------------------------------------------------------------------------
def _int8_expert(w13, w2):
    w13 = np.asarray(w13, dtype=np.int8)
    w2 = np.asarray(w2, dtype=np.int8)
    return synth.Expert(fmt=synth.FMT_INT8, w13=w13, s13=np.ones(w13.shape[0], np.float32),
                        w2=w2, s2=np.ones(w2.shape[0], np.float32))


def _layer(x, experts, E, k, I, S=0, router_w=None, router_b=None):
    x = np.atleast_2d(np.asarray(x, dtype=np.float32))
    T, d = x.shape
    if router_w is None:
        router_w = np.zeros((E, d), np.float32)
    return synth.LayerInputs(name="hand", T=T, d=d, E=E, k=k, I=I, S=S,
                             x=synth.f32_to_bf16_bits(x), router_w=np.asarray(router_w, np.float32),
                             router_b=router_b, experts=experts)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _hand_layer(g, scale_down=(1, 2, 3)):
    rc = g["routed_case"]
    experts = [_int8_expert(g["w13"], np.asarray(g["w2"]) * m) for m in scale_down[:rc["E"]]]
    return _layer(g["x"], experts, E=rc["E"], k=rc["k"], I=g["I"])


# ---------------------------------------------------------------------------
# routing: worked example, brute force, ties, margins
# ---------------------------------------------------------------------------
def test_routing_flip_worked_example(golden_dir):
    g = _load(golden_dir, "routing_flip.json")
    for case in g["cases"]:
        z = np.array([case["logits"]])
        assert O.topk(z, 1)[0, 0] == case["top1"], case["note"]
        assert O.gates(z, O.topk(z, 1))[0, 0] == 1.0
    z = np.array([g["cases"][0]["logits"]])
    idx = O.topk(z, 2)
    assert list(idx[0]) == [0, 1]
    ga = 1.0 / (1.0 + math.exp(z[0, 1] - z[0, 0]))
    np.testing.assert_allclose(O.gates(z, idx)[0], [ga, 1.0 - ga], rtol=0, atol=1e-15)


@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (128, 8), (5, 5), (16, 1)])
def test_topk_matches_stable_argsort(E, k):
    rng = np.random.default_rng(E * 100 + k)
    z = rng.standard_normal((200, E))
    z[:50] = np.round(z[:50] * 2) / 2          # many exact ties
    ref = np.argsort(-z, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(O.topk(z, k), ref)


def test_topk_ties_go_to_lower_index():
    z = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    assert list(O.topk(z, 2)[0]) == [1, 2]
    assert list(O.topk(z, 4)[0]) == [1, 2, 4, 0]


def test_margin():
    z = np.array([[0.0, 2.0, 1.5, -1.0]])
    assert O.topk_margin(z, 1)[0] == 0.5
    assert O.topk_margin(z, 2)[0] == 1.5
    assert math.isinf(O.topk_margin(z, 4)[0])


# ---------------------------------------------------------------------------
# router logits with a bias
# ---------------------------------------------------------------------------
def test_router_logits_with_bias_hand_case(golden_dir):
    """Hand-worked logits, selection and gates with a non-zero bias and E != d."""
    g = _load(golden_dir, "router_bias.json")
    layer = _layer(g["x"], [], E=g["E"], k=g["k"], I=1, router_w=g["router_w"],
                   router_b=np.asarray(g["router_b"], np.float32))
    r = O.route(layer)
    np.testing.assert_array_equal(r["logits"], g["logits"])
    np.testing.assert_array_equal(r["idx"], g["idx"])
    np.testing.assert_allclose(r["gates"], g["gates"], rtol=1e-15, atol=0)


def test_router_logits_library_cross_check():
    """z = x Wr^T + b against torch's float64 linear layer on random inputs."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    T, d, E = 37, 96, 11
    x_bits = synth.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    w = rng.standard_normal((E, d)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    x64 = torch.from_numpy(synth.bf16_bits_as_f32(x_bits).astype(np.float64))
    ref = torch.nn.functional.linear(x64, torch.from_numpy(w.astype(np.float64)),
                                     torch.from_numpy(b.astype(np.float64))).numpy()
    np.testing.assert_allclose(O.router_logits(x_bits, w, b), ref, rtol=1e-13, atol=1e-13)
    ref0 = torch.nn.functional.linear(x64, torch.from_numpy(w.astype(np.float64))).numpy()
    np.testing.assert_allclose(O.router_logits(x_bits, w, None), ref0, rtol=1e-13, atol=1e-13)


def test_rel_l2_hand_value(golden_dir):
    c = _load(golden_dir, "router_bias.json")["rel_l2_case"]
    assert abs(O.rel_l2(c["a"], c["b"]) - c["value"]) < 1e-15
    assert O.rel_l2(c["b"], c["b"]) == 0.0
    # a second case: ||(0, 3, 4)|| / ||(0, 0, 10)|| = 5 / 10
    assert abs(O.rel_l2([0.0, 3.0, 14.0], [0.0, 0.0, 10.0]) - 0.5) < 1e-15


# ---------------------------------------------------------------------------
# gates
# ---------------------------------------------------------------------------
def test_gates_sum_to_one_and_match_softmax_over_selected():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((300, 64)) * 3
    for k in (1, 2, 6, 64):
        idx = O.topk(z, k)
        g = O.gates(z, idx)
        np.testing.assert_allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
        # closed form: softmax restricted to the selected logits
        zs = np.take_along_axis(z, idx.astype(np.int64), axis=1)
        ref = np.exp(zs - zs.max(axis=1, keepdims=True))
        ref /= ref.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(g, ref, rtol=1e-13, atol=0)
        assert np.all(np.diff(g, axis=1) <= 1e-15)  # slots in descending logit order
    assert np.all(O.gates(z, O.topk(z, 1)) == 1.0)


# ---------------------------------------------------------------------------
# schedule
# ---------------------------------------------------------------------------
def _random_idx(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (37, 8, 2), (64, 128, 8), (300, 7, 7), (513, 64, 6)])
def test_schedule_invariants(T, E, k):
    idx = _random_idx(T, E, k, T + E + k)
    s = O.schedule(idx, E)
    counts, offsets, st, inv = s["counts"], s["offsets"], s["sorted_token"], s["inv_pos"]
    assert counts.sum() == T * k
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[E] == T * k
    assert np.all(np.diff(offsets) == counts)
    # bijection: every slot filled once; permute then unpermute is the identity
    assert sorted(inv.ravel().tolist()) == list(range(T * k))
    for t in range(T):
        for j in range(k):
            p = inv[t, j]
            assert st[p] == t
            assert offsets[idx[t, j]] <= p < offsets[idx[t, j] + 1]
    # tokens strictly ascending inside each expert's segment
    for e in range(E):
        seg = st[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_schedule_positions_by_counting():
    """Brute force by the counting definition: pos(t, j) = offsets[e] +
    #{t' < t routed to e}, with offsets[e] = #{tasks of experts below e}."""
    T, E, k = 45, 9, 3
    idx = _random_idx(T, E, k, 7)
    s = O.schedule(idx, E)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            below = int(np.sum(idx < e))
            earlier = sum(1 for tp in range(t) if e in idx[tp])
            assert s["inv_pos"][t, j] == below + earlier


# ---------------------------------------------------------------------------
# dequantisation
# ---------------------------------------------------------------------------
def test_dequant_int8_closed_form():
    rng = np.random.default_rng(3)
    q = rng.integers(-127, 128, size=(5, 7)).astype(np.int8)
    s = rng.random(5).astype(np.float32)
    got = O.dequantize(O.FMT_INT8, q, s, 5, 7)
    for n in range(5):
        for kk in range(7):
            assert got[n, kk] == float(q[n, kk]) * float(s[n])


def test_int4_nibbles_by_hand():
    # 0x7F: low nibble 0xF = -1 (even k), high nibble 0x7 = +7 (odd k)
    # 0x80: low 0 , high 0x8 = -8;   0x19: low 9 = -7, high 1
    q = O.unpack_int4(np.array([[0x7F, 0x80, 0x19]], np.uint8), 6)
    assert q.tolist() == [[-1, 7, 0, -8, -7, 1]]


def test_int4_pack_roundtrip_and_group_scales():
    rng = np.random.default_rng(4)
    q = rng.integers(-8, 8, size=(3, 256)).astype(np.int8)
    np.testing.assert_array_equal(O.unpack_int4(synth.pack_int4(q), 256), q)
    # one distinct bf16 scale per (row, group of 128); q = 1 exposes the scale layout
    s_bits = synth.f32_to_bf16_bits(np.array([[0.5, 2.0], [0.25, 8.0], [1.0, 3.0]], np.float32))
    ones = synth.pack_int4(np.ones((3, 256), np.int8))
    w = O.dequantize(O.FMT_INT4, ones, s_bits, 3, 256)
    np.testing.assert_array_equal(w[:, :128], np.repeat([[0.5], [0.25], [1.0]], 128, axis=1))
    np.testing.assert_array_equal(w[:, 128:], np.repeat([[2.0], [8.0], [3.0]], 128, axis=1))


def test_e4m3_decode_golden(golden_dir):
    g = _load(golden_dir, "e4m3_codes.json")
    for code, val in g["codes"].items():
        assert O.decode_e4m3(np.array([int(code, 16)], np.uint8))[0] == val, code
    for code in g["nan_codes"]:
        assert np.isnan(O.decode_e4m3(np.array([int(code, 16)], np.uint8))[0])
    nz = O.decode_e4m3(np.array([int(g["negative_zero"], 16)], np.uint8))[0]
    assert nz == 0.0 and math.copysign(1.0, nz) < 0


def test_e4m3_decode_all_codes_vs_library():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.decode_e4m3(codes)
    both_nan = np.isnan(ref) & np.isnan(got)
    np.testing.assert_array_equal(got[~both_nan], ref[~both_nan])
    assert both_nan.sum() == 2


def test_fp8_dequant_closed_form():
    codes = np.array([[0x38, 0x40, 0xB8, 0x01]], np.uint8)
    s = np.array([0.5], np.float32)
    np.testing.assert_array_equal(O.dequantize(O.FMT_FP8, codes, s, 1, 4),
                                  [[0.5, 1.0, -0.5, 2.0 ** -10]])


# ---------------------------------------------------------------------------
# expert FFN and the whole layer
# ---------------------------------------------------------------------------
def test_hand_expert_ffn(golden_dir):
    g = _load(golden_dir, "hand_expert.json")
    w13 = np.asarray(g["w13"], np.float64)
    w2 = np.asarray(g["w2"], np.float64)
    y = O.expert_ffn(np.asarray([g["x"]], np.float64), w13, w2, g["I"])
    np.testing.assert_allclose(y[0], g["y"], rtol=1e-15, atol=1e-15)


def test_hand_routed_layer(golden_dir):
    g = _load(golden_dir, "hand_expert.json")
    rc = g["routed_case"]
    layer = _hand_layer(g)
    r = O.forward(layer, logits=np.asarray([rc["logits"]], np.float32))
    assert list(r["idx"][0]) == rc["idx"]
    np.testing.assert_allclose(r["gates"][0], rc["gates"], rtol=1e-15)
    np.testing.assert_allclose(r["out"][0], rc["out"], rtol=1e-14)


def test_E1_k1_is_the_dense_swiglu_ffn():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN (library cross-check)."""
    torch = pytest.importorskip("torch")
    L = synth.make_layer("tiny", T=16, E=1, k=1, I=128, d=256)
    r = O.forward(L)
    assert np.all(r["gates"] == 1.0)
    w13, w2 = O.dequantize_expert(L.experts[0], L.d, L.I)
    x = torch.from_numpy(O.bf16_to_f64(L.x))
    W1, W3 = torch.from_numpy(w13[:L.I]), torch.from_numpy(w13[L.I:])
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(x, W1)) * torch.nn.functional.linear(x, W3),
        torch.from_numpy(w2)).numpy()
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


def test_k_equals_E_uniform_gates_is_mean_of_experts():
    E = 4
    L = synth.make_layer("tiny", T=8, E=E, k=E, I=128, d=256)
    L.router_w = np.zeros_like(L.router_w)          # all logits equal -> gates 1/E
    r = O.forward(L)
    np.testing.assert_allclose(r["gates"], 1.0 / E, rtol=1e-15)
    assert np.all(r["idx"] == np.arange(E))          # ties resolved by index
    x = O.bf16_to_f64(L.x)
    dense = [O.expert_ffn(x, *O.dequantize_expert(ex, L.d, L.I), L.I) for ex in L.experts]
    np.testing.assert_allclose(r["out"], np.mean(dense, axis=0), rtol=1e-12, atol=1e-13)


def test_shared_expert_adds_with_weight_one():
    L = synth.make_layer("tiny", T=8, E=1, k=1, I=128, d=256, S=1)
    L.experts[1] = L.experts[0]                     # shared expert = routed expert
    r = O.forward(L)
    x = O.bf16_to_f64(L.x)
    y = O.expert_ffn(x, *O.dequantize_expert(L.experts[0], L.d, L.I), L.I)
    np.testing.assert_allclose(r["out"], 2.0 * y, rtol=1e-13, atol=1e-13)


def test_token_subset_matches_full_forward():
    L = synth.make_layer("tiny", T=24)
    full = O.forward(L)
    sub = [0, 5, 23, 11]
    part = O.forward(L, tokens=sub)
    np.testing.assert_array_equal(part["idx"], full["idx"][sub])
    np.testing.assert_allclose(part["out"], full["out"][sub], rtol=1e-13, atol=1e-13)


def test_from_logits_mode_uses_supplied_logits():
    L = synth.make_layer("tiny", T=10)
    z = np.random.default_rng(0).standard_normal((10, L.E)).astype(np.float32)
    r = O.route(L, logits=z)
    np.testing.assert_array_equal(r["idx"], np.argsort(-z.astype(np.float64), axis=1, kind="stable")[:, :L.k])


# ---------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# ---------------------------------------------------------------------------
def _pins_pass(golden_dir):
    checks = [test_hand_expert_ffn, test_hand_routed_layer, test_routing_flip_worked_example,
              test_e4m3_decode_golden, test_router_logits_with_bias_hand_case, test_rel_l2_hand_value]
    for chk in checks:
        try:
            chk(golden_dir)
        except (AssertionError, ValueError):
            return False
    try:
        test_topk_ties_go_to_lower_index()
        test_gates_sum_to_one_and_match_softmax_over_selected()
        test_schedule_positions_by_counting()
        test_int4_nibbles_by_hand()
        test_int4_pack_roundtrip_and_group_scales()
        test_shared_expert_adds_with_weight_one()
        test_dequant_int8_closed_form()
        test_router_logits_library_cross_check()
    except (AssertionError, ValueError):
        return False
    return True


def test_pins_pass_unmutated(golden_dir):
    assert _pins_pass(golden_dir)


MUTATIONS = {
    "gate_up_swapped": ("expert_ffn", lambda xr, w13, w2, I: (O.silu(xr @ w13[I:].T) * (xr @ w13[:I].T)) @ w2.T),
    "no_activation": ("silu", lambda a: a),
    "sigmoid_instead_of_silu": ("silu", lambda a: 1.0 / (1.0 + np.exp(-a))),
    "gates_not_renormalised": ("gates", lambda z, idx: np.take_along_axis(
        np.exp(z - z.max(1, keepdims=True)) / np.exp(z - z.max(1, keepdims=True)).sum(1, keepdims=True),
        np.asarray(idx, np.int64), axis=1)),
    "ties_to_higher_index": ("topk", lambda z, k: np.array(
        [sorted(range(z.shape[1]), key=lambda e: (-z[t, e], -e))[:k] for t in range(z.shape[0])], np.int32)),
    "e4m3_bias_8": ("decode_e4m3", lambda c: O.__dict__["_orig_decode_e4m3"](c) / 2.0),
    "int4_nibbles_swapped": ("unpack_int4", lambda p, K: O.__dict__["_orig_unpack_int4"](
        ((np.asarray(p, np.uint8) >> 4) | (np.asarray(p, np.uint8) << 4)).astype(np.uint8), K)),
    "schedule_tokens_descending": ("schedule", lambda idx, E: O.__dict__["_orig_schedule"](idx[::-1], E)),
    "router_bias_dropped": ("router_logits", lambda x, w, b: O.__dict__["_orig_router_logits"](x, w, None)),
    "router_bias_negated": ("router_logits", lambda x, w, b: O.__dict__["_orig_router_logits"](
        x, w, None if b is None else -np.asarray(b, np.float32))),
    "router_product_negated": ("router_logits", lambda x, w, b: O.__dict__["_orig_router_logits"](
        x, -np.asarray(w, np.float32), b)),
    "router_x_read_as_low_half": ("bf16_to_f64", lambda bits: (np.asarray(bits, np.uint16).astype(np.uint32))
                                  .view(np.float32).astype(np.float64)),
    "rel_l2_without_sqrt": ("rel_l2", lambda a, b: float(((np.asarray(a, np.float64) - np.asarray(b, np.float64)) ** 2)
                                                        .sum()) / max(float((np.asarray(b, np.float64) ** 2).sum()), 1e-300)),
    "rel_l2_relative_to_a": ("rel_l2", lambda a, b: O.__dict__["_orig_rel_l2"](b, a)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, golden_dir, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setitem(O.__dict__, "_orig_" + attr, getattr(O, attr))
    monkeypatch.setattr(O, attr, fn)
    assert not _pins_pass(golden_dir), f"planted mistake '{name}' went unnoticed"
