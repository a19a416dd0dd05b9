"""qmoe_route_topk_noalloc (routing with the library's fixed scratch array,
no handle, no allocation) against qmoe_route on the same inputs.

Both run the same router kernel with the same d-split, so expert indices
and gates must agree bit for bit.  Two consecutive calls with different
activations check that nothing from the first call (the partial logits
left in the shared scratch array) leaks into the second.  The file is collected last so it
also runs after every other GPU test has used the library in this process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from quantized_top_routed_b200 import qmoe, synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qmoe.load()


def _dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to("cuda")


def _route_handle(dl, x, T):
    L = dl.layer
    r = dict(idx=torch.empty((T, L.k), dtype=torch.int32, device="cuda"),
             gates=torch.empty((T, L.k), dtype=torch.float32, device="cuda"),
             counts=torch.empty(L.E, dtype=torch.int32, device="cuda"),
             offsets=torch.empty(L.E + 1, dtype=torch.int32, device="cuda"),
             sorted_token=torch.empty(T * L.k, dtype=torch.int32, device="cuda"),
             inv_pos=torch.empty((T, L.k), dtype=torch.int32, device="cuda"))
    qmoe.qmoe_route(dl.handle, x, None, T, r["idx"], r["gates"], r["counts"], r["offsets"], r["sorted_token"],
                    r["inv_pos"], torch.cuda.current_stream())
    torch.cuda.synchronize()
    return r["idx"].cpu().numpy(), r["gates"].cpu().numpy()


def _route_noalloc(L, w, b, x, T):
    idx = torch.full((T, L.k), -1, dtype=torch.int32, device="cuda")
    gates = torch.full((T, L.k), float("nan"), dtype=torch.float32, device="cuda")
    qmoe.qmoe_route_topk_noalloc(x, w, b, T, L.d, L.E, L.k, idx, gates, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return idx.cpu().numpy(), gates.cpu().numpy()


@pytest.mark.parametrize("name,T,kw", [
    ("decode", 256, {}),                                  # d-split router, 8 token tiles
    ("tiny", 77, {}),                                     # ragged last token tile
    ("decode", 1000, dict(E=40, k=5, I=128)),             # E not a multiple of 32, ragged T
    ("fine", 300, {}),                                    # router bias present
])
def test_noalloc_matches_route_on_two_consecutive_calls(name, T, kw):
    L = synth.make_layer(name, T=T, seed=11, **kw)
    dl = qmoe.DeviceLayer(L)
    try:
        w = _dev(L.router_w)
        b = _dev(L.router_b) if L.router_b is not None else None
        x1 = dl.x
        x2 = _dev(synth.make_layer(name, T=T, seed=12, **kw).x)
        for x in (x1, x2):
            ref_idx, ref_g = _route_handle(dl, x, T)
            idx, g = _route_noalloc(L, w, b, x, T)
            np.testing.assert_array_equal(idx, ref_idx)
            np.testing.assert_array_equal(g, ref_g)
        # the two inputs route differently, so the second call did not reuse the first's result
        assert not np.array_equal(_route_noalloc(L, w, b, x1, T)[0], _route_noalloc(L, w, b, x2, T)[0])
    finally:
        dl.close()


def test_noalloc_rejects_sizes_over_the_scratch():
    L = synth.make_layer("tiny", T=8, seed=1)
    w = _dev(L.router_w)
    T = qmoe.QMOE_ROUTE_STATIC_MAX_LOGITS // L.E + 1
    x = torch.zeros((8, L.d), dtype=torch.int16, device="cuda")   # never read: rejected first
    idx = torch.zeros((8, L.k), dtype=torch.int32, device="cuda")
    g = torch.zeros((8, L.k), dtype=torch.float32, device="cuda")
    with pytest.raises(qmoe.QmoeError, match="exceeds the fixed routing scratch"):
        qmoe.qmoe_route_topk_noalloc(x, w, None, T, L.d, L.E, L.k, idx, g)
