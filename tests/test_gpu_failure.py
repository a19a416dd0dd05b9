"""Failure detection of the grouped GEMMs, on a B200, without faulting the GPU.

Every barrier wait inside the grouped GEMM kernels is bounded.  Lowering the
bound far below the kernels' normal waits (qmoe_set_wait_limit) makes a wait
run out on purpose: the kernel must stop cleanly (drain its copies and MMAs,
free its tensor memory), raise the handle's error word, and leave the context
usable.  The test checks that qmoe_check_error then reports QMOE_ERR_TIMEOUT,
that the report clears, and that the next forward at the default bound
matches the fp64 oracle.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle.qmoe_oracle as O  # noqa: E402
from quantized_top_routed_b200 import qmoe, synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qmoe.load()


def _forward(dl, T):
    out = torch.empty((T, dl.layer.d), dtype=torch.int16, device="cuda")
    qmoe.qmoe_forward(dl.handle, dl.x, T, out, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return O.bf16_to_f64(out.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(T=64)),                       # INT8, 128-row token blocks
    ("decode", dict(T=32, d=512, I=256)),       # INT4 with per-stage scaling, 16-row token blocks
])
def test_wait_limit_runs_out_and_the_handle_recovers(name, kw):
    L = synth.make_layer(name, **kw)
    dl = qmoe.DeviceLayer(L)
    try:
        qmoe.qmoe_check_error(dl.handle)                 # clean start
        qmoe.qmoe_set_wait_limit(dl.handle, 100)         # far below one DRAM round trip
        _forward(dl, L.T)
        with pytest.raises(qmoe.QmoeError) as ei:
            qmoe.qmoe_check_error(dl.handle)
        assert ei.value.status == qmoe.QMOE_ERR_TIMEOUT
        qmoe.qmoe_check_error(dl.handle)                 # the report was cleared
        qmoe.qmoe_set_wait_limit(dl.handle, 0)           # default bound again
        got = _forward(dl, L.T)
        qmoe.qmoe_check_error(dl.handle)
        # the oracle evaluated on the GPU's own expert choice (routing is
        # compared separately by the parity tests)
        idx = torch.empty((L.T, L.k), dtype=torch.int32, device="cuda")
        scratch = [torch.empty((L.T, L.k), dtype=torch.float32, device="cuda"),
                   torch.empty(L.E, dtype=torch.int32, device="cuda"),
                   torch.empty(L.E + 1, dtype=torch.int32, device="cuda"),
                   torch.empty(L.T * L.k, dtype=torch.int32, device="cuda"),
                   torch.empty((L.T, L.k), dtype=torch.int32, device="cuda")]
        qmoe.qmoe_route(dl.handle, dl.x, None, L.T, idx, *scratch, torch.cuda.current_stream())
        torch.cuda.synchronize()
        ref = O.forward(L, idx_override=idx.cpu().numpy())
        assert O.rel_l2(got, ref["out"]) <= 1e-2
        assert float(np.abs(got - ref["out"]).max()) <= 3e-2
    finally:
        dl.close()
