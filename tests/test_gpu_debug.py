"""The QMOE_DEBUG build of the library on a B200.

That build checks every index the kernels take from data (expert ids, token
rows, schedule positions, the grouped GEMMs' tile tables) before using it; a
failed check skips the access and raises QMOE_ERR_BOUNDS instead of
faulting.  On valid inputs no check may fail, and the outputs must be the
same bits as the product build's: the checks add no arithmetic.  The debug
library runs in a child process, because QMOE_DEBUG=1 selects it when the
binding first loads.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from quantized_top_routed_b200 import qmoe, synth  # noqa: E402

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# INT8 with 128-row token blocks; INT4 with per-stage scaling; shared experts
# and a Zipf load; two weight formats in one layer.
CASES = [("tiny", {"T": 200}),
         ("decode", {"T": 64, "d": 512, "I": 256}),
         ("fine", {"T": 96, "d": 256, "E": 8, "k": 2, "I": 256, "S": 2}),
         ("mixed", {"T": 128, "d": 256, "E": 8, "k": 2, "I": 256})]

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from quantized_top_routed_b200 import qmoe, synth
assert qmoe.load().qmoe_debug_build() == 1, "the debug library was not loaded"
cases = json.loads(sys.argv[2])
for i, (name, kw) in enumerate(cases):
    L = synth.make_layer(name, **kw)
    dl = qmoe.DeviceLayer(L)
    out = torch.empty((L.T, L.d), dtype=torch.int16, device="cuda")
    qmoe.qmoe_forward(dl.handle, dl.x, L.T, out, torch.cuda.current_stream())
    torch.cuda.synchronize()
    qmoe.qmoe_check_error(dl.handle)          # raises on QMOE_ERR_BOUNDS
    np.save(sys.argv[3] + f"/debug_{i}.npy", out.cpu().numpy())
    dl.close()
print("child ok")
"""


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_debug_build_passes_its_checks_and_matches_the_product_bits(tmp_path):
    assert qmoe.load().qmoe_debug_build() == 0
    want = []
    for name, kw in CASES:
        L = synth.make_layer(name, **kw)
        dl = qmoe.DeviceLayer(L)
        try:
            out = torch.empty((L.T, L.d), dtype=torch.int16, device="cuda")
            qmoe.qmoe_forward(dl.handle, dl.x, L.T, out, torch.cuda.current_stream())
            torch.cuda.synchronize()
            qmoe.qmoe_check_error(dl.handle)
            want.append(out.cpu().numpy())
        finally:
            dl.close()
    env = dict(os.environ, QMOE_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, json.dumps(CASES), str(tmp_path)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    for i, (name, _) in enumerate(CASES):
        got = np.load(tmp_path / f"debug_{i}.npy")
        assert np.array_equal(got, want[i]), f"{name}: the debug build's output differs from the product build's"
