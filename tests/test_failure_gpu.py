"""The failure path of the library's bounded waits, on the GPU, without faulting or hanging it.

Every wait inside the kernels gives up after a limit, records GDN_ERR_TIMEOUT in the device
status word and returns.  ``gdn_selftest_wait_timeout`` launches a kernel whose wait (on a
barrier that nothing arrives on) runs out after 1 ms; the host must then read the error, clear
it, and the device must still compute correctly."""
import time

import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200._abi import GDN_ERR_TIMEOUT
from gated_deltanet_linear_eqs_b200.inputs import make_inputs
from tests._metrics import S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_device_stays_usable():
    api.gdn_read_device_status(reset=True)            # start from a clear word
    t0 = time.perf_counter()
    api.gdn_selftest_wait_timeout(1_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert api.gdn_read_device_status(reset=True) == GDN_ERR_TIMEOUT
    assert api.gdn_read_device_status(reset=False) == 0
    assert elapsed < 5.0                               # gave up; did not hang
    inp = make_inputs(1, 100, 2, 64, 64, seed=31, with_s0=True)
    g = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    y, sf = api.gdn_prefill(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["s0"])
    torch.cuda.synchronize()
    yr, sr = oracle.forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["s0"])
    assert max_rel(y, yr) <= Y_TOL and frob_rel(sf, sr) <= S_TOL
    assert api.gdn_read_device_status(reset=False) == 0
