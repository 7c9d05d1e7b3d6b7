"""GPU parity of gdn_prefill_segmented (through the C ABI) against the fp64 token loop: the
segment maps, their scan and the pass from every segment's start state must reproduce the
unsegmented recurrence.  Bars: y max|dy|/max|y_ref| <= 1e-2, final state relative Frobenius
<= 1e-3."""
import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import make_inputs
from tests._metrics import S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,H,d,P,dtype", [
    (1, 1000, 2, 128, 4, "bf16"),   # ragged last segment and chunk
    (2, 333, 1, 64, 3, "bf16"),
    (1, 4096, 4, 128, 8, "bf16"),
    (1, 300, 2, 64, 5, "fp32"),     # the token-loop path
    (1, 100, 2, 128, 8, "bf16"),    # more segments asked for than chunks: two result
    (2, 200, 2, 128, 1, "bf16"),    # one segment: the plain prefill
])
def test_segmented_prefill_matches_token_loop(B, T, H, d, P, dtype):
    inp = make_inputs(B, T, H, d, d, dtype=dtype, seed=T + P, with_s0=True)
    g = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    y, sf = api.gdn_prefill_segmented(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["s0"],
                                      num_segments=P, scale=0.9)
    torch.cuda.synchronize()
    yr, sr = oracle.forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["s0"],
                            scale=0.9)
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(sf, sr) <= S_TOL
    assert api.gdn_read_device_status(reset=False) == 0
