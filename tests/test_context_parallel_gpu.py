"""The exchange step of a sequence split along time (context parallelism), through the bf16
kernels on one GPU: every segment's affine map S -> M S + N from two gdn_prefill runs (v = 0
from S0 = I, then S0 = 0), the maps composed from S0 in segment order, and every segment run
from its start state -- the steps dist.context_parallel_prefill takes on each rank, here for all
P segments in one process (no collective).  y and the final state are compared with the fp64
token loop over the whole sequence; the by-product errors are printed for the record."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.dist import segment_map, start_states
from gated_deltanet_linear_eqs_b200.inputs import make_inputs
from tests._metrics import S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P", [2, 4, 8])
@pytest.mark.parametrize("decay", ["benchmark", "slow"])
def test_context_parallel_maps_through_kernels(P, decay):
    B, T, H, d = 1, 4096, 4, 128
    inp = make_inputs(B, T, H, d, d, seed=50 + P, with_s0=True)
    if decay == "slow":
        rng = np.random.default_rng(P)
        inp["alpha"] = torch.from_numpy(rng.uniform(0.97, 0.9995, (B, T, H)).astype(np.float32))
    g = {n: t.cuda() for n, t in inp.items() if isinstance(t, torch.Tensor)}
    L = T // P
    sl = lambda x, r: x[:, r * L:(r + 1) * L].contiguous()
    maps = [segment_map(*(sl(g[n], r) for n in ("q", "k", "v", "alpha", "beta")))
            for r in range(P)]
    starts = start_states([m for m, _ in maps], [n for _, n in maps], g["s0"])
    ys = []
    for r in range(P):
        y, _ = api.gdn_prefill(*(sl(g[n], r) for n in ("q", "k", "v", "alpha", "beta")),
                               starts[r].contiguous())
        ys.append(y)
    torch.cuda.synchronize()
    y = torch.cat(ys, 1)
    yr, sr = oracle.forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["s0"])
    ey, es = max_rel(y, yr), frob_rel(starts[-1], sr)
    print(f"P={P} {decay}: y {ey:.2e}, final state {es:.2e}")
    assert ey <= Y_TOL
    assert es <= S_TOL
