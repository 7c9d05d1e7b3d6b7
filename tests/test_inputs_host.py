"""The seeded input recipe (gated_deltanet_linear_eqs_b200/inputs.py): the documented workload
shapes and values that both the CUDA path and the oracle receive."""
import numpy as np
import torch

from gated_deltanet_linear_eqs_b200.inputs import (cu_seqlens_from, make_decode_step_inputs,
                                                   make_inputs, make_varlen_inputs,
                                                   varlen_lengths)


def test_varlen_lengths_of_the_packed_workload():
    """Seed 0 gives the four documents the benchmark names; the lengths sum to 32768 and are not
    multiples of the 64-token chunk."""
    lengths = varlen_lengths(32768, 4, seed=0)
    assert lengths == [16749, 4122, 7000, 4897]
    assert sum(lengths) == 32768 and all(x % 64 for x in lengths)
    cu = cu_seqlens_from(lengths)
    assert cu.dtype == torch.int32 and cu.tolist() == [0, 16749, 20871, 27871, 32768]


def test_inputs_are_seeded_and_rounded_once():
    a = make_inputs(1, 70, 2, 64, 64, seed=3, with_s0=True, with_dy=True)
    b = make_inputs(1, 70, 2, 64, 64, seed=3, with_s0=True, with_dy=True)
    for n in ("q", "k", "v", "alpha", "beta", "s0", "dy"):
        assert torch.equal(a[n], b[n]), n
    assert a["q"].dtype == torch.bfloat16 and a["alpha"].dtype == torch.float32
    # alpha = exp(-softplus(N(0,1))) and beta = sigmoid(N(0,1)) lie strictly inside (0, 1)
    for n in ("alpha", "beta"):
        x = a[n].numpy()
        assert np.all(x > 0) and np.all(x < 1), n
    assert abs(float(a["s0"].std()) - 0.02) < 0.005
    c = make_inputs(1, 70, 2, 64, 64, seed=4)
    assert not torch.equal(a["q"], c["q"])


def test_varlen_and_decode_layouts():
    d = make_varlen_inputs([5, 0, 9], 2, 64, 64, seed=1)
    assert d["q"].shape == (1, 14, 2, 64) and d["s0"].shape == (3, 2, 64, 64)
    assert d["cu_seqlens"].tolist() == [0, 5, 5, 14]
    t = make_decode_step_inputs(4, 3, 128, 128, step=7)
    assert t["q"].shape == (4, 3, 128) and t["alpha"].shape == (4, 3)
    # fresh tokens per step: seed = 1 + step
    u = make_decode_step_inputs(4, 3, 128, 128, step=8)
    assert not torch.equal(t["q"], u["q"])
