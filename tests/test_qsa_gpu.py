"""GPU parity of the QSA block indexer (gdn_qsa_block_scores / gdn_qsa_select_blocks, through the
C ABI) against the fp64 oracle (oracle/qsa_indexer.py).

* pooled keys: max|dk|/max|k_ref| <= 1e-2 (they are stored in bf16); block bases exact;
* scores: every visible entry, max|dI|/max|I_ref| <= 1e-2 per document;
* selection: a top-k choice near a tie is decided by rounding, so the unique part is compared
  with the oracle -- every block whose oracle score lies farther than the score tolerance from
  the oracle's budget-th score must be selected exactly when the oracle selects it -- and the
  whole selection must be the exact top set (ties to the lower index) of the kernel's own
  scores, with the count min(budget, visible), sorted and -1 padded."""
import numpy as np
import pytest
import torch

import oracle.qsa_indexer as oq
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import make_qsa_inputs, varlen_lengths
from tests._metrics import max_rel

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _run(lengths, budget, seed, sample=None):
    inp = make_qsa_inputs(lengths, seed=seed)
    cu = inp["cu_seqlens"].numpy()
    g = {n: v.cuda() for n, v in inp.items()}
    maxlen = max(lengths) if lengths else 0
    sel, kh, base, sc = api.gdn_qsa_indexer(g["q"], g["k"], g["g"], g["cu_seqlens"], maxlen,
                                            budget=budget)
    torch.cuda.synchronize()
    kh_r, base_r = oq.pooled_keys(inp["k"], inp["g"], cu)
    np.testing.assert_array_equal(base.cpu().numpy(), base_r)
    nb = int(base_r[-1])
    if nb:
        assert max_rel(kh[:nb], kh_r) <= TOL
    sc = sc.cpu().double().numpy()
    sel = sel.cpu().numpy()
    sc_r = oq.block_scores(inp["q"], kh_r, base_r, cu)
    T = int(cu[-1])
    toks = range(T) if sample is None else sample
    for n in range(len(lengths)):  # scores, per document
        a, b = int(cu[n]), int(cu[n + 1])
        got = [sc[t, :len(sc_r[t])] for t in range(a, b)]
        ref = [sc_r[t] for t in range(a, b)]
        if any(len(r) for r in ref):
            den = max(np.abs(r).max() for r in ref if len(r))
            err = max(np.abs(x - r).max() for x, r in zip(got, ref) if len(r))
            assert err / den <= TOL, (n, err / den)
    for t in range(T):  # the selection is the exact top set of the kernel's own scores
        s = sc[t, :len(sc_r[t])]
        nk = min(budget, len(s))
        want = np.sort(np.lexsort((np.arange(len(s)), -s))[:nk])
        np.testing.assert_array_equal(sel[t, :nk], want)
        assert np.all(sel[t, nk:] == -1)
    for t in toks:  # the unique part agrees with the oracle's selection
        r = sc_r[t]
        if len(r) <= budget:
            np.testing.assert_array_equal(sel[t, :len(r)], np.arange(len(r)))
            continue
        ref_sel = oq.select_blocks(r, budget)
        kth = np.sort(r)[::-1][budget - 1]
        den = np.abs(r).max()
        clear = np.abs(r - kth) > TOL * den
        chosen = np.zeros(len(r), bool)
        chosen[sel[t][sel[t] >= 0]] = True
        ref_chosen = np.zeros(len(r), bool)
        ref_chosen[ref_sel[ref_sel >= 0]] = True
        np.testing.assert_array_equal(chosen[clear], ref_chosen[clear])


@pytest.mark.parametrize("lengths,budget", [
    ([7, 0, 130, 64, 3, 257], 8),
    ([1, 2, 3, 4, 5], 512),          # nothing or few blocks visible: everything selected
    ([600], 16),                     # several 128-block product tiles, ragged last tile
    ([33, 900, 31], 100),
])
def test_qsa_indexer_small(lengths, budget):
    _run(lengths, budget, seed=sum(lengths) + budget)


def test_qsa_indexer_long_varlen():
    """The long varlen workload's stream (T = 32768, 4 seeded documents) with the pages' budget
    of 512 blocks: pooled keys and every visible score in full; the selection's validity on
    every token and its agreement with the oracle on 2048 sampled tokens (the last of every
    document among them)."""
    lengths = varlen_lengths(32768, 4, seed=0)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rng = np.random.default_rng(0)
    sample = sorted(set(rng.integers(0, 32768, 2048).tolist()) | {int(c) - 1 for c in cu[1:]})
    _run(lengths, 512, seed=0, sample=sample)


def test_qsa_long_document_rejected_on_device():
    """A document longer than max_doc_len is recorded in the device status word and its scores
    are not written; the call itself returns OK (the lengths are only known on the device)."""
    inp = make_qsa_inputs([40, 12], seed=1)
    g = {n: v.cuda() for n, v in inp.items()}
    api.gdn_read_device_status(reset=True)
    api.gdn_qsa_block_scores(g["q"], g["k"], g["g"], g["cu_seqlens"], 16)
    torch.cuda.synchronize()
    assert api.gdn_read_device_status(reset=True) == 1  # GDN_ERR_INVALID_ARG
