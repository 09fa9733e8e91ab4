"""Per-step policy ("BlockSparseAttention - ComfyUI Built-in Node
Documentation", general inputs start_percent / end_percent / dense_blocks /
min_tokens and "constraints and limitations"; "minimax-h3-chunk-star7" README,
"Hybrid").

CPU: the oracle's restatement is pinned to the values the pages state
(tests/golden/policy_examples.txt), and the library's bsa_policy_decide must
return the oracle's decision on a grid of inputs, errors included.
GPU: bsa.run_step takes the sparse path exactly as run_layer does, and a dense
decision gives dense softmax attention over every row.
"""
import itertools
import math
import os
import random

import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
from oracle import policy as opol

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "policy_examples.txt")


def _golden():
    lines = [l.split("#")[0].strip() for l in open(GOLDEN)]
    return [l for l in lines if l]


def test_oracle_defaults_match_the_pages():
    pol = opol.Policy()
    for line in _golden():
        if line.startswith("default "):
            _, name, value = line.split()
            assert getattr(pol, name) == type(getattr(pol, name))(float(value) if "." in value else int(value))


def test_oracle_dense_blocks_example():
    for line in _golden():
        if line.startswith("dense_blocks"):
            spec = line.split('"')[1]
            kind, *blocks = line.split('"')[2].split()
            want = opol.BLOCK if kind == "dense" else opol.SPARSE
            pol = opol.Policy(start_percent=0.0, dense_blocks=spec)
            for b in blocks:
                assert opol.decide(pol, 20000, int(b), 0.5) == want, (spec, b)


def test_oracle_hybrid_four_steps():
    for line in _golden():
        if line.startswith("hybrid"):
            _, n, kind, *steps = line.split()
            want = opol.HYBRID if kind == "dense" else opol.SPARSE
            pol = opol.Policy(start_percent=0.0, hybrid=True)
            for s1 in steps:                              # the pages count steps from 1
                assert opol.decide(pol, 20000, 0, 0.5, int(s1) - 1, int(n)) == want


def test_oracle_window_and_length_edges():
    pol = opol.Policy()
    assert opol.decide(pol, 12288, 0, 0.2) == opol.SPARSE           # window closed at start
    assert opol.decide(pol, 12288, 0, math.nextafter(0.2, 0.0)) == opol.WINDOW
    assert opol.decide(pol, 12288, 0, 1.0) == opol.SPARSE           # and at end
    assert opol.decide(pol, 12287, 0, 0.5) == opol.SHORT
    assert opol.decide(opol.Policy(dense_blocks="3"), 20000, -1, 0.5) == opol.SPARSE   # no block index
    with pytest.raises(ValueError):
        opol.decide(opol.Policy(hybrid=True), 20000, 0, 0.5)                 # step unknown


SPECS = ["", "0, 1, 47-49", " 5 ", "2-2,7", "1,,3,", "0-3, 10-12, 40", "x", "3-1", "1-", "-2", "4 5", "1-2-3"]


def _c_decide(pol, *args):
    cpol = bsa.make_policy(pol.start_percent, pol.end_percent, pol.min_tokens, pol.hybrid, pol.hybrid_guard_steps,
                           pol.dense_blocks)
    try:
        return bsa.bsa_policy_decide(cpol, *args)
    except bsa.BsaError as e:
        assert e.status == 1                                              # BSA_ERR_INVALID_ARG
        return "error"


def _o_decide(pol, *args):
    try:
        return opol.decide(pol, *args)
    except ValueError:
        return "error"


def test_library_policy_matches_oracle():
    rng = random.Random(5)
    cases = 0
    for spec in SPECS:
        for hybrid, guard in ((False, 1), (True, 1), (True, 2), (True, 0)):
            for start, end in ((0.2, 1.0), (0.0, 0.0), (0.5, 0.3), (0.25, 0.75)):
                pol = opol.Policy(start, end, 1024, hybrid, guard, spec)
                for n_tok, blk, prog in itertools.product((1, 1023, 1024, 77000), (-1, 0, 2, 11, 48),
                                                          (0.0, 0.2, 0.3, 0.75, 1.0)):
                    n_steps = rng.choice([0, 1, 2, 4, 30])
                    step = rng.choice([-1, 0, 1, 2, 3, 29, 30])
                    args = (n_tok, blk, prog, step, n_steps)
                    assert _c_decide(pol, *args) == _o_decide(pol, *args), (pol, args)
                    cases += 1
    assert cases > 10000
    # invalid windows and progress
    for bad in (opol.Policy(start_percent=-0.1), opol.Policy(end_percent=1.5)):
        assert _c_decide(bad, 20000, 0, 0.5, -1, 0) == _o_decide(bad, 20000, 0, 0.5, -1, 0) == "error"
    assert _c_decide(opol.Policy(), 20000, 0, float("nan"), -1, 0) == "error"




@pytest.mark.gpu
def test_run_step_sparse_and_dense_paths():
    import oracle
    from workloads import Workload, make_qkv
    w = Workload("policy_step", B=1, H=2, N=2120, d=128, dtype="bf16", method="sol", q_block=64, k_block=64,
                 tau=1.3, prefix_len=200, dense_rows=(72, 200), grid=(3, 16, 40), seed=71)
    qc, kc, vc = make_qkv(w, "cpu")
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    p = bsa.params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    pol = bsa.make_policy(min_tokens=1024, hybrid=True, dense_blocks="3")
    # sparse: the same result as the plain hot path
    out_s = torch.empty_like(q)
    assert bsa.run_step(p, pol, q, k, v, out_s, buf, block_index=0, progress=0.5, step=1, n_steps=4) == \
        bsa.BSA_RUN_SPARSE
    ref = torch.empty_like(q)
    bsa.run_layer(p, q, k, v, ref, bsa.Buffers(p, q.device))
    assert torch.equal(out_s, ref)
    # dense (a guard step, a listed block, a short sequence): dense attention on every row
    dense_all = w.replace(tau=-math.inf, prefix_len=0, dense_rows=(0, 0))
    raw = [oracle.as_raw(t) for t in (qc, kc, vc)]
    res = oracle.routing(dense_all, *raw)
    want, _ = oracle.layer_rows(dense_all, *raw, res, oracle.all_tokens(dense_all))
    for kw, reason in ((dict(block_index=0, step=0), bsa.BSA_DENSE_HYBRID),
                       (dict(block_index=3, step=2), bsa.BSA_DENSE_BLOCK)):
        out_d = torch.empty_like(q)
        assert bsa.run_step(p, pol, q, k, v, out_d, buf, progress=0.5, n_steps=4, **kw) == reason
        got = out_d.float().cpu().permute(0, 2, 1, 3).reshape(-1, w.d).numpy()
        err = np.abs(got - want)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (reason, err.max(), err.mean())
