"""Boundary behaviour on the GPU: the split form of the fine-pass entry point,
and the kernels' bounded waits.

bsa_attention_prepare followed by bsa_attention_run must give, bit for bit,
what bsa_attention gives.  The bounded-wait self-test makes one wait run out
(an mbarrier nothing arrives on, a short limit): the kernel must return on its
own, report code 7 (timeout) through the workspace status word, and leave the
context usable for the next launch.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
from workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

CASES = [
    Workload("split_sinks_extra", B=1, H=2, N=2120, d=128, dtype="bf16", method="sol", q_block=64, k_block=64,
             tau=1.3, prefix_len=200, dense_rows=(72, 200), extra_tokens=64, grid=(3, 16, 40), seed=61),
    Workload("split_f32", B=1, H=2, N=1024, d=64, dtype="f32", method="sol", q_block=64, k_block=64, tau=1.0,
             seed=62),
    Workload("split_sla", B=1, H=2, N=2880, d=128, dtype="bf16", method="sla", q_block=128, k_block=64,
             keep_percent=15.0, centroid=0, grid=(4, 24, 30), seed=63),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_prepare_then_run_equals_attention(w):
    q, k, v = (t.cuda() for t in make_qkv(w, "cpu"))
    p = bsa.params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    bsa.bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count)
    bsa.bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, buf.extra_idx,
                   buf.extra_count, buf.ws)
    args = (buf.kbar, buf.vbar, buf.blk_count, buf.row_ptr, buf.col_idx, buf.extra_idx, buf.extra_count)
    out_a, out_b = torch.empty_like(q), torch.empty_like(q)
    lse_a, lse_b = torch.empty_like(buf.lse), torch.empty_like(buf.lse)
    bsa.bsa_attention(p, q, k, v, *args, out_a, lse_a, buf.ws)
    bsa.bsa_attention_prepare(p, q, k, v, *args, out_b, lse_b, buf.ws)
    bsa.bsa_attention_run(p, q, k, v, *args, out_b, lse_b, buf.ws)
    assert bsa.bsa_device_status(buf.ws) == 0
    assert torch.equal(out_a, out_b)
    assert torch.equal(lse_a, lse_b)


def _modified_centroids_needed(w, extra_idx, extra_count):
    """Entries the modified-centroid arrays need: per query block, the blocks its
    extra tokens came from that keep at least one token."""
    ei, ec = extra_idx.cpu().numpy(), extra_count.cpu().numpy()
    total = 0
    for r in range(ei.shape[0]):
        blk, cnt = np.unique(ei[r, :ec[r]] // 64, return_counts=True)
        total += int(np.sum(np.minimum(64, w.N - 64 * blk) - cnt > 0))
    return total


def _layer_with_capacity(w, q, k, v, per_row):
    p = bsa.params_for(w, q)
    p.modcent_per_row = per_row
    buf = bsa.Buffers(p, q.device)
    out = torch.empty_like(q)
    bsa.run_layer(p, q, k, v, out, buf)
    return buf, out, bsa.bsa_device_status(buf.ws)


def test_modified_centroid_capacity():
    """A capacity that holds exactly the entries the inputs need gives, bit for bit,
    the worst-case capacity's result; a smaller one is reported through the status
    word (BSA_ERR_CAPACITY) without a fault, and the next call runs clean."""
    w = CASES[0].replace(name="capacity", extra_tokens=256, N=3000, grid=(3, 20, 50), prefix_len=0,
                         dense_rows=(0, 0), seed=64)
    q, k, v = (t.cuda() for t in make_qkv(w, "cpu"))
    buf0, out0, st0 = _layer_with_capacity(w, q, k, v, 0)
    assert st0 == 0
    need = _modified_centroids_needed(w, buf0.extra_idx, buf0.extra_count)
    assert need > w.rows                                   # several per query block
    per_row = -(-need // w.rows)
    buf1, out1, st1 = _layer_with_capacity(w, q, k, v, per_row)
    assert st1 == 0
    assert torch.equal(out0, out1)
    _, out2, st2 = _layer_with_capacity(w, q, k, v, 1)
    assert st2 == bsa.BSA_ERR_CAPACITY
    assert bool(torch.isfinite(out2.float()).all())
    _, out3, st3 = _layer_with_capacity(w, q, k, v, per_row)
    assert st3 == 0
    assert torch.equal(out0, out3)


@pytest.mark.parametrize("case", ["extra_dense_hc1", "b2_ragged_hc2"])
def test_layer_from_host_memory_equals_device_layer(case):
    """bsa_layer_host (heads in chunks, copies on their own streams overlapping the
    kernels) gives, bit for bit, what the whole layer run on device arrays gives:
    heads are independent, and with at most 256 key blocks the dense rows are not
    split over keys, so every chunk computes exactly what the whole layer does."""
    w, hc = {
        "extra_dense_hc1": (CASES[0], 1),
        "b2_ragged_hc2": (Workload("host_b2", B=2, H=5, N=1500, d=128, dtype="bf16", method="sol", q_block=64,
                                   k_block=64, tau=1.0, grid=(3, 10, 50), seed=65), 2),
    }[case]
    qc, kc, vc = make_qkv(w, "cpu")
    q, k, v = (t.cuda() for t in (qc, kc, vc))
    p = bsa.params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    ref = torch.empty_like(q)
    bsa.run_layer(p, q, k, v, ref, buf)
    assert bsa.bsa_device_status(buf.ws) == 0
    hq, hk, hv = (t.contiguous().pin_memory() for t in (qc, kc, vc))
    hout = torch.full(hq.shape, float("nan"), dtype=hq.dtype).pin_memory()
    hl = bsa.HostLayer(p, q.device, hc)
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(2):                                   # twice: the second call reuses every buffer
        bsa.bsa_layer_host(p, hq, hk, hv, hout, hl, None, cin, cout)
        assert bsa.bsa_device_status(hl.buf.ws) == 0     # synchronises the stream the call ended on
        assert torch.equal(hout, ref.cpu())
        hout.fill_(float("nan"))
    bsa.bsa_layer_host(p, hq, hk, hv, hout, hl)          # one stream for everything
    assert bsa.bsa_device_status(hl.buf.ws) == 0
    assert torch.equal(hout, ref.cpu())


def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    bsa.bsa_selftest_bounded_wait(ws, 2_000_000)          # about 1 ms at the B200's clock
    stop.record()
    assert bsa.bsa_device_status(ws) == 7                 # BSA_DEV_TIMEOUT
    assert start.elapsed_time(stop) < 1000.0
    assert bsa.bsa_device_status(ws) == 0                 # read-and-clear
    # the context is still usable
    x = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 499500.0


def test_bounded_wait_rejects_bad_limits():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(bsa.BsaError):
        bsa.bsa_selftest_bounded_wait(ws, 0)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_selftest_bounded_wait(ws, 3_000_000_000)
