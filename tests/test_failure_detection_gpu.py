"""Failure detection on the GPU without a fault: a bounded wait that runs out.

dsa_set_wait_budget_ns shortens the budget of the indexer's pipeline waits to 1 ns, so the first
wait of a launch that is not already complete gives up. The launch must then record
DSA_ERR_DEVICE_TIMEOUT (with the indexer's location tag) in the workspace's status word, every
role must end (the teardown still lets in-flight copies and MMAs land under its own budget), the
host reads the status through dsa_get_device_status, and the context stays usable: the next call
with the default budget is clean and selects what the oracle selects.
"""
import pytest
import torch

import synthetic
from tests.dsa_cases import RowOracle, check_selection

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_long_indexer_b200")


def test_a_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    cfg = synthetic.config("prefill_4k")
    seed = 41
    g = synthetic.gen_all(cfg, seed, "cuda")
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    dsa.dsa_set_wait_budget_ns(1)
    try:
        dsa.indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"], cfg.topk,
                         ws)
        torch.cuda.synchronize()
        status, detail = dsa.dsa_get_device_status(ws.buf)
    finally:
        dsa.dsa_set_wait_budget_ns(0)
    assert status == dsa.DSA_ERR_DEVICE_TIMEOUT
    assert detail >> 16 == 1                            # recorded by the indexer kernel's waits
    assert dsa.dsa_get_device_status(ws.buf)[0] == dsa.DSA_OK      # cleared by the read
    idx = dsa.indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"],
                           cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    ro = RowOracle(cfg, seed)
    idx_h = idx.cpu().numpy()[0]
    for i in synthetic.sample_rows(cfg.n_q, 24, seed, extra=[0, cfg.n_q - 1]):
        _, scores = ro.indexer(0, i)
        check_selection(idx_h[i], scores, cfg.topk, i)
