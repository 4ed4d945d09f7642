"""The bounded-wait path of the kernels, made to run out on purpose without
faulting or hanging anything: the statistics kernel's first wait (for its
key tiles) gets a 1 ns limit through cobs_set_wait_limit_ns, so every CTA gives
up at its first retry, records COBS_ERR_TIMEOUT in the status word, lets the
copies it started land (that wait keeps the full limit), frees its tensor
memory and returns.  A normal call on a re-initialised workspace must then
pass and give the records an undisturbed build gives."""

import pytest
import torch

import block_sparse_long_cobs_b200 as cb
from harness import Problem
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["single_32k", "tiny_4k"])
def test_stats_wait_that_runs_out_reports_timeout(name):
    w = WORKLOADS[name].scaled(seq_len=4096)
    p = Problem(w)
    p.build_stats()
    torch.cuda.synchronize()
    want = p.stats.clone()
    assert p.device_status() == 0
    p.stats.fill_(7)
    cb.cobs_set_wait_limit_ns(1)
    try:
        p.build_stats()
        torch.cuda.synchronize()
    finally:
        cb.cobs_set_wait_limit_ns(0)
    assert p.device_status() == cb.COBS_ERR_TIMEOUT
    cb.cobs_workspace_init(p.ws, p.ws_bytes)
    p.build_stats()
    torch.cuda.synchronize()
    assert p.device_status() == 0
    assert torch.equal(p.stats, want)
