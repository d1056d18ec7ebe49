"""Failure handling without faulting the GPU: a bounded device wait that runs out, the host
watchdog, and an allocation that cannot succeed.  Each leaves the context usable, checked
by a forward that still matches the oracle afterwards."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import StcaModel
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"


def _forward_still_matches_oracle():
    wl = make_stca(2, users=2, L=300, n_items=5000)
    m = StcaModel(wl)
    x = m.inputs(wl)
    z = torch.empty((x["t_tot"], wl["cfg"]["d"]), device=dev)
    B.check(m.forward(x, z))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    assert R.row_rel_err(z.cpu().numpy(), R.stca_forward(wl)[0]) <= 2e-2


def test_bounded_wait_times_out_and_the_watchdog_reports_it():
    s = torch.cuda.Stream()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    B.check(B.stca_k_wait_selftest(err, s))
    # the kernel waits about 2 s before giving up: a short watchdog deadline passes first
    assert B.stca_stream_wait(s, 100) == B.ERR_TIMEOUT
    assert B.stca_stream_wait(s, 20_000) == B.OK
    assert err.item() == B.ERR_TIMEOUT
    assert B.stca_stream_wait(s, 0) == B.OK   # nothing left to wait for
    _forward_still_matches_oracle()


def test_allocation_failure_is_reported_and_leaks_nothing():
    free0, _ = torch.cuda.mem_get_info()
    cfg = B.StcaConfig(mode=B.MODE_STCA, M=3, d=512, H=8, hidden=1024, dtype=B.BF16, score=B.SOFTMAX,
                       time_buckets=16, max_users=1 << 20, max_tokens=(1 << 31) - 1, max_targets=1 << 24,
                       dedup=2, ln_eps=1e-5)
    h = ctypes.c_void_p()
    rc = B.lib().stca_create(ctypes.byref(cfg), ctypes.byref(h))
    assert rc in (B.ERR_CUDA, B.ERR_CAPACITY, B.ERR_INVALID_ARG) and h.value is None
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) < (256 << 20)
    _forward_still_matches_oracle()
