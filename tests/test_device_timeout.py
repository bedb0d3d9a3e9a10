"""The bounded device-side waits give up, report, and leave the stream usable.

Every barrier wait of the tensor-core kernels is bounded; when the limit runs
out the kernel records MLS_DEVFLAG_TIMEOUT, sets its abort flag and returns,
so a lost arrival never hangs the GPU.  mls_selftest_wait_timeout runs the
loss statistics kernel with its load warp issuing no loads -- barriers that
nothing completes -- and a 1 ms limit.  Nothing traps, faults or waits
without bound.
"""
import time

import pytest
import torch

from lm_head_loss_junction_b200 import _lib, multiexit_loss_workspace, new_status, status_read
from lm_head_loss_junction_b200 import workloads as wl
from tests.test_parity_loss import _check_all

pytestmark = pytest.mark.gpu


def _selftest(d, limit_ns, st):
    cfg = d.cfg
    y = torch.from_numpy(d.y).cuda()
    h = [t.cuda() for t in d.o]
    W = [t.cuda() for t in d.W]
    losses = torch.empty(2 * cfg.M, dtype=torch.float32, device="cuda")
    stats = torch.empty((3 * cfg.M - 1, cfg.T), dtype=torch.float32, device="cuda")
    fwd_b, _ = multiexit_loss_workspace(cfg.T, cfg.D, cfg.V, torch.bfloat16)
    ws = torch.empty(fwd_b, dtype=torch.uint8, device="cuda")
    return _lib.lib().mls_selftest_wait_timeout(
        cfg.M, cfg.T, cfg.V, _lib.i64_array(cfg.D), y.data_ptr(), _lib.ptr_array([t.data_ptr() for t in h]),
        _lib.ptr_array([t.data_ptr() for t in W]), losses.data_ptr(), stats.data_ptr(), ws.data_ptr(), fwd_b,
        int(limit_ns), st.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_wait_gives_up_reports_timeout_and_stream_stays_usable():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=300, V=1024)
    d = wl.make_inputs(cfg, with_tables=False)
    st = new_status()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert _selftest(d, 1_000_000, st) == 0                  # launched
    code, word = status_read(st)                             # synchronises
    elapsed = time.perf_counter() - t0
    assert code == 6 and (word & _lib.MLS_DEVFLAG_TIMEOUT), (code, word)
    assert elapsed < 2.0, elapsed                            # the 1 ms limit, not the library's 4 s
    assert status_read(st) == (0, 0)                         # the read cleared the word
    # the same stream, the ordinary calls: parity with the oracle as usual
    _check_all(d, cfg.alpha_d)


def test_selftest_argument_checks():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=128, V=256)
    d = wl.make_inputs(cfg, with_tables=False)
    st = new_status()
    assert _selftest(d, 10, st) == 1                         # limit below 1 us: MLS_ERR_INVALID_ARG
    assert _selftest(d, 5_000_000_000, st) == 1              # above the library's own 4 s
    assert status_read(st) == (0, 0)                         # nothing ran
