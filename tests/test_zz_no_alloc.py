"""The allocation-free junction backward entry point, called through the C ABI.

mls_junction_bwd_noalloc serves callers that cannot allocate device memory at
the point of the call -- programs whose device memory is owned by another
allocator, or latency-critical code that must not call cudaMalloc/cudaFree
(both can synchronise the device): it takes its scratch from a fixed array
inside the library.  This test runs it twice in a row on different shapes --
so stale scratch contents from the first call would show in the second -- and
checks each result against the ordinary entry point with a caller-supplied
workspace.  The file name makes pytest collect it last.
"""
import pytest
import torch

from lm_head_loss_junction_b200 import _lib, junction_bwd
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import assert_grad_close

pytestmark = pytest.mark.gpu


def _noalloc(x, o, E, dy, dE, accumulate):
    T, D = o.shape
    V, delta = E.shape
    do = torch.empty_like(o)
    de = torch.empty((T, delta), dtype=o.dtype, device=o.device)
    st = torch.zeros(1, dtype=torch.int32, device=o.device)
    code = _lib.lib().mls_junction_bwd_noalloc(
        x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V, delta, dy.data_ptr(), do.data_ptr(), de.data_ptr(),
        dE.data_ptr(), int(accumulate), _lib.MLS_BF16 if o.dtype == torch.bfloat16 else _lib.MLS_F32,
        st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert code == 0, _lib.STATUS_NAMES.get(code, code)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return do, de, dE


def _case(name, j, small):
    cfg = wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_heads=False)
    x = torch.from_numpy(d.x).cuda()
    return x, d.o[j].cuda(), d.E[j + 1].cuda(), wl.make_grad(cfg, j).cuda()


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        ("main3", 1, dict(batch=2, seq=700, V=512), True),      # Zipf ids: many tokens per id
        ("proxy2", 0, dict(batch=1, seq=300, V=4096), False),   # uniform ids, other shape
    ]
    for name, j, small, accumulate in cases:
        x, o, E, dy = _case(name, j, small)
        base = torch.randn(E.shape, dtype=torch.float32, device="cuda")
        dE_ref = base.clone()
        do_ref, de_ref, _ = junction_bwd(x, o, E, dy, dE=dE_ref, accumulate_dE=accumulate)
        dE_new = base.clone()
        do_new, de_new, _ = _noalloc(x, o, E, dy, dE_new, accumulate)
        assert_grad_close(do_new, do_ref, f"{name} do")
        assert_grad_close(de_new, de_ref, f"{name} de")
        assert_grad_close(dE_new - base, dE_ref - base, f"{name} dE")


def test_noalloc_rejects_sizes_beyond_its_array():
    x, o, E, dy = _case("proxy2", 0, dict(batch=1, seq=64, V=256))
    T, D = o.shape
    V_big = 4 << 20                       # the id tables alone would exceed the fixed array
    dE = torch.zeros(1, dtype=torch.float32, device="cuda")
    lib = _lib.lib()
    stream = torch.cuda.current_stream().cuda_stream
    code = lib.mls_junction_bwd_noalloc(
        x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V_big, E.shape[1], dy.data_ptr(),
        torch.empty_like(o).data_ptr(), None, dE.data_ptr(), 0, _lib.MLS_BF16, None, stream)
    assert code == 2                      # MLS_ERR_UNSUPPORTED, nothing launched
    # argument errors are reported first, as mls_junction_bwd reports them
    code = lib.mls_junction_bwd_noalloc(
        x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V_big, E.shape[1], None,
        torch.empty_like(o).data_ptr(), None, dE.data_ptr(), 0, _lib.MLS_BF16, None, stream)
    assert code == 1                      # MLS_ERR_INVALID_ARG: dy is NULL
