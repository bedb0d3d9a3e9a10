"""The C-ABI library loads, exports every symbol include/mls.h declares, and
rejects bad arguments synchronously (validation runs before any device call,
so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from lm_head_loss_junction_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mls.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mls_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), f"{n} missing from libmls.so"
    assert set(names) == set(_lib.PROTOTYPES), "binding prototypes out of sync with include/mls.h"


def test_status_strings_and_version():
    lib = _lib.lib()
    assert lib.mls_version() >= 100
    for code in range(8):
        assert lib.mls_status_string(code)


FAKE = 0x10000  # never dereferenced: validation fails first


def _loss_fwd(M=2, T=256, V=1024, D=(512, 1024), dt=_lib.MLS_BF16, h=None, W=None, ws=FAKE, ws_bytes=1 << 40,
              y=FAKE, alpha=0.3):
    lib = _lib.lib()
    h = h if h is not None else [FAKE] * M
    W = W if W is not None else [FAKE] * M
    return lib.mls_multiexit_loss_fwd(M, T, V, _lib.i64_array(D), y, _lib.ptr_array(h), _lib.ptr_array(W),
                                      alpha, dt, FAKE, FAKE, ws, ws_bytes, None, None)


def test_loss_argument_errors():
    assert _loss_fwd(M=0, D=()) == 1
    assert _loss_fwd(M=5, D=(64, 128, 192, 256, 320)) == 2           # more exits than supported
    assert _loss_fwd(D=(1024, 512)) == 1                             # widths must increase
    assert _loss_fwd(D=(512, 512)) == 1
    assert _loss_fwd(T=0) == 1
    assert _loss_fwd(y=None) == 1
    assert _loss_fwd(h=[FAKE, None]) == 1
    assert _loss_fwd(V=1000) == 2                                    # bf16 path needs V % 128 == 0
    assert _loss_fwd(D=(500, 1024)) == 2                             # bf16 path needs D % 64 == 0
    assert _loss_fwd(h=[FAKE + 8, FAKE]) == 2                        # misaligned
    assert _loss_fwd(ws=None) == 3
    assert _loss_fwd(ws_bytes=16) == 3
    assert _loss_fwd(alpha=float("nan")) == 1


def test_loss_valid_call_without_gpu_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _loss_fwd() == 7
    assert _loss_fwd(V=1000, dt=_lib.MLS_F32) == 7                   # fp32 path accepts any V


def test_junction_argument_errors():
    lib = _lib.lib()
    f = lib.mls_junction_fwd
    assert f(None, 8, FAKE, 64, FAKE, 10, 64, FAKE, None, _lib.MLS_BF16, None, None) == 1
    assert f(FAKE, 0, FAKE, 64, FAKE, 10, 64, FAKE, None, _lib.MLS_BF16, None, None) == 1
    assert f(FAKE, 8, FAKE, 60, FAKE, 10, 64, FAKE, None, _lib.MLS_BF16, None, None) == 2
    assert f(FAKE, 8, FAKE, 64, FAKE, 10, 62, FAKE, None, _lib.MLS_F32, None, None) == 2
    assert f(FAKE, 8, FAKE + 4, 64, FAKE, 10, 64, FAKE, None, _lib.MLS_BF16, None, None) == 2
    assert f(FAKE, 8, FAKE, 64, FAKE, 10, 64, None, None, _lib.MLS_BF16, None, None) == 1
    fv = lib.mls_junction_fwd_variant
    assert fv(FAKE, 8, FAKE, 64, FAKE, 10, 64, FAKE, None, 8, _lib.MLS_BF16, None, None) == 1   # unknown bit
    b = lib.mls_junction_bwd
    # dE requested without workspace
    assert b(FAKE, 8, FAKE, 64, FAKE, 10, 64, FAKE, FAKE, None, FAKE, 0, None, 0, _lib.MLS_BF16, None,
             None) == 3


def test_loss_options_reject_nonfinite_weights():
    lib = _lib.lib()
    opts = _lib.loss_options([1.0, float("nan")])
    code = lib.mls_multiexit_loss_fwd_opts(2, 256, 1024, _lib.i64_array([512, 1024]), FAKE,
                                           _lib.ptr_array([FAKE, FAKE]), _lib.ptr_array([FAKE, FAKE]), 0.3,
                                           _lib.MLS_BF16, FAKE, FAKE, FAKE, 1 << 40, ctypes.byref(opts), None, None)
    assert code == 1
    bad = _lib.LossOptions(None, 7)
    code = lib.mls_multiexit_loss_fwd_opts(2, 256, 1024, _lib.i64_array([512, 1024]), FAKE,
                                           _lib.ptr_array([FAKE, FAKE]), _lib.ptr_array([FAKE, FAKE]), 0.3,
                                           _lib.MLS_BF16, FAKE, FAKE, FAKE, 1 << 40, ctypes.byref(bad), None, None)
    assert code == 1                                                 # unknown distillation kind
    bad = _lib.LossOptions(None, 0, 3)
    code = lib.mls_multiexit_loss_fwd_opts(2, 256, 1024, _lib.i64_array([512, 1024]), FAKE,
                                           _lib.ptr_array([FAKE, FAKE]), _lib.ptr_array([FAKE, FAKE]), 0.3,
                                           _lib.MLS_BF16, FAKE, FAKE, FAKE, 1 << 40, ctypes.byref(bad), None, None)
    assert code == 1                                                 # teacher_grad must be 0 or 1


def test_agreement_argument_errors():
    lib = _lib.lib()
    one = lib.mls_exit_agreement(1, 16, 256, _lib.i64_array([64]), _lib.ptr_array([FAKE]), _lib.ptr_array([FAKE]),
                                 _lib.MLS_BF16, FAKE, FAKE, None, None, FAKE, 1 << 30, None, None)
    assert one == 1                                                  # needs a smaller exit
    nostats = lib.mls_exit_agreement(2, 16, 256, _lib.i64_array([64, 128]), _lib.ptr_array([FAKE, FAKE]),
                                     _lib.ptr_array([FAKE, FAKE]), _lib.MLS_BF16, None, FAKE, None, None, FAKE,
                                     1 << 30, None, None)
    assert nostats == 1


def test_workspace_queries():
    import torch
    from lm_head_loss_junction_b200 import junction_bwd_workspace, multiexit_loss_workspace
    f, b = multiexit_loss_workspace(8192, [1024, 2304, 4352], 49152, torch.bfloat16)
    # a bounded piece of G' (one 16384-column chunk of every exit), not all of it
    assert 3 * 8192 * 16384 * 2 <= b <= 3 << 29
    assert f >= (49152 // 128) * 5 * 8192 * 4
    f32f, f32b = multiexit_loss_workspace(256, [64, 128, 192], 512, torch.float32)
    assert f32b == 3 * 256 * 512 * 4
    assert junction_bwd_workspace(32768, 49152) >= 5 * 32768 * 4
    with pytest.raises(_lib.MLSError):
        multiexit_loss_workspace(10, [64, 64], 128, torch.bfloat16)


def test_multi_junction_argument_errors():
    lib = _lib.lib()
    D = _lib.i64_array([64, 128, 192])
    P = lambda *v: _lib.ptr_array(list(v))   # noqa: E731
    f = lib.mls_junction_fwd_multi
    ok = (FAKE, 8, 10, 2, D, P(FAKE, FAKE), P(FAKE, FAKE), P(FAKE, FAKE), None, _lib.MLS_BF16, None, None)
    assert f(*ok) == 7 or f(*ok) == 0                                  # valid: no device here
    assert f(FAKE, 8, 10, 0, D, P(FAKE), P(FAKE), P(FAKE), None, _lib.MLS_BF16, None, None) == 1
    assert f(FAKE, 8, 10, 4, D, P(FAKE), P(FAKE), P(FAKE), None, _lib.MLS_BF16, None, None) == 2
    assert f(FAKE, 8, 10, 2, _lib.i64_array([64, 64, 192]), P(FAKE, FAKE), P(FAKE, FAKE), P(FAKE, FAKE), None,
             _lib.MLS_BF16, None, None) == 1                            # widths must increase
    assert f(FAKE, 8, 10, 2, D, P(FAKE, FAKE), P(FAKE, FAKE), P(FAKE, None), None, _lib.MLS_BF16, None,
             None) == 1                                                 # missing output
    assert f(FAKE, 8, 10, 2, D, P(FAKE, FAKE + 4), P(FAKE, FAKE), P(FAKE, FAKE), None, _lib.MLS_BF16, None,
             None) == 2                                                 # misaligned input
    b = lib.mls_junction_bwd_multi
    # a table gradient without workspace
    assert b(FAKE, 8, 10, 2, D, P(FAKE, FAKE), P(FAKE, FAKE), P(FAKE, FAKE), P(FAKE, FAKE), None,
             P(None, FAKE), 0, None, 0, _lib.MLS_BF16, None, None) == 3
    n = ctypes.c_size_t()
    assert lib.mls_junction_bwd_multi_workspace(8192, 49152, 2, ctypes.byref(n)) == 0
    single = ctypes.c_size_t()
    lib.mls_junction_bwd_workspace(8192, 49152, ctypes.byref(single))
    assert single.value < n.value < 2 * single.value                   # one id grouping for both tables
