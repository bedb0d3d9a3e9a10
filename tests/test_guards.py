"""Out-of-bounds write detection without a sanitizer: every output buffer of
the C ABI calls sits between guard regions filled with a known bit pattern,
and every input is compared with a copy taken before the call.  A kernel that
writes one element past (or before) its output, or into an input, changes a
guard or an input and fails here.  Shapes are ragged on purpose (token counts
that are not multiples of the 128-token tile, a vocabulary that ends in half
a tile, junction widths that leave lanes idle)."""
import math

import pytest
import torch

from lm_head_loss_junction_b200 import (junction_bwd, junction_bwd_workspace, junction_fwd, multiexit_loss_bwd,
                                        multiexit_loss_fwd, multiexit_loss_workspace)
from lm_head_loss_junction_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD_BYTES = 4096                     # keeps every inner buffer 256-byte aligned
PATTERN = 0x5A


class Guarded:
    """A tensor of `shape` with GUARD_BYTES of pattern on both sides."""

    def __init__(self, shape, dtype):
        esize = torch.empty(0, dtype=dtype).element_size()
        g = GUARD_BYTES // esize
        n = math.prod(shape)
        self.raw = torch.empty(n * esize + 2 * GUARD_BYTES, dtype=torch.uint8, device="cuda")
        self.raw.fill_(PATTERN)
        self.n_bytes = n * esize
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.n_bytes].view(dtype).view(shape)
        assert self.t.data_ptr() % 256 == 0 and g * esize == GUARD_BYTES

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[GUARD_BYTES + self.n_bytes:]
        return bool(torch.all(head == PATTERN)) and bool(torch.all(tail == PATTERN))


def _inputs(cfg):
    d = wl.make_inputs(cfg)
    x = torch.from_numpy(d.x).cuda()
    y = torch.from_numpy(d.y).cuda()
    o = [t.cuda() for t in d.o]
    E = [t.cuda() for t in d.E]
    W = [t.cuda() for t in d.W]
    return d, x, y, o, E, W


def _snapshot(ts):
    return [t.clone() for t in ts]


def _unchanged(ts, snap):
    return all(torch.equal(a.view(torch.uint8) if a.dtype != torch.int32 else a,
                           b.view(torch.uint8) if b.dtype != torch.int32 else b) for a, b in zip(ts, snap))


CASES = [
    ("main3", dict(batch=1, seq=333, V=640)),        # ragged token tile, vocabulary ends in half a tile
    ("suite4", dict(batch=1, seq=130, V=384)),
    ("proxy2", dict(batch=3, seq=55, V=256)),
    ("tiny3", None),                                   # fp32 path
]


def _cfg(name, small):
    return wl.CONFIGS[name] if small is None else wl.small_variant(wl.CONFIGS[name], **small)


@pytest.mark.parametrize("name,small", CASES)
def test_junction_writes_stay_in_bounds(name, small):
    cfg = _cfg(name, small)
    d, x, y, o, E, W = _inputs(cfg)
    T = cfg.T
    for j in range(cfg.M - 1):
        ins = [x, o[j], E[j + 1]]
        snap = _snapshot(ins)
        D, Dn, dl = cfg.D[j], cfg.D[j + 1], cfg.deltas[j + 1]
        yo = Guarded((T, Dn), o[j].dtype)
        sc = Guarded((T,), torch.float32)
        junction_fwd(x, o[j], E[j + 1], out=yo.t, scale_out=sc.t)
        assert yo.intact() and sc.intact(), "junction forward wrote outside its outputs"
        dy = wl.make_grad(cfg, j).cuda()
        snap_dy = dy.clone()
        do = Guarded((T, D), o[j].dtype)
        de = Guarded((T, dl), o[j].dtype)
        dE = Guarded((cfg.V, dl), torch.float32)
        ws = Guarded((junction_bwd_workspace(T, cfg.V),), torch.uint8)
        junction_bwd(x, o[j], E[j + 1], dy, do_out=do.t, de_out=de.t, dE=dE.t, workspace=ws.t)
        assert do.intact() and de.intact() and dE.intact() and ws.intact(), \
            "junction backward wrote outside its outputs or workspace"
        assert _unchanged(ins, snap) and torch.equal(dy, snap_dy), "junction wrote into an input"


@pytest.mark.parametrize("name,small", CASES)
@pytest.mark.parametrize("opts", [dict(), dict(distill="reverse_kl", teacher_grad=True),
                                  dict(distill="js", teacher_grad=True), dict(distill="accept", teacher_grad=True)])
def test_loss_writes_stay_in_bounds(name, small, opts):
    cfg = _cfg(name, small)
    d, x, y, o, E, W = _inputs(cfg)
    M, T, V = cfg.M, cfg.T, cfg.V
    fb, bb = multiexit_loss_workspace(T, list(cfg.D), V, o[0].dtype)
    rows = 4 * M - 2 if (opts.get("distill") in ("js", "accept") and M > 1) else 3 * M - 1
    ins = [y] + o + W
    snap = _snapshot(ins)
    losses = Guarded((2 * M,), torch.float32)
    stats = Guarded((rows, T), torch.float32)
    wsf = Guarded((fb,), torch.uint8)
    fwd_opts = {k: v for k, v in opts.items()}
    multiexit_loss_fwd(y, o, W, 0.3, losses=losses.t, stats=stats.t, workspace=wsf.t, **fwd_opts)
    assert losses.intact() and stats.intact() and wsf.intact(), "loss forward wrote outside its buffers"
    dh = [Guarded((T, cfg.D[m]), o[m].dtype) for m in range(M)]
    dW = [Guarded((V, cfg.D[m]), torch.float32) for m in range(M)]
    wsb = Guarded((bb,), torch.uint8)
    snap_stats = stats.t.clone()
    multiexit_loss_bwd(y, o, W, stats.t, 0.3, 1.0, dh=[g.t for g in dh], dW=[g.t for g in dW], workspace=wsb.t,
                       **opts)
    assert all(g.intact() for g in dh + dW) and wsb.intact(), "loss backward wrote outside its buffers"
    assert torch.equal(stats.t, snap_stats), "loss backward wrote into the statistics"
    assert _unchanged(ins, snap), "loss wrote into an input"
    if M > 1 and cfg.dtype == "bf16":
        import ctypes
        from lm_head_loss_junction_b200 import _lib
        n = ctypes.c_size_t()
        code = _lib.lib().mls_exit_agreement_workspace(M, T, _lib.i64_array(list(cfg.D)), V, _lib.MLS_BF16,
                                                       ctypes.byref(n))
        assert code == 0
        wsa = Guarded((n.value,), torch.uint8)
        metrics = Guarded((3 * (M - 1),), torch.float32)
        per_token = Guarded((3 * (M - 1), T), torch.float32)
        top1 = Guarded((M, T), torch.int32)
        code = _lib.lib().mls_exit_agreement(M, T, V, _lib.i64_array(list(cfg.D)),
                                             _lib.ptr_array([t.data_ptr() for t in o]),
                                             _lib.ptr_array([t.data_ptr() for t in W]), _lib.MLS_BF16,
                                             stats.t.data_ptr(), metrics.t.data_ptr(), per_token.t.data_ptr(),
                                             top1.t.data_ptr(), wsa.t.data_ptr(), n.value, None, None)
        assert code == 0
        assert metrics.intact() and per_token.intact() and top1.intact() and wsa.intact(), \
            "agreement pass wrote outside its buffers"
        assert _unchanged(ins, snap), "agreement pass wrote into an input"
