"""Checks of the seeded input generator (no method arithmetic lives there)."""
import json
import os

import numpy as np
import torch

from lm_head_loss_junction_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def test_configs_match_the_pages_shapes():
    fig = json.load(open(GOLDEN))
    main = wl.CONFIGS["main3"]
    assert list(main.D) == fig["widths"]["value"]
    assert main.deltas == (1024, 1280, 2048)
    # the two small heads add about 0.16B parameters; one 2304-wide bf16 head is about 0.23 GB
    small = main.V * (main.D[0] + main.D[1])
    assert abs(small / fig["small_heads_params"]["value"] - 1) < fig["small_heads_params"]["approx_rel"]
    one = main.V * fig["one_head_bytes"]["width"] * fig["one_head_bytes"]["bytes_per_param"]
    assert abs(one / fig["one_head_bytes"]["value"] - 1) < fig["one_head_bytes"]["approx_rel"]
    for k in wl.CONFIG_ORDER:
        c = wl.CONFIGS[k]
        assert all(a < b for a, b in zip(c.D, c.D[1:])), "widths strictly increase"
        assert sum(c.deltas) == c.D[-1]
        assert c.alpha_d == fig["alpha_d"]["value"]


def test_inputs_are_deterministic_and_shaped():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=2, seq=16, V=256)
    a = wl.make_inputs(cfg)
    b = wl.make_inputs(cfg)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.y, b.y)
    for m in range(cfg.M):
        assert a.o[m].dtype == torch.bfloat16 and tuple(a.o[m].shape) == (32, cfg.D[m])
        assert tuple(a.E[m].shape) == (256, cfg.deltas[m])
        assert tuple(a.W[m].shape) == (256, cfg.D[m])
        assert torch.equal(a.o[m], b.o[m]) and torch.equal(a.W[m], b.W[m])
    assert a.x.min() >= 0 and a.x.max() < 256


def test_targets_are_next_tokens_within_each_sequence():
    cfg = wl.small_variant(wl.CONFIGS["proxy2"], batch=3, seq=10, V=64)
    d = wl.make_inputs(cfg, with_heads=False, with_tables=False)
    x = d.x.reshape(3, 10)
    y = d.y.reshape(3, 10)
    assert np.array_equal(y[:, :-1], x[:, 1:])
    assert y.min() >= 0 and y.max() < 64


def test_zipf_ids_are_rank_ordered():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=4, seq=4096, V=1000)
    d = wl.make_inputs(cfg, with_heads=False, with_tables=False)
    cnt = np.bincount(d.x, minlength=1000)
    # probability of rank k is proportional to k^-1.1: id 0 is the most frequent
    assert cnt[0] == cnt.max()
    p0 = 1.0 / np.sum(np.arange(1, 1001, dtype=np.float64) ** -1.1)
    assert abs(cnt[0] / d.x.size - p0) < 0.02


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is halfway between two bf16 values: ties go to the even one (1.0)
    a = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    t = wl.to_storage(a, "bf16").to(torch.float64).numpy()
    assert t[0] == 1.0 and t[1] == 1.0 + 2.0 ** -6
