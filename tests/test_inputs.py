"""The seeded input recipe shared by the tests and the bench (CPU): the same
seed gives the same bits, q, k, v, dout are drawn in that order from one
generator, the Q/K gain scales q and k only, and sampled rows are sorted,
distinct and in range."""

import numpy as np
import torch

from exact_io_aware_56_b200 import DECODE_WORKLOADS, WORKLOADS, make_decode_inputs, make_inputs, sample_rows


def test_same_seed_same_bits_other_seed_other_bits():
    a = make_inputs(1, 2, 1, 33, 64, 7)
    b = make_inputs(1, 2, 1, 33, 64, 7)
    c = make_inputs(1, 2, 1, 33, 64, 8)
    for n in ("q", "k", "v", "dout"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])
    assert tuple(a["q"].shape) == (1, 2, 33, 64) and tuple(a["k"].shape) == (1, 1, 33, 64)


def test_draw_order_and_gain():
    g = torch.Generator().manual_seed(11)
    draws = [torch.randn(1, 4, 50, 64, generator=g), torch.randn(1, 2, 50, 64, generator=g),
             torch.randn(1, 2, 50, 64, generator=g), torch.randn(1, 4, 50, 64, generator=g)]
    one = make_inputs(1, 4, 2, 50, 64, 11)
    two = make_inputs(1, 4, 2, 50, 64, 11, qk_gain=2.0, with_dout=False)
    for n, x in zip(("q", "k", "v", "dout"), draws):
        assert torch.equal(one[n], x.to(torch.bfloat16)), n
    # Scaling by 2 commutes with rounding to bf16, so the gain is exact.
    assert torch.equal(two["q"], 2 * one["q"]) and torch.equal(two["k"], 2 * one["k"])
    assert torch.equal(two["v"], one["v"]) and "dout" not in two


def test_decode_inputs_order():
    g = torch.Generator().manual_seed(5)
    want = [torch.randn(2, 4, 3, 64, generator=g), torch.randn(2, 2, 40, 64, generator=g),
            torch.randn(2, 2, 40, 64, generator=g)]
    got = make_decode_inputs(2, 4, 2, 3, 40, 64, 5)
    for n, x in zip(("q", "k", "v"), want):
        assert torch.equal(got[n], x.to(torch.bfloat16)), n


def test_workload_table_recipe():
    # Seeds 1000 + index (the two d = 64 variants share one draw); Q/K gain 2
    # only for the peaky 8192-token workload; decode seeds 1100 + index.
    seeds = {w.name: w.seed for w in WORKLOADS.values()}
    assert seeds["fwd_b1_h1_n128_d64"] == 1000
    assert seeds["fwdbwd_b4_h16_n2048_d64"] == seeds["fwdbwd_b4_h16_n2048_d64_causal"] == 1001
    assert [w.name for w in WORKLOADS.values() if w.qk_gain != 1.0] == ["fwdbwd_b2_h16_n8192_d128_causal_peaky"]
    assert sorted(w.seed for w in DECODE_WORKLOADS.values()) == [1100, 1101, 1102]


def test_sample_rows():
    r = sample_rows(8192, 256, 3)
    assert len(r) == 256 and np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < 8192
    assert np.array_equal(r, sample_rows(8192, 256, 3))
    assert np.array_equal(r, np.sort(np.random.default_rng(1003).choice(8192, 256, replace=False)))
