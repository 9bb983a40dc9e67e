"""Host-side launch planning of the QLoRA linear (no GPU needed): the fused GEMMs' K-split
choice and the launch counts, read through qlora_linear_plan.

The split rule is the library's documented one. Every CTA of the fused GEMM fills an SM, so s
splits of a grid of `tiles` tiles run in ceil(tiles * s / 148) waves. Each wave costs its
ceil(kb / s) k-blocks plus a fixed 4. The rule takes the cheapest s (the smallest on ties),
with at least 4 k-blocks per split. The tests restate that rule and also check invariants that
hold for any sensible split.
"""

import math

import pytest

from bit_nf4_quantized_dq_b200 import binding

SMS = 148
OVERHEAD = 4


def bn_for(cols):
    if cols >= 256:
        return 256
    if cols > 64:
        return 128
    if cols > 32:
        return 64
    if cols > 16:
        return 32
    return 16


def cost(tiles, kb, s):
    per = math.ceil(kb / s)
    used = math.ceil(kb / per)
    return math.ceil(tiles * used / SMS) * (per + OVERHEAD), used


def expected_splits(tiles, kb):
    if tiles >= SMS:
        return 1
    best, best_cost = 1, math.ceil(tiles / SMS) * (kb + OVERHEAD)
    for s in range(2, max(1, kb // 4) + 1):
        c, used = cost(tiles, kb, s)
        if c < best_cost:
            best, best_cost = used, c
    return best


SHAPES = [
    # (M tokens, K in, N out, r)
    (1, 5120, 5120, 64), (16, 5120, 5120, 64), (48, 4096, 11008, 16), (200, 5120, 13824, 64),
    (256, 5120, 5120, 64), (512, 4096, 4096, 64), (512, 11008, 4096, 64), (8192, 5120, 5120, 64),
    (8192, 5120, 13824, 64), (8192, 13824, 5120, 64), (3000, 3000, 4000, 8), (100, 8192, 22016, 256),
]


@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_fused_split_choice_follows_the_cost_rule(M, K, N, r):
    plan = binding.linear_plan(M, K, N, r)
    bn = bn_for(M)
    fwd_tiles = math.ceil(N / 128) * math.ceil(M / bn)
    dx_tiles = math.ceil(K / 128) * math.ceil(M / bn)
    assert plan["fwd_splits"] == expected_splits(fwd_tiles, math.ceil(K / 64))
    assert plan["dx_splits"] == expected_splits(dx_tiles, math.ceil(N / 64))


@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_split_invariants(M, K, N, r):
    plan = binding.linear_plan(M, K, N, r)
    bn = bn_for(M)
    for splits, tiles, kb in ((plan["fwd_splits"], math.ceil(N / 128) * math.ceil(M / bn), math.ceil(K / 64)),
                              (plan["dx_splits"], math.ceil(K / 128) * math.ceil(M / bn), math.ceil(N / 64))):
        assert splits >= 1
        per = math.ceil(kb / splits)
        assert (splits - 1) * per < kb                       # no empty split
        if splits > 1:
            assert per >= 4                                  # at least 4 k-blocks per split
            assert tiles < SMS                               # only grids smaller than the GPU split
            assert cost(tiles, kb, splits)[0] <= cost(tiles, kb, 1)[0]


def test_large_token_counts_never_split():
    for N, K in ((5120, 5120), (13824, 5120), (5120, 13824), (22016, 8192)):
        plan = binding.linear_plan(8192, K, N, 64)
        assert plan["fwd_splits"] == 1 and plan["dx_splits"] == 1


def test_launch_counts():
    # forward: t, finalize, fused (+ split reduce); backward: B^T, t split, u, finalize, fused dX
    # (+ split reduce), dA, finalize, dB, finalize
    for M, K, N, r in SHAPES:
        plan = binding.linear_plan(M, K, N, r)
        assert plan["fwd_launches"] == 3 + (plan["fwd_splits"] > 1)
        assert plan["bwd_launches"] == 9 + (plan["dx_splits"] > 1)
