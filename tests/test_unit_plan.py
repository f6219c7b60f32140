"""Host logic of the tensor-core product over calibration tokens: how its work
is cut into units (no GPU needed).  The decode below restates, for the test,
how each unit's CTA pair finds its tile and token stages; the checks are that
every (tile, stage) is covered exactly once, that no part is empty or short,
and that the last round of units is spread over every cluster."""
import itertools

import pytest

import post_weight_quantization_07_b200 as oc

BK = 128  # tokens per stage


def decode(plan, n_tok, n_tiles, u):
    kcs, n_kc, k, full, units = plan
    stages_total = (n_tok + BK - 1) // BK
    b, part, kk = u, 0, 1
    if u >= full:
        kk = k
        b = full + (u - full) // k
        part = (u - full) % k
    tile = b % n_tiles
    c0 = (b // n_tiles) * kcs
    ln = min(stages_total, c0 + kcs) - c0
    return tile, c0 + ln * part // kk, c0 + ln * (part + 1) // kk


@pytest.mark.parametrize("n_tok,n_tiles,clusters", list(itertools.product(
    [100, 1000, 8192, 8192 + 33, 32768, 65536, 131072 + 777], [1, 3, 16, 136, 256, 1540], [1, 7, 70, 74])))
def test_units_cover_every_stage_once(n_tok, n_tiles, clusters):
    plan = oc.oc_test_unit_plan(n_tok, n_tiles, clusters)
    kcs, n_kc, k, full, units = plan
    stages_total = (n_tok + BK - 1) // BK
    assert min(8, stages_total) <= kcs <= 64 and n_kc * kcs >= stages_total > (n_kc - 1) * kcs
    assert units == full + (n_kc * n_tiles - full) * k
    seen = {}
    ncl = min(clusters, units)
    load = [0] * ncl
    for u in range(units):
        tile, a, b = decode(plan, n_tok, n_tiles, u)
        assert b > a
        if k > 1 and u >= full:
            assert b - a >= 8
        for s in range(a, b):
            seen[(tile, s)] = seen.get((tile, s), 0) + 1
        load[u % ncl] += b - a
    assert len(seen) == n_tiles * stages_total and set(seen.values()) == {1}
    # the busiest cluster carries at most one part of a chunk more than an even share
    assert max(load) <= n_tiles * stages_total / ncl + kcs / k + 1e-9 or k == 1


def test_cross_product_slice_is_balanced():
    # a 4096-feature cross-product slice: 256 tiles, 8192 tokens, 70 clusters:
    # 210 whole chunks and the other 46 tiles in thirds (235 stages on the
    # busiest cluster against an even share of 234.06)
    kcs, n_kc, k, full, units = oc.oc_test_unit_plan(8192, 256, 70)
    assert (kcs, n_kc, k, full, units) == (64, 1, 3, 210, 348)
    load = [0] * 70
    for u in range(units):
        _, a, b = decode((kcs, n_kc, k, full, units), 8192, 256, u)
        load[u % 70] += b - a
    assert max(load) == 235


def test_unit_plan_rejects_bad_arguments():
    with pytest.raises(oc.OcError):
        oc.oc_test_unit_plan(0, 16, 70)
    with pytest.raises(oc.OcError):
        oc.oc_test_unit_plan(8192, 16, 0)
