"""Work decomposition of the tensor-core conv, checked on the host through
sige_conv_schedule (the functions the kernel runs at launch): every tile is in
exactly one tile group, the K splits of a unit sit where their sum can find
them, and the shared-memory carve-up fits.  No GPU needed.

SIGE tile-based sparse convolution ("Sparse Engine SIGE": gather the active
blocks, run the layer on the stacked blocks, scatter); the split of the block
convolution over CTAs is this implementation's."""
import numpy as np
import pytest

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs

NONE, PAIR, CLUSTER, GLOBAL = 0, 1, 2, 3


def _layers():
    out = [("resblock 256x256 C128 b8", 3, 1, 1, 128, 128, 8, 256, 256)]
    for i, (h, w, c, b) in enumerate(inputs.CFG4_LAYERS):
        out.append((f"sd{i}", 3, 1, 1, c, c, b, h, w))
    for i, (h, w, ci, co, k, s, b) in enumerate(inputs.CFG5_LAYERS):
        out.append((f"gaugan{i}", k, s, k // 2, ci, co, b, h, w))
    # the other layouts: POS (odd b), row-batched POS with b = 6 and at stride 2
    out += [("pos b3", 3, 1, 1, 256, 128, 3, 48, 48), ("rows b6", 3, 1, 1, 128, 256, 6, 48, 48),
            ("rows b2 s2", 3, 2, 1, 256, 128, 2, 64, 64)]
    return out


LAUNCHES = [(148, 1), (148, 2), (146, 2), (148, 4), (144, 4), (132, 4)]


def _tile_counts(cap):
    g = list(range(0, min(cap, 160) + 1))
    g += list(range(161, cap + 1, max(1, cap // 97)))
    return sorted(set(g + [cap]))


@pytest.mark.parametrize("name,k,s,p,ci,co,b,H,W", _layers())
def test_schedule_invariants(name, k, s, p, ci, co, b, H, W):
    cd = sige.conv_desc(k, s, p, ci, co, b)
    Ho, Wo = (H + 2 * p - k) // s + 1, (W + 2 * p - k) // s + 1
    cap = -(-Ho // b) * -(-Wo // b)
    for grid, cl in LAUNCHES:
        for G in _tile_counts(cap):
            d = sige.sige_conv_schedule(cd, G, grid, cl)
            T, TB, S, U = d["T"], d["tile_groups"], d["splits"], d["units"]
            ctx = (name, grid, cl, G, d)
            # every tile in exactly one group; units = groups x channel tiles x splits
            assert TB * T >= G and (TB - 1) * T < max(G, 1), ctx
            assert U == TB * d["cout_tiles"] * S, ctx
            assert d["cout_tiles"] == -(-co // 128) and d["k_chunks"] == k * k * ci // 64, ctx
            # each split keeps at least one k-chunk; a split launch fits in one round
            assert 1 <= S <= d["k_chunks"], ctx
            if S > 1:
                assert U <= grid, ctx
            if cl >= 4:
                assert S & (S - 1) == 0 and cl % S == 0, ctx
            # layout and accumulator columns
            lay = d["layout"]
            assert lay == (0 if (b == 8 and s == 1) else 2 if (b % 2 == 0 and 8 * b <= 256) else 1), ctx
            assert d["unit_cols"] == (64 * T if lay == 0 else b * b * T) and d["unit_cols"] <= 512, ctx
            if lay == 2:
                assert T == 8, ctx
            if lay == 1:
                assert T % 16 == 0, ctx
            # shared memory: control, >= 2 weight stages, the halo stages at the top
            assert d["weight_stages"] >= 2, ctx
            assert 4096 + d["weight_stages"] * 16384 <= d["halo_offset"], ctx
            assert d["halo_offset"] + d["halo_bytes"] <= d["smem_bytes"] <= 227 * 1024, ctx
            # how the split is summed
            kind = d["split_sum"]
            assert (kind == NONE) == (S == 1), ctx
            if kind == PAIR:
                assert cl == 2 and S == 2 and d["unit_cols"] <= 64, ctx
            if kind == CLUSTER:
                assert cl % S == 0 and (d["unit_cols"] // S) % 4 == 0, ctx
                assert d["reduce_scatter_bytes"] == d["unit_cols"] * 512 <= d["halo_bytes"], ctx
                u = np.arange(U)
                cta = u % grid
                # a CTA's member index (cluster rank mod S) is the unit's split index
                assert np.array_equal((cta % cl) % S, u % S), ctx
                # the S units of a tile group run in one round, in one cluster
                u0 = u - u % S
                assert np.array_equal(cta // cl, (u0 % grid) // cl), ctx
                assert np.array_equal(u // grid, u0 // grid), ctx
            if kind == GLOBAL:
                assert cl < 2 or cl % S != 0 or (d["unit_cols"] // S) % 4 != 0 or \
                    d["unit_cols"] * 512 > d["halo_bytes"], ctx


def test_k_split_ranges_partition():
    # split q of a unit covers k-chunks [q KC / S, (q + 1) KC / S)
    for name, k, s, p, ci, co, b, H, W in _layers():
        cd = sige.conv_desc(k, s, p, ci, co, b)
        for grid, cl in LAUNCHES:
            d = sige.sige_conv_schedule(cd, 1, grid, cl)
            S, KC = d["splits"], d["k_chunks"]
            bounds = [q * KC // S for q in range(S + 1)]
            assert bounds[0] == 0 and bounds[-1] == KC and all(b1 > b0 for b0, b1 in zip(bounds, bounds[1:]))


def test_cluster_size_rule():
    # a sparse launch asks for clusters of 4 exactly where one tile would split
    # K at least 4 ways; the bench layer keeps its clusters of two
    for name, k, s, p, ci, co, b, H, W in _layers():
        cd = sige.conv_desc(k, s, p, ci, co, b)
        d1 = sige.sige_conv_schedule(cd, 1, 148, 1)
        d = sige.sige_conv_schedule(cd, 1, 148, 2)
        assert d["cluster_for_sparse"] == (4 if d1["splits"] >= 4 else 2), name
    cd = sige.conv_desc(3, 1, 1, 128, 128, 8)
    d = sige.sige_conv_schedule(cd, 51, 148, 2)
    assert (d["layout"], d["T"], d["splits"], d["units"], d["split_sum"], d["cluster_for_sparse"]) == (0, 1, 2, 102, PAIR, 2)


def test_schedule_rejects_bad_arguments():
    cd = sige.conv_desc(3, 1, 1, 128, 128, 8)
    for tiles, grid, cl in [(-1, 148, 2), (5, 0, 1), (5, 148, 0), (5, 147, 2)]:
        with pytest.raises(sige.SigeError):
            sige.sige_conv_schedule(cd, tiles, grid, cl)
    with pytest.raises(sige.SigeError):
        sige.sige_conv_schedule(sige.conv_desc(3, 1, 1, 48, 64, 8), 5, 148, 2)   # C_in not a multiple of 64
