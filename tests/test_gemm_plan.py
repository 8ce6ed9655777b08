"""The tensor-core GEMM's tile scheduler, checked on the host over many shapes.

tp_gemm_plan reports the work units the persistent GEMM kernels hand out,
computed by the same host code the launchers use.  Whatever the shape, tile
kind, shard width, SM count and scratch, the plan must compute every output
element exactly once over the whole K range:

* the tiles cover [0, M) x [0, N) exactly once, 8-column aligned, and no
  tile crosses a column-shard boundary (a shard's tiles write its own
  columns: the column split of "图解Transformer并行计算" §1.2);
* each tile's units cover its K blocks [0, ceil(K / 64)) exactly once, in
  order: one whole unit, or K slices with distinct partial-tile indices
  that fit the scratch (split only in the last, short wave, or every tile
  when there are fewer tiles than persistent CTAs), each slice at least 32
  K blocks deep (16 for a GEMM of fewer than four waves);
* every unit is a tile of the grid and the unit count matches the plan.
"""
import random

import pytest

from megatron_tensor_transformer_logical_b200 import binding as L

KINDS = (128, 192, 256, 512)


def _check_plan(M, N, K, n_shard, kind, sms, scratch):
    units = L.tp_gemm_plan(M, N, K, n_shard, kind, sms, scratch)
    kb_total = -(-K // 64)
    rows = 256 if kind == 512 else 128
    cols = 256 if kind == 512 else kind
    shard = n_shard if (n_shard > 0 and n_shard % 8 == 0 and N % n_shard == 0) else 0
    by_tile = {}
    for u in units:
        by_tile.setdefault(u["tile"], []).append(u)
        assert u["rows"] == rows
        assert 0 <= u["kb0"] < u["kb1"] <= kb_total
    # K coverage per tile, and the shape of the split
    parts = []
    split_tiles = []
    for tile, us in by_tile.items():
        first = us[0]
        assert all((v["m0"], v["n0"], v["n_end"]) == (first["m0"], first["n0"], first["n_end"])
                   for v in us), "units of one tile disagree on its coordinates"
        if len(us) == 1:
            assert us[0]["part"] == -1 and (us[0]["kb0"], us[0]["kb1"]) == (0, kb_total)
        else:
            split_tiles.append(tile)
            assert all(v["part"] >= 0 for v in us)
            assert [(v["kb0"], v["kb1"]) for v in us] == sorted((v["kb0"], v["kb1"]) for v in us)
            edges = [us[0]["kb0"]] + [v["kb1"] for v in us]
            assert edges[0] == 0 and edges[-1] == kb_total
            assert all(us[i]["kb1"] == us[i + 1]["kb0"] for i in range(len(us) - 1))
            parts += [v["part"] for v in us]
    assert len(parts) == len(set(parts))
    if parts:
        assert scratch, "K slices need the last-wave scratch"
        assert max(parts) + 1 == len(parts)
        assert len(parts) * rows * cols * 4 <= sms * 128 * 256 * 4
        n_tiles = len(by_tile)
        slots = sms // 2 if kind == 512 else sms
        if n_tiles < slots:
            # fewer tiles than workers: every tile is split, within the workers
            assert sorted(split_tiles) == list(range(n_tiles))
            assert len(parts) <= slots
        else:
            # only the last tiles (the short last wave) are split, at most half a wave
            assert sorted(split_tiles) == list(range(n_tiles - len(split_tiles), n_tiles))
            assert 2 * len(split_tiles) <= slots
            assert len(split_tiles) == n_tiles % slots
        # every slice is at least 32 K blocks deep (16 when the GEMM has
        # fewer than four waves of tiles)
        depth = 16 if n_tiles < 4 * slots else 32
        assert all(v["kb1"] - v["kb0"] >= depth for t in split_tiles for v in by_tile[t][:-1])
    # spatial coverage: per row band, the column ranges partition [0, N)
    bands = {}
    for tile, us in by_tile.items():
        u = us[0]
        assert u["m0"] % rows == 0 and 0 <= u["m0"] < M
        assert u["n0"] % 8 == 0 and u["n0"] < u["n_end"] <= N
        assert u["n_end"] - u["n0"] <= cols
        if shard:
            s0 = (u["n0"] // shard) * shard
            assert u["n_end"] <= s0 + shard, "tile crosses a shard boundary"
        bands.setdefault(u["m0"], []).append((u["n0"], u["n_end"]))
    assert sorted(bands) == list(range(0, M, rows))
    for m0, spans in bands.items():
        spans.sort()
        assert spans[0][0] == 0 and spans[-1][1] == N
        assert all(spans[i][1] == spans[i + 1][0] for i in range(len(spans) - 1))


LAYER_SHAPES = [  # the 175B-shaped layer's GEMMs (M, N, K, shard width)
    (2048, 36864, 12288, 1536), (2048, 12288, 12288, 0), (12288, 12288, 2048, 0),
    (12288, 36864, 2048, 1536), (2048, 12288, 36864, 0), (2048, 49152, 12288, 6144),
    (2048, 12288, 49152, 0), (49152, 12288, 2048, 0), (12288, 49152, 2048, 6144),
    (2048, 51200, 12288, 6400),
]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("scratch", [True, False])
def test_layer_gemm_plans(kind, scratch):
    for M, N, K, sh in LAYER_SHAPES:
        _check_plan(M, N, K, sh, kind, 148, scratch)


def test_random_gemm_plans():
    rng = random.Random(20261202)
    for _ in range(400):
        M = rng.choice([1, 7, 127, 128, 129, 255, 256, 300, 1000, 2048, 4099])
        N = 8 * rng.randint(1, 900)
        K = rng.choice([1, 63, 64, 65, 1000, 2048, 4096, 12288])
        t = rng.choice([1, 2, 3, 4, 5, 8, 64])
        n_shard = N // t if N % t == 0 else rng.choice([0, 24])
        _check_plan(M, N, K, n_shard, rng.choice(KINDS), rng.choice([2, 3, 8, 132, 148]),
                    rng.random() < 0.7)


def test_short_last_wave_is_split():
    """A GEMM whose last wave is short (here 28 of 148 tiles, as the 175B
    layer's N = 12288 GEMMs) gets its last tiles cut into K slices when the
    scratch is there, and runs whole tiles without it."""
    units = L.tp_gemm_plan(2048, 12288, 49152, 0, 256, 148, True)
    assert len(units) == 740 + 28 * 5
    assert sum(u["part"] >= 0 for u in units) == 28 * 5
    units = L.tp_gemm_plan(2048, 12288, 49152, 0, 256, 148, False)
    assert len(units) == 768 and all(u["part"] == -1 for u in units)


def test_tile_starved_gemm_is_split():
    """A wgrad of the GPT-2-small MLP (M = 3072, N = 768, K = 8192): 72 tiles
    of 128 x 256 for 148 SMs, so every tile is cut into two K slices of 64
    blocks (144 units); without the scratch the 72 tiles run whole."""
    units = L.tp_gemm_plan(3072, 768, 8192, 0, 256, 148, True)
    assert len(units) == 144 and all(u["part"] >= 0 for u in units)
    assert {u["kb1"] - u["kb0"] for u in units} == {64}
    units = L.tp_gemm_plan(3072, 768, 8192, 0, 256, 148, False)
    assert len(units) == 72


def test_short_gemm_splits_its_last_wave_finer():
    """The GPT-2-small MLP's second GEMM (M = 8192, N = 768, K = 3072):
    192 tiles on 148 SMs, 1.3 waves; the 44 tiles of the last wave are cut
    into three slices of 16 K blocks."""
    units = L.tp_gemm_plan(8192, 768, 3072, 0, 256, 148, True)
    assert len(units) == 148 + 44 * 3
    assert {u["kb1"] - u["kb0"] for u in units if u["part"] >= 0} == {16}


def test_invalid_plan_requests():
    for args in [(0, 8, 8, 0, 256, 148), (8, 8, 0, 0, 256, 148), (8, 8, 8, 0, 100, 148),
                 (8, 8, 8, 0, 256, 1)]:
        with pytest.raises(L.TPError):
            L.tp_gemm_plan(*args, True)
