"""The prefill GEMM's work schedule, on CPU: the library walks each CTA's
items with the same code the kernel runs, so these checks hold for the
launch itself. Every (tile, 128-k block) pair is covered exactly once; with
stream-K a tile is cut at most once, its later part the first item of the
phase of CTA c and its earlier part the last item of CTA c - 1 (the pair that
meets in workspace slot c); whole tiles keep the strided order; the CTAs'
k-block loads differ by at most one k-block."""

import pytest

SHAPES = [
    (512, 4096, 14336),    # 224 tiles on 148 CTAs
    (2048, 4096, 14336),   # 896 tiles: 6 full waves and 8 tiles
    (8192, 4096, 14336),   # 3584 tiles: 3% of the schedule idle (whole tiles)
    (4096, 4096, 14336),   # 1792 tiles: 7% idle
    (300, 1056, 4000),     # ragged M, K (9 blocks, the last part-filled) and N
    (17, 64, 128),         # one tile
    (1000, 14336, 4096),   # 128 tiles: fewer than the CTAs
    (4000, 4096, 1200),    # 160 tiles: 12 over one wave
]


def _schedule(lbq, M, K, N, sk):
    grid, nkb, first = lbq.lbq_debug_gemm_schedule(M, K, N, sk, 0)
    per_cta = [first] + [lbq.lbq_debug_gemm_schedule(M, K, N, sk, c)[2] for c in range(1, grid)]
    return grid, nkb, per_cta


@pytest.mark.parametrize("M,K,N", SHAPES)
@pytest.mark.parametrize("sk", [0, 1])
def test_schedule_covers_every_block_once(M, K, N, sk):
    import bit_weight_only_pack_b200 as lbq
    grid, nkb, per_cta = _schedule(lbq, M, K, N, sk)
    tiles = ((M + 255) // 256) * ((N + 127) // 128)
    assert nkb == (K + 127) // 128 and grid == min(tiles, 148)
    seen = {}
    for c, items in enumerate(per_cta):
        for (tile, kb0, kb1, part) in items:
            assert 0 <= tile < tiles and 0 <= kb0 < kb1 <= nkb
            assert part == (1 if kb0 > 0 else (2 if kb1 < nkb else 0))
            for kb in range(kb0, kb1):
                assert (tile, kb) not in seen, f"block ({tile}, {kb}) twice"
                seen[(tile, kb)] = c
    assert len(seen) == tiles * nkb


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_cut_tiles_meet_between_neighbours(M, K, N):
    import bit_weight_only_pack_b200 as lbq
    grid, nkb, per_cta = _schedule(lbq, M, K, N, 1)
    parts_of = {}
    for c, items in enumerate(per_cta):
        for i, (tile, kb0, kb1, part) in enumerate(items):
            parts_of.setdefault(tile, []).append((c, i, kb0, kb1, part))
            if part == 1:  # a later part opens the CTA's stream-K phase: only whole tiles before it
                assert all(p == 0 for (_, _, _, p) in items[:i])
                prev = per_cta[c - 1][-1]
                assert c > 0 and prev[0] == tile and prev[3] == 2 and prev[2] == kb0
            if part == 2:  # an earlier part ends the CTA's items and its later part opens CTA c + 1's phase
                assert i == len(items) - 1
                nxt = [it for it in per_cta[c + 1] if it[0] == tile]
                assert len(nxt) == 1 and nxt[0][3] == 1 and nxt[0][1] == kb1
    assert all(len(v) <= 2 for v in parts_of.values())


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_stream_k_balances_the_last_waves(M, K, N):
    import bit_weight_only_pack_b200 as lbq
    grid, nkb, per_cta = _schedule(lbq, M, K, N, 1)
    _, _, whole = _schedule(lbq, M, K, N, 0)
    load = [sum(kb1 - kb0 for (_, kb0, kb1, _) in items) for items in per_cta]
    load_whole = [sum(kb1 - kb0 for (_, kb0, kb1, _) in items) for items in whole]
    cut = any(p != 0 for items in per_cta for (_, _, _, p) in items)
    ws = lbq.lbq_workspace_size(1, M, K, N, 128 if K % 128 == 0 else 32, lbq.MODES["asym"])
    assert (ws > 0) == cut
    if cut:
        assert max(load) - min(load) <= 1
        assert max(load) < max(load_whole)
        # one flag per CTA (rounded to 256 bytes) and one FP32 tile of 256 x 128 per CTA
        assert ws == (grid * 4 + 255) // 256 * 256 + grid * 256 * 128 * 4
        if K % 64 == 0:
            assert lbq.lbq_workspace_size(2, M, K, N, 0, lbq.MODES["lut3"]) == ws
    else:
        assert load == load_whole
    # the rule: cut where the last wave leaves at least 5% of the schedule's SM
    # time idle (and 4 k-blocks per SM)
    tiles = ((M + 255) // 256) * ((N + 127) // 128)
    rem, waves = tiles % grid, -(-tiles // grid)
    assert cut == (tiles > grid and rem > 0 and nkb * (grid - rem) >= 4 * grid and 20 * (grid - rem) >= grid * waves)
    if (M, K, N) in [(512, 4096, 14336), (2048, 4096, 14336), (4096, 4096, 14336)]:
        assert cut
    if (M, K, N) == (8192, 4096, 14336):
        assert not cut


def test_whole_tile_schedule_is_the_strided_order():
    import bit_weight_only_pack_b200 as lbq
    grid, nkb, per_cta = _schedule(lbq, 2048, 4096, 14336, 0)
    for c, items in enumerate(per_cta):
        assert [t for (t, _, _, _) in items] == list(range(c, 896, grid))
        assert all((kb0, kb1, p) == (0, nkb, 0) for (_, kb0, kb1, p) in items)


@pytest.mark.parametrize("n_tiles,m_tiles", [(112, 32), (112, 8), (112, 2), (33, 5), (7, 13), (10, 16), (112, 9), (1, 1)])
def test_banded_tile_order_is_a_bijection(n_tiles, m_tiles):
    """The kernel's tile order: bands of 8 token tiles, channel tiles outer
    inside a band; every (channel tile, token tile) once, a partial last band
    included, and the plain token-inner order when there are at most 8 token
    tiles."""
    import bit_weight_only_pack_b200 as lbq
    got = [lbq.lbq_debug_tile_coords(t, n_tiles, m_tiles) for t in range(n_tiles * m_tiles)]
    assert sorted(got) == [(a, b) for a in range(n_tiles) for b in range(m_tiles)]
    if m_tiles <= 8:
        assert got == [(t // m_tiles, t % m_tiles) for t in range(n_tiles * m_tiles)]
    else:  # the first band: 8 token tiles of channel tile 0, then of channel tile 1, ...
        assert got[:16] == [(0, b) for b in range(8)] + [(1, b) for b in range(8)]
