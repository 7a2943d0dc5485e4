"""Coverage of the tensor-core epilogue's output writes, on the CPU.

The tests restate the index arithmetic of ns_gemm_tc_kernel (the tile order of a launch and,
per tile, which 32 x 32 sub-tiles each epilogue warp stores directly or at the mirrored
position) and check, for every stored form and warp layout, that each 32 x 32 block of the
output is written exactly once: the whole matrix for a plain product and for the whole
symmetric form (upper triangle directly, strictly-lower blocks by mirror), and exactly the
256-blocks on or above the diagonal for the upper-block form. Tile counts must match the
problem tables' counts. Ragged sizes, every combination of 256 x 256 and 256 x 512 tiles with
four or eight epilogue warps, and both CTAs of a pair are covered.
"""
import pytest

TILE_M = 256
GROUP_M = 8   # raster group of row blocks (tile_sched.cuh)


def cdiv(a, b):
    return -(-a // b)


def ctrunc(a, b):
    """C integer division (truncation toward zero)."""
    q = abs(a) // abs(b)
    return q if (a >= 0) == (b > 0) else -q


def sym_tiles(m, tn):
    tm, tnn = cdiv(m, TILE_M), cdiv(m, tn)
    return sum(tnn - (bi * TILE_M) // tn for bi in range(tm))


def decode(l, sym, tiles_m, tiles_n, tn):
    if sym:
        bi = 0
        while True:
            first = (bi * TILE_M) // tn
            cnt = tiles_n - first
            if l < cnt:
                return bi, first + l
            l -= cnt
            bi += 1
    per_group = GROUP_M * tiles_n
    g = l // per_group
    first = g * GROUP_M
    gsize = min(GROUP_M, tiles_m - first)
    r = l - g * per_group
    return first + r % gsize, r // gsize


def ch_of(i, sub, wide, epi):
    if wide:
        return ((i >> 2) << 3) + (sub << 2) + (i & 3)
    return (sub << 2) + i if epi == 8 else i


def writes(M, N, sym, tn, epi):
    """Every (row block, column block) of 32 x 32 written by one launch of one problem."""
    wide = tn == 512
    tiles_m, tiles_n = cdiv(M, TILE_M), cdiv(N, tn)
    n_tiles = sym_tiles(M, tn) if sym else tiles_m * tiles_n
    warp_chunks = tn // 32 // (epi // 4)
    out = []
    tiles = set()
    for l in range(n_tiles):
        bi, bj = decode(l, sym, tiles_m, tiles_n, tn)
        assert bi < tiles_m and bj < tiles_n and (bi, bj) not in tiles
        tiles.add((bi, bj))
        for rank in range(2):
            for quarter in range(4):
                for sub in range(epi // 4):
                    r0 = bi * TILE_M + rank * 128 + quarter * 32
                    col0 = bj * tn
                    lo = hi = 0
                    if r0 < M and col0 < N:
                        hi = min(tn // 32, (N - col0 + 31) // 32)
                        first = r0 if sym == 1 else (bi * TILE_M if sym else col0)
                        lo = min(hi, max(0, ctrunc(first - col0, 32)))
                    chs = [ch_of(i, sub, wide, epi) for i in range(warp_chunks)]
                    assert chs == sorted(chs)
                    i_lo = sum(c < lo for c in chs)
                    i_hi = sum(c < hi for c in chs)
                    for i in range(i_lo, i_hi):
                        c0 = col0 + chs[i] * 32
                        out.append((r0 // 32, c0 // 32))
                        if sym == 1 and c0 >= r0 + 32:
                            out.append((c0 // 32, r0 // 32))
    return out, n_tiles, len(tiles)


def blocks_in(M, N, keep):
    return sorted((rb, cb) for rb in range(cdiv(M, 32)) for cb in range(cdiv(N, 32)) if keep(rb, cb))


LAYOUTS = [(256, 4), (256, 8), (512, 8)]   # (tile columns, epilogue warps) the kernel runs
SIZES = [1, 17, 32, 33, 255, 256, 257, 300, 520, 768, 1000, 1024, 2100, 3000]


@pytest.mark.parametrize("tn,epi", LAYOUTS)
@pytest.mark.parametrize("m", SIZES)
def test_symmetric_whole_form_writes_every_block_once(tn, epi, m):
    out, n_tiles, distinct = writes(m, m, 1, tn, epi)
    assert distinct == n_tiles
    assert sorted(out) == blocks_in(m, m, lambda rb, cb: True)


@pytest.mark.parametrize("tn,epi", [(256, 4), (256, 8)])
@pytest.mark.parametrize("m", SIZES)
def test_upper_block_form_writes_the_blocks_on_and_above_the_diagonal_once(tn, epi, m):
    out, _, _ = writes(m, m, 2, tn, epi)
    assert sorted(out) == blocks_in(m, m, lambda rb, cb: cb // 8 >= rb // 8)


@pytest.mark.parametrize("tn,epi", LAYOUTS)
@pytest.mark.parametrize("shape", [(1, 7), (7, 1), (33, 17), (300, 701), (768, 2304), (2100, 2600),
                                   (2600, 2100), (1024, 4096), (4096, 1100), (2049, 513)])
def test_plain_product_writes_every_block_once(tn, epi, shape):
    M, N = shape
    out, n_tiles, distinct = writes(M, N, 0, tn, epi)
    assert distinct == n_tiles == cdiv(M, TILE_M) * cdiv(N, tn)
    assert sorted(out) == blocks_in(M, N, lambda rb, cb: True)
