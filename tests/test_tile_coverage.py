"""Host-side check of the Newton-Schulz kernel's storage rule for its symmetric
intermediates (CPU only).

The kernel stores A = X X^T and B' = a I + b A + c A A as their 256x256 blocks
(I, J) with J >= I, and a consumer reads a k-block below the diagonal as the
transpose of a stored block.  This test restates the kernel's tile
enumeration (ns_gemm.cu: tile_of, with the row tile tm of a symmetric output
starting at the column tile that holds column tm * tile_m; 256x512 tiles in
two N = 256 halves, a half skipped when it starts past the matrix or below the
diagonal block: half_ok) and its per-k-block operand rule (a_major /
b_major), and checks, for both tile modes and both tile widths on the
producing and the consuming side and for ragged sizes, that the computed
halves cover each output block exactly once (symmetric outputs: the upper
blocks), that every element a consumer reads was stored, that the square
stage's epilogue reads A only from stored blocks, and that a consumer's rows
never straddle two 256-blocks.
"""
import numpy as np
import pytest

BN, BK, BLK = 256, 64, 256


def tiles(stage, rows, cols, tile_m, tile_n=BN):
    """The computed N = 256 halves (m0, n0, a_up, b_up) of a stage's tiles."""
    tall = rows > cols
    s = min(rows, cols)
    if stage in ("gram", "square"):
        M = N = s
        sym = True
    else:
        M, N = rows, cols
        sym = False
    a_up = stage == "square" or (stage == "apply" and not tall)
    b_up = stage == "square" or (stage == "apply" and tall)
    tiles_n = -(-N // tile_n)
    out = []
    for tm in range(-(-M // tile_m)):
        m0 = tm * tile_m
        first = (m0 // tile_n) if sym else 0
        for tn in range(first, tiles_n):
            for h in range(tile_n // BN):
                n0 = tn * tile_n + h * BN
                if n0 < N and (not sym or n0 >= (m0 & ~(BLK - 1))):
                    out.append((m0, n0, a_up, b_up))
    return out


def stored_mask(rows, cols, tile_m, tile_n=BN):
    s = min(rows, cols)
    mask = np.zeros((s, s), np.int32)
    for m0, n0, _, _ in tiles("gram", rows, cols, tile_m, tile_n):
        mask[m0:m0 + tile_m, n0:n0 + BN] += 1
    return mask


MODES = [(128, BN), (256, BN), (256, 2 * BN)]   # one CTA, CTA pair, CTA pair with 256x512 tiles


def check_reads(rows, cols, producer, consumer):
    s = min(rows, cols)
    count = stored_mask(rows, cols, *producer)
    assert count.max() <= 1, (rows, cols, producer)    # no block written twice
    stored = count > 0
    tile_m, tile_n = consumer
    pair = tile_m == 256
    rows_a, rows_b = 128, (128 if pair else 256)
    for stage in ("square", "apply"):
        for m0, n0, a_up, b_up in tiles(stage, rows, cols, tile_m, tile_n):
            if stage == "square":
                # The epilogue adds b A_ij of its own output block.
                assert stored[m0:m0 + tile_m, n0:n0 + BN].all(), (rows, cols, m0, n0)
            for rank in ((0, 1) if pair else (0,)):
                for up, r0, nr, origin in ((a_up, m0 + rank * rows_a, rows_a, m0),
                                           (b_up, n0 + rank * rows_b, rows_b, n0)):
                    if not up or r0 >= s:
                        continue
                    blk = origin // BLK
                    assert r0 // BLK == blk and (r0 + nr - 1) // BLK == blk
                    for k0 in range(0, s, BK):
                        transposed = k0 // BLK < blk
                        rr = slice(r0, min(r0 + nr, s))
                        kk = slice(k0, min(k0 + BK, s))
                        sub = stored[kk, rr] if transposed else stored[rr, kk]
                        assert sub.all(), (rows, cols, stage, m0, n0, rank, k0, transposed)


@pytest.mark.parametrize("rows,cols", [(64, 64), (200, 200), (256, 256), (300, 700), (700, 300), (513, 513),
                                       (768, 2304), (3072, 768), (1000, 1000), (129, 513), (520, 260),
                                       (2048, 1000), (4096, 4096)])
@pytest.mark.parametrize("producer", MODES)
@pytest.mark.parametrize("consumer", MODES)
def test_every_read_of_a_symmetric_operand_hits_a_stored_block(rows, cols, producer, consumer):
    check_reads(rows, cols, producer, consumer)


@pytest.mark.parametrize("mode", MODES)
def test_stored_blocks_are_the_upper_256_blocks(mode):
    for n in (1000, 1300, 2560, 4096):
        mask = stored_mask(n, n, *mode)
        i, j = np.indices(mask.shape)
        assert np.array_equal(mask, ((j // BLK) >= (i // BLK)).astype(np.int32)), (n, mode)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("rows,cols", [(300, 700), (2056, 2100), (4096, 2304), (2560, 2560)])
def test_apply_halves_cover_the_output_once(mode, rows, cols):
    cover = np.zeros((rows, cols), np.int32)
    for m0, n0, _, _ in tiles("apply", rows, cols, *mode):
        cover[m0:m0 + mode[0], n0:n0 + BN] += 1
    assert (cover == 1).all()


def test_wide_tiles_skip_the_lower_half_on_odd_row_tiles():
    """256x512 tiles of a symmetric output: a row tile starting in the second
    half of a 512-column tile computes only that half."""
    halves = tiles("square", 1024, 1024, 256, 2 * BN)
    assert (256, 0, True, True) not in halves and (256, 256, True, True) in halves
    assert len(halves) == 4 + 3 + 2 + 1


def test_reading_lower_blocks_directly_would_miss():
    """The rule is needed: reading every k-block directly touches unstored blocks."""
    stored = stored_mask(300, 700, 128) > 0   # A is 300 x 300: blocks [0, 256) and [256, 300)
    assert not stored[BLK:, :BLK].any()
    assert stored[:BLK, BLK:].all()
