"""Host-side check of the Newton-Schulz kernel's storage rule for its symmetric
intermediates (CPU only).

The kernel stores A = X X^T, P = b I + c A and B' = a I + A P as their 256x256
blocks (I, J) with J >= I, and a consumer reads a k-block below the diagonal as
the transpose of a stored block.  This test restates the kernel's tile
enumeration (ns_gemm.cu: tile_of, with the row tile tm of a symmetric output
starting at column tile tm * tile_m / 256) and its per-k-block operand rule
(a_major / b_major) and checks, for both tile modes on the producing and the
consuming side and for ragged sizes, that every element a consumer reads was
stored, and that a consumer's rows never straddle two 256-blocks.
"""
import numpy as np
import pytest

BN, BK, BLK = 256, 64, 256


def tiles(stage, rows, cols, tile_m):
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
    tiles_n = -(-N // BN)
    out = []
    for tm in range(-(-M // tile_m)):
        first = (tm * tile_m) // BLK if sym else 0
        for tn in range(first, tiles_n):
            out.append((tm * tile_m, tn * BN, a_up, b_up))
    return out


def stored_mask(rows, cols, tile_m):
    s = min(rows, cols)
    mask = np.zeros((s, s), bool)
    for m0, n0, _, _ in tiles("gram", rows, cols, tile_m):
        mask[m0:m0 + tile_m, n0:n0 + BN] = True
    return mask


def check_reads(rows, cols, producer_tile_m, consumer_tile_m):
    s = min(rows, cols)
    stored = stored_mask(rows, cols, producer_tile_m)
    pair = consumer_tile_m == 256
    rows_a, rows_b = 128, (128 if pair else 256)
    for stage in ("square", "apply"):
        for m0, n0, a_up, b_up in tiles(stage, rows, cols, consumer_tile_m):
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
@pytest.mark.parametrize("producer_tile_m", [128, 256])
@pytest.mark.parametrize("consumer_tile_m", [128, 256])
def test_every_read_of_a_symmetric_operand_hits_a_stored_block(rows, cols, producer_tile_m, consumer_tile_m):
    check_reads(rows, cols, producer_tile_m, consumer_tile_m)


def test_stored_blocks_are_the_upper_256_blocks():
    for tile_m in (128, 256):
        mask = stored_mask(1000, 1000, tile_m)
        i, j = np.indices(mask.shape)
        assert np.array_equal(mask, (j // BLK) >= (i // BLK))


def test_reading_lower_blocks_directly_would_miss():
    """The rule is needed: reading every k-block directly touches unstored blocks."""
    stored = stored_mask(300, 700, 128)   # A is 300 x 300: blocks [0, 256) and [256, 300)
    assert not stored[BLK:, :BLK].any()
    assert stored[:BLK, BLK:].all()
