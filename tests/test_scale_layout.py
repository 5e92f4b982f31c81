"""CPU checks of the test side's tiled scale-layout index function.

The GPU parity tests compare scale bytes through ``gpu_helpers.tiled_scales``;
these checks fix its structure without a GPU: each 512-byte atom covers 128
rows by 4 consecutive blocks; inside it, row r's 4 bytes sit in 16-byte chunk
r % 32, at slot (r // 32) % 4; atoms follow in row-tile-major order.  The map is
a bijection onto the padded byte range that ``nvfp4_scales_bytes`` reports."""
import numpy as np
import pytest

from gpu_helpers import tiled_scales, untile_scales


def _pad(R, KB):
    return -(-R // 128) * 128, -(-KB // 4) * 4


@pytest.mark.parametrize("R,KB", [(1, 1), (127, 5), (128, 4), (130, 80), (300, 7), (256, 320)])
def test_round_trip_and_padding_zero(R, KB):
    rng = np.random.default_rng(R * 1000 + KB)
    s = rng.integers(1, 256, size=(R, KB), dtype=np.uint8)       # no zeros: padding is the only 0
    t = tiled_scales(s)
    R128, KB4 = _pad(R, KB)
    assert t.size == R128 * KB4
    assert np.array_equal(untile_scales(t, R, KB), s)
    assert int((t == 0).sum()) == R128 * KB4 - R * KB


def _tags(R, KB):
    """Tile the tag row * KB + block of every scale, carried as two byte planes."""
    idx = np.arange(R * KB, dtype=np.int64)
    lo = tiled_scales((idx & 0xFF).astype(np.uint8).reshape(R, KB)).astype(np.int64)
    hi = tiled_scales((idx >> 8).astype(np.uint8).reshape(R, KB)).astype(np.int64)
    return hi * 256 + lo


@pytest.mark.parametrize("R,KB", [(128, 4), (256, 12), (384, 8)])
def test_full_tiles_are_a_permutation(R, KB):
    tags = _tags(R, KB)
    assert tags.size == R * KB
    assert np.array_equal(np.sort(tags), np.arange(R * KB))


def test_atom_structure_by_explicit_walk():
    """Walk one 2 x 3 grid of atoms byte by byte, naming each byte's (row, block)
    from the atom description rather than the closed-form index."""
    R, KB = 256, 12
    tags = _tags(R, KB)
    pos = 0
    for row_tile in range(R // 128):
        for block_group in range(KB // 4):
            for chunk in range(32):                                # 16-byte chunk = row % 32
                for slot in range(4):                              # 4-byte slot = (row // 32) % 4
                    row = row_tile * 128 + slot * 32 + chunk
                    for j in range(4):                             # block within the group
                        blk = block_group * 4 + j
                        assert tags[pos] == row * KB + blk, (pos, row, blk)
                        pos += 1
    assert pos == R * KB


def test_padded_size_matches_library():
    import nvfp4_block_scaled_21_b200 as nv
    for R, KB in [(1, 1), (8, 320), (130, 5), (8192, 320)]:
        R128, KB4 = _pad(R, KB)
        assert nv.scales_bytes(R, KB * 16) == R128 * KB4


@pytest.mark.parametrize("R,KB", [(16, 16), (64, 16), (130, 5), (257, 8)])
def test_smoke_untiling_inverts_the_test_layout(R, KB):
    """smoke() reads the GPU's scale bytes back with its own loop; it must be
    the inverse of the tests' tiling."""
    import __graft_entry__
    rng = np.random.default_rng(R + KB)
    s = rng.integers(0, 256, size=(R, KB), dtype=np.uint8)
    assert np.array_equal(__graft_entry__._untile_scales(tiled_scales(s), R, KB * 16), s)
