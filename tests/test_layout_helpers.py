"""Pins for the test-side layout readers (CPU only): they must agree with a
brute-force loop over the layout include/nvfp4.h states in words."""
import numpy as np

import oracle
from tests import _helpers as H


def _brute_offset(r, j, K):
    # "((r/128) * (K/64) + j/4) * 512 + (r%32) * 16 + ((r/32)%4) * 4 + j%4"
    return ((r // 128) * (K // 64) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4


def test_sf_logical_matches_brute_force_and_is_a_bijection():
    for rows, K in ((1, 64), (130, 192), (256, 320)):
        padded = (rows + 127) // 128 * 128
        nbytes = padded * K // 16
        buf = np.arange(nbytes, dtype=np.int64)
        seen = set()
        for r in range(padded):
            for j in range(K // 16):
                o = _brute_offset(r, j, K)
                assert 0 <= o < nbytes and o not in seen
                seen.add(o)
        assert len(seen) == nbytes
        # each logical (r, j) reads byte _brute_offset(r, j)
        byte_buf = (buf % 251).astype(np.uint8)
        log = H.sf_logical(byte_buf, rows, K)
        for r in range(rows):
            for j in range(K // 16):
                assert log[r, j] == byte_buf[_brute_offset(r, j, K)]
        pad = H.sf_padding_rows(byte_buf, rows, K)
        assert pad.size == (padded - rows) * (K // 16)


def test_unpack_inverts_oracle_pack():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 16, size=(5, 64)).astype(np.uint8)
    np.testing.assert_array_equal(H.unpack_codes(oracle.pack_codes(codes)), codes)
