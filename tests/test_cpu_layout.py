"""Host-side cache layout helpers (pure index arithmetic), CPU only."""
import numpy as np
import pytest

from rank_latent_kv_lk_b200.layout import CacheGeometry, chunk_bytes, tile_index


@pytest.mark.parametrize("rb", [4, 8, 12, 16, 24, 32, 48, 64])
def test_tile_index_is_a_permutation_of_each_block(rb):
    T = 64
    idx = tile_index(T, rb)
    assert sorted(idx.reshape(-1).tolist()) == list(range(T * rb))
    # a 16-token block occupies one contiguous 16 * rb byte range
    for blk in range(T // 16):
        sub = idx[blk * 16:(blk + 1) * 16]
        assert sub.min() == blk * 16 * rb and sub.max() == (blk + 1) * 16 * rb - 1


@pytest.mark.parametrize("rb", [8, 12, 32])
def test_tile_index_matches_chunk_major_rule(rb):
    cs = chunk_bytes(rb)
    idx = tile_index(32, rb)
    for t in (0, 5, 15, 16, 31):
        for k in range(rb):
            assert idx[t, k] == (t // 16) * 16 * rb + (k // cs) * 16 * cs + (t % 16) * cs + k % cs
    # consecutive tokens read the same chunk at consecutive cs-byte addresses
    assert np.all(np.diff(idx[:16, 0]) == cs)


def test_pack_unpack_roundtrip_ragged():
    rng = np.random.default_rng(0)
    g = CacheGeometry(3, [8, 24, 64], 48, "i4", 16)
    lens = [0, 17, 48]
    rows = [[rng.integers(0, 256, (lens[b], r // 2), dtype=np.uint8) for r in g.ranks] for b in range(3)]
    scales = [[rng.standard_normal((lens[b], ng)).astype(np.float16) for ng in g.ng] for b in range(3)]
    c, s = g.pack(rows, scales)
    assert c.size == g.codes_bytes and s.size == g.scales_elems
    r2, s2 = g.unpack(c, s, lens)
    for b in range(3):
        for h in range(3):
            assert np.array_equal(r2[b][h], rows[b][h])
            assert np.array_equal(s2[b][h], scales[b][h])


def test_plane_offsets_follow_the_header_formula():
    g = CacheGeometry(2, [16, 32, 8], 32, "i8")
    assert g.code_plane(0, 0) == (0, 16 * 32)
    assert g.code_plane(0, 2) == ((16 + 32) * 32, 8 * 32)
    assert g.code_plane(1, 1) == ((56 + 16) * 32, 32 * 32)
    assert g.scale_plane(1, 2) == ((1 * 3 + 2) * 32, 32)


@pytest.mark.parametrize("kind,ranks", [("i8", [8, 12, 32, 64]), ("i4", [8, 24, 64])])
def test_v_role_dimension_major_roundtrip(kind, ranks):
    rng = np.random.default_rng(1)
    g = CacheGeometry(2, ranks, 48, kind, 16, role="v")
    lens = [33, 48]
    rb = [r if kind == "i8" else r // 2 for r in ranks]
    rows = [[rng.integers(0, 256, (lens[b], n), dtype=np.uint8) for n in rb] for b in range(2)]
    scales = [[rng.standard_normal((lens[b], ng)).astype(g.scale_dtype) for ng in g.ng] for b in range(2)]
    c, s = g.pack(rows, scales)
    r2, _ = g.unpack(c, s, lens)
    for b in range(2):
        for h in range(len(ranks)):
            assert np.array_equal(r2[b][h], rows[b][h])
    # the header's placement: int8 dim d of token t at (t/16)*16*rb + d*16 + t%16;
    # int4 byte (t/16)*16*rb + d*8 + (t%16)/2, low nibble = even token
    off, _ = g.code_plane(1, 1)
    t, d = 37, 5
    if kind == "i8":
        assert c[off + (t // 16) * 16 * rb[1] + d * 16 + t % 16] == rows[1][1][t, d]
    else:
        byte = c[off + (t // 16) * 16 * rb[1] + d * 8 + (t % 16) // 2]
        nib = (byte >> 4) if t % 2 else (byte & 0xF)
        src = rows[1][1][t, d // 2]
        assert nib == ((src >> 4) if d % 2 else (src & 0xF))
