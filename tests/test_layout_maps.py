"""Host-side checks of the two token orders the library stores (CPU only).

The attention kernel reads a score tile with the .16x256b TMEM load: thread t
of a warp, in a 16-lane group, holds lanes t/4 and t/4 + 8 and, in its
registers 4k + e (row t/4) and 4k + 2 + e (row t/4 + 8), the columns
8k + 2g + e (g = t % 4, k = 0..15, e = 0..1).  It writes P~ back with the
mirror store (.16x256b.x4, k = 0..3), one 32-bit word (four e4m3 keys) per
register, and the PV product reads column c of that A operand as the K
indices 4c..4c+3.  These tests replay that bookkeeping in plain Python and
check that the stored K^ row order and V^T token order in tests/parity.py are
exactly the ones it needs.
"""
import numpy as np

from tests import parity as P


def test_maps_are_blockwise_permutations():
    for Np in (128, 384, 1024):
        for m in (P.key_interleave(Np), P.value_interleave(Np)):
            assert sorted(m.tolist()) == list(range(Np))
            assert (m // 128 == np.arange(Np) // 128).all()      # never leaves its block


def test_value_map_is_an_involution():
    m = P.value_interleave(256)
    assert (m[m] == np.arange(256)).all()
    assert not (m == np.arange(256)).all()


def test_score_load_gives_each_thread_32_consecutive_keys():
    # stored K^ row n of a block = score column n of the tile
    col_token = P.key_interleave(128)
    for g in range(4):
        regs = {}
        for k in range(16):
            for e in range(2):
                regs[4 * k + e] = col_token[8 * k + 2 * g + e]          # row t/4
                regs[4 * k + 2 + e] = col_token[8 * k + 2 * g + e]      # row t/4 + 8
        # the kernel's x0[j] (row 0) is register 4*(j//2) + j%2
        x0_tokens = [regs[4 * (j // 2) + j % 2] for j in range(32)]
        x1_tokens = [regs[4 * (j // 2) + 2 + j % 2] for j in range(32)]
        assert x0_tokens == list(range(32 * g, 32 * g + 32))
        assert x1_tokens == x0_tokens


def test_p_store_and_pv_k_order_match_the_value_map():
    # thread g's word i (keys 32g + 4i .. +3, i = 0..7) goes to register 4k+e
    # with word index 2k+e (row 0), hence to TMEM column 8k + 2g + e
    k_index_token = np.full(128, -1)
    for g in range(4):
        for k in range(4):
            for e in range(2):
                word = 2 * k + e
                col = 8 * k + 2 * g + e
                for j in range(4):
                    k_index_token[4 * col + j] = 32 * g + 4 * word + j
    assert sorted(k_index_token.tolist()) == list(range(128))
    # V^T byte p of a block must hold the token that K index p multiplies
    assert (k_index_token == P.value_interleave(128)).all()


def test_packed_int4_layout_golden():
    """Two INT4 values per byte, low nibble first, two's complement: hand-worked
    bytes (1 | -1 << 4 = 0xF1, 7 | -7 << 4 = 0x97, -8 | 0 = 0x08, 0 | 3 = 0x30)."""
    got = P.pack_int4(np.array([[1, -1, 7, -7, -8, 0, 0, 3]]))
    assert got.tolist() == [[0xF1, 0x97, 0x08, 0x30]]


def test_exported_layout_matches_the_documented_orders():
    """sage2_layout_info() (host only) gives the constants and the two token
    orders that the GPU payload tests hold the kernels to."""
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as qa
    lay = qa.sage2_layout_info()
    assert lay["version"] == qa.sage2_version()
    assert (lay["block_rows"], lay["tile_keys"], lay["int4_max"], lay["int8_max"]) == (128, 128, 7, 127)
    assert (lay["p_scale"], lay["v_scale_div"], lay["packed_low_first"]) == (448.0, 448.0, 1)
    assert lay["key_perm"] == P.key_interleave(128).tolist()
    assert lay["value_perm"] == P.value_interleave(128).tolist()
