"""Host check of the GEMV kernels' table-lookup address arithmetic, restated
in Python with an exact emulation of the PTX byte permute (prmt, default
mode: a selector nibble with its top bit set replicates the sign bit of the
chosen byte).  Every table address a lane can form -- every weight byte,
every lane, every stored position, full panels and every narrow width --
must stay inside one 64 KB table buffer, and the 32 lanes of a warp must hit
32 different banks at every step (for narrow panels: as far as the repeated
table copies allow).  No GPU is used."""

import numpy as np
import pytest

TABLE_BYTES = 65536


def prmt(a, b, sel):
    """PTX prmt.b32 d, a, b, sel (default mode)."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    d = 0
    for k in range(4):
        nib = (sel >> (4 * k)) & 0xF
        byte = src[nib & 7]
        if nib & 8:
            byte = 0xFF if byte & 0x80 else 0x00
        d |= byte << (8 * k)
    return d


def addr_sel(j):
    return (4 + j) | (j << 4) | ((12 + j) << 8) | ((12 + j) << 12)


def full_offsets(lane):
    L = (4 * lane) * 0x01010101
    return [((L + (16 * m) * 0x01010101 + 0x0C080400) & 0x7C7C7C7C) & 0xFFFFFFFF for m in range(8)]


def narrow_offsets_dup(lane, Bp):
    copies, r = 32 // Bp, lane % Bp
    base = Bp * ((lane // Bp) % copies)
    out = []
    for m in range(8):
        word = 0
        for jj in range(4):
            u = 4 * m + jj
            q = (r + u) % Bp
            q = base + q if u < Bp else 0
            word |= (4 * q) << (8 * jj)
        out.append(word)
    return out


def test_prmt_emulation():
    assert prmt(0x44332211, 0x88776655, 0x3210) == 0x44332211
    assert prmt(0x44332211, 0x88776655, 0x7654) == 0x88776655
    assert prmt(0x000000FF, 0, 0x8888) == 0xFFFFFFFF            # sign replicated
    assert prmt(0x0000007F, 0, 0x8888) == 0


@pytest.mark.parametrize("second_token", [0, 128])
def test_full_panel_addresses_stay_in_the_buffer_and_hit_distinct_banks(second_token):
    for u in range(32):
        m, j = divmod(u, 4)
        banks = set()
        for lane in range(32):
            off = full_offsets(lane)[m]
            assert ((off >> (8 * j)) & 0xFF) == 4 * ((lane + u) % 32)       # byte group (lane + u) mod 32
            for b in (0, 1, 0x7F, 0x80, 0xFE, 0xFF):
                w = b << (8 * j)
                a = prmt(w, off, addr_sel(j)) + second_token
                assert a == 256 * b + 4 * ((lane + u) % 32) + second_token
                assert 0 <= a and a + 4 <= TABLE_BYTES
            banks.add((prmt(0xFF << (8 * j), off, addr_sel(j)) // 4) % 32)
        assert len(banks) == 32


@pytest.mark.parametrize("Bp", [4, 8, 12, 16, 20, 24, 28])
def test_narrow_panel_addresses_stay_in_the_buffer(Bp):
    copies = 32 // Bp
    for u in range(Bp):
        m, j = divmod(u, 4)
        slots = []
        for lane in range(32):
            off = narrow_offsets_dup(lane, Bp)[m]
            q = (off >> (8 * j)) & 0xFF
            assert q % 4 == 0 and q // 4 < copies * Bp <= 32
            assert (q // 4) % Bp == (lane % Bp + u) % Bp                    # the lane's byte group
            for b in (0, 0x80, 0xFF):
                a = prmt(b << (8 * j), off, addr_sel(j))
                assert a == 256 * b + q and a + 4 + 128 <= TABLE_BYTES
            slots.append(q // 4)
        # lanes sharing a slot: at most ceil(32 / (copies * Bp)) ... bounded by the copies available
        worst = max(slots.count(s) for s in set(slots))
        assert worst <= -(-32 // (copies * Bp)) + (1 if (32 // Bp) * Bp < 32 else 0)
        if 32 % Bp == 0:
            assert worst == 1                                               # conflict-free


def test_repeated_narrow_columns_cover_the_copies():
    """column c of a narrow panel's table (c >= its width) repeats column
    c mod width for the first floor(32/Bp) copies, and is zero past them."""
    for Bp in (4, 8, 12, 16, 20, 24, 28):
        w = 8 * Bp
        for c in range(256):
            if c < w:
                src = c
            elif c < (256 // w) * w:
                src = c % w
            else:
                src = None
            copies = 32 // Bp
            slot_group = c // 8
            if src is not None:
                assert slot_group < copies * Bp
            else:
                assert slot_group >= copies * Bp


def z_slot(t):
    """Slot of panel column t in the z buffer: the low four columns of each
    8-column group first (group q at 4q), the high four after them (128 + 4q)."""
    return (128 if t & 4 else 0) + 4 * (t >> 3) + (t & 3)


def test_z_layout_gives_contiguous_build_reads():
    """The table build's lane q reads its group's z as two 16-byte words at
    4q and 128 + 4q: they must hold columns 8q..8q+3 and 8q+4..8q+7 in order,
    and a warp's 32 words must be consecutive (4 wavefronts per read).  The
    z stores (thread t writes column t) then hit each bank twice: one extra
    wavefront per warp and panel, the price of the contiguous reads."""
    assert sorted(z_slot(t) for t in range(256)) == list(range(256))
    inv = {z_slot(t): t for t in range(256)}
    for q in range(32):
        assert [inv[4 * q + i] for i in range(4)] == [8 * q + i for i in range(4)]
        assert [inv[128 + 4 * q + i] for i in range(4)] == [8 * q + 4 + i for i in range(4)]
    for base in (0, 128):
        words = [base + 4 * q for q in range(32)]
        assert words == list(range(base, base + 128, 4))                  # 512 consecutive bytes
    for w in range(8):
        banks = [z_slot(32 * w + i) % 32 for i in range(32)]
        assert max(banks.count(b) for b in set(banks)) == 2
