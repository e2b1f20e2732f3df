"""The K-split (stream-K) work partition of the decode GEMM, checked on the
CPU: the formulas below restate the kernel's (contiguous balanced ranges of
(tile, K-step) units per CTA; the CTA holding a unit; the workspace slot a
split tile's partial goes to) and are checked for full coverage and for the
writer and the reader of every partial agreeing on its slot."""
import pytest


def unit_begin(c, U, G):
    return c * U // G


def cta_of_unit(u, U, G):
    return ((u + 1) * G + U - 1) // U - 1


def items(c, U, G, kt):
    u, end = unit_begin(c, U, G), unit_begin(c + 1, U, G)
    out = []
    while u < end:
        tp = u // kt
        kb = u - tp * kt
        ke = min(kt, kb + (end - u))
        out.append((tp, kb, ke))
        u += ke - kb
    return out


@pytest.mark.parametrize("tiles,kt,G", [(96, 20, 148), (96, 20, 96), (1, 20, 20), (1, 3, 3), (7, 5, 148),
                                        (200, 20, 148), (3, 1, 3), (13, 7, 148), (1000, 20, 148), (96, 68, 148),
                                        (96, 20, 296), (96, 68, 296), (40, 3, 296)])
def test_partition(tiles, kt, G):
    U = tiles * kt
    G = min(G, U)
    seen = [0] * U
    writer_slot = {}
    for c in range(G):
        its = items(c, U, G, kt)
        assert len(its) >= 1
        for idx, (tp, kb, ke) in enumerate(its):
            for k in range(kb, ke):
                seen[tp * kt + k] += 1
            c_first = cta_of_unit(tp * kt, U, G)
            c_last = cta_of_unit(tp * kt + kt - 1, U, G)
            assert c_first <= c <= c_last
            if c_first != c_last:
                # only the first and last items of a range can be partial
                assert idx in (0, len(its) - 1)
                writer_slot[(tp, c)] = 2 * c + (0 if idx == 0 else 1)
            else:
                assert (kb, ke) == (0, kt)
    assert all(v == 1 for v in seen)
    for tp in range(tiles):
        c_first = cta_of_unit(tp * kt, U, G)
        c_last = cta_of_unit(tp * kt + kt - 1, U, G)
        if c_first == c_last:
            continue
        for c in range(c_first, c_last + 1):
            reader = 2 * c + (0 if unit_begin(c, U, G) >= tp * kt else 1)
            assert writer_slot[(tp, c)] == reader
            assert reader < 2 * G


def test_cta_of_unit_inverts_unit_begin():
    for U in (1, 7, 1920, 9999):
        for G in (1, 3, 148, 296):
            if G > U:
                continue
            for u in range(U):
                c = cta_of_unit(u, U, G)
                assert unit_begin(c, U, G) <= u < unit_begin(c + 1, U, G)
