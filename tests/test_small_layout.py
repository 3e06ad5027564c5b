"""Host-side check of the single-CTA Newton solve's shared-memory layout (csrc/pn_small.cuh).

The kernel keeps every per-step array in chunk-interleaved rows (row m * ntiles + k for step m of
32-step chunk k), so a ragged last chunk still owns 32 rows; the step inputs keep B*T rows in
natural order.  This restates that layout and the size formula SmallCfg::smem_bytes uses, and
walks every index the kernel's phases form for a range of shapes, checking each access (and each
16-byte vector access's alignment) against its region.  A layout change in the kernel has to
change this file too.
"""
import pytest

L = 32
NW = 8


def regions(DP, R, B, T):
    NCS, WR = R + 1, R * DP
    nch = (T + L - 1) // L
    ntiles, nbt = B * nch, B * T
    nrows = L * ntiles
    out, off = {}, 0
    for name, size in (("sWf", DP * WR), ("sWb", DP * WR), ("sRed", NW), ("sS0", B * DP), ("sU", nbt * WR),
                       ("sS", nrows * DP), ("sCf", nrows * NCS * DP), ("sBv", nrows * DP),
                       ("sAgg", ntiles * (DP * DP + DP)), ("sCar", ntiles * DP)):
        out[name] = (off, size)
        off += size
    smem_bytes = 4 * (2 * DP * WR + NW + B * DP + nbt * WR + nrows * (DP + NCS * DP + DP)
                      + ntiles * (DP * DP + 2 * DP))
    assert smem_bytes == 4 * off
    return out, nch, ntiles, nrows


@pytest.mark.parametrize("DP,R", [(4, 1), (8, 1), (4, 3), (8, 3)])
@pytest.mark.parametrize("B,T", [(1, 1), (1, 31), (1, 1024), (2, 70), (3, 77), (2, 300), (4, 64), (3, 200),
                                 (1, 33)])
def test_every_access_stays_in_its_region(DP, R, B, T):
    NCS, WR = R + 1, R * DP
    reg, nch, ntiles, nrows = regions(DP, R, B, T)

    def chk(name, idx, n=1):
        off, size = reg[name]
        assert 0 <= idx and idx + n <= size, (name, idx, n, size)
        if n == 4:
            assert (off + idx) % 4 == 0, (name, off, idx)

    def row_of(b, t):
        return (t % L) * ntiles + b * nch + t // L

    rows = set()
    for b in range(B):          # phase 1 and the result copy
        for t in range(T):
            r = row_of(b, t)
            rows.add(r)
            chk("sU", (b * T + t) * WR + WR - 1)
            for ci in range(DP):
                chk("sS", r * DP + ci)
                chk("sBv", r * DP + ci)
                for q in range(NCS):
                    chk("sCf", (r * NCS + q) * DP + ci)
            if t > 0:
                chk("sS", row_of(b, t - 1) * DP + DP - 1)
    assert len(rows) == B * T   # one row per step
    for e in range(nrows * DP):     # the initial guess covers every row
        r = e // DP
        assert (r % ntiles) // nch < B
        chk("sS", e)
    for k in range(ntiles):     # phases 2 and 3
        t0 = (k % nch) * L
        for m in range(min(L, T - t0)):
            r = m * ntiles + k
            assert r == row_of(k // nch, t0 + m)
            for e in range(0, NCS * DP, 4):
                chk("sCf", r * NCS * DP + e, 4)
            for e in range(0, DP, 4):
                chk("sBv", r * DP + e, 4)
                chk("sS", r * DP + e, 4)
        for e in range(0, DP * DP + DP, 4):
            chk("sAgg", k * (DP * DP + DP) + e, 4)
        chk("sCar", k * DP + DP - 1)
