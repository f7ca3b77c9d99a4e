"""The tensor-core kernel's launch schedule, checked on the CPU (no GPU).

The kernel's CTA c owns the tiles [T c / C, T (c + 1) / C) of the row-major tile
order v = i tiles_c + j and walks them in M-groups of R row tiles, round by
round, team by team (team t takes column blocks t, t + teams, ...), row by row.
This test restates that walk independently and checks that the schedule
brings exactly those tiles, in that order, in copies of consecutive chunks
that never wrap the ring, never overwrite a copy still outstanding, keep fewer
than 64 copies outstanding, and are released exactly batch_tiles times.
"""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import _lib as lib
from lossless_bf16_weight_nwc_b200 import synth

KMAX_OUTSTANDING = 48


def blob_of(rows, cols, tile_cols=512, lmax=0, seed=0):
    w = synth.matrix(synth.MatrixSpec("w", rows, cols, "normal", 0.02, seed), seed)
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols)
    try:
        return lib.nwc_compress_host(plan, w)
    finally:
        lib.nwc_plan_destroy(plan)


def header(blob):
    h = blob[:128].view(np.uint32)
    q = blob[:128].view(np.uint64)
    rows, cols = int(q[2]), int(q[3])
    tile_cols = int(h[9])
    tiles_r, tiles_c = int(q[5]), int(q[6])
    index = blob[384:384 + 4 * (tiles_r * tiles_c + 1)].view(np.uint32).astype(np.int64)
    return rows, cols, tile_cols, tiles_r, tiles_c, index


def walk(tiles_r, tiles_c, ctas, R, TT):
    """Per CTA, its present tiles (blob index u) in the kernel's order."""
    T = tiles_r * tiles_c
    out = []
    for c in range(ctas):
        a, b = T * c // ctas, T * (c + 1) // ctas
        i0, i1 = a // tiles_c, (b - 1) // tiles_c
        seq = []
        for ig in range(i0, i1 + 1, R):
            rg = min(R, i1 + 1 - ig)
            for rho in range((tiles_c + TT - 1) // TT):
                for t in range(TT):
                    j = rho * TT + t
                    if j >= tiles_c:
                        break
                    for r in range(rg):
                        v = (ig + r) * tiles_c + j
                        if a <= v < b:
                            seq.append(j * tiles_r + ig + r)
        out.append(seq)
    return out


CASES = [(8, 512, 512), (300, 2000, 512), (1024, 1024, 512), (77, 1032, 512), (129, 296, 256),
         (40, 200, 128), (17, 136, 64), (4100, 96, 512), (2048, 4096, 512), (1024, 4096, 512),
         (4096, 14336, 512), (520, 14336, 512), (20000, 1024, 512)]


@pytest.mark.parametrize("rows,cols,tile_cols", CASES)
@pytest.mark.parametrize("sms,smem", [(148, 232448), (132, 232448), (7, 232448), (148, 200000)])
def test_tc_schedule_invariants(rows, cols, tile_cols, sms, smem):
    blob = blob_of(rows, cols, tile_cols)
    _, _, _, tiles_r, tiles_c, index = header(blob)
    try:
        info, cta, bat, ring, tb = lib.nwc_tc_schedule_describe(blob, sms, smem)
    except lib.NwcError as e:
        assert e.status == 2                     # UNSUPPORTED: no layout fits
        return
    T = tiles_r * tiles_c
    C, R, TT, BT = info["ctas"], info["rows"], info["teams"], info["batch_tiles"]
    ring_bytes = info["ring_bytes"]
    assert C == min(T, sms, 256) and info["tiles"] == T
    assert 1 <= TT <= 8 and 1 <= R <= 16 and R * TT <= 16 and TT <= tiles_c
    assert info["smem_bytes"] <= smem
    assert info["a_offset"] % 1024 == 0 and info["b_offset"] % 1024 == 0
    assert info["b_offset"] == info["a_offset"] + 2 * TT * R * 1024
    assert info["ring_offset"] >= info["b_offset"] + 2 * TT * 8192
    chunk = 16 * np.diff(index)
    per_cta = -(-T // C)
    assert ring_bytes >= min(R + 2 * BT, per_cta) * chunk.max()
    seen = np.zeros(T, dtype=np.int64)
    for c, seq in enumerate(walk(tiles_r, tiles_c, C, R, TT)):
        b0, b1 = int(cta[c]), int(cta[c + 1])
        order = []
        vstart = []
        vhead = 0
        for k in range(b1 - b0):
            off16, nbytes, at, need = (int(v) for v in bat[b0 + k])
            # consecutive chunks starting at chunk off16
            u0 = int(np.searchsorted(index, off16))
            assert index[u0] == off16
            n = int(np.searchsorted(index, off16 + nbytes // 16)) - u0
            assert 1 <= n <= BT and 16 * (index[u0 + n] - index[u0]) == nbytes
            assert at % 16 == 0 and at + nbytes <= ring_bytes
            assert need <= k and need >= k - KMAX_OUTSTANDING + 1
            # first in, first out: the copy's bytes overlap no copy issued
            # after the released ones [0, need)
            pos = vhead if vhead % ring_bytes + nbytes <= ring_bytes else \
                vhead + ring_bytes - vhead % ring_bytes
            assert pos % ring_bytes == at
            for q in range(need, k):
                assert vstart[q][0] + vstart[q][1] <= pos or pos + nbytes <= vstart[q][0] + ring_bytes
                assert pos - vstart[q][0] < ring_bytes
            vstart.append((pos, nbytes))
            vhead = pos + nbytes
            for q in range(n):
                u = u0 + q
                order.append(u)
                assert ring[u] == at + 16 * (index[u] - index[u0])
                assert tb[u] & 0x0FFFFFFF == k
                assert tb[u] >> 28 == (BT - n if q == 0 else 0)
        assert order == seq, c
        for u in seq:
            seen[u] += 1
    assert (seen == 1).all()


def test_tc_shape_takes_the_fewest_rounds():
    """A 4096 x 4096 matrix gives each of 148 CTAs 28 tiles over at most 5 row
    tiles: one M-group of 5 rows with 3 teams takes 3 rounds of column blocks,
    where 4 rows x 4 teams would take 2 groups x 2 rounds."""
    info = lib.nwc_tc_schedule_describe(blob_of(4096, 4096))[0]
    assert (info["rows"], info["teams"]) == (5, 3)
    tall = lib.nwc_tc_schedule_describe(blob_of(20000, 1024))[0]
    assert tall["rows"] * tall["teams"] >= 14
