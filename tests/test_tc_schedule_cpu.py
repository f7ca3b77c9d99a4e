"""The tensor-core kernel's launch schedules, checked on the CPU (no GPU).

The kernel splits K into ksplit column ranges and the row tiles into
ctas / ksplit row ranges (part k of n over m items: [m k / n, m (k + 1) / n));
CTA c = rs ksplit + ks owns row range rs x column range ks and walks it in
M-groups of R row tiles, round by round, team by team (team t takes column
blocks j_lo + t, j_lo + t + teams, ...), row by row.  This test restates that
walk independently and checks that each schedule (one per accumulator width)
brings exactly those tiles' lane lengths and streams (the chunk after its raw
plane), in that order, one copy per tile, never wrapping the ring, never
overwriting a copy still outstanding, keeping fewer than 64 copies
outstanding, and that every tile belongs to exactly one CTA.
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


def walk(tiles_r, tiles_c, ctas, R, TT, KS):
    """Per CTA, its tiles (blob index u) in the kernel's order."""
    assert ctas % KS == 0
    RS = ctas // KS
    out = []
    for c in range(ctas):
        ks, rs = c % KS, c // KS
        i_lo, i_hi = tiles_r * rs // RS, tiles_r * (rs + 1) // RS
        j_lo, j_hi = tiles_c * ks // KS, tiles_c * (ks + 1) // KS
        seq = []
        ig = i_lo
        while ig < i_hi:
            rg = min(R, i_hi - ig)
            j0 = j_lo
            while j0 < j_hi:
                for t in range(TT):
                    if j0 + t >= j_hi:
                        break
                    seq += [(j0 + t) * tiles_r + ig + r for r in range(rg)]
                j0 += TT
            ig += R
        out.append(seq)
    return out


CASES = [(8, 512, 512), (300, 2000, 512), (1024, 1024, 512), (77, 1032, 512), (129, 296, 256),
         (40, 200, 128), (17, 136, 64), (4100, 96, 512), (2048, 4096, 512), (1024, 4096, 512),
         (4096, 14336, 512), (520, 14336, 512), (20000, 1024, 512)]


@pytest.mark.parametrize("rows,cols,tile_cols", CASES)
@pytest.mark.parametrize("sms,smem", [(148, 232448), (132, 232448), (7, 232448), (148, 200000)])
@pytest.mark.parametrize("rows_of_x", [1, 32, 64])
def test_tc_schedule_invariants(rows, cols, tile_cols, sms, smem, rows_of_x):
    blob = blob_of(rows, cols, tile_cols)
    _, _, _, tiles_r, tiles_c, index = header(blob)
    try:
        info, cta, bat, ring, tb = lib.nwc_tc_schedule_describe(blob, sms, smem, rows_of_x)
    except lib.NwcError as e:
        assert e.status == 2                     # UNSUPPORTED: no layout fits
        return
    T = tiles_r * tiles_c
    C, R, TT, N, SB = info["ctas"], info["rows"], info["teams"], info["n"], info["x_stages"]
    KS = info["ksplit"]
    ring_bytes = info["ring_bytes"]
    raw = 8 * tile_cols
    # The split stays within the scratch slots: at most tiles_c / 4 parts.
    assert KS == 1 or 2 <= KS <= tiles_c // 4
    assert C % KS == 0 and C // KS == min(tiles_r, min(sms, 256) // KS)
    assert info["tiles"] == T and info["batch_tiles"] == 1
    assert N == (16 if rows_of_x <= 16 else 32 if rows_of_x <= 32 else 64)
    assert 1 <= TT <= 15 and 1 <= R <= 16 and R * TT <= 30 and TT * N <= 512
    assert TT <= -(-tiles_c // KS)
    assert SB in (1, 2) and info["smem_bytes"] <= smem
    assert info["a_offset"] % 1024 == 0 and info["b_offset"] % 1024 == 0
    NA = info["a_stages"]
    assert SB <= NA <= 3
    assert info["b_offset"] == info["a_offset"] + NA * TT * R * 1024
    assert info["ring_offset"] >= info["b_offset"] + TT * SB * N * 128
    streams = 16 * np.diff(index) - raw
    per_cta = -(-tiles_r // (C // KS)) * -(-tiles_c // KS)
    assert ring_bytes >= min(R + 2, per_cta) * streams.max()
    seen = np.zeros(T, dtype=np.int64)
    for c, seq in enumerate(walk(tiles_r, tiles_c, C, R, TT, KS)):
        b0, b1 = int(cta[c]), int(cta[c + 1])
        assert b1 - b0 == len(seq)
        vstart = []
        vhead = 0
        for k, u in enumerate(seq):
            off16, nbytes, at, need = (int(v) for v in bat[b0 + k])
            # the tile's lane lengths and streams: after its raw plane
            assert off16 == index[u] + raw // 16 and nbytes == 16 * index[u + 1] - 16 * off16
            assert at % 16 == 0 and at + nbytes <= ring_bytes
            assert need <= k and need >= k - KMAX_OUTSTANDING + 1
            pos = vhead if vhead % ring_bytes + nbytes <= ring_bytes else \
                vhead + ring_bytes - vhead % ring_bytes
            assert pos % ring_bytes == at
            for q in range(need, k):                    # no overlap with outstanding copies
                assert pos - vstart[q][0] < ring_bytes
                assert vstart[q][0] + vstart[q][1] <= pos or pos + nbytes <= vstart[q][0] + ring_bytes
            vstart.append((pos, nbytes))
            vhead = pos + nbytes
            assert ring[u] == at and tb[u] == k
            seen[u] += 1
    assert (seen == 1).all()


def rounds(info, tiles_r, tiles_c):
    KS, RS = info["ksplit"], info["ctas"] // info["ksplit"]
    rows_c, cols_c = -(-tiles_r // RS), -(-tiles_c // KS)
    return -(-rows_c // info["rows"]) * -(-cols_c // info["teams"])


def test_tc_shape_prefers_two_x_stages_then_the_fewest_rounds():
    """A 4096 x 4096 matrix (512 x 8 tiles) on 148 SMs.  With accumulators of
    16 or 32 columns the x stages are small: two per team, K split in two, 74
    row ranges of 6 or 7 row tiles x 4 column blocks, one M-group of 7 rows and
    4 teams, every decode warp one tile with its streams resident.  At 64
    columns two x stages per team take 64 KiB: they are kept (with one, a
    team's next x chunk waits for its last MMAs), and the shape with every
    warp's streams resident is then 4 teams of 4 rows without a split, in two
    rounds."""
    blob = blob_of(4096, 4096)
    _, _, _, _, _, index = header(blob)
    streams = int((16 * np.diff(index) - 4096).max())
    for rows_of_x in (1, 17):
        info = lib.nwc_tc_schedule_describe(blob, rows_of_x=rows_of_x)[0]
        assert (info["ksplit"], info["ctas"], info["rows"], info["teams"]) == (2, 148, 7, 4)
        assert info["x_stages"] == 2 and rounds(info, 512, 8) == 1
        assert info["ring_bytes"] >= 28 * streams
    info = lib.nwc_tc_schedule_describe(blob, rows_of_x=64)[0]
    assert (info["ksplit"], info["ctas"], info["rows"], info["teams"]) == (1, 148, 4, 4)
    assert info["x_stages"] == 2 and rounds(info, 512, 8) == 2
    assert info["ring_bytes"] >= 18 * streams


@pytest.mark.parametrize("rows,cols,best", [(14336, 4096, 4), (4096, 14336, 4), (1024, 4096, 1),
                                            (20000, 1024, 2)])
def test_tc_shape_rounds_meet_the_bound(rows, cols, best):
    """The fewest rounds any rectangle split can give: at least the tiles of
    the largest rectangle over 30 decode warps."""
    blob = blob_of(rows, cols)
    tiles_r, tiles_c = rows // 8, cols // 512
    info = lib.nwc_tc_schedule_describe(blob, rows_of_x=64)[0]
    assert rounds(info, tiles_r, tiles_c) == best
    assert best >= -(-(tiles_r * tiles_c) // (148 * 30))
