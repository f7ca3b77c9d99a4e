"""The launch schedule (host logic, no GPU): which bytes each bulk copy moves,
where they land in a CTA's shared-memory ring, and which earlier copies must
have been released first.  The kernels follow it blindly, so every property the
pipeline relies on is checked here, on blobs of several shapes and devices."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

K_SLOTS = 64          # barrier slots per CTA (kernels.cuh)
K_MAX_LAG = 48        # tiles a consumer's next wait may lie past its last release (kernels.cuh)
K_MAX_CTAS = 256
K_XSTAGE = {1: 8448, 16: 33024}  # shared memory for x by rows of x per launch (kernels.cuh)
K_RING_SLACK = 512    # shared memory after the ring that readers may touch (kernels.cu)
B200_SMS, B200_SMEM = 148, 232448


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


def blob_of(lib, rows, cols, tile_cols=512, lmax=0, kind="normal", seed=0):
    w = synth.matrix(synth.MatrixSpec("w", rows, cols, kind, 0.02, 0), seed)
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols)
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    return blob


def index_of(blob):
    tiles_r = int.from_bytes(blob[40:48].tobytes(), "little")
    tiles_c = int.from_bytes(blob[48:56].tobytes(), "little")
    n = tiles_r * tiles_c
    return np.frombuffer(blob[384:384 + 4 * (n + 1)].tobytes(), dtype=np.uint32).astype(np.int64)


def check_schedule(lib, blob, sms, smem, rows_of_x=1):
    info, cta, bat, ring = lib.nwc_schedule_describe(blob, sms, smem, rows_of_x)
    index = index_of(blob)
    n_tiles = len(index) - 1
    C, T, R = info["ctas"], info["batch_tiles"], info["ring_bytes"]
    assert info["tiles"] == n_tiles
    assert C == min(n_tiles, sms, K_MAX_CTAS)
    assert 2 <= T <= 8
    assert R % 16 == 0 and info["smem_bytes"] <= smem
    assert info["xstage_bytes"] == K_XSTAGE[1 if rows_of_x <= 4 else 16]
    assert cta[0] == 0 and cta[C] == info["batches"] == len(bat)
    max_out = K_SLOTS - -(-K_MAX_LAG // T)
    for c in range(C):
        first, last = n_tiles * c // C, n_tiles * (c + 1) // C
        b0, b1 = int(cta[c]), int(cta[c + 1])
        assert b1 - b0 == -(-(last - first) // T)
        prev_need = 0
        for k in range(b1 - b0):
            src, nbytes, at, need = (int(v) for v in bat[b0 + k])
            q0, q1 = first + k * T, min(first + (k + 1) * T, last)
            # The copy moves exactly the batch's chunks.
            assert src == index[q0] and nbytes == 16 * (index[q1] - index[q0])
            # It lands 16-byte aligned, inside the ring, without wrapping.
            assert at % 16 == 0 and at + nbytes <= R
            for q in range(q0, q1):
                assert ring[q] == at + 16 * (index[q] - index[q0])
            # Releases are awaited in order, never for itself or later batches,
            # and enough of them to bound the outstanding copies.
            assert prev_need <= need <= k
            assert k - need < max_out
            prev_need = need
            # Room: no batch still outstanding at issue time shares a byte.
            for m in range(need, k):
                _, mb, mat, _ = (int(v) for v in bat[b0 + m])
                assert mat + mb <= at or at + nbytes <= mat, (c, k, m)


@pytest.mark.parametrize("rows,cols,tile_cols", [(4096, 4096, 512), (1024, 1024, 512),
                                                 (14336, 512, 512), (77, 1030, 256),
                                                 (1000, 1026, 128), (4100, 96, 64), (8, 64, 64)])
def test_schedule_invariants_b200(lib, rows, cols, tile_cols):
    blob = blob_of(lib, rows, cols, tile_cols)
    for rows_of_x in (0, 1, 4, 5, 16):
        check_schedule(lib, blob, B200_SMS, B200_SMEM, rows_of_x)


def test_schedule_classes_differ_in_ring(lib):
    """Launches of up to 4 rows of x reserve less shared memory for x, so their
    ring is larger by up to the difference (a ring never exceeds what the CTA's
    tiles need)."""
    blob = blob_of(lib, 4096, 4096)
    small, _, _, _ = lib.nwc_schedule_describe(blob, B200_SMS, B200_SMEM, 1)
    large, _, _, _ = lib.nwc_schedule_describe(blob, B200_SMS, B200_SMEM, 16)
    assert 0 < small["ring_bytes"] - large["ring_bytes"] <= K_XSTAGE[16] - K_XSTAGE[1]
    assert small["smem_bytes"] <= large["smem_bytes"] <= B200_SMEM


@pytest.mark.parametrize("sms,smem", [(1, B200_SMEM), (3, 100_000), (148, 120_000),
                                      (1000, B200_SMEM), (7, 80_000)])
def test_schedule_invariants_other_devices(lib, sms, smem):
    # Small rings force wrap-around and waits on many releases; many SMs hit
    # the CTA cap.
    blob = blob_of(lib, 2048, 2048, 512, lmax=12, kind="student_t5", seed=3)
    check_schedule(lib, blob, sms, smem)
    if smem >= 100_000:
        check_schedule(lib, blob, sms, smem, 16)


def test_schedule_tight_ring_serialises(lib):
    """A ring with room for one batch only makes every copy wait for the
    release of the one before it."""
    blob = blob_of(lib, 64, 4096, 512, lmax=12, kind="student_t5", seed=3)
    info, _, bat, _ = lib.nwc_schedule_describe(blob, 1, B200_SMEM)
    T = info["batch_tiles"]
    index = index_of(blob)
    max_chunk = int(16 * np.diff(index).max())
    ring_offset = -(-(-(-(16384 + 8 + 2 * K_SLOTS * 8) // 16) * 16 + K_XSTAGE[1]) // 128) * 128
    smem = ring_offset + T * max_chunk + K_RING_SLACK  # ring of one worst-case batch + read slack
    assert 2 * int(bat[:-1, 1].min()) > T * max_chunk + 16  # the last batch may be short
    info, _, bat, _ = lib.nwc_schedule_describe(blob, 1, smem)
    assert info["ring_bytes"] == T * max_chunk
    assert [int(v) for v in bat[:-1, 3]] == list(range(len(bat) - 1))
    check_schedule(lib, blob, 1, smem)


def test_schedule_errors(lib):
    blob = blob_of(lib, 64, 1024)
    with pytest.raises(lib.NwcError):
        lib.nwc_schedule_describe(blob[:200], B200_SMS, B200_SMEM)
    with pytest.raises(lib.NwcError):
        lib.nwc_schedule_describe(blob, 0, B200_SMEM)
    with pytest.raises(lib.NwcError):  # more rows than one launch takes
        lib.nwc_schedule_describe(blob, B200_SMS, B200_SMEM, 17)
    with pytest.raises(lib.NwcError):  # a 64 KiB decode table alone does not fit
        lib.nwc_schedule_describe(blob, B200_SMS, 60_000)
