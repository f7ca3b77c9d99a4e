"""A second, pure-Python reader of the NWB1 blob format (test helper), with 1,
2 or 4 bit streams per lane, and of its variant NWE1 (verbatim runs for rare
exponents).

Written from the format statement alone, in a different language and style
from the oracle's C++ decoder, so that the encoder is checked against the
format and not only against its own decoder.  Slow; small blobs only."""
import struct

import numpy as np


def parse(blob: bytes):
    b = bytes(blob)
    (magic, version, hdr, lmax, rows, cols, tile_rows, tile_cols, tiles_r, tiles_c,
     filler, zero, lens_off, index_off, tiles_off, total, coded_bits) = struct.unpack_from(
        "<IIIIQQIIQQIIQQQQQ", b, 0)
    assert magic in (0x3142574E, 0x3145574E) and version == 1 and hdr == 128, "header"
    assert total == len(b), "total bytes"
    verbatim = magic == 0x3145574E  # NWE1: offset 60 holds the kept exponents
    streams = 1 if verbatim else zero + 1   # bit streams per lane and tile
    assert streams in (1, 2, 4), "streams per lane"
    lens = list(b[lens_off:lens_off + 256])
    n_tiles = tiles_r * tiles_c
    index = struct.unpack_from(f"<{n_tiles + 1}I", b, index_off)
    return dict(lmax=lmax, rows=rows, cols=cols, tile_rows=tile_rows, tile_cols=tile_cols,
                tiles_r=tiles_r, tiles_c=tiles_c, filler=filler, lens=lens,
                index=index, tiles_off=tiles_off, total=total, coded_bits=coded_bits,
                streams=streams, verbatim=verbatim, kept=zero if verbatim else None,
                verbatim_runs=struct.unpack_from("<Q", b, 104)[0] if verbatim else None)


def codebook(lens):
    """{bitstring: symbol} by the canonical rule: sort by (length, symbol)."""
    order = sorted((l, s) for s, l in enumerate(lens) if l)
    book, value, prev = {}, None, None
    for l, s in order:
        value = 0 if value is None else (value + 1) << (l - prev)
        prev = l
        book[format(value, f"0{l}b")] = s
    return book


def sequence_bits(area: bytes) -> str:
    """Bit i of the sequence is bit 31 - i % 32 of little-endian word i // 32."""
    out = []
    for w in struct.unpack(f"<{len(area) // 4}I", area):
        out.append(format(w, "032b"))
    return "".join(out)


def decode(blob: bytes) -> np.ndarray:
    h = parse(blob)
    b = bytes(blob)
    book = codebook(h["lens"])
    rows, cols, tr, tc = h["rows"], h["cols"], h["tile_rows"], h["tile_cols"]
    out = np.zeros((rows, cols), dtype=np.uint16)
    per_lane = 2 * tr * (tc // 64)
    S = h["streams"]
    n_streams = 32 * S
    for u in range(h["tiles_r"] * h["tiles_c"]):
        i, j = u % h["tiles_r"], u // h["tiles_r"]
        c0 = h["tiles_off"] + 16 * h["index"][u]
        c1 = h["tiles_off"] + 16 * h["index"][u + 1]
        raw = b[c0:c0 + tr * tc]
        head = c0 + tr * tc
        runs = {}                   # NWE1: (row, group) -> its 64 verbatim exponent bytes
        if h["verbatim"]:
            flags = b[head:head + 16]
            at = head + 16
            for r in range(tr):
                for m in range(tc // 64):
                    if flags[r] >> m & 1:
                        runs[(r, m)] = b[at:at + 64]
                        at += 64
            head = at
        lane_len = b[head:head + n_streams]
        bits = sequence_bits(b[head + n_streams:c1])
        start = 0
        for sigma in range(n_streams):
            # Stream sigma: lane sigma // S, the lane's symbol pairs q with q % S == sigma % S.
            t = sigma // S
            s = bits[start:start + 8 * lane_len[sigma]]
            start += 8 * lane_len[sigma]
            p = 0
            for k in [k for k in range(per_lane) if (k // 2) % S == sigma % S]:
                r = t // 4
                c = 64 * (k // 16) + 16 * (t % 4) + k % 16
                if (r, k // 16) in runs:
                    sym = runs[(r, k // 16)][c - 64 * (k // 16)]
                else:
                    q = p + 1
                    while s[p:q] not in book:
                        q += 1
                        assert q - p <= h["lmax"], "no code"
                    sym = book[s[p:q]]
                    p = q
                rb = raw[(k // 16) * 512 + 16 * t + k % 16]
                row, col = i * tr + r, j * tc + c
                if row < rows and col < cols:
                    out[row, col] = ((rb >> 7) << 15) | (sym << 7) | (rb & 0x7F)
                else:
                    assert sym == h["filler"] and rb == 0, "filler"
            assert set(s[p:]) <= {"0"} and len(s) - p < 8, "lane padding"
        assert set(bits[start:]) <= {"0"}, "area padding"
    return out
