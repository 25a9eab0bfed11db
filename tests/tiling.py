"""Test-side model of the tiled layouts: GGUF-style bytes -> tiled bytes, written
from the layout description in include/ntx.h (the NTX_*_T comment) with numpy,
separately from the library's repack kernel, so the kernel's output can be
checked byte for byte against the documented layout."""
import numpy as np

Q8_0, Q4_0, Q4_K, Q6_K, Q5_K = 0, 1, 2, 3, 4


def _fields(qtype, host, rows, cols):
    """Logical fields of a GGUF-style matrix: codes [rows, cols] and scale arrays."""
    b = host.reshape(rows, -1)
    if qtype == Q8_0:
        blk = b.reshape(rows, cols // 32, 34)
        return dict(code=blk[:, :, 2:].view(np.int8).reshape(rows, cols).astype(np.int32),
                    d=blk[:, :, 0:2].copy().view(np.uint16)[:, :, 0])
    if qtype == Q4_0:
        blk = b.reshape(rows, cols // 32, 18)
        c = blk[:, :, 2:].astype(np.int32)
        code = np.concatenate([c & 15, c >> 4], axis=2).reshape(rows, cols)
        return dict(code=code, d=blk[:, :, 0:2].copy().view(np.uint16)[:, :, 0])
    if qtype == Q6_K:
        blk = b.reshape(rows, cols // 256, 210).astype(np.int32)
        code = np.zeros((rows, cols // 256, 256), np.int32)
        for e in range(256):
            h, t = e >> 7, e & 127
            lo = (blk[:, :, 64 * h + t] & 15) if t < 64 else (blk[:, :, 64 * h + t - 64] >> 4)
            hi = (blk[:, :, 128 + 32 * h + (t & 31)] >> (2 * (t >> 5))) & 3
            code[:, :, e] = lo | (hi << 4)
        sc = b.reshape(rows, cols // 256, 210)[:, :, 192:208]
        d = b.reshape(rows, cols // 256, 210)[:, :, 208:210].copy().view(np.uint16)[:, :, 0]
        return dict(code=code.reshape(rows, cols), sc=sc.copy(), d=d)
    bb = 176 if qtype == Q5_K else 144
    blk = b.reshape(rows, cols // 256, bb).astype(np.int32)
    code = np.zeros((rows, cols // 256, 256), np.int32)
    for e in range(256):
        c, r = e >> 6, e & 63
        if qtype == Q5_K:
            # fp16 d | fp16 dmin | 12 B scales | 32 B fifth bits | 128 B low nibbles
            byte = blk[:, :, 48 + 32 * c + (r & 31)]
            b5 = (blk[:, :, 16 + (r & 31)] >> (2 * c + (r >> 5))) & 1
            code[:, :, e] = ((byte & 15) if r < 32 else (byte >> 4)) | (b5 << 4)
        else:
            byte = blk[:, :, 16 + 32 * c + (r & 31)]
            code[:, :, e] = (byte & 15) if r < 32 else (byte >> 4)
    s = blk[:, :, 4:16]
    sc = np.zeros((rows, cols // 256, 8), np.int32)
    mn = np.zeros((rows, cols // 256, 8), np.int32)
    for j in range(8):
        if j < 4:
            sc[:, :, j] = s[:, :, j] & 63
            mn[:, :, j] = s[:, :, j + 4] & 63
        else:
            sc[:, :, j] = (s[:, :, j + 4] & 15) | ((s[:, :, j - 4] >> 6) << 4)
            mn[:, :, j] = (s[:, :, j + 4] >> 4) | ((s[:, :, j] >> 6) << 4)
    raw = b.reshape(rows, cols // 256, bb)
    return dict(code=code.reshape(rows, cols), sc=sc, mn=mn, d=raw[:, :, 0:2].copy().view(np.uint16)[:, :, 0],
                dmin=raw[:, :, 2:4].copy().view(np.uint16)[:, :, 0])


def _h16(v):
    return [int(v) & 0xFF, int(v) >> 8]


def tile(qtype, host, rows, cols):
    """Tiled bytes (uint8 array of rows * row_bytes) of a GGUF-style matrix."""
    assert rows % 16 == 0
    f = _fields(qtype, host, rows, cols)
    code = f["code"]
    out = []
    uk = 32 if qtype in (Q8_0, Q4_0) else 256
    for g in range(rows // 16):
        r0 = 16 * g
        for u in range(cols // uk):
            c0 = uk * u
            unit = []
            if qtype == Q8_0:
                for lane in range(32):
                    gid, tig = lane >> 2, lane & 3
                    for reg in range(4):
                        row = r0 + gid + 8 * (reg & 1)
                        for j in range(4):
                            unit.append(code[row, c0 + 16 * (reg >> 1) + 4 * tig + j] & 0xFF)
                for gid in range(8):
                    unit += _h16(f["d"][r0 + gid, u]) + _h16(f["d"][r0 + gid + 8, u])
            elif qtype == Q4_0:
                for lane in range(32):
                    gid, tig = lane >> 2, lane & 3
                    for hi in range(2):
                        row = r0 + gid + 8 * hi
                        for j in range(4):
                            c = c0 + 4 * tig + j
                            unit.append(code[row, c] | (code[row, c + 16] << 4))
                for gid in range(8):
                    unit += _h16(f["d"][r0 + gid, u]) + _h16(f["d"][r0 + gid + 8, u])
            elif qtype == Q6_K:
                for m in range(8):
                    for lane in range(32):
                        gid, tig = lane >> 2, lane & 3
                        cc = c0 + 32 * m + 4 * tig
                        a = [code[r0 + gid, cc:cc + 4], code[r0 + gid + 8, cc:cc + 4], code[r0 + gid, cc + 16:cc + 20]]
                        a3 = code[r0 + gid + 8, cc + 16:cc + 20]
                        for w in range(3):
                            for j in range(4):
                                unit.append(int(a[w][j]) | (((int(a3[j]) >> (2 * w)) & 3) << 6))
                for gid in range(8):
                    for par in range(2):
                        for hi in range(2):
                            for mm in range(8):
                                unit.append(int(f["sc"][r0 + gid + 8 * hi, u, 2 * mm + par]))
                for gid in range(8):
                    unit += _h16(f["d"][r0 + gid, u]) + _h16(f["d"][r0 + gid + 8, u])
            else:
                for m in range(8):
                    for lane in range(32):
                        gid, tig = lane >> 2, lane & 3
                        for hi in range(2):
                            row = r0 + gid + 8 * hi
                            for j in range(4):
                                c = c0 + 32 * m + 4 * tig + j
                                unit.append((code[row, c] & 15) | ((code[row, c + 16] & 15) << 4))
                    if qtype == Q5_K:
                        # fifth bits: per gid words H0 (row gid), H1 (row gid + 8); the bit of
                        # column 4 t + j at 8 j + 2 t, of column 16 + 4 t + j at 8 j + 2 t + 1
                        for gid in range(8):
                            for hi in range(2):
                                row = r0 + gid + 8 * hi
                                for j in range(4):
                                    v = 0
                                    for t in range(4):
                                        c = c0 + 32 * m + 4 * t + j
                                        v |= ((code[row, c] >> 4) & 1) << (2 * t)
                                        v |= ((code[row, c + 16] >> 4) & 1) << (2 * t + 1)
                                    unit.append(v)
                for gid in range(8):
                    V = lambda m, b: int((f["mn"] if b & 2 else f["sc"])[r0 + gid + 8 * (b & 1), u, m])
                    for wn in range(4):
                        for b in range(4):
                            unit.append((V(2 * wn, b) & 15) | ((V(2 * wn + 1, b) & 15) << 4))
                    for wh in range(2):
                        for b in range(4):
                            unit.append(sum(((V(4 * wh + t, b) >> 4) & 3) << (2 * t) for t in range(4)))
                for gid in range(8):
                    unit += _h16(f["d"][r0 + gid, u]) + _h16(f["d"][r0 + gid + 8, u])
                    unit += _h16(f["dmin"][r0 + gid, u]) + _h16(f["dmin"][r0 + gid + 8, u])
            out.append(np.array(unit, dtype=np.uint8))
    return np.concatenate(out)
