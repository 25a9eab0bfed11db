"""Test-side packers: logical quant values -> block bytes.

Written from the block layouts alone (the inverse direction of the oracle's
decoders, in separate code), so a misplaced bit or index in either side makes
the round-trip tests fail.
"""
import numpy as np


def f16_bits(v: float) -> int:
    return int(np.array(v, dtype=np.float16).view(np.uint16))


def pack_q8_0(d_bits: int, q) -> bytes:
    q = [int(v) for v in q]
    assert len(q) == 32 and all(-128 <= v <= 127 for v in q)
    return bytes([d_bits & 0xFF, d_bits >> 8]) + bytes([v & 0xFF for v in q])


def pack_q4_0(d_bits: int, q) -> bytes:
    q = [int(v) for v in q]
    assert len(q) == 32 and all(0 <= v <= 15 for v in q)
    return bytes([d_bits & 0xFF, d_bits >> 8]) + bytes([q[j] | (q[j + 16] << 4) for j in range(16)])


def pack_q4_k(d_bits: int, dmin_bits: int, sc, m, q) -> bytes:
    sc, m, q = [int(v) for v in sc], [int(v) for v in m], [int(v) for v in q]
    assert len(sc) == 8 and len(m) == 8 and len(q) == 256
    assert all(0 <= v < 64 for v in sc + m) and all(0 <= v < 16 for v in q)
    s = [0] * 12
    for j in range(8):
        if j < 4:
            s[j] |= sc[j]
            s[j + 4] |= m[j]
        else:
            s[j + 4] |= (sc[j] & 15) | ((m[j] & 15) << 4)
            s[j - 4] |= (sc[j] >> 4) << 6
            s[j] |= (m[j] >> 4) << 6
    codes = [0] * 128
    for e in range(256):
        chunk, r = divmod(e, 64)
        byte = 32 * chunk + (r % 32)
        codes[byte] |= q[e] if r < 32 else (q[e] << 4)
    return bytes([d_bits & 0xFF, d_bits >> 8, dmin_bits & 0xFF, dmin_bits >> 8] + s + codes)


def pack_q6_k(d_bits: int, sc, q) -> bytes:
    sc, q = [int(v) for v in sc], [int(v) for v in q]
    assert len(sc) == 16 and len(q) == 256 and all(0 <= v < 64 for v in q)
    ql = [0] * 128
    qh = [0] * 64
    for e in range(256):
        h, t = divmod(e, 128)
        lo, hi = q[e] & 15, q[e] >> 4
        if t < 64:
            ql[64 * h + t] |= lo
        else:
            ql[64 * h + t - 64] |= lo << 4
        qh[32 * h + t % 32] |= hi << (2 * (t // 32))
    return bytes(ql + qh + [v & 0xFF for v in sc] + [d_bits & 0xFF, d_bits >> 8])


def pack_q5_k(d_bits: int, dmin_bits: int, sc, m, q) -> bytes:
    sc, m, q = [int(v) for v in sc], [int(v) for v in m], [int(v) for v in q]
    assert len(sc) == 8 and len(m) == 8 and len(q) == 256
    assert all(0 <= v < 64 for v in sc + m) and all(0 <= v < 32 for v in q)
    # scales and mins exactly as Q4_K: reuse that packer's 12 bytes
    s = list(pack_q4_k(0, 0, sc, m, [0] * 256)[4:16])
    qh = [0] * 32
    qs = [0] * 128
    for e in range(256):
        chunk, r = divmod(e, 64)
        upper, lane = divmod(r, 32)
        qs[32 * chunk + lane] |= (q[e] & 15) << (4 * upper)
        qh[lane] |= (q[e] >> 4) << (2 * chunk + upper)
    return bytes([d_bits & 0xFF, d_bits >> 8, dmin_bits & 0xFF, dmin_bits >> 8] + s + qh + qs)


def pack_f16(bits) -> bytes:
    return b"".join(bytes([int(v) & 0xFF, int(v) >> 8]) for v in bits)


def pack_f32(values) -> bytes:
    return np.array(values, dtype=np.float32).tobytes()


def logical_weights(qtype: int, fields: dict) -> list:
    """Exact (Fraction) weights of one block from its logical fields."""
    from fractions import Fraction as Fr

    def f16(bits):
        return Fr(float(np.array(bits, dtype=np.uint16).view(np.float16)))

    if qtype == 0:
        d = f16(fields["d"])
        return [d * v for v in fields["q"]]
    if qtype == 1:
        d = f16(fields["d"])
        return [d * (v - 8) for v in fields["q"]]
    if qtype == 2:
        d, dmin = f16(fields["d"]), f16(fields["dmin"])
        return [d * fields["sc"][e // 32] * fields["q"][e] - dmin * fields["m"][e // 32] for e in range(256)]
    if qtype == 3:
        d = f16(fields["d"])
        return [d * fields["sc"][e // 16] * (fields["q"][e] - 32) for e in range(256)]
    if qtype == 4:
        d, dmin = f16(fields["d"]), f16(fields["dmin"])
        return [d * fields["sc"][e // 32] * fields["q"][e] - dmin * fields["m"][e // 32] for e in range(256)]
    if qtype == 5:
        return [f16(b) for b in fields["bits"]]
    if qtype == 6:
        return [Fr(float(v)) for v in np.array(fields["values"], dtype=np.float32)]
    raise ValueError(qtype)


def random_fields(qtype: int, rng: np.random.Generator, d_range=(1e-3, 1e-2)) -> dict:
    d = f16_bits(rng.uniform(*d_range))
    if qtype == 0:
        return {"d": d, "q": rng.integers(-127, 128, 32)}
    if qtype == 1:
        return {"d": d, "q": rng.integers(0, 16, 32)}
    if qtype == 2:
        return {"d": d, "dmin": f16_bits(rng.uniform(*d_range)), "sc": rng.integers(0, 64, 8),
                "m": rng.integers(0, 64, 8), "q": rng.integers(0, 16, 256)}
    if qtype == 3:
        return {"d": d, "sc": rng.integers(-127, 128, 16), "q": rng.integers(0, 64, 256)}
    if qtype == 4:
        return {"d": d, "dmin": f16_bits(rng.uniform(*d_range)), "sc": rng.integers(0, 64, 8),
                "m": rng.integers(0, 64, 8), "q": rng.integers(0, 32, 256)}
    if qtype == 5:
        # finite binary16 patterns of both signs, subnormals included
        bits = rng.integers(0, 0x7C00, 1) | (rng.integers(0, 2, 1) << 15)
        return {"bits": bits}
    if qtype == 6:
        return {"values": rng.standard_normal(1).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30)}
    raise ValueError(qtype)


def pack(qtype: int, f: dict) -> bytes:
    if qtype == 0:
        return pack_q8_0(f["d"], f["q"])
    if qtype == 1:
        return pack_q4_0(f["d"], f["q"])
    if qtype == 2:
        return pack_q4_k(f["d"], f["dmin"], f["sc"], f["m"], f["q"])
    if qtype == 3:
        return pack_q6_k(f["d"], f["sc"], f["q"])
    if qtype == 4:
        return pack_q5_k(f["d"], f["dmin"], f["sc"], f["m"], f["q"])
    if qtype == 5:
        return pack_f16(f["bits"])
    if qtype == 6:
        return pack_f32(f["values"])
    raise ValueError(qtype)


def parse_golden(path: str):
    """Blocks of a tests/golden/*_blocks.txt fixture: list of (title, bytes, [Fraction])."""
    from fractions import Fraction as Fr

    def expand(tokens, item):
        out = []
        i = 0
        while i < len(tokens):
            t = tokens[i]
            if t.startswith("("):
                depth, j, group = 0, i, []
                while True:
                    tok = tokens[j]
                    depth += tok.count("(") - tok.count(")")
                    group.append(tok)
                    if depth == 0:
                        break
                    j += 1
                text = " ".join(group)
                inner, rep = text[1:].rsplit(")", 1)
                n = int(rep[1:]) if rep.startswith("*") else 1
                out += expand(inner.split(), item) * n
                i = j + 1
                continue
            n = 1
            if "*" in t:
                a, t = t.split("*", 1)
                n = int(a)
            out += item(t) * n
            i += 1
        return out

    def byte_item(t):
        return [int(t, 16)]

    def val_item(t):
        if ".." in t:
            a, b = t.split("..")
            a, b = int(a), int(b)
            step = 1 if b >= a else -1
            return [Fr(v) for v in range(a, b + step, step)]
        return [Fr(t)]

    blocks = []
    title = None
    raw = None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "block":
            title = rest
        elif key == "bytes":
            raw = bytes(expand(rest.split(), byte_item))
        elif key == "expect":
            blocks.append((title, raw, expand(rest.split(), val_item)))
    return blocks
