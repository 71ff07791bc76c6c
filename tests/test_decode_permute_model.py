"""A CPU model of the byte-permute group decode, checked against the
per-element table decode on every scale byte and every code in every position.

The fp16 operand decoders (if4_decode_f16, the fused-decode linear) and the
round trip's bf16 output decode a group without a table load per element.  They
round the group's eight magnitudes once, t[m] = out(fl32(base[m] * eff)) for
m = 0..7 (base: the FP4 magnitudes, or the INT4 magnitudes fl32(k * fl(6/7))),
and split them into a low-byte and a high-byte plane of 8 bytes each.  Each
element's magnitude index is formed eight nibbles at a time: m = n & 7 for
FP4, and for INT4 (two's complement) m = n & 7 for n < 8 and 8 - (n & 7)
above.  A byte permute (prmt) picks four elements' bytes from each plane.  A
second permute of the code word and its 4-bit shift puts every element's sign
bit at bit 7 of its high byte, and a third interleaves the planes into
16-bit pairs.  Rounding is symmetric in sign, so -t[m] is the rounded
negative value.  INT4 code 8 (k = -8, which the encoder never emits) has m = 8,
which the planes cannot hold.  It is flagged (bit 3 of m), and the kernels
decode such a group with the per-element table.

This models the permute and nibble arithmetic bit for bit (prmt in its
default mode, sign-replicating selector bit included) and checks it against
decoding each element from its nibble alone.  It does not run the kernels
(the GPU parity tests do)."""
import numpy as np
import pytest

F32 = np.float32
C67 = F32(6.0) / F32(7.0)                                     # fl(6/7)
FP4_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=F32)
INT4_MAG = (np.arange(8, dtype=F32) * C67).astype(F32)        # fl32(k * fl(6/7))


def e4m3_value(sb):
    """Magnitude of E4M3 byte sb (bit 7 ignored: it selects INT4)."""
    b = sb & 0x7F
    e, m = b >> 3, b & 7
    if e == 0:
        return F32(m / 8.0 * 2.0 ** -6)
    return F32((1 + m / 8.0) * 2.0 ** (e - 7))


def out16(x, kind):
    """16-bit pattern of binary32 values x rounded to fp16 or bf16 (RN-even)."""
    x = np.asarray(x, dtype=F32)
    if kind == "f16":
        with np.errstate(over="ignore"):                     # beyond 65504: +-inf
            return x.astype(np.float16).view(np.uint16).astype(np.uint32)
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (r & 0xFFFF).astype(np.uint32)


def prmt(a, b, c):
    """PTX prmt.b32 default mode: byte i of the result is byte (c_i & 7) of
    the 8-byte value {b, a}, or that byte's bit 7 replicated when c_i & 8."""
    a, b, c = (np.asarray(v, dtype=np.uint64) for v in (a, b, c))
    ab = a | (b << np.uint64(32))
    d = np.zeros(np.broadcast(a, b, c).shape, dtype=np.uint64)
    for i in range(4):
        sel = (c >> np.uint64(4 * i)) & np.uint64(0xF)
        byte = (ab >> (np.uint64(8) * (sel & np.uint64(7)))) & np.uint64(0xFF)
        rep = np.where((byte & np.uint64(0x80)) != 0, np.uint64(0xFF), np.uint64(0))
        byte = np.where((sel & np.uint64(8)) != 0, rep, byte)
        d |= byte << np.uint64(8 * i)
    return d.astype(np.uint32)


def reference_decode(w, sb, eff, kind):
    """Per-element table decode of the 8 nibbles of each word w: the signed
    value of the nibble (FP4 or INT4 by bit 7 of sb), times eff in binary32,
    rounded to 16 bits.  Returns [len(w), 8] patterns."""
    w = np.asarray(w, dtype=np.uint32)
    n = (w[:, None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
    if sb & 0x80:
        k = ((n ^ 8).astype(np.int64) - 8).astype(F32)
        q = (k * C67).astype(F32)
    else:
        q = np.where(n >= 8, -FP4_MAG[n & 7], FP4_MAG[n & 7]).astype(F32)
    return out16((q * eff).astype(F32), kind)


def permute_decode(w, sb, eff, kind):
    """The kernels' steps.  Returns ([len(w), 4] 16-bit pairs, flagged)."""
    w = np.asarray(w, dtype=np.uint32)
    base = INT4_MAG if sb & 0x80 else FP4_MAG
    t = out16((base * eff).astype(F32), kind)                 # t[0..7]
    p = [t[2 * j] | (t[2 * j + 1] << 16) for j in range(4)]   # 4 16-bit pairs
    lo0, hi0 = prmt(p[0], p[1], 0x6420), prmt(p[0], p[1], 0x7531)
    lo1, hi1 = prmt(p[2], p[3], 0x6420), prmt(p[2], p[3], 0x7531)
    im = np.uint32(0xFFFFFFFF) if sb & 0x80 else np.uint32(0)
    s = (w >> 3) & np.uint32(0x11111111)
    m = w & np.uint32(0x77777777)
    mag = ((m ^ ((s * np.uint32(7)) & im)) + (s & im)).astype(np.uint32)
    flagged = (mag & np.uint32(0x88888888)) != 0
    w4 = (w << np.uint32(4)).astype(np.uint32)
    out = []
    for h in range(2):
        sel = mag >> np.uint32(16 * h)
        lo4 = prmt(lo0, lo1, sel)
        sg = prmt(w4, w, 0x5140 if h == 0 else 0x7362) & np.uint32(0x80808080)
        hi4 = prmt(hi0, hi1, sel) | sg
        out.append(prmt(lo4, hi4, 0x5140))
        out.append(prmt(lo4, hi4, 0x7362))
    return np.stack(out, axis=1), flagged


def _split(pairs):
    return np.stack([pairs & 0xFFFF, pairs >> 16], axis=2).reshape(pairs.shape[0], 8)


def _words(seed):
    # every nibble value at every position (16 rotations), then random words
    rot = np.array([sum(((i + j) % 16) << (4 * i) for i in range(8)) for j in range(16)],
                   dtype=np.uint64).astype(np.uint32)
    rng = np.random.default_rng(seed)
    return np.concatenate([rot, rng.integers(0, 2 ** 32, 48, dtype=np.uint64).astype(np.uint32)])


@pytest.mark.parametrize("kind", ["f16", "bf16"])
@pytest.mark.parametrize("ts", [1.0, 0.3719, 3.0e-3, 211.5])
def test_permute_decode_equals_table_decode_every_scale_byte(kind, ts):
    words = _words(int(ts * 1000) + (kind == "bf16"))
    n_flagged = 0
    for sb in range(256):
        eff = F32(e4m3_value(sb) * F32(ts))
        ref = reference_decode(words, sb, eff, kind)
        got, flagged = permute_decode(words, sb, eff, kind)
        nib = (words[:, None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
        # flagged exactly when an INT4 group's word holds code 8
        assert np.array_equal(flagged, bool(sb & 0x80) & (nib == 8).any(axis=1)), sb
        ok = ~flagged
        n_flagged += int(flagged.sum())
        assert np.array_equal(_split(got)[ok], ref[ok]), (kind, ts, sb)
    assert n_flagged > 0


def test_permute_decode_pins_signs_and_zero_scale():
    # FP4 -0 (code 8) keeps its sign under every scale, zero scale included
    w = np.array([0x88888888, 0x0F0F0F0F, 0xF0F0F0F0], dtype=np.uint32)
    for sb in (0x00, 0x38, 0x7E):
        got, _ = permute_decode(w, sb, e4m3_value(sb), "f16")
        ref = reference_decode(w, sb, e4m3_value(sb), "f16")
        assert np.array_equal(_split(got), ref)
        assert (_split(got)[0] == 0x8000).all()


def test_prmt_model_selector_semantics():
    # byte i of {b, a} by selector nibble; bit 3 replicates the byte's sign
    a, b = 0x83828180, 0x07060504
    assert int(prmt(a, b, 0x3210)) == a and int(prmt(a, b, 0x7654)) == b
    assert int(prmt(a, b, 0x0000)) == 0x80808080
    assert int(prmt(a, b, 0x8888)) == 0xFFFFFFFF
    assert int(prmt(a, b, 0xCCCC)) == 0x00000000
