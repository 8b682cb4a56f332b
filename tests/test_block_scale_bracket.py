"""The quantizer kernels form the block scale without a division in almost
every block: with il = RN(RN(1/(6g)) * (1 - 2^-20)) and ih = RN(RN(1/(6g)) *
(1 + 2^-20)), the bytes e4m3(RN(b * il)) and e4m3(RN(b * ih)) bracket
e4m3(RN(b / (6g))); where they agree that byte is taken, else the quotient is
divided out.  This CPU test restates that rule in float32 numpy (each
operation is one correctly rounded IEEE op) and checks it against the
oracle's definition -- e4m3 of the correctly rounded quotient -- for every
BF16 block amax up to the tensor amax, over many global scales, including
exact ties on E4M3 midpoints."""
import numpy as np

import oracle as O

F32 = np.float32


def _bf16(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def _check_amax(amax_bits):
    amax = _bf16([amax_bits])[0]
    g = F32(amax / F32(2688.0))
    k6 = F32(F32(6.0) * g)
    b = _bf16(np.arange(0, amax_bits + 1, dtype=np.uint32))          # every block amax <= amax
    exact = O.e4m3_encode_array((b / k6).astype(np.float32))
    if not k6 >= np.finfo(np.float32).tiny:
        return exact.size, 0                                          # kernels always divide here
    inv = F32(F32(1.0) / k6)
    il = F32(inv * F32(1.0 - 2.0 ** -20))
    ih = F32(inv * F32(1.0 + 2.0 ** -20))
    lo = O.e4m3_encode_array((b * il).astype(np.float32))
    hi = O.e4m3_encode_array((b * ih).astype(np.float32))
    agree = lo == hi
    bad = np.nonzero(agree & (lo != exact))[0]
    assert bad.size == 0, f"amax {amax:a}: bracket agrees but differs from the quotient at b={b[bad[0]]:a}"
    return exact.size, int((~agree).sum())


def test_bracket_rule_matches_correctly_rounded_quotient():
    rng = np.random.default_rng(2024)
    amaxes = list(rng.integers(0x0080, 0x7F80, size=120)) + [0x3F80, 0x40C0, 0x4340, 0x43E0, 0x0080, 0x0100,
                                                             0x7F7F, 0x3C00, 0x3B4D, 0x40AF]
    total = slow = 0
    for ab in amaxes:
        n, s = _check_amax(int(ab))
        total += n
        slow += s
    assert total > 1_000_000
    assert slow < total * 0.01          # the division is the exception


def test_bracket_rule_subnormal_global_scale_always_divides():
    # amax at the bottom of the BF16 range: 6 g is subnormal in FP32
    n, _ = _check_amax(0x0001)
    assert n == 2


# ---- the quotient table of the one-tensor kernel ---------------------------------------
#
# For a BF16 block amax b = m_b 2^(e_b - 127) (m_b = 1 + i/128) and a normal
# 6g = m_k 2^(e_k - 127), the kernel takes the bits of RN(b / 6g) as
# qtab[i] + (e_b << 23), qtab[i] = bits(RN((1 + i/128) / m_k)) - (e_k << 23),
# clamped at 0 as a signed integer.  Restated here in float32 numpy and checked
# against e4m3 of the correctly rounded quotient for every BF16 block amax up
# to the tensor amax (zero, BF16 subnormals and quotients below 2^-126
# included), at tensor amaxes whose g is at least 2^-64.

def _table_rule(b_bits, k6):
    kb = np.array([k6], np.float32).view(np.uint32)[0]
    mk = np.array([(kb & 0x807FFFFF) | (127 << 23)], np.uint32).view(np.float32)[0]
    num = ((np.uint32(127) << 23) | (np.arange(128, dtype=np.uint32) << 16)).view(np.float32)
    q = (num / mk).astype(np.float32)                                  # correctly rounded
    qtab = q.view(np.uint32).astype(np.int64) - int(kb & 0x7F800000)
    f = (np.asarray(b_bits, np.uint32) << 16)                           # FP32 bits of the BF16 amax
    bits = qtab[(f >> 16) & 0x7F] + (f & 0x7F800000).astype(np.int64)
    bits = np.maximum(bits, 0).astype(np.uint32)
    return O.e4m3_encode_array(bits.view(np.float32))


def test_quotient_table_matches_correctly_rounded_quotient():
    rng = np.random.default_rng(2025)
    amaxes = list(rng.integers(0x2600, 0x7F80, size=120)) + [0x2600, 0x3F80, 0x40C0, 0x4340, 0x43E0, 0x7F7F,
                                                             0x3C00, 0x3B4D, 0x40AF, 0x2580]
    total = 0
    for ab in amaxes:
        amax = _bf16([ab])[0]
        g = F32(amax / F32(2688.0))
        assert g >= 2.0 ** -64
        k6 = F32(F32(6.0) * g)
        bits = np.arange(0, int(ab) + 1, dtype=np.uint32)              # every block amax <= amax
        exact = O.e4m3_encode_array((_bf16(bits) / k6).astype(np.float32))
        got = _table_rule(bits, k6)
        bad = np.nonzero(got != exact)[0]
        assert bad.size == 0, f"amax {amax:a}: table rule differs at b={_bf16(bits[bad[:1]])[0]:a}"
        total += bits.size
    assert total > 1_000_000
