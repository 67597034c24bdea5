"""Exhaustive CPU checks of two exactness arguments behind the kernels'
operand encodings (plain arithmetic, no kernel involved; the kernels'
results are compared with the oracle in the GPU tests).

1. Activations as two e4m3 pieces (the opt-in tcgen05 decode kernel): with a
   token scaled by a power of two so that its max |x| lies in [128, 256),
   p0 = rn_e4m3(x) and p1 = rn_e4m3(x - p0) sum back to every bf16 value x
   exactly when |x| >= 2^-9 * max (8 significant bits = 4 + 4), and to within
   2^-10 absolute (half the smallest e4m3 subnormal step) below that.
2. The residual decode (both decode kernels and the tcgen05 prefill kernel):
   OR-ing a 2-bit field at bit 2i into the fp16 pattern of 1024 gives
   1024 + 4^i q exactly, and one fused multiply-add by 4^-i with
   -(1024 * 4^-i + z) gives q - z exactly; the 3-bit high bit placed two bits
   above the field keeps it exact (q <= 7).
"""
import numpy as np
import torch


def _every_bf16_below(limit):
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    y = (bits << 16).view(np.float32)
    return y[np.isfinite(y) & (np.abs(y) < limit)]


def test_two_e4m3_pieces_hold_bf16():
    y = _every_bf16_below(256.0)
    t = torch.from_numpy(y)
    p0 = t.to(torch.float8_e4m3fn).to(torch.float32)
    p1 = (t - p0).to(torch.float8_e4m3fn).to(torch.float32)   # t - p0 is exact in fp32
    s = p0.double() + p1.double()
    err = (s - t.double()).abs().numpy()
    for row_max in (128.0, 192.0, 255.0):
        near = np.abs(y) >= row_max * 2.0 ** -9
        assert (err[near] == 0).all(), row_max
    assert err.max() <= 2.0 ** -10
    # and the bound is reached: the pieces are not exact for every value
    assert err.max() == 2.0 ** -10


def test_magic_number_decode_is_exact():
    for bits in (2, 3):
        qmax = 3 if bits == 2 else 7
        for i in range(4):
            for q in range(qmax + 1):
                lo, hi = q & 3, q >> 2
                # fp16 pattern of 1024 is 0x6400; field bits 2i (+ high bit 2i+2), mantissa unit 1
                pattern = 0x6400 | (lo << (2 * i)) | (hi << (2 * i + 2))
                v = np.array([pattern], np.uint16).view(np.float16)[0]
                assert float(v) == 1024 + 4 ** i * q
                for z in range(qmax + 1):
                    nz = np.float16(-(1024 * 4.0 ** -i + z))
                    assert float(nz) == -(1024 * 4.0 ** -i + z)            # representable
                    m = np.float16(4.0 ** -i)
                    fma = np.float16(float(v) * float(m) + float(nz))    # one rounding
                    assert float(fma) == q - z
