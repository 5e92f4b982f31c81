"""Four fp32 rows whose NVFP4 results depend on how the scale and element
quotients are formed (shared by the oracle pins and the GPU parity test).

Each row is 1x32.  Block 0 holds the tensor amax 2688 g, so the tensor scale
is exactly g; block 1 holds the probe values.

A: g = 0.100250244140625; block 1 = [6g, 2.5g, -2.5g, 0, ...].  Its scale is
   E4M3 1.0, so d = g, and x = 2.5g is the midpoint between the E2M1 values 2
   and 3 when divided exactly, while fl32(1/g) exceeds 1/g by enough that
   fl32(x * fl32(1/g)) = 2.5000002: the reciprocal-then-multiply element step
   gives 3.0, an exact division would give the even neighbour 2.0.
B: g = 0.07904052734375; block 1 = [1.0625 * 6g, 0.5g, 0, ...].  bamax/(6g)
   is exactly 1.0625, the midpoint between the E4M3 values 1.0 and 1.125, so
   the correctly rounded quotient ties to the even code 1.0 (0x38), while
   bamax * fl32(1/(6g)) rounds to 1.0625001 and would give 1.125 (0x39).
C: g = 5592469 * 2^-28 (amax 2688 g rounded to fp32 gives back g), so that
   6g lies exactly half an ulp below fl32(6g) = (2^23 + 96) * 2^-26 and rounds
   up to it; block 1 = [1.0625 * fl32(6g), g/4, 0, ...].  The quotient by the
   rounded fl32(6g) is exactly the E4M3 midpoint 1.0625 (code 1.0, 0x38); by
   the unrounded 6g it would be 1.0625001 (code 1.125, 0x39).
D: amax = 294.8681640625, g = fl32(amax / 2688); block 1 = [fl32(1.125 *
   fl32(6g)), x, -x, 0, ...] with x = 0.30852556228637695.  Its scale is E4M3
   1.125 and d = fl32(1.125 g) is rounded; x * fl32(1/d) is exactly 2.5 (a tie,
   code 2.0), while the reciprocal of the unrounded 1.125 g would give
   2.5000002 (code 3.0).
"""
import numpy as np


def vectors():
    f = np.float32
    a, b = np.zeros((1, 32), f), np.zeros((1, 32), f)
    ga, gb = f(0.100250244140625), f(0.07904052734375)
    a[0, 0], a[0, 16], a[0, 17], a[0, 18] = f(2688) * ga, f(6) * ga, f(2.5) * ga, -f(2.5) * ga
    b[0, 0], b[0, 16], b[0, 17] = f(2688) * gb, f(1.0625) * f(6 * gb), f(0.5) * gb
    c, d = np.zeros((1, 32), f), np.zeros((1, 32), f)
    gc = f(np.ldexp(5592469, -28))
    c[0, 0], c[0, 16], c[0, 17] = f(2688) * gc, f(1.0625) * f(f(6) * gc), f(0.25) * gc
    d[0, 0] = f(294.8681640625)
    gd = f(d[0, 0] / f(2688))
    xd = f(0.30852556228637695)
    d[0, 16], d[0, 17], d[0, 18] = f(1.125) * f(f(6) * gd), xd, -xd
    return (a, ga), (b, gb), (c, gc), (d, gd)
