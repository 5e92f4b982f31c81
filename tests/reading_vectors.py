"""Two fp32 rows whose NVFP4 results depend on how the scale and element
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
"""
import numpy as np


def vectors():
    f = np.float32
    a, b = np.zeros((1, 32), f), np.zeros((1, 32), f)
    ga, gb = f(0.100250244140625), f(0.07904052734375)
    a[0, 0], a[0, 16], a[0, 17], a[0, 18] = f(2688) * ga, f(6) * ga, f(2.5) * ga, -f(2.5) * ga
    b[0, 0], b[0, 16], b[0, 17] = f(2688) * gb, f(1.0625) * f(6 * gb), f(0.5) * gb
    return (a, ga), (b, gb)
