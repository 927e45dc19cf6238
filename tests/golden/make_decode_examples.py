"""Write decode_examples.txt from the two-counter closed form.

Closed form of one C-BSG bipolar XNOR count ("Precision As You Need", key
design 1, with the two enable-gated counters read as in the oracle): with
n = C[a, L] ones in A's stream and C[b, m] = #{l < m : r_l <= b},
    count = C[b, n] + (L - n) - C[b, L - n].
For the natural-order first Sobol dimension, r_l - 1 is the 8-bit reversal
of l.  Only the standard library is used; nothing here calls the oracle or
the CUDA library.
"""
import os

P = 8
Q = 1 << P


def rev(l):
    return int(format(l, f"0{P}b")[::-1], 2)


def C(b, m):
    return sum(1 for l in range(m) if rev(l) + 1 <= b)


def count(a, b, L):
    n = C(a, L)
    return C(b, n) + (L - n) - C(b, L - n)


CASES = [(192, 192, 256), (255, 255, 256), (1, 255, 256), (128, 200, 64),
         (200, 128, 64), (160, 96, 96), (96, 160, 192), (130, 130, 128),
         (0, 77, 64), (256, 77, 64), (64, 64, 1), (250, 7, 255)]

if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "decode_examples.txt"), "w") as f:
        f.write("# a b L count   (a, b levels in [0, 256]; x = level - 128)\n")
        f.write("# written by make_decode_examples.py from the closed form\n")
        for a, b, L in CASES:
            f.write(f"{a} {b} {L} {count(a, b, L)}\n")
