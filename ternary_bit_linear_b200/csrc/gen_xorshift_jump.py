"""Writes tq_xorshift_jump.h, the jump-ahead tables of the stochastic-flip
kernel (tq_train.cuh).

xorshift64 (G. Marsaglia, "Xorshift RNGs", J. Stat. Softw. 8(14), 2003; shift
triple 13, 7, 17) is linear over GF(2): one step is x -> A x for a 64 x 64
bit matrix A, so the state n steps ahead is A^n x.  A matrix is stored as its
64 columns, column b being the image of bit b.  The kernel gives each lane a
run of kRun consecutive weights; these powers let it start every run at the
right point of the one sequential stream:

    chunk[j] = A^(kChunk * 2^j)   j < 26   (start of a CTA's first chunk)
    warp[w]  = A^(kWarpRun * w)   w < 8    (warp w inside a chunk)
    lane[b][l] = column b of A^(kRun * l)  (lane l inside a warp; stored
                                            column-major for shared memory)

    python gen_xorshift_jump.py > tq_xorshift_jump.h
"""
import sys

RUN = 64                 # weights per lane
WARP_RUN = 32 * RUN      # weights per warp
WARPS = 8
CHUNK = WARPS * WARP_RUN  # weights per CTA pass (16384)
CHUNK_BITS = 26          # chunks < 2^26: up to 2^40 weights
MASK = (1 << 64) - 1


def step(x):
    x ^= (x << 13) & MASK
    x ^= x >> 7
    x ^= (x << 17) & MASK
    return x


def apply(cols, v):
    r = 0
    b = 0
    while v:
        if v & 1:
            r ^= cols[b]
        v >>= 1
        b += 1
    return r


def mul(a, b):  # a o b
    return [apply(a, c) for c in b]


def power(cols, e):
    result = [1 << b for b in range(64)]
    base = cols
    while e:
        if e & 1:
            result = mul(result, base)
        base = mul(base, base)
        e >>= 1
    return result


def tables():
    A = [step(1 << b) for b in range(64)]
    chunk = [power(A, CHUNK << j) for j in range(CHUNK_BITS)]
    warp = [power(A, WARP_RUN * w) for w in range(WARPS)]
    lane_m = [power(A, RUN * l) for l in range(32)]
    lane = [[lane_m[l][b] for l in range(32)] for b in range(64)]
    return chunk, warp, lane


def fmt(rows):
    out = []
    for row in rows:
        vals = ["0x%016xull" % v for v in row]
        lines = ["        " + ", ".join(vals[i:i + 4]) for i in range(0, len(vals), 4)]
        out.append("    {\n" + ",\n".join(lines) + "}")
    return "{\n" + ",\n".join(out) + "}"


def header():
    chunk, warp, lane = tables()
    return f"""// tq_xorshift_jump.h -- written by gen_xorshift_jump.py; do not edit.
//
// Powers of the GF(2) transition matrix A of xorshift64 (shift triple 13, 7,
// 17), each as 64 columns (column b = image of bit b):
//   TQ_XS_CHUNK[j]   = A^({CHUNK} * 2^j), j < {CHUNK_BITS}
//   TQ_XS_WARP[w]    = A^({WARP_RUN} * w), w < {WARPS}
//   TQ_XS_LANE[b][l] = column b of A^({RUN} * l), l < 32
#pragma once

#define TQ_XS_RUN {RUN}
#define TQ_XS_WARPS {WARPS}
#define TQ_XS_CHUNK_BITS {CHUNK_BITS}

#define TQ_XS_CHUNK_INIT {fmt(chunk)}

#define TQ_XS_WARP_INIT {fmt(warp)}

#define TQ_XS_LANE_INIT {fmt(lane)}
""".replace("\n    ", "\\\n    ").replace("{\\\n", "{\\\n")


if __name__ == "__main__":
    sys.stdout.write(header())
