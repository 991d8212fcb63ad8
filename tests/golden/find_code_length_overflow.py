"""Write code_length_overflow.txt: byte blocks whose DEFLATE code-length tree
would be deeper than its 7-bit limit at gzip level 1, so that compressing them
runs the length-limiting repair (RFC 1951 section 3.2.7 caps code-length codes
at 7 bits).  Random skewed blocks almost never reach it; a seeded hill climb
on the oracle's unclamped tree depth finds such blocks in a few hundred steps.

Only the oracle is called.  The file holds inputs, not expected outputs: the
tests compare the oracle's stream for them with the host zlib at test time.

    python tests/golden/find_code_length_overflow.py
"""
import os
import random
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import deflate1  # noqa: E402


def climb(b: int, seed: int, need_dynamic: bool, max_steps: int = 20000):
    rnd = random.Random(seed)
    weights = [rnd.random() ** 6 for _ in range(256)]
    best_x = bytearray(rnd.choices(range(256), weights, k=b))
    best = deflate1.tree_depths(bytes(best_x))[2]
    for _ in range(max_steps):
        x = bytearray(best_x)
        for _ in range(rnd.randint(1, 8)):
            p = rnd.randrange(b)
            r = rnd.random()
            if r < 0.4:
                x[p] = rnd.randrange(256)
            elif r < 0.7:
                x[p] = x[rnd.randrange(b)]
            else:
                q = rnd.randrange(b)
                ln = rnd.randint(1, 16)
                x[p:p + ln] = x[q:q + ln]
                x = x[:b] + bytearray(max(0, b - len(x)))
        d = deflate1.tree_depths(bytes(x))[2]
        if d >= best:
            best, best_x = d, x
            if d > 7 and (not need_dynamic or deflate1.deflate1_raw(bytes(x))[1] == "dynamic"):
                return bytes(x)
    return None


def main():
    found = []
    # At 128 bytes the fixed block usually wins, so the repaired lengths only
    # enter the block-type decision; larger blocks also send them.
    plan = ((128, range(1, 7), False), (256, range(1, 7), True), (1024, range(1, 4), True))
    for b, seeds, need_dynamic in plan:
        for seed in seeds:
            x = climb(b, seed, need_dynamic)
            if x is not None:
                found.append((b, seed, x))
    path = os.path.join(HERE, "code_length_overflow.txt")
    with open(path, "w") as f:
        f.write("# Blocks whose code-length Huffman tree exceeds 7 bits before the\n")
        f.write("# length-limiting repair (RFC 1951 section 3.2.7), found by\n")
        f.write("# tests/golden/find_code_length_overflow.py with the oracle only.\n")
        f.write("# Format: <block size> <seed> <hex bytes>\n")
        for b, seed, x in found:
            f.write(f"{b} {seed} {x.hex()}\n")
    print(f"wrote {len(found)} blocks to {path}")


if __name__ == "__main__":
    main()
