"""Write the stochastic-rounding fixtures whose values depend on the hash.

Calls only the oracle; its SplitMix64 hash is pinned to published vectors.
Run from the repository root:  python tests/golden/make_sr_fixtures.py

sr_boundary_step.txt: a step at which element (i=1, j=0) of tile (b=0, h=0)
    draws u == 0.5 exactly (the fraction of a tie).
sr_clamp_steps.txt: steps at which element (0,0) draws u < 5*2^-20 (rounds up
    past +qmax) and element (0,1) draws u >= 1 - 5*2^-20 (stays below -qmax).
"""
import os
import sys

sys.path.insert(0, os.getcwd())
import oracle  # noqa: E402

SEED = 0x5EED
HERE = os.path.dirname(os.path.abspath(__file__))
L = oracle.lib()


def first_step(i, j, pred):
    step = 0
    while not pred(L.orc_hash(SEED, step, 0, 0, i, j) >> 41):
        step += 1
    return step


tie = first_step(1, 0, lambda u23: u23 == (1 << 22))
up = first_step(0, 0, lambda u23: u23 < 40)
down = first_step(0, 1, lambda u23: u23 >= (1 << 23) - 40)
with open(os.path.join(HERE, "sr_boundary_step.txt"), "w") as f:
    f.write("# Written by tests/golden/make_sr_fixtures.py from the oracle's hash:\n"
            "# element (i=1, j=0) of tile (b=0, h=0) draws u == 0.5 exactly, the\n"
            "# fraction at a tie; stochastic rounding must then round down.\n")
    f.write("seed %d\nstep %d\n" % (SEED, tie))
with open(os.path.join(HERE, "sr_clamp_steps.txt"), "w") as f:
    f.write("# Written by tests/golden/make_sr_fixtures.py from the oracle's hash:\n"
            "# step_up: element (0,0) of tile (0,0) draws u < 5*2^-20;\n"
            "# step_down: element (0,1) of tile (0,0) draws u >= 1 - 5*2^-20.\n")
    f.write("seed %d\nstep_up %d\nstep_down %d\n" % (SEED, up, down))
print(tie, up, down)
