"""Host model of the two-group inner product's hand-off (k_inner_ws): the
producer group regenerates digit j's 'a' words into ring buffer j mod RING
and arrives on FULL[s]; the consumer group syncs on FULL[s], reads the
buffer and, if digit j + RING exists, arrives on EMPTY[s], on which the
producer syncs before refilling.  A named-barrier phase completes when both
groups have arrived.  The model checks, under every interleaving order it
tries, that the steps never deadlock, that no group arrives twice on one
barrier within a phase, and that no buffer is refilled before it is read --
for the ring depth the kernel is compiled with and for other depths."""
import os
import random
import re

import pytest

from tests.conftest import ROOT


def kernel_ring():
    src = open(os.path.join(ROOT, "key_switching_b200", "csrc", "kernels.cu")).read()
    return int(re.search(r"#define PC_WS_RING (\d+)", src).group(1))


def steps(beta, ring):
    prod, cons = [], []
    for j in range(beta):
        s = j % ring
        if j >= ring:
            prod.append(("sync", ("EMPTY", s)))
        prod.append(("write", j))
        prod.append(("arrive", ("FULL", s)))
    for j in range(beta):
        s = j % ring
        cons.append(("sync", ("FULL", s)))
        cons.append(("read", j))
        if j + ring < beta:
            cons.append(("arrive", ("EMPTY", s)))
    return {"P": prod, "C": cons}


def run(beta, ring, pick):
    prog = steps(beta, ring)
    pc = {"P": 0, "C": 0}
    arrived, waiting, buf = {}, {}, {}
    while pc["P"] < len(prog["P"]) or pc["C"] < len(prog["C"]):
        for who in pick():
            if who in waiting or pc[who] >= len(prog[who]):
                continue
            op, arg = prog[who][pc[who]]
            if op in ("arrive", "sync"):
                a = arrived.setdefault(arg, set())
                assert who not in a, f"{who} arrives twice on {arg} in one phase"
                a.add(who)
                if len(a) == 2:  # phase complete: release the waiter
                    arrived[arg] = set()
                    for w in [w for w, b in waiting.items() if b == arg]:
                        del waiting[w]
                        pc[w] += 1
                    pc[who] += 1
                elif op == "sync":
                    waiting[who] = arg
                else:
                    pc[who] += 1
            elif op == "write":
                assert arg % ring not in buf, f"digit {arg} overwrites unread digit {buf.get(arg % ring)}"
                buf[arg % ring] = arg
                pc[who] += 1
            else:
                assert buf.pop(arg % ring, None) == arg, f"digit {arg} not in its buffer when read"
                pc[who] += 1
            break
        else:
            raise AssertionError(f"deadlock: beta={beta} ring={ring} at {pc}, waiting {waiting}")


@pytest.mark.parametrize("ring", sorted({2, 3, 4, 6, kernel_ring()}))
def test_hand_off_completes_for_every_digit_count(ring):
    for beta in range(1, 65):
        run(beta, ring, lambda: ["P", "C"])
        run(beta, ring, lambda: ["C", "P"])
        rnd = random.Random(beta)
        for _ in range(10):
            run(beta, ring, lambda: rnd.sample(["P", "C"], 2))


def test_model_catches_a_missing_wait():
    # a producer that refills without waiting on EMPTY must be caught
    global steps
    orig = steps

    def bad(beta, ring):
        p = orig(beta, ring)
        p["P"] = [s for s in p["P"] if s[0] != "sync"]
        return p
    steps = bad
    try:
        with pytest.raises(AssertionError):
            run(8, 2, lambda: ["P", "C"])
    finally:
        steps = orig


def test_barrier_ids_fit_the_hardware():
    ring = kernel_ring()
    assert 2 + 2 * ring - 1 <= 15  # FULL 2 .. ring+1, EMPTY ring+2 .. 2 ring+1
