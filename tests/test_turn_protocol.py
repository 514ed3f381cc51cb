"""Model check of the exponential-pass turns of the D = 64 forward kernel.

The two softmax warps that share an SM sub-partition alternate their
exponential passes: stream 1's pass r waits for stream 0's pass r (while
stream 0 has a pass r), stream 0's pass r waits for stream 1's pass r - 1
(while stream 1 has one).  Each warp signals one mbarrier per stream, one
phase per pass, and waits by phase parity.  A parity wait is only correct if
the awaited barrier has not already completed the phase after the awaited one;
this test runs the rule over random tile counts and random interleavings and
checks that this never happens and that no interleaving deadlocks.
"""

import random


def run(t0, t1, rng):
    total = (t0, t1)
    done = [0, 0]  # passes completed (= phases completed on the stream's barrier)
    while done[0] < t0 or done[1] < t1:
        ready = []
        for s in (0, 1):
            r = done[s]
            if r >= total[s]:
                continue
            o = 1 - s
            want = r if s == 1 else r - 1
            if 0 <= want < total[o]:
                # parity wait on phase `want`: wrong if phase want + 1 is complete too
                assert done[o] <= want + 1, (t0, t1, s, r, done)
                if done[o] < want + 1:
                    continue
            ready.append(s)
        assert ready, ("deadlock", t0, t1, done)
        done[rng.choice(ready)] += 1


def test_turns_never_alias_or_deadlock():
    rng = random.Random(1)
    for _ in range(5000):
        run(rng.randint(0, 40), rng.randint(0, 40), rng)
