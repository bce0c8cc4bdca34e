"""The oracle's pins catch planted mistakes (no GPU).

oracle/mutation_check.py builds copies of the oracle with one plausible mistake
each (dropped terms, wrong signs, bounds, indices, rounding) and runs the pin
suite against every copy; each mistake that changes an output must make a pin
fail.  About a minute of CPU time.
"""
from oracle import mutation_check


def test_every_observable_planted_mistake_fails_a_pin():
    assert mutation_check.run() == 0
