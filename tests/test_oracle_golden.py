"""The oracle still produces the digests stored in tests/golden/oracle_small.txt.

Those digests were written by tests/golden/make_golden.py, which calls only the
oracle; a change of the oracle's arithmetic must regenerate them in the same
commit, naming the passage that justifies it.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))


def test_oracle_matches_stored_digests(orc):
    import make_golden
    stored = [l.strip() for l in open(os.path.join(HERE, "golden", "oracle_small.txt"))
              if l.strip() and not l.startswith("#")]
    assert make_golden.digest_lines() == stored
