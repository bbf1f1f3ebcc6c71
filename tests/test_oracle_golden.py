"""CPU: the oracle's outputs on a tiny seeded case match the digests stored in
tests/golden/oracle_digests.json (written by tests/golden/make_oracle_digests.py,
which calls only oracle/). This guards against unnoticed changes to the oracle's
arithmetic; the pins of its correctness are in tests/test_oracle_*.py."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_oracle_digests  # noqa: E402


def test_oracle_outputs_match_the_stored_digests():
    with open(os.path.join(HERE, "golden", "oracle_digests.json")) as f:
        stored = json.load(f)
    now = make_oracle_digests.compute()
    assert now["case"] == stored["case"]
    changed = sorted(k for k in stored["digests"] if stored["digests"][k] != now["digests"].get(k))
    assert not changed, f"oracle outputs changed: {changed}"
