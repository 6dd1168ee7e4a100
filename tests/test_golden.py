"""The stored tiny-workload fixture (written by tests/golden/make_golden.py from the oracle)
still matches the oracle bit for bit, and its split layout is the 'ceil first' rule."""
import json
import os

from tests.golden.make_golden import build

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_gqa_fixture_matches_oracle():
    with open(os.path.join(HERE, "tiny_gqa.json")) as f:
        stored = json.load(f)
    assert build() == stored
    # 2 splits per request, first split ceil(n/2) pages: (2,1), (4,4), (7,6), (8,8) pages
    sizes = [[b[1] - b[0], b[2] - b[1]] for b in stored["split_page_start"]]
    assert sizes == [[2, 1], [4, 4], [7, 6], [8, 8]]
