"""Host logic of the per-CTA timeline tool (no GPU): the summary and the
residency table computed from a timeline array."""
import numpy as np

from key_switching_b200 import timeline


def _tl(roles, recs):
    """recs: role -> list of (start ns, end ns, sm)"""
    a = np.zeros((roles, 16, 3), dtype=np.uint64)
    for r, lst in recs.items():
        for i, (s, e, sm) in enumerate(lst):
            a[r, i] = (s, e, sm)
    return a


def test_summary_is_relative_to_the_first_cta():
    names = ("a", "b", "c")
    tl = _tl(3, {0: [(10_000, 14_000, 0), (11_000, 19_000, 1)], 2: [(15_000, 23_000, 1)]})
    summ, rows = timeline.summarize(tl, names, bin_us=4.0)
    assert list(summ) == ["a", "c"]  # role b ran no CTA
    a, c = summ["a"], summ["c"]
    assert (a["ctas"], a["sms"]) == (2, 2) and (c["ctas"], c["sms"]) == (1, 1)
    assert a["first_start_us"] == 0.0 and a["last_start_us"] == 1.0
    assert a["first_end_us"] == 4.0 and a["last_end_us"] == 9.0
    assert a["cta_us_min"] == 4.0 and a["cta_us_max"] == 8.0 and a["cta_us_median"] == 6.0
    assert c["first_start_us"] == 5.0 and c["last_end_us"] == 13.0
    # resident CTAs at t = 0, 4, 8, 12, 16 us (a CTA counts on [start, end))
    assert [t for t, _ in rows] == [0.0, 4.0, 8.0, 12.0, 16.0]
    assert [r["a"] for _, r in rows] == [1, 1, 1, 0, 0]
    assert [r["c"] for _, r in rows] == [0, 0, 1, 1, 0]


def test_empty_timeline():
    assert timeline.summarize(np.zeros((8, 4, 3), dtype=np.uint64), tuple("abcdefgh")) == ({}, [])
