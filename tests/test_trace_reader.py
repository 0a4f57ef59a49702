"""The cycle-trace reader (threshold_gated_block_b200/trace.py) on a hand-made
trace: phase lengths are the differences of the stamps it is given, kept and
skipped steps apart, and the steady-state median leaves out the first two and
the last step of each slot."""
import numpy as np

from threshold_gated_block_b200 import trace as T


def _synthetic(nblk=6, skew=0):
    """A trace whose waiter and MMA warps read clocks `skew` cycles ahead of warp 0."""
    tr = np.zeros(2048, dtype=np.int64)
    for w in range(12):
        tr[3 + w] = 500 + (skew if w in (T.MMA_WARP, T.WAIT_WARP) else 0)
    t = 1000
    for j in range(nblk):
        for s in range(2):
            kept = (j % 2 == 0)
            base = T.SOFTMAX + (s * T.STEPS + j) * 8
            tr[T.WAIT + s * T.STEPS + j] = t - 7 + skew
            tr[base + 0] = t
            tr[base + 1] = t + 10
            tr[base + 2] = t + 90
            tr[base + 3] = t + 100
            tr[base + 4] = t + 150
            if kept:
                tr[base + 5] = t + 950
                tr[base + 6] = t + 1000
                tr[base + 7] = t + 1040
            else:
                tr[base + 7] = t + 170
            end = tr[base + 7]
            m = T.MMA + (s * T.STEPS + j) * 4
            tr[m + 0] = end + 300 + skew
            if kept:
                tr[m + 1] = end + 350 + skew
                tr[m + 2] = end + 380 + skew
            tr[m + 3] = end + 400 + skew
        t += 3000
    return tr


def test_phases_are_stamp_differences():
    rows = T.phases(_synthetic(), [6, 6])
    assert len(rows) == 12
    kept = [r for r in rows if r["kept"]][0]["ph"]
    assert kept["fence"] == 10 and kept["load"] == 80 and kept["max"] == 10 and kept["gate"] == 50
    assert kept["exp"] == 800 and kept["P store"] == 50 and kept["announce"] == 40 and kept["to MMA"] == 300
    assert kept["V wait"] == 50 and kept["PV issue"] == 30 and kept["QK issue"] == 20
    skipped = [r for r in rows if not r["kept"]][0]["ph"]
    assert "exp" not in skipped and skipped["announce"] == 20 and skipped["QK issue"] == 100
    first = rows[0]["ph"]
    assert first["period"] == 3000 and first["to softmax"] == 7


def test_warp_clock_offsets_are_removed():
    a = T.phases(_synthetic(skew=0), [6, 6])
    b = T.phases(_synthetic(skew=1850), [6, 6])
    assert [r["ph"] for r in a] == [r["ph"] for r in b]


def test_summary_uses_the_steady_state_only():
    rows = T.phases(_synthetic(), [6, 6])
    summ = T.summarize(rows)
    # steps 2..4 of each slot: 2 and 4 kept, 3 skipped
    assert summ["kept"]["steps"] == 4 and summ["skipped"]["steps"] == 2
    assert summ["kept"]["exp"] == 800 and summ["skipped"]["announce"] == 20
