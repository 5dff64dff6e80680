"""Host logic of the phase-timeline tool (ternary_weight_linear_fwd_b200.timeline): grouping CTA records
into launches and the phase medians, on hand-made records (CPU only; the stamps themselves come from the
test build's kernels on a GPU)."""
import numpy as np

from ternary_weight_linear_fwd_b200 import timeline as tl


def _rec(kind, key, cta, grid, stamps):
    r = np.zeros(10, dtype=np.int64)
    r[0], r[1] = kind, (key << 32) | (cta << 16) | grid
    r[2:2 + len(stamps)] = stamps
    return r


def test_gemv_launches_and_phases():
    """Two launch shapes alternating (K = 2560 then 6912), 3 CTAs each, records shuffled: every phase and
    the release gap come out as built."""
    recs = []
    t = 1000
    for launch in range(6):
        K = 2560 if launch % 2 == 0 else 6912
        for c in range(3):
            e = t + 10 * c
            # entry, wait returned (+200), quantised (+300), landed (+5), contracted (+400), stored (+50)
            recs.append(_rec(1, K, c, 3, [e, e + 200, e + 500, e + 505, e + 905, e + 955]))
        t += 2000
    rng = np.random.default_rng(0)
    rec = np.array(recs)[rng.permutation(len(recs))]
    launches = tl._launches(rec, end_col=7)
    assert len(launches) == 6 and all(len(L) == 3 for L in launches)
    assert [int(L[0, 1] >> 32) for L in launches] == [2560, 6912] * 3
    out = tl._gemv_summary(rec)
    for k in ("K=2560", "K=6912"):
        s = out[k]
        assert s["dependency_wait_returned"] == 200 and s["x_quantised"] == 300 and s["weights_landed"] == 5
        assert s["contracted"] == 400 and s["stored"] == 50
        # previous launch's last store (t - 2000 + 20 + 955) to this launch's first wait return (t + 200)
        assert s["previous_store_to_wait_return"] == 2000 + 200 - 975
        assert s["period"] == 2000


def test_pair_phases_skip_unreached_stamps():
    """Pair records: stamps relative to each CTA's entry, zeros (phases a CTA never reached, such as the
    MMA issue on rank 1) left out, first and last launch dropped, the spread of the entries."""
    recs = []
    t = 0
    for launch in range(5):
        for c in range(4):
            e = t + 100 * c
            mma = e + 700 if c % 2 == 0 else 0  # rank 1 issues no MMA
            recs.append(_rec(2, 256, c, 4, [e, e + 80, e + 150, e + 220, mma, e + 745, e + 900, e + 910]))
        t += 5000
    out = tl._pair_summary(np.array(recs))
    assert out["set_up"] == 80 and out["producer_past_wait"] == 150 and out["first_stage_landed"] == 220
    assert out["first_tile_mmas_issued"] == 700
    assert out["first_accumulator_ready"] == 745 and out["last_epilogue_done"] == 900 and out["end"] == 910
    assert out["entry_spread"] == 300
