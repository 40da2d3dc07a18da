"""Accuracy against storage for the group sizes and axes of the 4-bit compression, from the
oracle alone ("FlexGen" README mirror, out-of-memory tips: weight compression saves about
70 % of weight memory; group size and axis are readings, g in {32, 64, 128}, along the output
channel or along the input dimension).

Storage is (0.5 + 4/g) bytes per element (codes plus an fp16 {min, scale} pair per group).
Checked: the error falls as groups shrink; with 1 % of columns scaled x50, groups along the input dimension
(each inside one column) keep the other columns' error low, where groups along the output
channel mix an outlier column into 1 of every few groups.  ``python -m pytest -s`` prints
the table."""
import numpy as np
import pytest

import fg_synth
import oracle


def _errors(w, g, axis):
    K, N = w.shape
    codes, params = oracle.quantize_pack(w, g, axis)
    wh = oracle.dequantize(codes, params, K, N, g, axis).astype(np.float64)
    wf = w.astype(np.float64)
    e = np.abs(wh - wf)
    nbytes = codes.nbytes + params.nbytes
    return float(np.sqrt(np.mean(e ** 2)) / np.sqrt(np.mean(wf ** 2))), float(e.max() / np.abs(wf).max()), nbytes / w.size


@pytest.mark.parametrize("dist,scale", [("normal", 0.02), ("outlier", 0.02)])
def test_accuracy_against_bytes(dist, scale):
    K, N = 1024, 1024
    w = fg_synth.tensor(77, 3, (K, N), dist, scale)
    rows = []
    for axis in (1, 0):
        prev = None
        for g in (128, 64, 32):
            rel_rms, rel_max, bpe = _errors(w, g, axis)
            assert bpe == pytest.approx(0.5 + 4.0 / g)
            rows.append((dist, "output channel" if axis == 1 else "input dim", g, bpe, rel_rms, rel_max))
            if prev is not None:
                assert rel_rms < prev          # smaller groups, smaller error
            prev = rel_rms
    for r in rows:
        print(f"{r[0]:8s} groups along {r[1]:14s} g {r[2]:3d}: {r[3]:.4f} B/elem "
              f"({100 * (1 - r[3] / 2):.1f} % below fp16), rel. RMS error {r[4]:.4f}, rel. max error {r[5]:.4f}")
    if dist == "outlier":
        # grouping inside a column keeps outlier columns from widening other columns' steps
        by = {(r[1], r[2]): r[4] for r in rows}
        for g in (32, 64, 128):
            assert by[("input dim", g)] < by[("output channel", g)]
