"""The parity tests' tie checks, exercised on the CPU.

``TileStats`` accepts a code or metadata value that differs from the float32
oracle only where the fp64 oracle puts the value at a rounding boundary.
Here the "GPU" result is the float32 oracle's own output with one planted
change: a flip at a genuine tie must pass, the same flip anywhere else must
fail, and a difference without the source rows must fail too.
"""

import math

import numpy as np

from oracle import kvq_oracle as o
from parity_helpers import TIE_EPS, TileStats

BITS, ITERS = 4, 4


def _tile(seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, 128))
    x[:, rng.choice(128, 3, replace=False)] *= 12.0
    return x.astype(np.float16)


def _add(st, x, codes, s_t, z_t, c_t, ref, with_src=True):
    rot, _ = o.dequantize_tile(codes, s_t, z_t, c_t)
    st.add(codes, np.stack([s_t, z_t], axis=1), c_t, rot.astype(np.float32), ref,
           src=(x, BITS, ITERS, 0) if with_src else None)


def _find_code_tie():
    for seed in range(200):
        x = _tile(seed)
        p = o.quantize_tile(x, BITS, ITERS, return_parts=True)
        v = (p["y"] - p["z"][:, None]) / p["s"][:, None]
        dist = np.abs(v - np.floor(v) - 0.5)
        delta = TIE_EPS * (np.abs(p["y"]) + np.abs(p["z"][:, None])) / p["s"][:, None]
        i, j = np.unravel_index(np.argmin(dist / delta), v.shape)
        if dist[i, j] <= delta[i, j] and 0 < math.floor(v[i, j]) < (1 << BITS) - 2:
            far = np.unravel_index(np.argmax(dist), v.shape)
            return x, (i, j), far, v
    raise AssertionError("no tie found in 200 seeded tiles")


def test_code_flip_at_a_tie_passes_and_elsewhere_fails():
    x, (i, j), far, v = _find_code_tie()
    ref = o.quantize_tile(x, BITS, ITERS, dtype=np.float32)
    lo = math.floor(v[i, j])
    other = lo if ref["codes"][i, j] == lo + 1 else lo + 1
    codes = ref["codes"].copy()
    codes[i, j] = other
    st = TileStats()
    _add(st, x, ref["codes"], ref["s_t"], ref["z_t"], ref["c_t"], ref)  # an identical tile: 99.99% needs > 1e4 codes
    _add(st, x, codes, ref["s_t"], ref["z_t"], ref["c_t"], ref)
    st.check()
    assert st.code_diffs == 1 and not st.untied
    # the same kind of flip away from a tie (a code off by one, still within
    # every other bar) is rejected
    codes = ref["codes"].copy()
    fi, fj = far
    codes[fi, fj] = codes[fi, fj] + 1 if codes[fi, fj] < (1 << BITS) - 1 else codes[fi, fj] - 1
    bad = TileStats()
    _add(bad, x, ref["codes"], ref["s_t"], ref["z_t"], ref["c_t"], ref)
    _add(bad, x, codes, ref["s_t"], ref["z_t"], ref["c_t"], ref)
    assert bad.untied and bad.max_code_diff == 1
    try:
        bad.check()
    except AssertionError as e:
        assert "not rounding ties" in str(e)
    else:
        raise AssertionError("a flip away from a tie passed")


def _one_ulp(h, up=True):
    b = int(np.array([h], dtype=np.float16).view(np.uint16)[0])
    b += 1 if (up == (float(h) >= 0)) else -1
    return np.array([b], dtype=np.uint16).view(np.float16)[0]


def test_metadata_ulp_at_a_tie_passes_and_elsewhere_fails():
    for seed in range(400):
        x = _tile(seed)
        ref = o.quantize_tile(x, BITS, ITERS, dtype=np.float32)
        p = o.quantize_tile(x, BITS, ITERS, return_parts=True)
        exact = p["s"] * p["r"]
        ymax = p["y"].max(axis=1)
        amp = (np.abs(ymax) + np.abs(p["z"])) / (ymax - p["z"])
        # the fp16 neighbour on the other side of the rounding boundary
        nb = np.array([_one_ulp(ref["s_t"][k], exact[k] > float(ref["s_t"][k])) for k in range(64)])
        mid = 0.5 * (ref["s_t"].astype(np.float64) + nb.astype(np.float64))
        rel = np.abs(exact - mid) / (TIE_EPS * amp * np.abs(exact))
        k = int(np.argmin(rel))
        if rel[k] <= 1.0:
            break
    else:
        raise AssertionError("no metadata tie found")
    s_t = ref["s_t"].copy()
    s_t[k] = nb[k]
    st = TileStats()
    _add(st, x, ref["codes"], s_t, ref["z_t"], ref["c_t"], ref)
    st.check()
    assert st.meta_diffs == 1
    far = int(np.argmax(rel))
    s_t = ref["s_t"].copy()
    s_t[far] = nb[far]
    bad = TileStats()
    _add(bad, x, ref["codes"], s_t, ref["z_t"], ref["c_t"], ref)
    assert bad.max_meta_ulp == 1 and bad.untied


def test_difference_without_source_rows_fails():
    x = _tile(3)
    ref = o.quantize_tile(x, BITS, ITERS, dtype=np.float32)
    c_t = ref["c_t"].copy()
    c_t[5] = _one_ulp(c_t[5])
    st = TileStats()
    _add(st, x, ref["codes"], ref["s_t"], ref["z_t"], c_t, ref, with_src=False)
    assert st.unchecked == 1
    try:
        st.check()
    except AssertionError as e:
        assert "without a tie check" in str(e)
    else:
        raise AssertionError("an unchecked difference passed")


def test_identical_tile_passes_without_source_rows():
    x = _tile(4)
    ref = o.quantize_tile(x, BITS, ITERS, dtype=np.float32)
    st = TileStats()
    _add(st, x, ref["codes"], ref["s_t"], ref["z_t"], ref["c_t"], ref, with_src=False)
    assert st.check() == 1.0 and st.exact_tiles == 1
