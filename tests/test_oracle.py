"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle_pins as pins
from oracle import oracle as orc


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_rejects_bad_arguments(oracle_lib):
    q = np.zeros((1, 2, 4), np.float32)
    c = np.zeros((1, 8, 4), np.float32)
    for g, w in ((0, 1), (2, -1)):
        with pytest.raises(RuntimeError):
            orc.lca(q, q[:, :, :2], c, c[:, :, :2], g=g, w=w, lib=oracle_lib)


def test_error_does_not_grow_with_length(oracle_lib):
    """Qualitative form of the page's bound (section 2, "Vantagens Teoricas"):
    the LCA-vs-dense error depends on within-group variation, not on L.  Here
    every group is a tight cluster (small fixed spread around a centre), and
    the error must not grow as L quadruples.  No constant is given on the
    page, so only the trend is checked, with generous slack."""
    rng = np.random.default_rng(21)
    d_c, d_r, g, H = 16, 8, 8, 2
    errs = []
    for L in (128, 512, 2048):
        nG = L // g
        centres_c = rng.standard_normal((nG, d_c))
        centres_k = rng.standard_normal((nG, d_r))
        C = (np.repeat(centres_c, g, 0) + 0.05 * rng.standard_normal((L, d_c))).astype(np.float32)
        K = (np.repeat(centres_k, g, 0) + 0.05 * rng.standard_normal((L, d_r))).astype(np.float32)
        qc = (rng.standard_normal((1, H, d_c)) * 0.3).astype(np.float32)
        qr = (rng.standard_normal((1, H, d_r)) * 0.3).astype(np.float32)
        lca = orc.lca(qc, qr, C[None], K[None], g=g, w=0, lib=oracle_lib).out
        dense = orc.mla(qc, qr, C[None], K[None], lib=oracle_lib)
        errs.append(float(np.abs(lca - dense).max()))
    assert errs[-1] < 4.0 * errs[0] + 1e-6, errs
