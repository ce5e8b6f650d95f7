"""The growing-score attention input used by the GPU rescale test is discriminating: an online softmax
with lazy rescaling (threshold 2^8, 128-key tiles) that forgets to rescale the output accumulator when the
reference maximum moves misses the exact softmax by far more than the parity tolerance, while the same
online softmax with the rescale matches it to rounding."""
import numpy as np
import pytest

from helpers import MAX_ABS_TOL, REL_L2_TOL, f64, growing_score_attn_inputs


def _online(q, k, v, scale, rows, rescale_o):
    out = []
    for t in rows:
        s = (k[:t + 1] @ q[t]) * scale * np.log2(np.e)
        m_ref, o, l = None, np.zeros(v.shape[1]), 0.0
        for j0 in range(0, t + 1, 128):
            sj = s[j0:j0 + 128]
            mx = sj.max()
            if m_ref is None:
                m_ref = mx
            elif mx > m_ref + 8.0:
                a = 2.0 ** (m_ref - mx)
                if rescale_o:
                    o *= a
                l *= a
                m_ref = mx
            p = 2.0 ** (sj - m_ref)
            o += p @ v[j0:j0 + len(sj)]
            l += p.sum()
        out.append(o / l)
    return np.array(out)


@pytest.mark.parametrize("d", [128, 256])
def test_growing_score_input_catches_a_missing_rescale(d):
    qb, kb, vb = growing_score_attn_inputs(d)
    q, k, v = f64(qb)[0, :, 0], f64(kb)[0, :, 0], f64(vb)[0, :, 0]
    scale = d ** -0.5
    rows = np.arange(0, q.shape[0], 29)
    exact = []
    for t in rows:
        s = (k[:t + 1] @ q[t]) * scale
        w = np.exp(s - s.max())
        exact.append(w @ v[:t + 1] / w.sum())
    exact = np.array(exact)
    good = _online(q, k, v, scale, rows, True)
    bad = _online(q, k, v, scale, rows, False)
    rel = lambda x: np.linalg.norm(x - exact) / np.linalg.norm(exact)
    assert rel(good) < 1e-12
    assert rel(bad) > 10 * REL_L2_TOL and np.abs(bad - exact).max() > MAX_ABS_TOL
