"""CPU check of the bound behind the long-row Stage 1 kernel's row-maximum pass, which reads only
the hi bf16 plane of each chunk summary: with hi = bf16(k̄) rounded to nearest, every element
satisfies |k̄ - hi| <= 2^-8 |k̄|, so |<q, k̄> - <q, hi>| <= 2^-8 sum |q_j| |k̄_j| <= 2^-8 |q| |k̄|
(Cauchy-Schwarz).  The kernel widens its cut by (2^-8 + 2^-10) xs |q| max|k̄_c| to cover the fp32
accumulation of both logits as well.  Checked here in float64 on random and on worst-case
aligned inputs (every residual with the sign of its q_j)."""
import numpy as np
import pytest
import torch


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("seed", range(5))
def test_hi_plane_logit_error_is_within_the_bound(seed):
    rng = np.random.default_rng(seed)
    d = 128
    for scale in (1e-3, 1.0, 37.0):
        q = _bf16(rng.standard_normal((64, d)))                        # queries are exact in bf16
        kb = (rng.standard_normal((256, d)) * scale).astype(np.float32).astype(np.float64)
        hi = _bf16(kb)
        assert np.all(np.abs(kb - hi) <= 2.0 ** -8 * np.abs(kb))
        err = np.abs(q @ kb.T - q @ hi.T)
        bound = 2.0 ** -8 * np.linalg.norm(q, axis=1)[:, None] * np.linalg.norm(kb, axis=1)[None, :]
        assert np.all(err <= bound)
        # worst case: a query whose signs follow the residuals of one summary
        r = kb[0] - hi[0]
        qa = _bf16(np.sign(r) + (r == 0))
        e = abs(float(qa @ kb[0] - qa @ hi[0]))
        assert e <= 2.0 ** -8 * np.linalg.norm(qa) * np.linalg.norm(kb[0])
        assert e <= (2.0 ** -8 + 2.0 ** -10) * np.linalg.norm(qa) * np.linalg.norm(kb[0])
