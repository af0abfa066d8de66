"""GPU parity of thinkv_classify_thoughts: tags bit-exact with the oracle's
classifier on the hand-worked examples, on random masses (many near the
thresholds), and on the top-k masses a decode call produced."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W

import harness as Hn
from test_oracle_classify import _golden

pytestmark = pytest.mark.gpu


def _gpu_tags(mass_np, tt, tr):
    from mixed_precision_paged_thinkv_b200.binding import classify_thoughts
    m = torch.as_tensor(np.ascontiguousarray(mass_np, dtype=np.float32), device="cuda")
    return classify_thoughts(m, tt, tr).cpu().numpy()


def test_golden_examples_on_gpu():
    for tt, tr, m, tag in _golden():
        assert int(_gpu_tags(m[None, :], tt, tr)[0]) == tag


@pytest.mark.parametrize("hq", [1, 7, 32, 64, 300])
def test_random_masses_bit_exact(hq):
    rng = np.random.default_rng(hq)
    n = 5000
    m = rng.random((n, hq)).astype(np.float32)
    # a third of the rows sit exactly on the thresholds' neighbourhood
    tt, tr = np.float32(0.62), np.float32(0.41)
    m[: n // 3] = (tt + (rng.integers(-3, 4, (n // 3, 1)) * np.float32(2 ** -24))).astype(np.float32)
    g = _gpu_tags(m, float(tt), float(tr))
    o = O.classify(m, float(tt), float(tr))
    assert np.array_equal(g, o)


def test_tags_from_decode_masses():
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    w = W.scaled(W.WORKLOADS["gpt-oss-20b"], batch=6, lengths=("uniform", 400, 1800))
    g = WorkloadRun(w)
    g.setup()
    _, mass = g.decode(0, topk=32)
    torch.cuda.synchronize()
    m = mass.cpu().numpy()
    tt, tr = float(np.quantile(m.mean(1), 0.7)), float(np.quantile(m.mean(1), 0.3))
    assert np.array_equal(_gpu_tags(m, tt, tr), O.classify(m, tt, tr))
