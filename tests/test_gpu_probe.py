"""The clock probe: monotonic samples, a plausible SM clock."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_clock_probe_samples(lib):
    n = 200
    s = torch.zeros(n, 2, dtype=torch.int64, device="cuda")
    lib.velox_clock_probe(s, n, 1000)
    torch.cuda.synchronize()
    a = s.cpu().numpy().astype(np.float64)
    assert np.all(np.diff(a[:, 0]) > 0) and np.all(np.diff(a[:, 1]) > 0)
    ghz = np.diff(a[:, 0]) / np.diff(a[:, 1])
    # an idle GPU: its clock, whatever the other users of the box left it at
    assert 0.3 < float(np.median(ghz)) < 2.5
    # the pause: about 1 us between samples, no more than a few
    assert 0.5e3 < float(np.median(np.diff(a[:, 1]))) < 20e3
