"""Host-side helpers of the package (CPU): the pooled audit ratios that
pipeline.audit_metrics forms from velox_route_audit's counts, against the
oracle's definition of the same ratios."""

import numpy as np
import torch

from oracle import audit as oa


def test_audit_metrics_match_the_oracle_pooling():
    from routed_block_sparse_b200.pipeline import audit_metrics
    r = np.random.default_rng(3)
    M, kg, kf = 143, 50, 80
    counts = np.stack([r.integers(0, 20, size=(3, 4)), r.integers(0, 20, size=(3, 4)),
                       r.integers(0, 50, size=(3, 4)), r.integers(0, 20, size=(3, 4)),
                       r.integers(0, 20, size=(3, 4)), r.integers(0, 30, size=(3, 4))], -1)
    got = audit_metrics(torch.from_numpy(counts.astype(np.int32)), M, kg, kf)
    ref = oa.metrics(counts, M, kg, kf)
    assert abs(got["R_geo"] - ref.R_geo) < 1e-12
    assert abs(got["R_50"] - ref.R_50) < 1e-12
    assert abs(got["recall_top_fuse_model"] - ref.recall_fuse_model) < 1e-12
    assert abs(got["recall_top_fuse_fused"] - ref.recall_fuse_fused) < 1e-12
    assert abs(got["changed_fraction"] - ref.changed) < 1e-12
