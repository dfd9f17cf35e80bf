"""The row-sharded helpers on one GPU (no process group: the combine steps are identities): the
shard g and record are those of the plain calls, and two row halves combined off-line give the
whole tensor's record."""
import pytest

import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import dist as mxdist, inputs

from gpu_helpers import assert_stats

pytestmark = pytest.mark.gpu


def test_sharded_helpers_single_process(cuda_device):
    x = inputs.workload3_tensor(0, 4, device=cuda_device)  # 4096 x 11008, Student-t rows
    g = mxdist.global_scale_sharded(x, "ue5m3")
    assert g == int(mx.global_scale(x, "ue5m3").item()) & 0xFFFF
    _, _, st = mxdist.quantize_with_stats_sharded(x, 32, "ue5m3", g)
    ref = mx.quantize_with_stats(x, 32, "ue5m3", g)[2].to_dict()
    assert_stats(st, ref, "sharded record")
    halves = [mx.quantize_with_stats(h, 32, "ue5m3", g)[2].to_dict()
              for h in (x[:2048], x[2048:])]
    comb = {k: halves[0][k] + halves[1][k] for k in ("sse_elem", "sse_max", "sse_zero", "numel",
                                                    "n_blocks", "n_zero_blocks", "n_scale_sat",
                                                    "n_elem_sat")}
    assert_stats(comb, ref, "two halves")
