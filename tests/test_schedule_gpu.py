"""The persistent schedule as it runs on the device: with the visit-counter
test hook of attn_fwd_options, every work item of attn_fwd_num_work_items must
be visited exactly once, for every mask, head map and CTA count (including
grids larger and smaller than the item count, where the split last round and
the long/short pairing of row units change)."""
import pytest
import torch

from exact_io_aware_72_b200 import fwd, num_work_items
from harness.inputs import make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [
    (1, 2, 2, 256), (1, 2, 2, 1000), (2, 8, 2, 1500), (1, 6, 2, 640), (1, 3, 3, 1000), (3, 2, 1, 257),
    (1, 16, 2, 4096),
])
@pytest.mark.parametrize("mask,window", [("causal", None), ("full", None), ("sliding_window", 300)])
@pytest.mark.parametrize("grid", [0, 1, 5, 37, 148])
def test_every_item_visited_once(cuda_ok, shape, mask, window, grid):
    B, Hq, Hkv, N = shape
    d = 64
    q, k, v = (t.cuda() for t in make_qkv(B, Hq, Hkv, N, d, sum(shape)))
    n = num_work_items(B, Hq, Hkv, N, d, mask, window)
    assert n > 0
    visits = torch.zeros(n, dtype=torch.int32, device="cuda")
    fwd(q, k, v, mask=mask, window=window, grid_ctas=grid, item_visits=visits)
    torch.cuda.synchronize()
    counts = torch.bincount(visits.cpu().long(), minlength=3)
    assert int(visits.min()) == 1 and int(visits.max()) == 1, f"visit counts: {counts.tolist()}"
