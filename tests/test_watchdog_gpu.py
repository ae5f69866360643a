"""Bounded device waits: a loader that issues no copies (a flag nothing else
sets) makes every consumer wait run out; the kernel stops early, reports
ATTN_ERR_TIMEOUT through attn_debug_error, and the context stays usable."""
import pytest
import torch

from exact_io_aware_72_b200 import attn as A
from harness.inputs import make_qkv
from tests.parity import check_case

pytestmark = pytest.mark.gpu


def test_stalled_loader_times_out_and_context_survives(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 2, 512, 128, 31))
    assert A.debug_error()[0] == 0
    A.fwd(q, k, v, mask="causal", inject_stall=True, wait_timeout_ns=20_000_000)
    st, code = A.debug_error()
    assert st == A.ATTN_ERR_TIMEOUT and code != 0
    assert A.debug_error()[0] == 0          # the word was cleared
    check_case(1, 2, 2, 512, 128, "causal", seed=31)
    assert A.debug_error()[0] == 0
