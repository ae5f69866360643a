"""The backward at the full sizes the benchmark times (same inputs, same
launches), against the fp64 backward oracle on whole heads, element by element
within the bound derived in tests/parity_bwd.py.

dense (B=2, 32/32 heads, N=8192, d=128, causal, sharp rows): two whole heads,
dQ, dK and dV (with one query head per KV head, a head's dK and dV come from it
alone).  gqa (B=1, 64/8, N=16384): dQ of one whole query head (its dK and dV
sum over the group's eight query heads; that sum is checked at small sizes).
"""
import pytest
import torch

from harness.inputs import MASK_NAMES, WORKLOADS, make_dout, make_workload
from oracle import attention_bwd_fp64 as G
from tests.parity_bwd import bounds, compare_bwd, run_cuda_bwd, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,heads,grads", [
    ("dense", [(0, 0), (1, 31)], ("dq", "dk", "dv")),
    ("gqa", [(0, 63)], ("dq",)),
])
def test_backward_workload_whole_heads(cuda_ok, name, heads, grads):
    w = WORKLOADS[name]
    q, k, v = make_workload(w, device="cuda")
    do = make_dout(w.B, w.Hq, w.N, w.d, w.seed, device="cuda")
    got = dict(zip(("dq", "dk", "dv"), run_cuda_bwd(q, k, v, do, w.mask, w.window, w.scale)))
    kind = MASK_NAMES[w.mask]
    g = w.Hq // w.Hkv
    for b, h in heads:
        hk = h // g
        qn, don = to_np(q[b:b + 1, h:h + 1]), to_np(do[b:b + 1, h:h + 1])
        kn, vn = to_np(k[b:b + 1, hk:hk + 1]), to_np(v[b:b + 1, hk:hk + 1])
        refs = dict(zip(("dq", "dk", "dv"), G.attention_bwd(qn, kn, vn, don, w.scale, kind, w.window)))
        bnds = dict(zip(("dq", "dk", "dv"), bounds(qn, kn, vn, don, w.scale, kind, w.window)))
        sel = {"dq": (b, h), "dk": (b, hk), "dv": (b, hk)}
        mine = [to_np(got[n][sel[n][0]:sel[n][0] + 1, sel[n][1]:sel[n][1] + 1]) for n in grads]
        worst = compare_bwd(grads, mine, [refs[n] for n in grads], [bnds[n] for n in grads], (name, b, h))
        print(f"\n{name} head ({b}, {h}): worst error / bound " +
              ", ".join(f"{n} {r:.3f}" for n, r in worst.items()))
    del q, k, v, do, got
    torch.cuda.empty_cache()
