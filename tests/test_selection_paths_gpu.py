"""The two kernel paths for selection and attention agree on the same inputs.

For few (batch, kv-head) units with bf16 data, socket_decode runs one fused
selection + attention kernel; otherwise it runs the top-k kernel and then an
attention kernel (socket_set_selection_path documents the rule).  Both are
parity-tested against the oracle elsewhere; here the same inputs go through
both, and the selections must be identical bit for bit (the same exact rule:
the k largest float32 scores, ties to the lower index, ascending) and the
outputs equal up to float32 summation order.  The cases cover several slices
per unit, one slice, per-head units, a threshold bin over the candidate
capacity (all scores tied), and a ragged tail.
"""
import pytest
import torch

import soft_lsh_top_b200 as sk
import workloads as wl
from parity import gpu_decode, gpu_hash

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = {
    "grouped_many_slices": (wl.Workload(name="paths_a", B=2, Hq=8, Hkv=2, N=40001, L=24, P=8, tau=0.3, k=900,
                                        seed=7301), False, False),
    "grouped_one_slice": (wl.Workload(name="paths_b", B=1, Hq=8, Hkv=1, N=1500, L=16, P=7, tau=0.5, k=97,
                                      seed=7302), False, False),
    "group8_ragged": (wl.Workload(name="paths_c", B=1, Hq=16, Hkv=2, N=33333, L=32, P=8, tau=0.25, k=2048,
                                  seed=7303), False, False),
    "per_head": (wl.Workload(name="paths_d", B=1, Hq=4, Hkv=2, N=20000, L=12, P=8, tau=0.4, k=512, seed=7304),
                 True, False),
    "all_ties_over_capacity": (wl.Workload(name="paths_e", B=1, Hq=4, Hkv=2, N=12000, L=5, P=8, tau=0.3, k=700,
                                           seed=7305), False, True),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_and_separate_paths_agree(case):
    w, per_head, ties = CASES[case]
    inp = wl.make_inputs(w, DEV)
    if ties:
        inp["q"].zero_()
        inp["V"].fill_(1.0)
    ids, vnorm = gpu_hash(inp, w)
    assert sk.socket_set_selection_path(sk.SOCKET_PATH_AUTO) == sk.SOCKET_PATH_AUTO
    try:
        idx_a, out_a, sc_a = gpu_decode(inp, w, ids, vnorm, per_head=per_head)
        sk.socket_set_selection_path(sk.SOCKET_PATH_SEPARATE)
        idx_s, out_s, sc_s = gpu_decode(inp, w, ids, vnorm, per_head=per_head)
    finally:
        sk.socket_set_selection_path(sk.SOCKET_PATH_AUTO)
    assert torch.equal(sc_a.view(torch.int32), sc_s.view(torch.int32))  # the same scoring kernels
    assert torch.equal(idx_a, idx_s)
    assert torch.all(idx_a[..., 1:] > idx_a[..., :-1])
    torch.testing.assert_close(out_a, out_s, rtol=1e-5, atol=1e-5)
