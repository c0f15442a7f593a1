"""The kernel paths of a decode step agree on the same inputs.

By shape, socket_decode runs the whole step in one kernel (small problems),
or a fused selection + attention kernel after the soft-table and scoring
kernels (few bf16 units), or four separate kernels (socket_set_selection_path
documents the rule and can force the separate kernels).  Every path is
parity-tested against the oracle elsewhere; here the same inputs go through
the shape's own path and through the separate kernels.  Scores must be
identical bit for bit (the same float32 operations in the same order), so
must the selections (the k largest scores, ties to the lower index,
ascending), and the outputs must agree up to float32 summation order.  The
cases cover several slices per unit, one slice, per-head units, a threshold
bin over the candidate capacity (all scores tied), a ragged tail, and the
one-kernel step with fp32 and bf16 data, hard LSH (tau = 0) and P < 4.
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
    # Many 32K-key slices per unit: the top-k CTAs of the separate path write
    # their own slices of the selection (candidates, and a threshold bin over
    # the candidate capacity).
    "many_slices_spread": (wl.Workload(name="paths_j", B=1, Hq=4, Hkv=2, N=300001, L=8, P=8, tau=0.3, k=1500,
                                       seed=7310), False, False),
    "many_slices_spread_all_ties": (wl.Workload(name="paths_k", B=1, Hq=4, Hkv=2, N=270000, L=5, P=8, tau=0.3,
                                                k=900, seed=7311), False, True),
    # The one-kernel step (N <= 8192, L <= 32, small G * L).
    "one_kernel_tiny_f32": (wl.TINY, False, False),
    "one_kernel_bf16_group4": (wl.Workload(name="paths_f", B=2, Hq=8, Hkv=2, N=6001, L=12, P=8, tau=0.3, k=500,
                                           seed=7306), False, False),
    "one_kernel_per_head": (wl.Workload(name="paths_g", B=1, Hq=8, Hkv=2, N=5000, L=20, P=6, tau=0.6, k=1000,
                                        seed=7307), True, False),
    "one_kernel_hard_lsh_p3": (wl.Workload(name="paths_h", B=1, Hq=2, Hkv=1, N=8192, L=32, P=3, tau=0.0, k=64,
                                           dtype="f32", seed=7308), False, False),
    "one_kernel_all_ties": (wl.Workload(name="paths_i", B=1, Hq=4, Hkv=2, N=3000, L=5, P=8, tau=0.3, k=333,
                                        seed=7309), False, True),
}

# The kernels each case takes by shape (socket_last_decode_path reports them).
ONE, FUSED = sk.SOCKET_STEP_ONE_KERNEL, sk.SOCKET_STEP_FUSED
EXPECTED_PATH = {name: (ONE if name.startswith("one_kernel") else FUSED) for name in CASES}


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
        assert sk.socket_last_decode_path() == EXPECTED_PATH[case]
        sk.socket_set_selection_path(sk.SOCKET_PATH_SEPARATE)
        idx_s, out_s, sc_s = gpu_decode(inp, w, ids, vnorm, per_head=per_head)
        assert sk.socket_last_decode_path() == sk.SOCKET_STEP_SEPARATE
    finally:
        sk.socket_set_selection_path(sk.SOCKET_PATH_AUTO)
    assert torch.equal(sc_a.view(torch.int32), sc_s.view(torch.int32))  # the same scoring kernels
    assert torch.equal(idx_a, idx_s)
    assert torch.all(idx_a[..., 1:] > idx_a[..., :-1])
    torch.testing.assert_close(out_a, out_s, rtol=1e-5, atol=1e-5)


def test_last_decode_path_is_per_thread():
    """socket_last_decode_path reports the calling host thread's own last
    decode: another thread that made none sees -1."""
    import threading

    w = CASES["one_kernel_bf16_group4"][0]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    gpu_decode(inp, w, ids, vnorm)
    assert sk.socket_last_decode_path() == sk.SOCKET_STEP_ONE_KERNEL
    seen = []
    t = threading.Thread(target=lambda: seen.append(sk.socket_last_decode_path()))
    t.start()
    t.join()
    assert seen == [-1]
