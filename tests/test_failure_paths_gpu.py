"""Failure detection without a GPU fault: the decode kernels' bounded waits
give up, report it in the workspace error word, and return; the context
stays usable.

socket_set_wait_limit(0) makes every bounded wait of the decode kernels give
up at once: the scoring kernel's and the attention kernel's waits for data
they have requested, and the fused selection + attention kernel's wait for
the threshold that the unit's last CTA publishes.  The kernels then set
their bit in the error word, wait (with the normal, long limit) for the
copies they have already issued to land, and return without results -- the
path a real expiry takes.  Nothing here traps, faults or hangs: no wait is
left on something that never arrives.

The shapes (N above the one-kernel step's limit, so that path, which has no
bounded waits, is not taken) run, by path: bf16 by shape -> soft tables,
scoring, fused selection + attention; bf16 forced separate and fp32 ->
soft tables, scoring, top-k, attention.
"""
import pytest
import torch

import soft_lsh_top_b200 as sk
import workloads as wl
from parity import gpu_hash

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GATHER, TABLE, SELECT = 0x1, 0x2, 0x4


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t


@pytest.mark.parametrize("dtype,path,N", [("bf16", "auto", 9000), ("bf16", "separate", 9000), ("f32", "auto", 9000),
                                          ("bf16", "separate", 9 * 32768 + 5)])
def test_expired_waits_are_reported_and_the_context_stays_usable(dtype, path, N):
    """The last case has nine 32K-key top-k slices per unit: each slice CTA
    waits for the unit's output slots (SELECT) before writing its part."""
    w = wl.Workload(name="expiry", B=1, Hq=4, Hkv=2, N=N, L=8, P=8, tau=0.4, k=300, dtype=dtype, seed=7100)
    mode = sk.SOCKET_PATH_AUTO if path == "auto" else sk.SOCKET_PATH_SEPARATE
    before = sk.socket_set_selection_path(mode)
    try:
        want = [GATHER]
        if dtype == "bf16" and path == "auto":
            want = [SELECT]  # the fused kernel's slices wait for the unit's threshold
        elif N > 8 * 32768:
            want = [GATHER, SELECT]
        _expire_and_recover(w, dtype, want)
    finally:
        sk.socket_set_selection_path(before)


def _expire_and_recover(w, dtype, want):
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    ws, idx, out = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, DEV)

    def run():
        sk.socket_decode(inp["q"], inp["W"], ids, vnorm, inp["K"], inp["V"], w.N, w.tau, w.k, ws, idx, out)

    run()
    torch.cuda.synchronize()
    assert sk.read_device_error(ws) == 0
    want_idx, want_out = idx.clone(), out.clone()

    previous = sk.socket_set_wait_limit(0)
    try:
        run()
        torch.cuda.synchronize()  # the kernels returned
        err = sk.read_device_error(ws)
    finally:
        sk.socket_set_wait_limit(previous)
    assert err & TABLE, hex(err)
    # The attention kernel's row gathers wait for their copies; the fused
    # kernel's slices, and the slices of a unit with many top-k slices, wait
    # for the unit's last CTA.
    for bit in want:
        assert err & bit, hex(err)

    idx.fill_(-1)
    out.fill_(float("nan"))
    run()
    torch.cuda.synchronize()
    assert sk.read_device_error(ws) == 0
    assert torch.equal(idx, want_idx)
    assert torch.equal(_bits(out), _bits(want_out))
