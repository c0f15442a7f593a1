"""Failure detection without a GPU fault: the decode kernels' bounded waits
give up, report it in the workspace error word, and return; the context
stays usable.

socket_set_wait_limit(0) makes every bounded wait of the decode kernels give
up at once: the scoring kernel's and the attention kernel's waits for data
they have requested, and the fused selection + attention kernel's wait for
the threshold that the unit's last CTA publishes (that kernel runs for these
few-unit bf16 shapes; fp32 keys take the separate top-k and attention
kernels).  The kernels then set their bit in the error word, wait (with the
normal, long limit) for the copies they have already issued to land, and
return without results -- the path a real expiry takes.  Nothing here traps,
faults or hangs: no wait is left on something that never arrives.
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


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_expired_waits_are_reported_and_the_context_stays_usable(dtype):
    w = wl.Workload(name="expiry", B=1, Hq=4, Hkv=2, N=5000, L=8, P=8, tau=0.4, k=300, dtype=dtype, seed=7100)
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
    # bf16: the fused kernel's slices wait for the unit's threshold; fp32: the
    # attention kernel's row gathers wait for their copies.
    assert err & (SELECT if dtype == "bf16" else GATHER), hex(err)

    idx.fill_(-1)
    out.fill_(float("nan"))
    run()
    torch.cuda.synchronize()
    assert sk.read_device_error(ws) == 0
    assert torch.equal(idx, want_idx)
    assert torch.equal(_bits(out), _bits(want_out))
