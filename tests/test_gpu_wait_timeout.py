"""Failure detection on the GPU without a GPU fault: a pipeline wait that runs out.

sap_test_arm_wait_timeout makes the next forward launch use a 20 ms wait limit and leave the
first V tile of its first CTA out (no copy is issued, so nothing is in flight).  In that CTA the
MMA issuer waits for the tile, and the producer waits for the tile's ring stage to be released;
whichever wait started first runs out at the limit and records its timeout bit in the device
error word (the two-tile kernel, with shared or per-tile K/V: the MMA issuer's; the one-tile
kernel: the producer's), the
other roles see the CTA's abort flag, and the CTA winds down (its issued MMAs and copies are
waited for before tensor memory and shared memory are released); every other CTA finishes
normally.  The call returns, the host reads SAP_ERR_DEVICE with the bit through
sap_device_status, and the next normal call on the same process passes parity: the context stays
usable.
"""
import math

import pytest

import oracle
import packed_sequence_causal_b200 as sap
import workloads
from gpu_helpers import Run, assert_close, assert_lse

pytestmark = pytest.mark.gpu

K_ERR_TIMEOUT_LOAD, K_ERR_TIMEOUT_MMA = 1 << 0, 1 << 1
K_ERR_TIMEOUT_ANY = 0xF  # load, MMA, softmax, epilogue waits


@pytest.mark.parametrize("hq,hkv,first", [(4, 2, K_ERR_TIMEOUT_MMA),    # two-tile forward kernel
                                           (4, 4, K_ERR_TIMEOUT_MMA),    # two-tile, K/V per tile (MHA)
                                           (3, 3, K_ERR_TIMEOUT_LOAD)])  # one-tile forward kernel
def test_wait_that_runs_out_is_reported_and_the_context_survives(hq, hkv, first):
    b = workloads.custom_batch([700, 324], hq, hkv, 128, seed=61, with_do=False)
    r = Run(b, 2)
    r.fwd()  # uploads the plan; normal call
    lib = sap.load_library()
    assert lib.sap_test_arm_wait_timeout(20_000_000) == 0
    sap.sap_attn_fwd(r.plan, r.q, r.k, r.v, r.scale, r.o, r.lse, r.ws_fwd)
    code = sap.sap_device_status()  # synchronises: the launch has ended
    assert code & first and code & ~K_ERR_TIMEOUT_ANY == 0, code
    assert sap.sap_device_status() == 0  # reading the word cleared it
    o, lse = r.fwd()  # the hook disarmed itself: a normal launch on the same context
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, 1.0 / math.sqrt(128))
    assert_close(o, ro, "O after a timed-out launch")
    assert_lse(lse, rl, "LSE after a timed-out launch")
