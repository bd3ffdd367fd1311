"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every pipeline wait in the library's kernels gives up after a limit, records
QLORA_ERR_TIMEOUT in the device error word, lets the kernel's other roles
stop, waits (bounded) for the copies and tensor-core work already in flight,
frees its tensor memory and returns.  The test hook qlora_debug_inject_stall
arms one launch in which a producer warp skips one signal (a flag that nothing
else sets), with a 1 ms limit, so that path runs for real: the call must come
back, the host must read the timeout, and the very next normal call on the
same context must match the oracle again.  Nothing here traps, faults or
spins without a bound.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import codebook as ocb
from oracle import codec as occ
from test_gpu_linear import Runner, full_check

pytestmark = pytest.mark.gpu

TIMEOUT = 7          # QLORA_ERR_TIMEOUT
LIMIT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    q.qlora_check_device_error()   # start from a clean error word
    yield q
    q.qlora_debug_inject_stall(None)


def expect_timeout(q):
    with pytest.raises(q.QLoraError) as e:
        q.qlora_check_device_error()
    assert e.value.status == TIMEOUT
    q.qlora_check_device_error()   # the word was cleared by the read


def test_quantizer_wait_runs_out_then_recovers(q):
    W = synthetic.normal((1024, 1024), 0.02, 901, torch.bfloat16)
    w = q.NF4Weight(1024, 1024)
    ws = torch.empty(q.qlora_quantize_workspace_bytes(1024, 1024), dtype=torch.uint8, device="cuda")
    Wd = W.cuda()
    q.qlora_debug_inject_stall("quantize", LIMIT_NS)
    q.qlora_quantize_nf4_dq(Wd, w, ws)
    expect_timeout(q)
    # the next call is a normal one and is bit-exact
    q.qlora_quantize_nf4_dq(Wd, w, ws)
    q.qlora_check_device_error()
    ref = occ.quantize(W.float().numpy(), ocb.nf4_codebook())
    assert np.array_equal(w.packed.cpu().numpy(), ref["packed"])
    assert np.array_equal(w.code2.cpu().numpy(), ref["e"])


@pytest.mark.parametrize("M", [200, 512])        # single-CTA engine, CTA-pair engine
@pytest.mark.parametrize("kind", ["fwd_fused", "bwd_fused"])
def test_fused_gemm_wait_runs_out_then_recovers(q, M, kind):
    case = synthetic.linear_case(M, 384, 512, 16, alpha=16.0, seed=910 + M)
    run = Runner(q, case)
    N, K, r = run.w.rows, run.w.cols, case["r"]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    q.qlora_debug_inject_stall(kind, LIMIT_NS)
    if kind == "fwd_fused":
        q.qlora_linear_fwd(run.w, run.X, M, run.A, run.B, r, case["scale"], Y, None, run.ws)
    else:
        q.qlora_linear_bwd(run.w, run.X, run.dY, M, run.A, run.B, r, case["scale"], None, dX, dA, dB, run.ws)
    expect_timeout(q)
    # the context is intact: normal calls on it match the oracle
    full_check(q, case, ydt=torch.bfloat16)
