"""Bounded waits on the GPU: a wait that cannot complete gives up and reports.

Every barrier wait in the kernels has a time bound; when it runs out the
kernel records ATTN_ERR_DEVICE_TIMEOUT in the device status word and winds
down (no copy left in flight, tensor memory freed) instead of spinning.
reserved[0] of an attn_prefill call makes the tensor-core kernel's softmax
warps first wait, with that bound in microseconds, on a barrier nothing
arrives at.  Nothing faults, traps or hangs: each wait ends after 1 ms, the
status word reports the timeout once, and the next call on the same context
is correct.
"""
import pytest
import torch

import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, poisoned_workspace, run_prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G", [1, 2])
def test_prefill_wait_timeout_is_reported_and_recovered(cuda_lib, G):
    p = W.random_prefill(900 + G, R=130, Hq=2 * G, Hkv=2, D=128, depth=300, sinks=True)
    (q, k, v, out), kw = A.problem_kwargs(p)
    out.fill_(float("nan"))
    args = A.make_args(q, k, v, out, **kw)
    args.reserved[0] = 1000
    ws = poisoned_workspace(A.workspace_size(args, A.OP_PREFILL))
    A.attn_prefill_args(args, ws=ws)
    torch.cuda.synchronize()
    with pytest.raises(A.AttnError) as e:
        A.check_device_status()
    assert e.value.status == -5          # ATTN_ERR_DEVICE_TIMEOUT
    A.check_device_status()              # reported once: the word was cleared
    assert torch.isnan(out).all()        # the CTAs gave up before writing
    # the context is still usable and the same call without the test is correct
    check(p, run_prefill(p), "prefill after a timed-out call")
