"""Failure detection on the GPU without a fault: a bounded pipeline wait on a
barrier that nothing arrives on gives up after its limit, the kernel reports
ATTN_DEV_TIMEOUT in the caller's status word, and the context stays usable
(a forward right after it matches the oracle)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import compare, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402
from exact_attention_145_b200 import _lib  # noqa: E402


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    lib = _lib.load()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.attn_selftest_wait_timeout(status.data_ptr(), stream) == _lib.ATTN_OK
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.ATTN_DEV_TIMEOUT
    w = W.WORKLOADS["tiny_mha_s128_d64"]
    d = W.make_prefill_inputs(w)
    o, lse = ea.attn_fwd(dev_bf16(d["q"]), dev_bf16(d["k"]), dev_bf16(d["v"]))
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(d["q"], d["k"], d["v"])
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "after timeout self-test")
