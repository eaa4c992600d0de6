"""The bounded-wait timeout path of the tensor-core forward, exercised without any fault.

Every device-side wait of the fused forward (an mbarrier phase, another CTA's published decay
prefix) gives up after a limit, records UA_ERR_TIMEOUT and tears its CTA down (abort flag, a
short pause for copies in flight, TMEM freed) instead of hanging.  Lowering the limit to 0
makes every wait that has to spin give up at its first check; the call must then report
UA_ERR_TIMEOUT through the status word, and with the default limit restored the next call
must be clean and give the same results as before."""
import pytest
import torch

from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua

pytestmark = pytest.mark.gpu


def _inputs(w):
    x = I.make_prefill_inputs(w)
    return {n: torch.from_numpy(a).cuda().to(torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32)
            for n, a in x.items()}


@pytest.mark.parametrize("d", [64, 128])
def test_zero_wait_limit_reports_timeout_and_leaves_the_context_usable(d):
    # 32 query tiles in one chain: the last CTAs wait on their predecessors' prefixes
    w = I.Workload("timeout", 1, 4096, 3 if d == 128 else 4, 1, d, "bf16", 4096 + d)
    x = _inputs(w)
    args = (x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    assert ua.get_device_status() == 0
    ref = ua.prefill_fwd(*args, scale=w.scale, theta=w.theta)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    try:
        ua.set_wait_limit_ns(0)
        ua.prefill_fwd(*args, scale=w.scale, theta=w.theta)
        torch.cuda.synchronize()
        code = ua.get_device_status()
    finally:
        ua.set_wait_limit_ns(ua.WAIT_LIMIT_DEFAULT_NS)
    assert code == 7, f"expected UA_ERR_TIMEOUT, status word {ua.STATUS.get(code, code)}"
    again = ua.prefill_fwd(*args, scale=w.scale, theta=w.theta)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    for n in ("o", "lse", "b_final"):
        assert torch.equal(again[n], ref[n]), n
