"""Failure detection on the GPU without a fault: the bounded wait of the
pipelined kernels, run against a barrier that nothing completes, gives up,
reports the timeout through the device status word, and leaves the context
usable (a normal index call succeeds afterwards)."""
import pytest
import torch

from synth import workloads as S
from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a GPU", allow_module_level=True)


def test_bounded_wait_reports_timeout_and_context_survives():
    from ivf_top_key_b200 import C, AiError
    assert C.ai_debug_wait_timeout(1 << 16) & 1 == 1  # bit 0: timeout
    with pytest.raises(AiError, match="ARG"):
        C.ai_debug_wait_timeout(0)
    # the context still works: a small index end to end
    wl = S.scaled(S.WORKLOADS["tiny_fp32_L4k"], L=1024, T=512)
    gpu, _ = P.make_pair(wl)
    kd, ks, _ = P.keys_inputs(wl, 0, 1024)
    gpu.append_keys(kd, ks)
    gpu.seal()
    qd, wd, _, _ = P.query_inputs(wl, 512, 1024)
    out = torch.empty((512, wl.k), dtype=torch.int32, device="cuda")
    gpu.route_refine(qd, wd, 512, wl.k, wl.budget, out=out)
    gpu.sync()
    assert int(out.min()) >= -1 and int(out.max()) < 1024
    gpu.close()
