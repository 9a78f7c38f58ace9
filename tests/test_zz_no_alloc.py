"""The allocation-free exhaustive selection gives the same top-k as the
handle-based exhaustive call on the same keys.

It exists for callers that cannot allocate device memory themselves (a
server drawing all memory from its own reserved pool, a latency-critical
path that must avoid cudaMalloc's implicit synchronisation).  Its only
scratch is a fixed array inside the library that every call shares, so the
test calls it twice in a row: the second call must not see leftovers of
the first.  Collected last on purpose (file name), and independent of what
ran before it.
"""
import numpy as np
import pytest
import torch

from synth import workloads as S
from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a GPU", allow_module_level=True)


def _compare(a, sa, b, sb, qv, wv, kv):
    """Same ids (as sets), scores within the parity tolerance; the kernels
    are the same, so they are expected to agree bit for bit."""
    for i in range(a.shape[0]):
        tol = P.score_tol(qv[i], wv[i], kv[np.maximum(b[i], 0)])
        assert set(a[i].tolist()) == set(b[i].tolist()), i
        assert np.all(np.abs(sa[i] - sb[i]) <= tol + 1e-6), i


def _noalloc(C, keys, code, qd, wd, pos0, k):
    T = qd.shape[0]
    out = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
    sc = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    status = torch.full((1,), 0x7777, dtype=torch.int32, device="cuda")
    C.ai_select_exhaustive_noalloc(keys, code, qd, wd, pos0, k, out, sc, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device flags raised"
    return out.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("dtype,d,H,n,T,k", [("bf16", 128, 32, 3000, 96, 100),
                                              ("bf16", 128, 64, 1200, 40, 64),
                                              ("fp32", 32, 4, 700, 50, 16)])
def test_noalloc_matches_handle_based_exhaustive(dtype, d, H, n, T, k):
    from ivf_top_key_b200 import C
    wl = S.scaled(S.WORKLOADS["glm_bf16_L128k"], L=n, T=T, d=d, H=H, M=64, key_dtype=dtype,
                  q_dtype=dtype, window=256, refit_period=0, budget=512, k=k)
    gpu, orc = P.make_pair(wl, max_keys=n)
    kd, ks, kv = P.keys_inputs(wl, 0, n)
    gpu.append_keys(kd, ks)
    pos0 = n - T
    qd, wd, qv, wv = P.query_inputs(wl, pos0, n)
    ref = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ref_sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    gpu.select_exhaustive(qd, wd, pos0, k, out=ref, out_scores=ref_sc)
    gpu.sync()
    code = C.DTYPES[dtype]
    for call in range(2):
        a, sa = _noalloc(C, kd, code, qd, wd, pos0, k)
        _compare(a, sa, ref.cpu().numpy(), ref_sc.cpu().numpy(), qv, wv, kv)
    gpu.close()


def test_noalloc_several_passes_then_a_smaller_call():
    """300,000 bf16 keys leave room for 13 score rows per pass, so 40
    queries take four passes (query, weight and output offsets move each
    pass).  The second call uses fewer keys (another row stride) and other
    queries, so scores left in the shared array by the first call would
    surface as a mismatch."""
    from ivf_top_key_b200 import C
    n, k = 300_000, 64
    wl = S.scaled(S.WORKLOADS["glm_bf16_L128k"], L=n, T=40, M=256, window=1024, refit_period=0,
                  budget=512, k=k)
    gpu, _ = P.make_pair(wl, max_keys=n)
    kd, ks, kv = P.keys_inputs(wl, 0, n)
    gpu.append_keys(kd, ks)
    for n_call, T in ((n, 40), (200_000, 37)):
        pos0 = n_call - T
        qd, wd, qv, wv = P.query_inputs(wl, pos0, n_call)
        # causal: queries below n_call see the same keys in the full store
        ref = torch.empty((T, k), dtype=torch.int32, device="cuda")
        ref_sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
        gpu.select_exhaustive(qd, wd, pos0, k, out=ref, out_scores=ref_sc)
        gpu.sync()
        a, sa = _noalloc(C, kd[:n_call], C.AI_BF16, qd, wd, pos0, k)
        _compare(a, sa, ref.cpu().numpy(), ref_sc.cpu().numpy(), qv, wv, kv)
    gpu.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from ivf_top_key_b200 import C, AiError
    keys = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((1, 32, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, 32), dtype=torch.float32, device="cuda")
    out = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(AiError, match="ARG"):
        # a key count above the documented maximum, passed without data
        C._check(C._lib.ai_select_exhaustive_noalloc(
            C._ptr(keys), C.AI_BF16, (1 << 20) + 1, 128, 32, C._ptr(q), C._ptr(w), 0, 1, 4,
            C._ptr(out), None, None, C._stream(None)))
