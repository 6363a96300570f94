"""kq_transform_quant_two_stage_static (the two-stage path with its workspace in
a static device array of the library) against kq_transform_quant_two_stage
with a caller workspace, through the C ABI: the same codes and scales, bit for
bit, on two successive calls.  Independent of the other test files (it makes
its own inputs and is the first user of the static array in its process)."""
import math

import numpy as np
import pytest

from kronecker_factored_transforms_b200.workloads import f32_to_bf16_bits


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def _inputs(T, n1, n2, scaled, seed):
    rng = np.random.default_rng(seed)
    n = n1 * n2
    P1 = np.eye(n1) + 0.1 * rng.standard_normal((n1, n1)) / math.sqrt(n1)
    P2 = np.eye(n2) + 0.1 * rng.standard_normal((n2, n2)) / math.sqrt(n2)
    x = 0.5 * rng.standard_t(3, size=(T, n))
    cinv = (1.0 / np.exp(rng.uniform(math.log(0.5), math.log(2.0), n))).astype(np.float32) if scaled else None
    bits = lambda a: f32_to_bf16_bits(a.astype(np.float32))
    return bits(x), bits(P1), bits(P2), cinv


def test_static_workspace_rejects_oversize(kq):
    """4 T n1 n2 above the static array: KQ_ERR_ARG before anything is launched."""
    f = kq.lib.kq_transform_quant_two_stage_static
    x, P1, P2, q, s = 0x1000000, 0x2000000, 0x3000000, 0x5000000, 0x6000000
    limit_T = kq.STATIC_WORKSPACE_BYTES // (4 * 256 * 256)
    assert f(x, P1, P2, None, 0.9, q, s, limit_T + 1, 256, 256, None) == kq.KQ_ERR_ARG
    assert f(x, P1, P2, None, 0.9, q, s, 4, 272, 256, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(None, None, None, None, 0.9, None, None, 0, 256, 256, None) == kq.KQ_OK  # empty: no-op


@pytest.mark.gpu
def test_static_workspace_matches_caller_workspace(kq):
    import torch
    dev16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    # the last case fills the static array to its last byte: T = 256 at 256 x 256
    cases = [(9, 256, 256, True), (40, 112, 256, False), (256, 256, 256, True)]
    for call, (T, n1, n2, scaled) in enumerate(cases):
        x, P1, P2, cinv = _inputs(T, n1, n2, scaled, seed=31 + call)
        n = n1 * n2
        assert 4 * T * n <= kq.STATIC_WORKSPACE_BYTES
        if call == 2:
            assert kq.kq_two_stage_workspace_bytes(T, n1, n2) == kq.STATIC_WORKSPACE_BYTES
        xd, p1, p2 = dev16(x), dev16(P1), dev16(P2)
        cd = None if cinv is None else torch.from_numpy(cinv).cuda()
        need = kq.kq_two_stage_workspace_bytes(T, n1, n2)
        ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
        q_ref = torch.empty((T, n // 2), dtype=torch.uint8, device="cuda")
        s_ref = torch.empty((T,), dtype=torch.float32, device="cuda")
        kq.kq_transform_quant_two_stage(xd, p1, p2, cd, 0.85, q_ref, s_ref, ws, need, T, n1, n2)
        q = torch.full((T, n // 2), 0x5A, dtype=torch.uint8, device="cuda")
        s = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
        kq.kq_transform_quant_two_stage_static(xd, p1, p2, cd, 0.85, q, s, T, n1, n2)
        torch.cuda.synchronize()
        assert kq.kq_device_error() == 0
        assert torch.equal(q, q_ref), "codes differ on call %d" % call
        assert torch.equal(s, s_ref), "scales differ on call %d" % call
