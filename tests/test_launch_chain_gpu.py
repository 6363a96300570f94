"""Back-to-back launches on one stream, where each kernel may be scheduled
while the previous one is still running (programmatic dependent launch).

Each kernel must touch global memory only after the previous kernel on the
stream has completed.  The chains below make that observable: a later call
overwrites an earlier call's input (write after read) or reads an earlier
call's output (read after write), and every output of the chain, launched
without a synchronisation in between, must equal the same call run alone.
(Codes reinterpreted as bf16 activations are arbitrary bit patterns, NaN and
infinity included; the kernels are deterministic, so the comparison is
bitwise.)
"""
import numpy as np
import pytest
import torch

from kronecker_factored_transforms_b200.workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("name,T1,T2,alpha", [
    ("hidden8192", 4096, 8192, None),         # batch, batch, then pair kernel (T3 = 2048): 64 x 128, cinv
    ("hidden8192", 2048, 8192, None),         # pair, batch, pair
    ("tiny", 16384, 32768, None),             # batch kernel with n2 = 16 padded to 64 columns
    ("llama7b_hidden", 1024, 4096, 2.0 ** -20)])  # warp-MMA kernel (alpha below 2^-19)
def test_transform_chain_war_and_raw(kq, name, T1, T2, alpha):
    w = make_workload(name, T=T1)
    alpha = w.alpha if alpha is None else alpha
    n1, n2, n = w.n1, w.n2, w.n
    xA0 = dev(w.x.view(np.int16))
    xB = dev(make_workload(name, T=T2, shard=1).x.view(np.int16))
    P1, P2 = dev(w.P1.view(np.int16)), dev(w.P2.view(np.int16))
    cinv = dev(w.cinv) if w.cinv is not None else None
    T3 = T2 * (n // 2) // (2 * n)                     # call 2's codes read as bf16 rows of n
    q1, s1 = torch.empty(T1 * n // 2, dtype=torch.uint8, device="cuda"), torch.empty(T1, device="cuda")
    s2 = torch.empty(T2, device="cuda")
    q3, s3 = torch.empty(T3 * n // 2, dtype=torch.uint8, device="cuda"), torch.empty(T3, device="cuda")
    xA = xA0.clone()
    q2 = xA.view(torch.uint8)[: T2 * n // 2]          # call 2 writes its codes over call 1's input

    def call1():
        kq.kq_transform_quant(xA, P1, P2, cinv, alpha, q1, s1, T1, n1, n2)

    def call2():
        kq.kq_transform_quant(xB, P1, P2, cinv, alpha, q2, s2, T2, n1, n2)

    def call3():
        kq.kq_transform_quant(q2, P1, P2, None, alpha, q3, s3, T3, n1, n2)

    kinds = [kq.kq_kernel_for(t, n1, n2, c, alpha) for t, c in ((T1, cinv is not None), (T2, cinv is not None),
                                                                (T3, False))]
    assert "unsupported" not in kinds

    def snap():
        return [t.clone() for t in (q1, s1, q2, s2, q3, s3)]

    # each call alone
    call1(); torch.cuda.synchronize()
    call2(); torch.cuda.synchronize()
    call3(); torch.cuda.synchronize()
    ref = snap()
    assert kq.kq_device_error() == 0
    # the same three back to back, repeated; call 1 needs its input back first
    for _ in range(3):
        for t in (q1, s1, s2, q3, s3):
            t.fill_(0)
        xA.copy_(xA0)
        torch.cuda.synchronize()
        call1(); call2(); call3()
        torch.cuda.synchronize()
        got = snap()
        for label, g, r in zip(("q1", "s1", "q2", "s2", "q3", "s3"), got, ref):
            assert torch.equal(g.view(torch.uint8), r.view(torch.uint8)), label
    assert kq.kq_device_error() == 0


def test_headwise_and_two_stage_chain(kq):
    """A per-head call, a two-stage call (itself two dependent kernels) and a
    per-head call that reads the two-stage codes, back to back."""
    rng = np.random.default_rng(7)
    Th, heads, D = 1024, 8, 128
    xh = dev((rng.standard_normal((Th, heads * D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
             .view(np.int16))
    Q, _ = np.linalg.qr(rng.standard_normal((D, D)))
    Ph = dev((Q.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16).view(np.int16))
    ws = make_workload("square65536", T=64)
    n1, n2, n = ws.n1, ws.n2, ws.n
    x2 = dev(ws.x.view(np.int16))
    P1, P2 = dev(ws.P1.view(np.int16)), dev(ws.P2.view(np.int16))
    cinv = dev(ws.cinv) if ws.cinv is not None else None
    wsb = kq.kq_two_stage_workspace_bytes(ws.T, n1, n2)
    work = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    qh1 = torch.empty(Th * heads * D // 2, dtype=torch.uint8, device="cuda")
    sh1 = torch.empty(Th * heads, device="cuda")
    q2 = torch.empty(ws.T * n // 2, dtype=torch.uint8, device="cuda")
    s2 = torch.empty(ws.T, device="cuda")
    Th3 = ws.T * n // 2 // (2 * heads * D)           # call 2's codes read as bf16 rows of heads * D
    qh3 = torch.empty(Th3 * heads * D // 2, dtype=torch.uint8, device="cuda")
    sh3 = torch.empty(Th3 * heads, device="cuda")

    def chain(sync):
        kq.kq_headwise_transform_quant(xh, Ph, 0.9, qh1, sh1, Th, heads, D)
        if sync:
            torch.cuda.synchronize()
        kq.kq_transform_quant_two_stage(x2, P1, P2, cinv, ws.alpha, q2, s2, work, wsb, ws.T, n1, n2)
        if sync:
            torch.cuda.synchronize()
        kq.kq_headwise_transform_quant(q2, Ph, 0.9, qh3, sh3, Th3, heads, D)
        torch.cuda.synchronize()
        return [t.clone() for t in (qh1, sh1, q2, s2, qh3, sh3)]

    ref = chain(True)
    for _ in range(3):
        for t in (qh1, sh1, q2, s2, qh3, sh3):
            t.fill_(0)
        got = chain(False)
        for label, g, r in zip(("qh1", "sh1", "q2", "s2", "qh3", "sh3"), got, ref):
            assert torch.equal(g.view(torch.uint8), r.view(torch.uint8)), label
    assert kq.kq_device_error() == 0


def test_chain_in_a_cuda_graph(kq):
    """The same kind of chain captured into a CUDA graph and replayed: every
    output equals the eager, synchronised result."""
    w = make_workload("llama7b_hidden", T=2048)      # 64 x 64, no cinv
    n1, n2, n = w.n1, w.n2, w.n
    x = dev(w.x.view(np.int16))
    P1, P2 = dev(w.P1.view(np.int16)), dev(w.P2.view(np.int16))
    T1 = w.T
    q1, s1 = torch.empty(T1 * n // 2, dtype=torch.uint8, device="cuda"), torch.empty(T1, device="cuda")
    T2 = T1 * (n // 2) // (2 * n)                     # call 1's codes read as bf16 rows of n
    q2, s2 = torch.empty(T2 * n // 2, dtype=torch.uint8, device="cuda"), torch.empty(T2, device="cuda")
    stream = torch.cuda.Stream()

    def chain():
        kq.kq_transform_quant(x, P1, P2, None, w.alpha, q1, s1, T1, n1, n2, stream=stream)
        kq.kq_transform_quant(q1, P1, P2, None, w.alpha, q2, s2, T2, n1, n2, stream=stream)

    with torch.cuda.stream(stream):
        chain()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (q1, s1, q2, s2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        chain()
    for _ in range(3):
        for t in (q1, s1, q2, s2):
            t.fill_(0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for label, a, b in zip(("q1", "s1", "q2", "s2"), (q1, s1, q2, s2), ref):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), label
    del g
    assert kq.kq_device_error() == 0
