"""The backward pass on the GPU against the float64 oracle's (which is pinned by finite
differences and by exact attention's gradient in the exact limits).  The oracle is fed
the GPU's own clustering (teacher forcing).  Tolerance: per tensor and (b,h),
max|g - g*| / max|g*| <= 1e-4 (float32) and <= 2e-2 (bfloat16 inputs and outputs)."""
import numpy as np
import pytest
import torch

from clustered_softmax_attention_b200 import muse as m
from clustered_softmax_attention_b200.inputs import draw_problem, round_to_bf16
from oracle import muse_oracle as mo

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _problem(seed, H, N, D, Dv, dt):
    rng = np.random.Generator(np.random.PCG64(seed))
    cast = round_to_bf16 if dt == "bf16" else (lambda a: a.astype(np.float32))
    parts = [draw_problem(rng, N, D, Dv, 24, 0.4 / np.sqrt(D)) for _ in range(H)]
    dO = rng.standard_normal((1, H, N, Dv))
    to = lambda a: torch.tensor(np.ascontiguousarray(a), dtype=torch.float32).to(TDT[dt]).cuda()
    Q, K, V = (to(np.stack([cast(p[k]) for p in parts])[None]) for k in range(3))
    return Q, K, V, to(cast(dO))


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("dt,N,D,Dv,Cq,Ck,s", [("f32", 512, 64, 64, 12, 16, 1.0),
                                               ("bf16", 1024, 64, 64, 32, 32, 1.0),
                                               ("f32", 384, 64, 128, 8, 20, 0.6),
                                               ("bf16", 512, 128, 64, 16, 10, 0.125),
                                               ("bf16", 256, 128, 128, 256, 16, 1.0)])
def test_backward_vs_oracle(dt, N, D, Dv, Cq, Ck, s, parity):
    Q, K, V, dO = _problem(50 + N + D, 2, N, D, Dv, dt)
    ql, _, qp, qo = m.muse_kmeans(Q, Cq, 4)
    kl, _, kp, ko = m.muse_kmeans(K, Ck, 4)
    dQ, dK, dV = m.muse_backward(Q, K, V, dO, qp, qo, kp, ko, s)
    assert m.muse_last_device_status() == 0
    Qf, Kf, Vf, dOf = _host(Q), _host(K), _host(V), _host(dO)
    for h in range(2):
        ref = mo.muse_backward_from_labels(Qf[0, h], Kf[0, h], Vf[0, h], ql[0, h].cpu().numpy(),
                                           kl[0, h].cpu().numpy(), Cq, Ck, s, dOf[0, h])
        for name, got, want in zip(("dQ", "dK", "dV"), (dQ, dK, dV), ref):
            err = mo.max_rel_err(_host(got)[0, h], want)
            parity(f"{name} h={h}", err, TOL[dt])
            assert err <= TOL[dt], (name, h, err)


def test_backward_is_deterministic():
    Q, K, V, dO = _problem(7, 2, 512, 64, 64, "bf16")
    _, _, qp, qo = m.muse_kmeans(Q, 16, 3)
    _, _, kp, ko = m.muse_kmeans(K, 16, 3)
    a = m.muse_backward(Q, K, V, dO, qp, qo, kp, ko)
    b = m.muse_backward(Q, K, V, dO, qp, qo, kp, ko)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert m.muse_last_device_status() == 0
