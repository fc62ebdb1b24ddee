"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait in the tensor-core kernels has a limit; past it the kernel records
MUSE_ERR_TIMEOUT in the device status word, winds every warp down (copies and MMAs in
flight drained, tensor memory freed) and returns, so the context stays usable.  Here the
refinement kernel is told never to load its value tiles -- the waits for them can only
run out -- with a 1 ms limit: the call must report MUSE_ERR_TIMEOUT, and the next normal
call on the same context must report MUSE_OK and reproduce the earlier output exactly."""
import numpy as np
import pytest
import torch

from clustered_softmax_attention_b200 import muse as m
from clustered_softmax_attention_b200.inputs import draw_problem, round_to_bf16

pytestmark = pytest.mark.gpu


def _problem(seed, H, N, D):
    rng = np.random.Generator(np.random.PCG64(seed))
    parts = [draw_problem(rng, N, D, D, 32, 0.4 / np.sqrt(D)) for _ in range(H)]
    return [torch.tensor(np.stack([round_to_bf16(p[k]) for p in parts])[None]).to(torch.bfloat16)
            .cuda().contiguous() for k in range(3)]


@pytest.mark.parametrize("wait_limit_ns", [1_000_000, 0])
def test_refinement_wait_runs_out_and_reports_timeout(wait_limit_ns, parity):
    # (0 keeps the default 2 s limit: every block of this 16-block grid waits it out once)
    Q, K, V = _problem(41, 1, 2048, 64)
    C, T = 32, 4
    ql, qc, qp, qo = m.muse_kmeans(Q, C, T)
    kl, kc, kp, ko = m.muse_kmeans(K, C, T)
    summ = m.muse_tilted_summaries(qc, K, V, kp, ko, C, 1.0, want_mu_v=False)
    args = (Q, K, V, qc, qp, qo, kp, ko, summ["logZ"], summ["mu_k"], 1.0)
    O_ref = m.muse_dipole_refine(*args)
    assert m.muse_last_device_status() == 0
    m.muse_set_test_hooks(m.MUSE_TEST_WITHHOLD_VALUES, wait_limit_ns)
    try:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        m.muse_dipole_refine(*args)
        ev1.record()
        st = m.muse_last_device_status()
        parity("timed-out call, ms", ev0.elapsed_time(ev1))
    finally:
        m.muse_set_test_hooks(0, 0)
    assert st == 6, m.STATUS.get(st, st)          # MUSE_ERR_TIMEOUT
    O = m.muse_dipole_refine(*args)
    assert m.muse_last_device_status() == 0        # the context is still usable
    assert torch.equal(O, O_ref)
