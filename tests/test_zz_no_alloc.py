"""muse_kmeans_noalloc: the K-means entry point for callers that cannot allocate
device memory (no workspace argument; scratch in a static device array inside the
library).  Its results must equal those of muse_kmeans, the entry point that takes
a caller-allocated workspace, on consecutive calls.

The shared scratch keeps the previous call's contents.  Both calls below take the
multi-launch kernels (float32 with D = 128, then bfloat16 with C > 128), which are the
ones that use the scratch, and the larger problem goes first, so the second call runs
over the first one's leftover counts, chunk bases and ranks: none of that may leak into
its result.

This file is collected last so that a run stopping at the first failure has run
every other test before it."""
import numpy as np
import pytest
import torch

from clustered_softmax_attention_b200 import muse as m
from clustered_softmax_attention_b200.inputs import draw_problem, round_to_bf16

pytestmark = pytest.mark.gpu


def _inputs(seed, H, N, D, dt):
    rng = np.random.Generator(np.random.PCG64(seed))
    cast = round_to_bf16 if dt == torch.bfloat16 else (lambda a: a.astype(np.float32))
    X = np.stack([cast(draw_problem(rng, N, D, D, 48, 0.4 / np.sqrt(D))[0])
                  for _ in range(H)])[None]
    return torch.tensor(X).to(dt).cuda().contiguous()


def _noalloc(X, C, iters):
    B, H, N, D = X.shape
    labels = torch.empty(B, H, N, dtype=torch.int32, device=X.device)
    cen = torch.empty(B, H, C, D, dtype=torch.float32, device=X.device)
    perm = torch.empty(B, H, N, dtype=torch.int32, device=X.device)
    offs = torch.empty(B, H, C + 1, dtype=torch.int32, device=X.device)
    rc = m.lib().muse_kmeans_noalloc(m._p(X), m.dims(X), C, iters, m._p(labels), m._p(cen),
                                     m._p(perm), m._p(offs), m._stream())
    assert rc == 0, m.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    return labels, cen, perm, offs


def _same(got, ref):
    for a, b in zip(got[:1] + got[2:], ref[:1] + ref[2:]):   # labels, perm, offsets
        assert torch.equal(a, b)
    torch.testing.assert_close(got[1], ref[1], rtol=2e-5, atol=2e-6)  # centroids


def test_noalloc_kmeans_equals_workspace_kmeans_on_consecutive_calls():
    cases = [(_inputs(31, 3, 3000, 128, torch.float32), 100, 4),   # 9000 rows, multi-launch
             (_inputs(32, 2, 2048, 64, torch.bfloat16), 200, 5)]   # 4096 rows, C > 128
    for X, C, iters in cases:            # two calls in a row; the second on stale scratch
        ref = m.muse_kmeans(X, C, iters)  # caller-allocated workspace
        _same(_noalloc(X, C, iters), ref)
    assert m.muse_last_device_status() == 0


def test_noalloc_kmeans_one_launch_path_has_no_scratch_limit():
    """bfloat16, D = 64, C <= 128 keeps its state on chip: a problem whose multi-launch
    scratch would exceed the array (B*H*N = 4M rows) is still accepted."""
    X = _inputs(33, 1, 65536, 64, torch.bfloat16).expand(1, 64, 65536, 64).contiguous()
    assert m.muse_workspace_size("muse_kmeans", m.dims(X), 128) > m.NOALLOC_SCRATCH_BYTES
    ref = m.muse_kmeans(X, 128, 2)
    _same(_noalloc(X, 128, 2), ref)
    assert m.muse_last_device_status() == 0


def test_noalloc_kmeans_refuses_more_than_its_scratch():
    d = m.MuseDims(16, 16, 65536, 128, 128, m.MUSE_BF16, 1.0)
    need = m.muse_workspace_size("muse_kmeans", d, 1024)
    assert need > m.NOALLOC_SCRATCH_BYTES
    fake = m.ctypes.c_void_p(1 << 20)   # never dereferenced: the size check fails first
    rc = m.lib().muse_kmeans_noalloc(fake, d, 1024, 3, fake, fake, fake, fake, m._stream())
    assert rc == 4
