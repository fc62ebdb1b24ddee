"""The C-ABI library: it loads, exports every declared entry point, sizes its
workspace, and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes

import pytest

from clustered_softmax_attention_b200 import muse as m


@pytest.fixture(scope="module")
def lib():
    return m.load_library()


def test_every_declared_entry_point_is_exported(lib):
    names = m.declared_entry_points()
    assert {"muse_kmeans", "muse_tilted_summaries", "muse_dipole_refine", "muse_forward",
            "muse_forward_ex", "muse_causal_blocks", "muse_retrieve_exact", "muse_workspace_size",
            "muse_status_string", "muse_last_device_status", "muse_causal_levels"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in m.STATUS.items():
        assert lib.muse_status_string(code).decode() == name
    assert lib.muse_status_string(99).decode() == "MUSE_ERR_UNKNOWN"


def _d(B=1, H=2, N=1024, D=64, Dv=64, dtype=m.MUSE_BF16, scale=1.0):
    return m.MuseDims(B, H, N, D, Dv, dtype, scale)


def test_workspace_sizes(lib):
    d = _d()
    for entry in ("muse_kmeans", "muse_tilted_summaries", "muse_dipole_refine", "muse_forward"):
        assert lib.muse_workspace_size(entry.encode(), d, 32, 32, 0, 0, 0) > 0, entry
    assert lib.muse_workspace_size(b"muse_causal_blocks", d, 32, 32, 128, 0, 0) > 0
    assert lib.muse_workspace_size(b"muse_causal_blocks", d, 32, 32, 100, 0, 0) == 0
    assert lib.muse_workspace_size(b"nope", d, 32, 32, 0, 0, 0) == 0
    assert lib.muse_workspace_size(b"muse_forward", _d(D=32), 32, 32, 0, 0, 0) == 0
    assert lib.muse_workspace_size(b"muse_forward", d, 0, 32, 0, 0, 0) == 0
    assert lib.muse_workspace_size(b"muse_forward", d, 2048, 32, 0, 0, 0) == 0
    # forward_ex: the forward pass's buffers plus the partially specialised dipole's
    # covariances, B*H*(Cq+Ck)*D*Dv floats and 256 bytes, plus the summary form's tilted
    # value means, B*H*Cq*Ck*Dv floats and 256 bytes
    assert (lib.muse_workspace_size(b"muse_forward_ex", d, 32, 32, 0, 0, 0)
            == lib.muse_workspace_size(b"muse_forward", d, 32, 32, 0, 0, 0) + 2 * 64 * 64 * 64 * 4 + 256
            + 2 * 32 * 32 * 64 * 4 + 256)
    # forward = two clusterings + refinement buffers: grows with N
    assert (lib.muse_workspace_size(b"muse_forward", _d(N=2048), 32, 32, 0, 0, 0)
            > lib.muse_workspace_size(b"muse_forward", d, 32, 32, 0, 0, 0))


def test_causal_levels(lib):
    assert lib.muse_causal_levels(16384, 512) == 5
    assert lib.muse_causal_levels(512, 512) == 0
    assert lib.muse_causal_levels(1536, 512) == 2
    assert lib.muse_causal_levels(0, 512) == 0


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def test_argument_validation_enqueues_nothing(lib):
    st = ctypes.c_void_p(0)
    f = FAKE
    # wrong dtype / shape
    assert lib.muse_forward(f, f, f, _d(dtype=7), 8, 8, 2, f, f, 1 << 30, st) == 3
    assert lib.muse_forward(f, f, f, _d(D=96), 8, 8, 2, f, f, 1 << 30, st) == 2
    assert lib.muse_forward(f, f, f, _d(Dv=32), 8, 8, 2, f, f, 1 << 30, st) == 2
    assert lib.muse_forward(f, f, f, _d(N=0), 8, 8, 2, f, f, 1 << 30, st) == 2
    # null / misaligned pointers, cluster counts, iterations
    assert lib.muse_forward(None, f, f, _d(), 8, 8, 2, f, f, 1 << 30, st) == 1
    assert lib.muse_forward(MISALIGNED, f, f, _d(), 8, 8, 2, f, f, 1 << 30, st) == 1
    assert lib.muse_forward(f, f, f, _d(), 0, 8, 2, f, f, 1 << 30, st) == 1
    assert lib.muse_forward(f, f, f, _d(N=64), 65, 8, 2, f, f, 1 << 30, st) == 1
    assert lib.muse_forward(f, f, f, _d(), 8, 8, 0, f, f, 1 << 30, st) == 1
    assert lib.muse_forward(f, f, f, _d(scale=float("nan")), 8, 8, 2, f, f, 1 << 30, st) == 1
    # workspace too small or missing
    assert lib.muse_forward(f, f, f, _d(), 8, 8, 2, f, f, 16, st) == 4
    assert lib.muse_forward(f, f, f, _d(), 8, 8, 2, f, None, 1 << 30, st) == 4
    assert lib.muse_kmeans(f, _d(), 8, 2, f, f, f, f, f, 0, st) == 4
    assert lib.muse_kmeans(f, _d(), 8, 2, None, f, f, f, f, 1 << 30, st) == 1
    assert lib.muse_kmeans(f, _d(), 8, 1001, f, f, f, f, f, 1 << 30, st) == 1
    assert lib.muse_tilted_summaries(f, f, None, f, f, _d(), 8, 8, f, None, f, None, f, 1 << 30,
                                     st) == 1
    assert lib.muse_dipole_refine(f, f, f, None, f, f, f, f, f, f, None, None, None, _d(), 8, 8,
                                  f, f, 1 << 30, st) == 1
    # mu_v and cov: both materialised or neither
    assert lib.muse_dipole_refine(f, f, f, None, f, f, f, f, f, f, f, f, None, _d(), 8, 8,
                                  f, f, 1 << 30, st) == 1
    assert lib.muse_dipole_refine(f, f, f, None, f, f, f, f, f, f, f, None, f, _d(), 8, 8,
                                  f, f, 1 << 30, st) == 1
    assert lib.muse_dipole_refine(f, f, f, MISALIGNED, f, f, f, f, f, f, f, f, f, _d(), 8, 8,
                                  f, f, 1 << 30, st) == 1
    assert lib.muse_causal_blocks(f, f, f, _d(), 100, 8, 8, 2, f, None, None, f, 1 << 30, st) == 2
    assert lib.muse_causal_blocks(f, f, f, _d(N=1000), 128, 8, 8, 2, f, None, None, f, 1 << 30,
                                  st) == 2
    assert lib.muse_causal_blocks(f, f, f, _d(), 128, 8, 8, 2, f, None, None, f, 0, st) == 4
    # option flags: unknown bits and contradictory pairs are refused before the workspace
    # is looked at (both ablations, both refinement forms, an ablation with a form)
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 16, f, f, 1 << 30, st) == 1
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 3, f, f, 1 << 30, st) == 1
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 12, f, f, 1 << 30, st) == 1
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 5, f, f, 1 << 30, st) == 1
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 10, f, f, 1 << 30, st) == 1
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 4, f, f, 16, st) == 4
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 8, f, f, 16, st) == 4
    assert lib.muse_forward_ex(f, f, f, _d(), 8, 8, 2, 1, f, f, 16, st) == 4
    assert lib.muse_forward_ex(f, f, f, _d(D=96), 8, 8, 2, 1, f, f, 1 << 30, st) == 2


def test_refine_form_query(lib):
    """muse_refine_form reports the library's own choice between the pair and the summary
    form of the refinement (host only)."""
    f = lib.muse_refine_form
    d64k = _d(H=16, N=65536, D=128, Dv=128)
    assert f(d64k, 256, 256, 0) == 1                          # long context: summary form
    assert f(d64k, 256, 256, m.MUSE_FLAG_REFINE_PAIR) == 0
    assert f(d64k, 256, 300, 0) == 0                          # Ck > 256: pair form only
    assert f(_d(H=8, N=8192), 128, 128, 0) == 0               # D = 64: pair form
    assert f(_d(H=8, N=8192), 128, 128, m.MUSE_FLAG_REFINE_SUMMARY) == 0
    small = _d(N=2048, D=128, Dv=128)
    assert f(small, 32, 32, 0) == 0                           # short: the pair form is cheaper
    assert f(small, 32, 32, m.MUSE_FLAG_REFINE_SUMMARY) == 1
    assert f(_d(N=2048, D=128, Dv=128, dtype=m.MUSE_F32), 32, 32, m.MUSE_FLAG_REFINE_SUMMARY) == 0
    assert f(small, 32, 32, m.MUSE_FLAG_REFINE_SUMMARY | m.MUSE_FLAG_REFINE_PAIR) == -1
    assert f(small, 32, 32, m.MUSE_FLAG_MONOPOLE) == -1
    assert f(_d(D=96), 32, 32, 0) == -1
    assert f(small, 0, 32, 0) == -1


def test_binding_refuses_mismatched_tensors():
    """The binding checks what the C ABI cannot (buffer extents): Q, K, V shapes, dtypes and
    the output's shape, before anything reaches the library."""
    import torch
    Q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="K: shape"):
        m.muse_forward(Q, torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16), Q, 8, 8, 2)
    with pytest.raises(ValueError, match="K: dtype"):
        m.muse_forward(Q, Q.float(), Q, 8, 8, 2)
    with pytest.raises(ValueError, match="V: shape"):
        m.muse_causal_blocks(Q, Q, torch.zeros(1, 2, 255, 64, dtype=torch.bfloat16), 128, 8, 8, 2)
    with pytest.raises(ValueError, match="out: shape"):
        m.muse_forward_ex(Q, Q, Q, 8, 8, 2, out=torch.zeros(1, 2, 256, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="k_offsets: shape"):
        m.muse_tilted_summaries(torch.zeros(1, 2, 8, 64), Q, Q,
                                torch.zeros(1, 2, 256, dtype=torch.int32),
                                torch.zeros(1, 2, 8, dtype=torch.int32), 8)
    # consistent tensors on the host: refused for not being on the GPU
    with pytest.raises(ValueError, match="CUDA"):
        m.muse_forward(Q, Q, Q, 8, 8, 2)


def test_noalloc_kmeans_refuses_a_multi_launch_problem_beyond_its_scratch(lib):
    """float32 inputs take the multi-launch kernels, whose scratch (ranks of every row)
    for B*H*N = 4M rows exceeds the 16 MiB array: refused before any CUDA call.  (The
    one-launch bfloat16 path has no such limit; that acceptance needs real buffers and is
    a GPU test.)"""
    d = _d(B=8, H=8, N=65536, D=64, dtype=m.MUSE_F32)
    assert lib.muse_workspace_size(b"muse_kmeans", d, 64, 0, 0, 0, 0) > m.NOALLOC_SCRATCH_BYTES
    assert lib.muse_kmeans_noalloc(FAKE, d, 64, 2, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0)) == 4
    d = _d(B=1, H=1, N=4096, D=128, dtype=m.MUSE_F32)
    assert lib.muse_kmeans_noalloc(FAKE, d, 5000, 2, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0)) == 1


def test_test_hooks_refuse_unknown_bits(lib):
    """Unknown hook bits are refused before the device is touched."""
    assert lib.muse_set_test_hooks(2, 0) == 1
    assert lib.muse_set_test_hooks(0xFFFF, 5) == 1


def test_backward_validation_and_workspace(lib):
    st = ctypes.c_void_p(0)
    f = FAKE
    d = _d()
    need = lib.muse_workspace_size(b"muse_backward", d, 16, 16, 0, 0, 0)
    # the materialised C_ij and its gradient: 2 B*H*Cq*Ck*Dv*D floats at least
    assert need >= 2 * 2 * 16 * 16 * 64 * 64 * 4
    assert lib.muse_workspace_size(b"muse_backward", d, 16, 0, 0, 0, 0) == 0
    assert lib.muse_backward(f, f, f, f, f, f, f, f, _d(dtype=5), 16, 16, f, f, f, f, need, st) == 3
    assert lib.muse_backward(f, f, f, None, f, f, f, f, d, 16, 16, f, f, f, f, need, st) == 1
    assert lib.muse_backward(f, f, f, f, f, f, f, f, d, 16, 16, f, f, MISALIGNED, f, need, st) == 1
    assert lib.muse_backward(f, f, f, f, f, f, f, f, d, 0, 16, f, f, f, f, need, st) == 1
    assert lib.muse_backward(f, f, f, f, f, f, f, f, d, 16, 16, f, f, f, f, need - 1, st) == 4
