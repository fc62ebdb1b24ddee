"""Python binding of libmuse.so (ctypes).  Argument marshalling only.

Every function here has the name of the C entry point it calls (include/muse.h)
and does nothing but check shapes, allocate the caller-owned outputs and
workspace with torch, and pass device pointers plus the current CUDA stream.
All arithmetic runs in the library's CUDA kernels; if the library is missing,
the import of this module fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmuse.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "muse.h")

MUSE_F32, MUSE_BF16 = 0, 1
NOALLOC_SCRATCH_BYTES = 16 << 20   # MUSE_NOALLOC_SCRATCH_BYTES of include/muse.h
STATUS = {0: "MUSE_OK", 1: "MUSE_ERR_INVALID_ARG", 2: "MUSE_ERR_SHAPE", 3: "MUSE_ERR_DTYPE",
          4: "MUSE_ERR_WORKSPACE", 5: "MUSE_ERR_CUDA", 6: "MUSE_ERR_TIMEOUT", 7: "MUSE_ERR_DEVICE"}


class MuseError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class MuseDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("D", ctypes.c_int), ("Dv", ctypes.c_int), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float)]


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "muse_kmeans": [_vp, MuseDims, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "muse_kmeans_noalloc": [_vp, MuseDims, _i, _i, _vp, _vp, _vp, _vp, _vp],
    "muse_tilted_summaries": [_vp, _vp, _vp, _vp, _vp, MuseDims, _i, _i, _vp, _vp, _vp, _vp,
                              _vp, _sz, _vp],
    "muse_dipole_refine": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           MuseDims, _i, _i, _vp, _vp, _sz, _vp],
    "muse_forward": [_vp, _vp, _vp, MuseDims, _i, _i, _i, _vp, _vp, _sz, _vp],
    "muse_forward_ex": [_vp, _vp, _vp, MuseDims, _i, _i, _i, ctypes.c_uint, _vp, _vp, _sz, _vp],
    "muse_causal_levels": [_i, _i],
    "muse_causal_blocks": [_vp, _vp, _vp, MuseDims, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz,
                           _vp],
    "muse_retrieve_exact": [_vp, _vp, _vp, MuseDims, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp,
                            _vp, _sz, _vp],
    "muse_workspace_size": [ctypes.c_char_p, MuseDims, _i, _i, _i, _i, _i],
    "muse_status_string": [_i],
    "muse_last_error_detail": [],
    "muse_last_device_status": [_vp],
    "muse_set_test_hooks": [ctypes.c_uint, ctypes.c_uint64],
    "muse_refine_form": [MuseDims, _i, _i, ctypes.c_uint],
    "muse_backward": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, MuseDims, _i, _i, _vp, _vp, _vp,
                      _vp, _sz, _vp],
}
_RES = {"muse_workspace_size": _sz, "muse_status_string": ctypes.c_char_p,
        "muse_causal_levels": _i, "muse_last_error_detail": ctypes.c_char_p}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m clustered_softmax_attention_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _RES.get(name, _i)
    return lib


_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load_library()
    return _LIB


def declared_entry_points(header: str = HEADER):
    """Names of the functions declared in include/muse.h."""
    text = open(header).read()
    return sorted(set(re.findall(r"^\s*(?:muse_status|size_t|int|const char \*)\s*\**(muse_\w+)\s*\(",
                                 text, flags=re.M)))


def _check(code: int, where: str):
    if code != 0:
        detail = lib().muse_last_error_detail().decode() if code == 5 else ""
        raise MuseError(code, where + (f" ({detail})" if detail else ""))


def _p(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MUSE_F32
    if t.dtype == torch.bfloat16:
        return MUSE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def dims(X: torch.Tensor, V: Optional[torch.Tensor] = None, scale: float = 1.0) -> MuseDims:
    B, H, N, D = X.shape
    Dv = V.shape[-1] if V is not None else D
    return MuseDims(B, H, N, D, Dv, _dtype_code(X), float(scale))


def _expect(t, shape, dtype, name):
    """Shape and dtype of an argument the library reads or writes with sizes taken from
    other arguments (a mismatch would make it read or write past the tensor)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _qkv(Q, K, V, out=None):
    """Q, K [B,H,N,D] and V [B,H,N,Dv] of one dtype on one device; out [B,H,N,Dv]."""
    if Q.dim() != 4:
        raise ValueError(f"Q: expected [B,H,N,D], got shape {tuple(Q.shape)}")
    B, H, N, D = Q.shape
    _expect(K, (B, H, N, D), Q.dtype, "K")
    if V.dim() != 4 or tuple(V.shape[:3]) != (B, H, N):
        raise ValueError(f"V: shape {tuple(V.shape)}, expected [{B},{H},{N},Dv]")
    _expect(V, V.shape, Q.dtype, "V")
    if not (Q.device == K.device == V.device):
        raise ValueError("Q, K, V must be on one device")
    _expect(out, (B, H, N, V.shape[3]), Q.dtype, "out")


def _contig(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def muse_workspace_size(entry: str, d: MuseDims, Cq: int, Ck: int = 0, block: int = 0,
                        k1: int = 0, k2: int = 0) -> int:
    return int(lib().muse_workspace_size(entry.encode(), d, Cq, Ck, block, k1, k2))


def workspace(entry: str, d: MuseDims, Cq: int, Ck: int = 0, block: int = 0, k1: int = 0,
              k2: int = 0, device="cuda") -> torch.Tensor:
    n = muse_workspace_size(entry, d, Cq, Ck, block, k1, k2)
    if n == 0:
        raise MuseError(2, f"muse_workspace_size({entry})")
    return torch.empty(n, dtype=torch.uint8, device=device)


def muse_status_string(code: int) -> str:
    return lib().muse_status_string(code).decode()


def muse_last_device_status() -> int:
    return int(lib().muse_last_device_status(_stream()))


MUSE_TEST_WITHHOLD_VALUES = 1


def muse_set_test_hooks(hooks: int = 0, wait_limit_ns: int = 0) -> None:
    """Failure-path testing aid: make the refinement kernel's bounded waits run out
    (see include/muse.h).  muse_set_test_hooks() restores normal operation."""
    _check(lib().muse_set_test_hooks(hooks, wait_limit_ns), "muse_set_test_hooks")


def muse_causal_levels(N: int, block: int) -> int:
    return int(lib().muse_causal_levels(N, block))


def muse_kmeans(X: torch.Tensor, C: int, iters: int, ws: Optional[torch.Tensor] = None):
    """K-means of every (b,h) row set of X [B,H,N,D]: (labels, centroids, perm, offsets)."""
    _contig(X)
    d = dims(X)
    B, H, N, D = X.shape
    dev = X.device
    labels = torch.empty(B, H, N, dtype=torch.int32, device=dev)
    cen = torch.empty(B, H, C, D, dtype=torch.float32, device=dev)
    perm = torch.empty(B, H, N, dtype=torch.int32, device=dev)
    offs = torch.empty(B, H, C + 1, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace("muse_kmeans", d, C)
    _check(lib().muse_kmeans(_p(X), d, C, iters, _p(labels), _p(cen), _p(perm), _p(offs), _p(ws),
                             ws.numel(), _stream()), "muse_kmeans")
    return labels, cen, perm, offs


def muse_tilted_summaries(q_centroids, K, V, k_perm, k_offsets, Ck: int, scale: float = 1.0,
                          want_mu_k: bool = True, want_mu_v: bool = True, want_cov: bool = False):
    """Stage 1 summaries: dict with logZ and the requested mu_k / mu_v / cov."""
    _qkv(K, K, V)
    B, H, N, D = K.shape
    _expect(q_centroids, (B, H, q_centroids.shape[2], D), torch.float32, "q_centroids")
    _expect(k_perm, (B, H, N), torch.int32, "k_perm")
    _expect(k_offsets, (B, H, Ck + 1), torch.int32, "k_offsets")
    _contig(q_centroids, K, V, k_perm, k_offsets)
    B, H, Cq, D = q_centroids.shape
    d = dims(K, V, scale)
    dev = K.device
    Dv = d.Dv
    out = {"logZ": torch.empty(B, H, Cq, Ck, dtype=torch.float32, device=dev)}
    if want_mu_k:
        out["mu_k"] = torch.empty(B, H, Cq, Ck, D, dtype=torch.float32, device=dev)
    if want_mu_v:
        out["mu_v"] = torch.empty(B, H, Cq, Ck, Dv, dtype=torch.float32, device=dev)
    if want_cov:
        out["cov"] = torch.empty(B, H, Cq, Ck, Dv, D, dtype=torch.float32, device=dev)
    ws = workspace("muse_tilted_summaries", d, Cq, Ck)
    _check(lib().muse_tilted_summaries(
        _p(q_centroids), _p(K), _p(V), _p(k_perm), _p(k_offsets), d, Cq, Ck, _p(out["logZ"]),
        _p(out.get("mu_k")), _p(out.get("mu_v")), _p(out.get("cov")), _p(ws), ws.numel(),
        _stream()), "muse_tilted_summaries")
    return out


def muse_dipole_refine(Q, K, V, q_centroids, q_perm, q_offsets, k_perm, k_offsets, logZ, mu_k,
                       scale: float = 1.0, mu_v=None, cov=None, q_labels=None):
    """Stage 2 refinement: O [B,H,N,Dv] in Q's dtype.  With mu_v and cov (materialised
    summaries) the library evaluates the refinement from them as given."""
    _qkv(Q, K, V)
    B, H, N, D = Q.shape
    Cq, Ck = q_centroids.shape[2], logZ.shape[3]
    Dv = V.shape[3]
    _expect(q_centroids, (B, H, Cq, D), torch.float32, "q_centroids")
    _expect(q_perm, (B, H, N), torch.int32, "q_perm")
    _expect(q_offsets, (B, H, Cq + 1), torch.int32, "q_offsets")
    _expect(k_perm, (B, H, N), torch.int32, "k_perm")
    _expect(k_offsets, (B, H, Ck + 1), torch.int32, "k_offsets")
    _expect(logZ, (B, H, Cq, Ck), torch.float32, "logZ")
    _expect(mu_k, (B, H, Cq, Ck, D), torch.float32, "mu_k")
    _expect(mu_v, (B, H, Cq, Ck, Dv), torch.float32, "mu_v")
    _expect(cov, (B, H, Cq, Ck, Dv, D), torch.float32, "cov")
    _expect(q_labels, (B, H, N), torch.int32, "q_labels")
    _contig(Q, K, V, q_centroids, q_perm, q_offsets, k_perm, k_offsets, logZ, mu_k, mu_v, cov,
            q_labels)
    d = dims(Q, V, scale)
    O = torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], d.Dv, dtype=Q.dtype, device=Q.device)
    ws = workspace("muse_dipole_refine", d, Cq, Ck)
    _check(lib().muse_dipole_refine(
        _p(Q), _p(K), _p(V), _p(q_labels), _p(q_centroids), _p(q_perm), _p(q_offsets),
        _p(k_perm), _p(k_offsets), _p(logZ), _p(mu_k), _p(mu_v), _p(cov), d, Cq, Ck, _p(O),
        _p(ws), ws.numel(), _stream()), "muse_dipole_refine")
    return O


def muse_forward(Q, K, V, Cq: int, Ck: int, iters: int, scale: float = 1.0,
                 out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """The whole acausal forward pass."""
    _qkv(Q, K, V, out)
    _contig(Q, K, V, out, ws)
    d = dims(Q, V, scale)
    if out is None:
        out = torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], d.Dv, dtype=Q.dtype, device=Q.device)
    if ws is None:
        ws = workspace("muse_forward", d, Cq, Ck)
    _check(lib().muse_forward(_p(Q), _p(K), _p(V), d, Cq, Ck, iters, _p(out), _p(ws), ws.numel(),
                              _stream()), "muse_forward")
    return out


MUSE_FLAG_MONOPOLE = 1
MUSE_FLAG_PARTIAL_DIPOLE = 2
MUSE_FLAG_REFINE_SUMMARY = 4
MUSE_FLAG_REFINE_PAIR = 8


def muse_forward_ex(Q, K, V, Cq: int, Ck: int, iters: int, scale: float = 1.0, flags: int = 0,
                    out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """muse_forward with option flags (MUSE_FLAG_MONOPOLE: the monopole-only ablation;
    MUSE_FLAG_PARTIAL_DIPOLE: the partially specialised dipole; MUSE_FLAG_REFINE_SUMMARY /
    MUSE_FLAG_REFINE_PAIR: the form of the full method's refinement)."""
    _qkv(Q, K, V, out)
    _contig(Q, K, V, out, ws)
    d = dims(Q, V, scale)
    if out is None:
        out = torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], d.Dv, dtype=Q.dtype, device=Q.device)
    if ws is None:
        ws = workspace("muse_forward_ex", d, Cq, Ck)
    _check(lib().muse_forward_ex(_p(Q), _p(K), _p(V), d, Cq, Ck, iters, flags, _p(out), _p(ws),
                                 ws.numel(), _stream()), "muse_forward_ex")
    return out


def muse_causal_blocks(Q, K, V, block: int, Cq: int, Ck: int, iters: int, scale: float = 1.0,
                       return_labels: bool = False, out: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None):
    """Causal MuSe (hierarchical block decomposition).  Labels are [B,H,L,N] (-1 = none)."""
    _qkv(Q, K, V, out)
    _contig(Q, K, V, out, ws)
    d = dims(Q, V, scale)
    B, H, N, _ = Q.shape
    if out is None:
        out = torch.empty(B, H, N, d.Dv, dtype=Q.dtype, device=Q.device)
    L = muse_causal_levels(N, block)
    ql = kl = None
    if return_labels and L > 0:
        ql = torch.empty(B, H, L, N, dtype=torch.int32, device=Q.device)
        kl = torch.empty(B, H, L, N, dtype=torch.int32, device=Q.device)
    if ws is None:
        n = muse_workspace_size("muse_causal_blocks", d, Cq, Ck, block)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=Q.device)
    _check(lib().muse_causal_blocks(_p(Q), _p(K), _p(V), d, block, Cq, Ck, iters, _p(out), _p(ql),
                                    _p(kl), _p(ws), ws.numel(), _stream()), "muse_causal_blocks")
    if return_labels:
        return out, ql, kl
    return out


def muse_retrieve_exact(Q, K, V, block: int, Cq: int, Ck: int, iters: int, k1: int, k2: int,
                        scale: float = 1.0, return_all: bool = False,
                        out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """Causal MuSe with top-k1 cluster / top-k2 block retrieval."""
    _qkv(Q, K, V, out)
    _contig(Q, K, V, out, ws)
    d = dims(Q, V, scale)
    B, H, N, _ = Q.shape
    if out is None:
        out = torch.empty(B, H, N, d.Dv, dtype=Q.dtype, device=Q.device)
    ql = kl = sel = None
    if return_all:
        ql = torch.empty(B, H, N, dtype=torch.int32, device=Q.device)
        kl = torch.empty(B, H, N, dtype=torch.int32, device=Q.device)
        sel = torch.empty(B, H, Cq, N // block, max(1, k1 * k2), 2, dtype=torch.int32,
                          device=Q.device)
    if ws is None:
        ws = workspace("muse_retrieve_exact", d, Cq, Ck, block, k1, k2)
    _check(lib().muse_retrieve_exact(_p(Q), _p(K), _p(V), d, block, Cq, Ck, iters, k1, k2, _p(ql),
                                     _p(kl), _p(sel), _p(out), _p(ws), ws.numel(), _stream()),
           "muse_retrieve_exact")
    if return_all:
        return out, ql, kl, sel
    return out


def muse_backward(Q, K, V, dO, q_perm, q_offsets, k_perm, k_offsets, scale: float = 1.0,
                  ws: Optional[torch.Tensor] = None):
    """Gradients (dQ, dK, dV) of sum(O * dO) for the acausal forward pass, clusterings fixed."""
    _qkv(Q, K, V, dO)
    B, H, N, D = Q.shape
    Cq, Ck = q_offsets.shape[2] - 1, k_offsets.shape[2] - 1
    for t, shape, name in ((q_perm, (B, H, N), "q_perm"), (q_offsets, (B, H, Cq + 1), "q_offsets"),
                           (k_perm, (B, H, N), "k_perm"), (k_offsets, (B, H, Ck + 1), "k_offsets")):
        _expect(t, shape, torch.int32, name)
    _contig(Q, K, V, dO, q_perm, q_offsets, k_perm, k_offsets, ws)
    d = dims(Q, V, scale)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    if ws is None:
        ws = workspace("muse_backward", d, Cq, Ck)
    _check(lib().muse_backward(_p(Q), _p(K), _p(V), _p(dO), _p(q_perm), _p(q_offsets), _p(k_perm),
                               _p(k_offsets), d, Cq, Ck, _p(dQ), _p(dK), _p(dV), _p(ws), ws.numel(),
                               _stream()), "muse_backward")
    return dQ, dK, dV
