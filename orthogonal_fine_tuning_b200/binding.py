"""Thin Python binding over the C ABI (include/oft.h): argument marshalling only.

Tensors are torch tensors on a CUDA device (torch provides device memory and
streams); every step of the path runs in liboft.so's kernels.  There is no CPU
fallback: importing this module fails if the library is missing, and every call
raises OFTError when the library returns an error code.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import _lib

_L = _lib.load()

_FMT = {"int4": _lib.OFT_W_INT4, "fp8": _lib.OFT_W_FP8, "mxfp4": _lib.OFT_W_MXFP4}


class OFTError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"oft error {code}: {msg}")
        self.code = code


def _check(rc: int):
    if rc != _lib.OFT_OK:
        raise OFTError(rc, _L.oft_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected a bf16 tensor, got {t.dtype}")
    return t


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Weight:
    """A frozen low-precision weight W^T [d_out][d_in] (or an expert bank)."""
    fmt: str
    codes: torch.Tensor
    scales: torch.Tensor
    d_in: int
    d_out: int
    group: int
    n_experts: int = 0

    def c(self) -> _lib.CWeight:
        return _lib.CWeight(_FMT[self.fmt], _ptr(self.codes), _ptr(self.scales), self.d_in, self.d_out, self.group,
                            self.n_experts)


def _split(sizes: Sequence[int]) -> _lib.CSplit:
    s = _lib.CSplit()
    s.n = len(sizes)
    for i, v in enumerate(sizes):
        s.sizes[i] = int(v)
    return s


def version() -> str:
    return _L.oft_version().decode()


def library_path() -> str:
    return _lib.LIB_PATH


def oft_check_device(stream=None) -> None:
    _check(_L.oft_check_device(_stream(stream)))


def oft_build_rotation(Q: torch.Tensor, b: int, R: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Q bf16 [..., b(b-1)/2] -> R fp32 [..., b, b]."""
    nq = b * (b - 1) // 2
    assert Q.shape[-1] == nq
    nblocks = Q.numel() // nq
    if R is None:
        R = torch.empty(*Q.shape[:-1], b, b, dtype=torch.float32, device=Q.device)
    _check(_L.oft_build_rotation(_ptr(_bits(Q)), nblocks, b, _ptr(R), _stream(stream)))
    return R


def oft_linear_fwd_workspace(M: int, W: Weight, splits: Sequence[int], b: int) -> int:
    cw, cs = W.c(), _split(splits)
    return int(_L.oft_linear_fwd_workspace(M, ctypes.byref(cw), ctypes.byref(cs), b))


def oft_linear_fwd_noalloc(X: torch.Tensor, W: Weight, splits: Sequence[int], b: int, R: torch.Tensor,
                           Y: torch.Tensor, stream=None) -> torch.Tensor:
    """oft_linear_fwd without a workspace: scratch lives in the library's fixed
    device array (OFT_NOALLOC_SCRATCH_BYTES).  Y must be preallocated; nothing
    is allocated by this call."""
    cw, cs = W.c(), _split(splits)
    _check(_L.oft_linear_fwd_noalloc(_ptr(_bits(X)), X.shape[0], ctypes.byref(cw), ctypes.byref(cs), b, _ptr(R),
                                     _ptr(Y), _stream(stream)))
    return Y


def oft_linear_bwd_workspace(M: int, W: Weight, splits: Sequence[int], b: int) -> int:
    cw, cs = W.c(), _split(splits)
    return int(_L.oft_linear_bwd_workspace(M, ctypes.byref(cw), ctypes.byref(cs), b))


def _ws(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    return ws


def oft_linear_fwd(X: torch.Tensor, W: Weight, splits: Sequence[int], b: int, R: torch.Tensor,
                   Y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, W.d_out, dtype=torch.bfloat16, device=X.device)
    cw, cs = W.c(), _split(splits)
    nbytes = int(_L.oft_linear_fwd_workspace(M, ctypes.byref(cw), ctypes.byref(cs), b))
    ws = _ws(nbytes, X.device, workspace)
    _check(_L.oft_linear_fwd(_ptr(_bits(X)), M, ctypes.byref(cw), ctypes.byref(cs), b, _ptr(R), _ptr(Y), _ptr(ws),
                             ws.numel(), _stream(stream)))
    return Y


def oft_linear_fwd_weight_side_workspace(W: Weight) -> int:
    cw = W.c()
    return int(_L.oft_linear_fwd_weight_side_workspace(ctypes.byref(cw)))


def oft_linear_fwd_weight_side(X: torch.Tensor, W: Weight, splits: Sequence[int], b: int, R: torch.Tensor,
                               Y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                               stream=None) -> torch.Tensor:
    """The same product as oft_linear_fwd with the rotation applied to the weight:
    Y_p = X (R_p deq(W_p))."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, W.d_out, dtype=torch.bfloat16, device=X.device)
    cw, cs = W.c(), _split(splits)
    nbytes = int(_L.oft_linear_fwd_weight_side_workspace(ctypes.byref(cw)))
    ws = _ws(nbytes, X.device, workspace)
    _check(_L.oft_linear_fwd_weight_side(_ptr(_bits(X)), M, ctypes.byref(cw), ctypes.byref(cs), b, _ptr(R), _ptr(Y),
                                         _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def oft_linear_bwd(dY: torch.Tensor, X: torch.Tensor, W: Weight, splits: Sequence[int], b: int, R: torch.Tensor,
                   dX: Optional[torch.Tensor] = None, dQ: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    M = X.shape[0]
    P, nb = len(splits), W.d_in // b
    if dX is None:
        dX = torch.empty(M, W.d_in, dtype=torch.bfloat16, device=X.device)
    if dQ is None:
        dQ = torch.empty(P, nb, b * (b - 1) // 2, dtype=torch.float32, device=X.device)
    cw, cs = W.c(), _split(splits)
    nbytes = int(_L.oft_linear_bwd_workspace(M, ctypes.byref(cw), ctypes.byref(cs), b))
    ws = _ws(nbytes, X.device, workspace)
    _check(_L.oft_linear_bwd(_ptr(_bits(dY)), _ptr(_bits(X)), M, ctypes.byref(cw), ctypes.byref(cs), b, _ptr(R),
                             _ptr(dX), _ptr(dQ), _ptr(ws), ws.numel(), _stream(stream)))
    return dX, dQ


def moe_chunked_oft_workspace(T: int, E: int, top_k: int, chunk: int, W: Weight, b: int) -> int:
    cw = W.c()
    return int(_L.moe_chunked_oft_workspace(T, E, top_k, chunk, ctypes.byref(cw), b))


def moe_fused_oft_workspace(T: int, E: int, top_k: int, chunk: int, W: Weight, b: int) -> int:
    cw = W.c()
    return int(_L.moe_fused_oft_workspace(T, E, top_k, chunk, ctypes.byref(cw), b))


def _moe_fwd(fused: bool, X, logits, W, b, Q, top_k, chunk, workspace, out, stream) -> dict:
    T, E = logits.shape
    dev = X.device
    n_chunks = (E + chunk - 1) // chunk
    o = out if out is not None else dict(
        Y=torch.empty(T, W.d_out, dtype=torch.bfloat16, device=dev),
        topk_idx=torch.empty(T, top_k, dtype=torch.int32, device=dev),
        topk_w=torch.empty(T, top_k, dtype=torch.float32, device=dev),
        offsets=torch.empty(E + 1 + 3, dtype=torch.int32, device=dev)[: E + 1],
        bucket=torch.empty(T * top_k, dtype=torch.int32, device=dev),
        chunk_table=torch.empty(n_chunks, chunk, dtype=torch.int32, device=dev),
        n_active=torch.empty(4, dtype=torch.int32, device=dev)[:1],
    )
    cw = W.c()
    size_fn = _L.moe_fused_oft_workspace if fused else _L.moe_chunked_oft_workspace
    run_fn = _L.moe_fused_oft_fwd if fused else _L.moe_chunked_oft_fwd
    nbytes = int(size_fn(T, E, top_k, chunk, ctypes.byref(cw), b))
    ws = _ws(nbytes, dev, workspace)
    _check(run_fn(
        _ptr(_bits(X)), T, _ptr(logits), E, top_k, chunk, ctypes.byref(cw), b, _ptr(_bits(Q)), _ptr(o["Y"]),
        _ptr(o["topk_idx"]), _ptr(o["topk_w"]), _ptr(o["offsets"]), _ptr(o["bucket"]), _ptr(o["chunk_table"]),
        _ptr(o["n_active"]), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_chunked_oft_fwd(X: torch.Tensor, logits: torch.Tensor, W: Weight, b: int, Q: torch.Tensor, top_k: int,
                        chunk: int, workspace: Optional[torch.Tensor] = None, out: Optional[dict] = None,
                        stream=None) -> dict:
    """Chunked MoE forward: each chunk of active experts is dequantised to a bf16
    buffer, then one grouped GEMM."""
    return _moe_fwd(False, X, logits, W, b, Q, top_k, chunk, workspace, out, stream)


def moe_fused_oft_fwd(X: torch.Tensor, logits: torch.Tensor, W: Weight, b: int, Q: torch.Tensor, top_k: int,
                      chunk: int, workspace: Optional[torch.Tensor] = None, out: Optional[dict] = None,
                      stream=None) -> dict:
    """The same MoE forward with the dequant fused into the grouped GEMM (no chunk buffer)."""
    return _moe_fwd(True, X, logits, W, b, Q, top_k, chunk, workspace, out, stream)


def moe_chunked_oft_bwd_workspace(T: int, E: int, top_k: int, chunk: int, W: Weight, b: int) -> int:
    cw = W.c()
    return int(_L.moe_chunked_oft_bwd_workspace(T, E, top_k, chunk, ctypes.byref(cw), b))


def moe_chunked_oft_bwd(dY: torch.Tensor, X: torch.Tensor, logits: torch.Tensor, W: Weight, b: int, Q: torch.Tensor,
                        top_k: int, chunk: int, want_dlogits: bool = True, workspace: Optional[torch.Tensor] = None,
                        out: Optional[dict] = None, stream=None) -> dict:
    """Adapter backward of the chunked MoE layer: dX bf16 [T][K], dQ fp32
    [E][2][K/b][b(b-1)/2] and (optionally) dlogits fp32 [T][E]."""
    T, E = logits.shape
    dev = X.device
    nb = W.d_in // b
    o = out if out is not None else dict(
        dX=torch.empty(T, W.d_in, dtype=torch.bfloat16, device=dev),
        dQ=torch.empty(E, 2, nb, b * (b - 1) // 2, dtype=torch.float32, device=dev),
        dlogits=torch.empty(T, E, dtype=torch.float32, device=dev) if want_dlogits else None,
    )
    cw = W.c()
    nbytes = int(_L.moe_chunked_oft_bwd_workspace(T, E, top_k, chunk, ctypes.byref(cw), b))
    ws = _ws(nbytes, dev, workspace)
    dl = o.get("dlogits")
    _check(_L.moe_chunked_oft_bwd(
        _ptr(_bits(dY)), _ptr(_bits(X)), T, _ptr(logits), E, top_k, chunk, ctypes.byref(cw), b, _ptr(_bits(Q)),
        _ptr(o["dX"]), _ptr(o["dQ"]), _ptr(dl) if dl is not None else None, _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_chunked_oft_layer_workspace(T: int, E: int, top_k: int, chunk: int, W: Weight, W_down: Weight, b: int) -> int:
    cw, cd = W.c(), W_down.c()
    return int(_L.moe_chunked_oft_layer_workspace(T, E, top_k, chunk, ctypes.byref(cw), ctypes.byref(cd), b))


def moe_chunked_oft_layer_fwd(X: torch.Tensor, logits: torch.Tensor, W: Weight, W_down: Weight, b: int,
                              Q: torch.Tensor, Q_down: torch.Tensor, top_k: int, chunk: int,
                              workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                              stream=None) -> torch.Tensor:
    """Full expert layer: Y bf16 [T][K] = sum_k w_tk ((silu(g) u) R_e,down) W_e,down, with
    [g | u] the chunked gate/up outputs of expert e."""
    T, E = logits.shape
    Y = out if out is not None else torch.empty(T, W.d_in, dtype=torch.bfloat16, device=X.device)
    cw, cd = W.c(), W_down.c()
    nbytes = int(_L.moe_chunked_oft_layer_workspace(T, E, top_k, chunk, ctypes.byref(cw), ctypes.byref(cd), b))
    ws = _ws(nbytes, X.device, workspace)
    _check(_L.moe_chunked_oft_layer_fwd(
        _ptr(_bits(X)), T, _ptr(logits), E, top_k, chunk, ctypes.byref(cw), ctypes.byref(cd), b, _ptr(_bits(Q)),
        _ptr(_bits(Q_down)), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def oft_dequant_weight(W: Weight, transpose: bool = False, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    if out is None:
        shape = (W.d_in, W.d_out) if transpose else (W.d_out, W.d_in)
        out = torch.empty(*shape, dtype=torch.bfloat16, device=W.codes.device)
    cw = W.c()
    _check(_L.oft_dequant_weight(ctypes.byref(cw), _ptr(out), int(bool(transpose)), _stream(stream)))
    return out


def oft_moe_chunk_dequant(W: Weight, chunk_table: torch.Tensor, chunk_idx: int, chunk: int,
                          transpose: bool = False, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One chunk of the MoE transient dequant: bf16 [chunk][N][K], or with transpose
    [chunk][2][K][N/2].  Slots whose table entry is -1 are left as they were."""
    N, K = W.d_out, W.d_in
    if out is None:
        shape = (chunk, 2, K, N // 2) if transpose else (chunk, N, K)
        out = torch.zeros(*shape, dtype=torch.bfloat16, device=W.codes.device)
    cw = W.c()
    _check(_L.oft_moe_chunk_dequant(ctypes.byref(cw), _ptr(chunk_table), int(chunk_idx), int(chunk),
                                    int(bool(transpose)), _ptr(out), _stream(stream)))
    return out


def oft_rotate(X: torch.Tensor, R: torch.Tensor, b: int, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """X bf16 [M][K], R fp32 [P][K/b][b][b] -> X R_p, bf16 [P][M][K]."""
    M, K = X.shape
    P = R.shape[0]
    if out is None:
        out = torch.empty(P, M, K, dtype=torch.bfloat16, device=X.device)
    _check(_L.oft_rotate(_ptr(_bits(X)), M, K, P, b, _ptr(R), _ptr(out), _stream(stream)))
    return out


def oft_cayley_backward(R: torch.Tensor, G: torch.Tensor, b: int, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    nblocks = R.numel() // (b * b)
    if out is None:
        out = torch.empty(*R.shape[:-2], b * (b - 1) // 2, dtype=torch.float32, device=R.device)
    _check(_L.oft_cayley_backward(_ptr(R), _ptr(G), nblocks, b, _ptr(out), _stream(stream)))
    return out


def oft_set_gemm_mode(mode: int) -> None:
    """GEMM inside the linear calls: 0 by size (default), 1 the one-CTA fused-dequant
    kernel, 2 the 2-SM pair fused-dequant kernel, 3 the bf16 weight copy and the plain
    GEMM on 2-SM pairs, 4 the same on one CTA per tile (same product).  Mode 0 runs
    forwards of up to 128 tokens on the small-M split-K kernel."""
    _check(_L.oft_set_gemm_mode(int(mode)))


def oft_debug_bounded_wait(timeout_us: int, stream=None) -> None:
    _check(_L.oft_debug_bounded_wait(int(timeout_us), _stream(stream)))


class profile:
    """Context manager: CUDA event pairs around every library launch, per kernel class.

    After the block, .ms[kind] is the summed device time and .launches[kind] the
    number of launches, for kind in gemm/rotate/dequant/cayley/grad/route."""

    def __init__(self, max_launches: int = 65536):
        self.max_launches = max_launches
        self.ms, self.launches, self.dropped = {}, {}, 0

    def __enter__(self):
        _check(_L.oft_profile_begin(self.max_launches))
        return self

    def __exit__(self, *exc):
        n = len(_lib.KERNEL_CLASSES)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int * n)()
        dropped = ctypes.c_int(0)
        _check(_L.oft_profile_end(ms, cnt, n, ctypes.byref(dropped)))
        self.ms = {k: float(ms[i]) for i, k in enumerate(_lib.KERNEL_CLASSES)}
        self.launches = {k: int(cnt[i]) for i, k in enumerate(_lib.KERNEL_CLASSES)}
        self.dropped = int(dropped.value)
        return False
