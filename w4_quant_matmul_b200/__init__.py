"""W4-G256 quantized matmul for B200 (sm_100a): Python binding.

Every function here marshals torch CUDA tensors into the C ABI of libw4.so
(``include/w4.h``) and raises ``W4Error`` on a non-OK status.  All arithmetic
runs in the library's CUDA kernels; torch only provides device memory and the
current stream.  There is no CPU path: without the built library, calls raise
``LibraryMissing``.

Entry points (same names as the C ABI):
    w4_pack(w)                              -> codes, d, m
    w4_pack_g32(w)                          -> codes, d, m   (groups of 32)
    w4_pack_codes(q)                        -> codes
    w4_unpack(codes, K)                     -> q
    w4_gemv(codes, d, m, x, out_dtype)      -> y
    w4_gemv_g32(codes, d, m, x, out_dtype)  -> y   (group-32 weights)
    w4a8_gemv(codes, d, m, qa, dx, bsum, out_dtype) -> y   (int8 activations, M <= 8)
    w4a8_gemv_bf16(codes, d, m, x, out_dtype) -> y   (x quantised inside, M <= 8)
    q8_quantize_act(x)                      -> qa, dx, bsum
    w4a8_mmq(codes, d, m, qa, dx, bsum, out_dtype) -> y
    w4a8_mmq_static(codes, d, m, qa, dx, bsum, out_dtype) -> y   (no workspace)
    w4a8_mmq_blockdots(codes, d, m, qa, dx, bsum, out_dtype) -> y, P   (test: int32 block products)
    w4a8_gemv_blockdots(codes, d, m, qa, dx, bsum, out_dtype) -> y, P  (test: int32 block products)
    w4a8_mmq_workspace_size(M, N, K)
    w4_check_device_error()
"""
from __future__ import annotations

from ._lib import (LibraryMissing, W4_OK, W4_OUT_BF16, W4_OUT_F32, load, status_string)

__all__ = [
    "W4Error", "LibraryMissing", "w4_pack", "w4_pack_g32", "w4_pack_codes", "w4_unpack",
    "w4_gemv", "w4_gemv_g32", "w4a8_gemv",
    "w4a8_gemv_bf16",
    "q8_quantize_act", "w4a8_mmq", "w4a8_mmq_static", "w4a8_mmq_workspace_size",
    "w4a8_mmq_blockdots", "w4a8_gemv_blockdots",
    "w4_check_device_error",
    "w4_abi_version", "lib",
]

GROUP = 256
GROUP32 = 32
BLOCK = 32


class W4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = int(code)
        msg = status_string(code)
        if code == 6:  # W4_ERR_CUDA
            msg += f" (cudaError {load().w4_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


def lib():
    """The loaded ctypes library (raw C ABI)."""
    return load()


def _torch():
    import torch
    return torch


def _check(code: int, what: str):
    if code != W4_OK:
        raise W4Error(code, what)


def _stream(stream=None) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> int:
    return t.data_ptr()


def _div(n: int, unit: int):
    """n / unit when exact, else None (any extent: the library then rejects n)."""
    return n // unit if n % unit == 0 else None


def _need(t, dtype, name: str, shape):
    """Check a tensor argument before its pointer crosses the C ABI, which
    sees only pointers and sizes: type, dtype, exact shape (None = any extent)
    and contiguity.  A plane with the wrong extent would otherwise be read or
    written out of bounds.  Placement is checked by _on_device, once every
    argument's shape has been."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(e is not None and e != s for e, s in zip(shape, t.shape)):
        want = "[" + ", ".join("*" if e is None else str(e) for e in shape) + "]"
        raise ValueError(f"{name} must have shape {want}, got {list(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(**tensors):
    """Every tensor must be a CUDA tensor on the current device, where the
    library launches its kernels."""
    torch = _torch()
    for name, t in tensors.items():
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    current = torch.cuda.current_device()
    for name, t in tensors.items():
        if t.device.index != current:
            raise ValueError(f"{name} is on {t.device}, not the current device cuda:{current}")


def _as_u16(t):
    torch = _torch()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16)
    return t


def w4_abi_version() -> int:
    return int(load().w4_abi_version())


def w4_check_device_error() -> None:
    """Synchronise and raise if a kernel reported a timed-out wait."""
    _check(load().w4_check_device_error(), "w4_check_device_error")


def _pack(fn: str, group: int, w, codes, d, m, stream):
    torch = _torch()
    _need(w, torch.float32, "w", (None, None))
    N, K = w.shape
    if codes is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    _need(codes, torch.uint8, "codes", (N, _div(K, 2)))
    if d is None:
        d = torch.empty((N, K // group), dtype=torch.float16, device=w.device)
    _need(d, torch.float16, "d", (N, _div(K, group)))
    if m is None:
        m = torch.empty((N, K // group), dtype=torch.float16, device=w.device)
    _need(m, torch.float16, "m", (N, _div(K, group)))
    _on_device(w=w, codes=codes, d=d, m=m)
    _check(getattr(load(), fn)(_ptr(w), N, K, _ptr(codes), _ptr(d), _ptr(m), _stream(stream)),
           fn)
    return codes, d, m


def w4_pack(w, codes=None, d=None, m=None, stream=None):
    """Quantise fp32 W[N,K] (K % 256 == 0) to W4-G256 planes.
    Returns (codes uint8[N,K/2], d fp16[N,K/256], m fp16[N,K/256])."""
    return _pack("w4_pack", GROUP, w, codes, d, m, stream)


def w4_pack_g32(w, codes=None, d=None, m=None, stream=None):
    """Quantise fp32 W[N,K] (K % 32 == 0) to group-32 planes (one d, m per
    32 weights).  Returns (codes uint8[N,K/2], d fp16[N,K/32], m fp16[N,K/32])."""
    return _pack("w4_pack_g32", GROUP32, w, codes, d, m, stream)


def w4_pack_codes(q, codes=None, stream=None):
    """One code per byte q uint8[N,K] -> packed codes uint8[N,K/2]."""
    torch = _torch()
    _need(q, torch.uint8, "q", (None, None))
    N, K = q.shape
    if codes is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=q.device)
    _need(codes, torch.uint8, "codes", (N, _div(K, 2)))
    _on_device(q=q, codes=codes)
    _check(load().w4_pack_codes(_ptr(q), N, K, _ptr(codes), _stream(stream)), "w4_pack_codes")
    return codes


def w4_unpack(codes, K: int, q=None, stream=None):
    """Packed codes uint8[N,K/2] -> one code per byte uint8[N,K]."""
    torch = _torch()
    _need(codes, torch.uint8, "codes", (None, _div(K, 2)))
    if K % 2:
        raise ValueError("codes must have K/2 columns")
    N = codes.shape[0]
    if q is None:
        q = torch.empty((N, K), dtype=torch.uint8, device=codes.device)
    _need(q, torch.uint8, "q", (N, K))
    _on_device(codes=codes, q=q)
    _check(load().w4_unpack(_ptr(codes), N, K, _ptr(q), _stream(stream)), "w4_unpack")
    return q


def _out_code(out_dtype, y=None) -> int:
    """Output code from out_dtype; with out_dtype None, y's dtype, else bf16."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = y.dtype if isinstance(y, torch.Tensor) else torch.bfloat16
    if out_dtype in (torch.float32, "f32", "fp32", W4_OUT_F32):
        return W4_OUT_F32
    if out_dtype in (torch.bfloat16, "bf16", W4_OUT_BF16):
        return W4_OUT_BF16
    raise ValueError(f"unsupported out_dtype {out_dtype}")


def _output(y, M: int, N: int, oc: int, like):
    """The caller's y checked against [M,N] and the output type, or a new one."""
    torch = _torch()
    dtype = torch.float32 if oc == W4_OUT_F32 else torch.bfloat16
    if y is None:
        y = torch.empty((M, N), dtype=dtype, device=like.device)
    _need(y, dtype, "y", (M, N))
    return y


def _weights(codes, d, m, K: int, group: int = GROUP) -> int:
    """Check the weight planes (d, m per `group` weights) for reduction
    length K; returns N."""
    torch = _torch()
    _need(codes, torch.uint8, "codes", (None, _div(K, 2)))
    N = codes.shape[0]
    _need(d, torch.float16, "d", (N, _div(K, group)))
    _need(m, torch.float16, "m", (N, _div(K, group)))
    return N


def _int8_acts(qa, dx, bsum):
    """Check int8 activation blocks (the output of q8_quantize_act); returns M, K."""
    torch = _torch()
    _need(qa, torch.int8, "qa", (None, None))
    M, K = qa.shape
    _need(dx, torch.float32, "dx", (M, _div(K, BLOCK)))
    _need(bsum, torch.int32, "bsum", (M, _div(K, BLOCK)))
    return M, K


def w4_gemv(codes, d, m, x, out_dtype=None, y=None, stream=None):
    """y[M,N] = x[M,K] @ dequant(W)^T for 1 <= M <= 8; x is bf16.
    out_dtype: torch.bfloat16 (default) or torch.float32; with a caller y and
    no out_dtype, y's dtype."""
    torch = _torch()
    _need(x, torch.bfloat16, "x", (None, None))
    M, K = x.shape
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, x)
    _on_device(codes=codes, d=d, m=m, x=x, y=y)
    _check(load().w4_gemv(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(x), M, _ptr(y), oc,
                          _stream(stream)), "w4_gemv")
    return y


def w4_gemv_g32(codes, d, m, x, out_dtype=None, y=None, stream=None):
    """w4_gemv for group-32 weights (w4_pack_g32 planes: d, m fp16[N,K/32]);
    y[M,N] = x[M,K] @ dequant(W)^T for 1 <= M <= 8, K % 32 == 0."""
    torch = _torch()
    _need(x, torch.bfloat16, "x", (None, None))
    M, K = x.shape
    N = _weights(codes, d, m, K, GROUP32)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, x)
    _on_device(codes=codes, d=d, m=m, x=x, y=y)
    _check(load().w4_gemv_g32(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(x), M, _ptr(y), oc,
                              _stream(stream)), "w4_gemv_g32")
    return y


def w4a8_gemv(codes, d, m, qa, dx, bsum, out_dtype=None, y=None, stream=None):
    """y[M,N] for 1 <= M <= 8 from W4-G256 weights and int8 activation blocks
    (the output of q8_quantize_act): exact int32 block dot products, scales in fp32."""
    M, K = _int8_acts(qa, dx, bsum)
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, qa)
    _on_device(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum, y=y)
    _check(load().w4a8_gemv(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx), _ptr(bsum),
                            M, _ptr(y), oc, _stream(stream)), "w4a8_gemv")
    return y


def w4a8_gemv_bf16(codes, d, m, x, out_dtype=None, y=None, stream=None):
    """w4a8_gemv with the quantiser folded in: bf16 x[M,K] (1 <= M <= 8) is
    quantised to int8 blocks inside the kernel; bit-identical to
    q8_quantize_act followed by w4a8_gemv."""
    torch = _torch()
    _need(x, torch.bfloat16, "x", (None, None))
    M, K = x.shape
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, x)
    _on_device(codes=codes, d=d, m=m, x=x, y=y)
    _check(load().w4a8_gemv_bf16(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(x), M, _ptr(y), oc,
                                 _stream(stream)), "w4a8_gemv_bf16")
    return y


def q8_quantize_act(x, qa=None, dx=None, bsum=None, stream=None):
    """bf16 x[M,K] (K % 32 == 0) -> (qa int8[M,K], dx fp32[M,K/32], bsum int32[M,K/32])."""
    torch = _torch()
    _need(x, torch.bfloat16, "x", (None, None))
    M, K = x.shape
    if qa is None:
        qa = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if dx is None:
        dx = torch.empty((M, K // BLOCK), dtype=torch.float32, device=x.device)
    if bsum is None:
        bsum = torch.empty((M, K // BLOCK), dtype=torch.int32, device=x.device)
    _need(qa, torch.int8, "qa", (M, K))
    _need(dx, torch.float32, "dx", (M, _div(K, BLOCK)))
    _need(bsum, torch.int32, "bsum", (M, _div(K, BLOCK)))
    _on_device(x=x, qa=qa, dx=dx, bsum=bsum)
    _check(load().q8_quantize_act(_ptr(x), M, K, _ptr(qa), _ptr(dx), _ptr(bsum),
                                  _stream(stream)), "q8_quantize_act")
    return qa, dx, bsum


def w4a8_mmq_workspace_size(M: int, N: int, K: int) -> int:
    return int(load().w4a8_mmq_workspace_size(M, N, K))


def w4a8_mmq(codes, d, m, qa, dx, bsum, out_dtype=None, y=None, workspace=None, stream=None):
    """y[M,N] from W4-G256 weights and int8 activation blocks (tensor cores).
    workspace: optional uint8 1-D device tensor of at least
    w4a8_mmq_workspace_size(M, N, K) bytes (allocated here when omitted)."""
    torch = _torch()
    M, K = _int8_acts(qa, dx, bsum)
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, qa)
    placed = dict(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum, y=y)
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace", (None,))
        placed["workspace"] = workspace
    _on_device(**placed)
    if workspace is None:
        ws_need = w4a8_mmq_workspace_size(M, N, K)
        if ws_need > 0:
            workspace = torch.empty(ws_need, dtype=torch.uint8, device=qa.device)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().w4a8_mmq(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx), _ptr(bsum),
                           M, _ptr(y), oc, ws_ptr, ws_bytes, _stream(stream)), "w4a8_mmq")
    return y


def w4a8_mmq_static(codes, d, m, qa, dx, bsum, out_dtype=None, y=None, stream=None):
    """The W4A8 product without a workspace, for callers that cannot allocate
    device memory: the split-K scratch is the library's static device array
    (shared by every call on the device; overlapping calls must be serialised).
    Raises W4Error (W4_ERR_WORKSPACE) for shapes whose scratch need exceeds it.
    The C entry point allocates nothing; this wrapper allocates only the output
    (through torch) when `y` is omitted, so a caller that cannot allocate
    passes its own `y`."""
    M, K = _int8_acts(qa, dx, bsum)
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, qa)
    _on_device(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum, y=y)
    _check(load().w4a8_mmq_static(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx),
                                  _ptr(bsum), M, _ptr(y), oc, _stream(stream)), "w4a8_mmq_static")
    return y


def w4a8_mmq_blockdots(codes, d, m, qa, dx, bsum, out_dtype=None, y=None, stream=None):
    """w4a8_mmq that also returns the exact int32 block products
    P[M, N, K/32] read back from the kernel's tensor-memory accumulators (for
    tests of the integer core; much slower than w4a8_mmq).  Returns (y, P)."""
    torch = _torch()
    M, K = _int8_acts(qa, dx, bsum)
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, qa)
    _on_device(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum, y=y)
    P = torch.empty((M, N, K // BLOCK), dtype=torch.int32, device=qa.device)
    ws_need = w4a8_mmq_workspace_size(M, N, K)
    ws = torch.empty(max(ws_need, 1), dtype=torch.uint8, device=qa.device) if ws_need else None
    _check(load().w4a8_mmq_blockdots(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx),
                                     _ptr(bsum), M, _ptr(y), oc, _ptr(P),
                                     P.numel() * 4, _ptr(ws) if ws is not None else None,
                                     ws_need, _stream(stream)), "w4a8_mmq_blockdots")
    return y, P


def w4a8_gemv_blockdots(codes, d, m, qa, dx, bsum, out_dtype=None, y=None, stream=None):
    """w4a8_gemv (M <= 8) that also returns the exact int32 block products
    P[M, N, K/32] its integer core formed (for tests).  Returns (y, P)."""
    torch = _torch()
    M, K = _int8_acts(qa, dx, bsum)
    N = _weights(codes, d, m, K)
    oc = _out_code(out_dtype, y)
    y = _output(y, M, N, oc, qa)
    _on_device(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum, y=y)
    P = torch.empty((M, N, K // BLOCK), dtype=torch.int32, device=qa.device)
    _check(load().w4a8_gemv_blockdots(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx),
                                      _ptr(bsum), M, _ptr(y), oc, _ptr(P), P.numel() * 4,
                                      _stream(stream)), "w4a8_gemv_blockdots")
    return y, P

