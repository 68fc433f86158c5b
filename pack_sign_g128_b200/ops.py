"""Thin torch-facing wrappers over the libw1 C ABI (argument marshalling only).

Tensors are CUDA tensors; 16-bit formats travel as their natural torch dtypes
(bf16 activations, fp16 scales / diagonals) and sign words as int32 (same bits
as the ABI's uint32).  Every call runs on the current torch CUDA stream and
raises W1Error on a non-OK status.  No computation happens here.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


# The raw handle of a device's current stream without building a Stream
# object (a few microseconds per call otherwise); the public call is the
# fallback where this torch build lacks it.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None, t: torch.Tensor | None = None) -> int:
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and t is not None and t.is_cuda:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream().cuda_stream


def sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return _lib.call("w1_sync_status", _stream(stream))


def set_knob(name: str, value: str | int | None) -> None:
    """Set a process-wide testing / tuning knob of the library (w1_set_knob);
    None restores the value the W1_* environment variable gave."""
    v = None if value is None else str(value).encode()
    _lib.check(_lib.call("w1_set_knob", name.encode(), v), f"w1_set_knob({name})")


def status_string(status: int) -> str:
    return _lib.call("w1_status_string", int(status)).decode()


def w1_pack(W: torch.Tensor, signs: torch.Tensor | None = None, scales: torch.Tensor | None = None,
            stream=None):
    """fp32 W [N, K] -> (signs int32 [N, K/32], scales fp16 [N, K/128])."""
    N, K = W.shape
    if W.dtype != torch.float32:
        raise TypeError("W must be float32")
    if signs is None:
        signs = torch.empty((N, K // 32), dtype=torch.int32, device=W.device)
    if scales is None:
        scales = torch.empty((N, K // 128), dtype=torch.float16, device=W.device)
    st = _lib.call("w1_pack", _ptr(W), N, K, _ptr(signs), _ptr(scales), _stream(stream, W))
    _lib.check(st, "w1_pack")
    return signs, scales


W1_GEMV_STATIC_WEIGHTS = 1


def w1_gemv(signs: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None,
            stream=None, static_weights: bool = False) -> torch.Tensor:
    """y [B, N] fp32 = x [B, K] bf16 times the 1-bit matrix (B <= 8).

    static_weights=True calls w1_gemv_ex with W1_GEMV_STATIC_WEIGHTS: the
    weights must not have been written by the kernel just before on the stream.
    """
    N, KW = signs.shape
    B = x.shape[0]
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    st = _lib.fn("w1_gemv_ex")(_ptr(signs), _ptr(scales), N, KW * 32, _ptr(x), B, _ptr(y),
                               W1_GEMV_STATIC_WEIGHTS if static_weights else 0, _stream(stream, x))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_gemv")
    return y


def _check_kron(H: torch.Tensor, R: torch.Tensor, K: int) -> None:
    if H.dim() != 2 or H.shape[0] != H.shape[1] or R.dim() != 2 or R.shape[0] != R.shape[1]:
        raise ValueError("H and R must be square matrices")
    if H.shape[0] * R.shape[0] != K:
        raise ValueError(f"n1 * n2 = {H.shape[0]} * {R.shape[0]} is not K = {K}")


def w1_okt_rotate(H: torch.Tensor, R: torch.Tensor, x: torch.Tensor, x_rot: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """x_rot [B, K] fp32 = (H kron R)^T x for every row of x [B, K] bf16.

    H fp32 [n1, n1] and R fp32 [n2, n2] are orthogonal, n1 * n2 = K."""
    n1, n2 = H.shape[0], R.shape[0]
    B, K = x.shape
    if x.dtype != torch.bfloat16 or H.dtype != torch.float32 or R.dtype != torch.float32:
        raise TypeError("x must be bfloat16, H and R float32")
    _check_kron(H, R, K)
    if x_rot is None:
        x_rot = torch.empty((B, K), dtype=torch.float32, device=x.device)
    st = _lib.fn("w1_okt_rotate")(_ptr(H), n1, _ptr(R), n2, _ptr(x), B, _ptr(x_rot), _stream(stream, x))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_okt_rotate")
    return x_rot


def w1_okt_gemv(signs: torch.Tensor, scales: torch.Tensor, H: torch.Tensor, R: torch.Tensor, x: torch.Tensor,
                y: torch.Tensor | None = None, x_rot: torch.Tensor | None = None, stream=None,
                static_weights: bool = False) -> torch.Tensor:
    """y [B, N] fp32 = the 1-bit matrix (packed in rotated coordinates) times
    (H kron R)^T x, x [B, K] bf16, B <= 8.  x_rot (fp32 [B, K]) receives the
    rotated activations; allocated here when omitted."""
    N, KW = signs.shape
    B, K = x.shape
    if x.dtype != torch.bfloat16 or H.dtype != torch.float32 or R.dtype != torch.float32:
        raise TypeError("x must be bfloat16, H and R float32")
    if KW * 32 != K:
        raise ValueError(f"x has K = {K} columns, the packed weights {KW * 32}")
    _check_kron(H, R, K)
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    if x_rot is None:
        x_rot = torch.empty((B, K), dtype=torch.float32, device=x.device)
    st = _lib.fn("w1_okt_gemv")(_ptr(signs), _ptr(scales), N, KW * 32, _ptr(H), H.shape[0], _ptr(R), R.shape[0],
                                _ptr(x), B, _ptr(x_rot), _ptr(y),
                                W1_GEMV_STATIC_WEIGHTS if static_weights else 0, _stream(stream, x))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_okt_gemv")
    return y


def measure_workspace(m: int, n: int, device=None) -> torch.Tensor:
    """Workspace for w1_residual / dbf_residual / w1_power_iteration on m x n."""
    nbytes = _lib.call("w1_measure_workspace_size", m, n)
    if nbytes == 0:
        raise ValueError("invalid measurement sizes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def w1_residual(W: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor, E: torch.Tensor | None = None,
                want_E: bool = True, workspace: torch.Tensor | None = None, stream=None):
    """(E fp32 [N, K] or None, sums fp64 [2] = (sum E^2, sum W^2)) for W and its packing."""
    N, K = W.shape
    if W.dtype != torch.float32:
        raise TypeError("W must be float32")
    if tuple(signs.shape) != (N, K // 32) or tuple(scales.shape) != (N, K // 128):
        raise ValueError("signs / scales do not match W's shape")
    if want_E and E is None:
        E = torch.empty((N, K), dtype=torch.float32, device=W.device)
    sums = torch.empty(2, dtype=torch.float64, device=W.device)
    if workspace is None:
        workspace = measure_workspace(N, K, W.device)
    st = _lib.fn("w1_residual")(_ptr(W), N, K, _ptr(signs), _ptr(scales), _ptr(E) if want_E else None, _ptr(sums),
                                _ptr(workspace), workspace.numel(), _stream(stream, W))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_residual")
    return (E if want_E else None), sums


def dbf_residual_workspace_size(m: int, r: int, n: int) -> int:
    return int(_lib.fn("dbf_residual_workspace_size")(m, r, n))


def dbf_residual(W: torch.Tensor, a: torch.Tensor, B1: torch.Tensor, mid: torch.Tensor, B2: torch.Tensor,
                 b: torch.Tensor, E: torch.Tensor | None = None, want_E: bool = True,
                 workspace: torch.Tensor | None = None, stream=None):
    """(E fp32 [m, n] or None, sums fp64 [2]) for W against diag(a) U diag(mid) V diag(b)."""
    m, n = W.shape
    r = mid.shape[0]
    if W.dtype != torch.float32:
        raise TypeError("W must be float32")
    if (a.shape[0] != m or b.shape[0] != n or tuple(B1.shape) != (m, r // 32)
            or tuple(B2.shape) != (r, n // 32)):
        raise ValueError("DBF operands do not match W's shape")
    if want_E and E is None:
        E = torch.empty((m, n), dtype=torch.float32, device=W.device)
    sums = torch.empty(2, dtype=torch.float64, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(dbf_residual_workspace_size(m, r, n), 1), dtype=torch.uint8, device=W.device)
    st = _lib.fn("dbf_residual")(_ptr(W), _ptr(a), _ptr(B1), _ptr(mid), _ptr(B2), _ptr(b), m, r, n,
                                 _ptr(E) if want_E else None, _ptr(sums), _ptr(workspace), workspace.numel(),
                                 _stream(stream, W))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "dbf_residual")
    return (E if want_E else None), sums


def w1_stream_probe(a: torch.Tensor, b: torch.Tensor | None, out: torch.Tensor, ctas: int, early: bool,
                    stream=None) -> None:
    """Launch the per-launch floor probe over a's and b's bytes (see include/w1.h)."""
    if out.dtype != torch.int32 or out.numel() < ctas:
        raise ValueError("out must be int32 with at least `ctas` elements")
    ab = a.numel() * a.element_size()
    bb = 0 if b is None else b.numel() * b.element_size()
    st = _lib.fn("w1_stream_probe")(_ptr(a), ab, _ptr(b) if b is not None else None, bb, ctas, 1 if early else 0,
                                    _ptr(out), _stream(stream, a))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_stream_probe")


def dbf_reproject_workspace_size(m: int, r: int, n: int) -> int:
    return int(_lib.fn("dbf_reproject_mid_workspace_size")(m, r, n))


def dbf_reproject_mid(W: torch.Tensor, a: torch.Tensor, B1: torch.Tensor, B2: torch.Tensor, b: torch.Tensor,
                      max_iter: int = 200, tol: float = 1e-13, workspace: torch.Tensor | None = None, stream=None):
    """Least-squares middle diagonal for fixed signs and outer scalers:
    (mid fp16 [r], mid fp64 [r], info int32 [2] = iterations, converged)."""
    m, n = W.shape
    r = B1.shape[1] * 32
    if W.dtype != torch.float32:
        raise TypeError("W must be float32")
    if a.shape[0] != m or b.shape[0] != n or B1.shape[0] != m or tuple(B2.shape) != (r, n // 32):
        raise ValueError("DBF operands do not match W's shape")
    mid = torch.empty(r, dtype=torch.float16, device=W.device)
    mid64 = torch.empty(r, dtype=torch.float64, device=W.device)
    info = torch.zeros(2, dtype=torch.int32, device=W.device)
    need = dbf_reproject_workspace_size(m, r, n)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=W.device)
    st = _lib.fn("dbf_reproject_mid")(_ptr(W), _ptr(a), _ptr(B1), _ptr(B2), _ptr(b), m, r, n, max_iter, tol,
                                      _ptr(mid), _ptr(mid64), _ptr(info), _ptr(workspace), workspace.numel(),
                                      _stream(stream, W))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "dbf_reproject_mid")
    return mid, mid64, info


def w1_power_iteration(A: torch.Tensor, v0: torch.Tensor, iters: int = 32, workspace: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Spectral norm estimate of A fp32 [m, n] (fp64 scalar tensor on the device)."""
    m, n = A.shape
    if A.dtype != torch.float32 or v0.dtype != torch.float32:
        raise TypeError("A and v0 must be float32")
    if v0.numel() != n:
        raise ValueError(f"v0 has {v0.numel()} entries, A has {n} columns")
    sigma = torch.empty((), dtype=torch.float64, device=A.device)
    if workspace is None:
        workspace = measure_workspace(m, n, A.device)
    st = _lib.fn("w1_power_iteration")(_ptr(A), m, n, _ptr(v0), iters, _ptr(sigma), _ptr(workspace),
                                       workspace.numel(), _stream(stream, A))
    if st != _lib.W1_OK:
        raise _lib.W1Error(st, "w1_power_iteration")
    return sigma


def gemm_workspace(M: int, K: int, device=None) -> torch.Tensor:
    """Workspace bytes for w1_gemm (fp16 copy of x, token scales)."""
    n = _lib.call("w1_gemm_workspace_size", M, K)
    if n == 0:
        raise ValueError("invalid w1_gemm sizes")
    return torch.empty(n + 256, dtype=torch.uint8, device=device)


def _aligned256(ws: torch.Tensor) -> int:
    p = ws.data_ptr()
    return (p + 255) // 256 * 256


def gemv_choice(N: int, K: int, B: int, static_weights: bool = False) -> str:
    """The kernel/K split w1_gemv chose for this shape ("" before the first call):
    "direct/<split>" (8 warps per CTA), "direct16/<split>", "tc/<split>", "ring/<split>"."""
    buf = ctypes.create_string_buffer(64)
    st = _lib.call("w1_gemv_choice", N, K, B, W1_GEMV_STATIC_WEIGHTS if static_weights else 0, buf, 64)
    _lib.check(st, "w1_gemv_choice")
    return buf.value.decode()


def gemv_set_choice(N: int, K: int, B: int, name: str, static_weights: bool = False) -> None:
    """Pin w1_gemv's kernel for this shape ("direct/1", "direct16/2", "tc/0", "ring/0")."""
    st = _lib.call("w1_gemv_set_choice", N, K, B, W1_GEMV_STATIC_WEIGHTS if static_weights else 0, name.encode())
    _lib.check(st, "w1_gemv_set_choice")


def w1_gemm(signs: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None,
            stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y [M, N] fp32 = x [M, K] bf16 times the 1-bit matrix (prefill).

    workspace: a gemm_workspace(M, K) buffer; allocated here when omitted.
    """
    N = signs.shape[0]
    K = signs.shape[1] * 32
    M = x.shape[0]
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = gemm_workspace(M, K, device=x.device)
    base = _aligned256(workspace)
    avail = workspace.numel() - (base - workspace.data_ptr())
    st = _lib.call("w1_gemm", _ptr(signs), _ptr(scales), N, K, _ptr(x), M, _ptr(y),
                   ctypes.c_void_p(base), avail, _stream(stream, x))
    _lib.check(st, "w1_gemm")
    return y


_MOE_WS_ALIGN = 1024  # w1_moe_grouped's workspace alignment


def moe_workspace(T: int, H: int, I: int, E: int, top_k: int, device=None) -> torch.Tensor:
    """Workspace for w1_moe_grouped (with slack: the call uses its 1024-byte aligned part)."""
    nbytes = _lib.call("w1_moe_workspace_size", T, H, I, E, top_k)
    if nbytes == 0:
        raise ValueError("invalid MoE sizes")
    return torch.empty(nbytes + _MOE_WS_ALIGN, dtype=torch.uint8, device=device or "cuda")


def _moe_ws_offset(workspace: torch.Tensor) -> int:
    p = workspace.data_ptr()
    return (p + _MOE_WS_ALIGN - 1) // _MOE_WS_ALIGN * _MOE_WS_ALIGN - p


def w1_moe_grouped(x: torch.Tensor, logits: torch.Tensor, gate, up, down, top_k: int,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Routed SwiGLU layer.  gate/up/down = (signs int32 [E, rows, K/32], scales fp16 [E, rows, K/128])."""
    T, H = x.shape
    E = logits.shape[1]
    I = gate[0].shape[1]
    if x.dtype != torch.bfloat16 or logits.dtype != torch.float32:
        raise TypeError("x must be bfloat16 and logits float32")
    if workspace is None:
        workspace = moe_workspace(T, H, I, E, top_k, x.device)
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=x.device)
    off = _moe_ws_offset(workspace)
    st = _lib.call("w1_moe_grouped", _ptr(x), _ptr(logits), T, H, I, E, top_k, _ptr(gate[0]), _ptr(gate[1]),
                   _ptr(up[0]), _ptr(up[1]), _ptr(down[0]), _ptr(down[1]), _ptr(out),
                   ctypes.c_void_p(_ptr(workspace) + off),
                   workspace.numel() * workspace.element_size() - off, _stream(stream, x))
    _lib.check(st, "w1_moe_grouped")
    return out


def moe_workspace_views(workspace: torch.Tensor, T: int, H: int, I: int, E: int, top_k: int) -> dict:
    """Typed views of the MoE workspace (routing, sorted order, h) for inspection."""
    R = T * top_k
    workspace = workspace[_moe_ws_offset(workspace):]  # the part the call used

    def up(v, a):
        return (v + a - 1) // a * a
    off = 256
    views = {}
    for name in ("ids", "wts", "pos", "sroute", "stok"):
        views[name] = workspace[off:off + 4 * R].view(torch.float32 if name == "wts" else torch.int32)
        off = up(off + 4 * R, 256)
    views["offsets"] = workspace[off:off + 4 * (E + 1)].view(torch.int32)
    off = up(off + 4 * (E + 1), 256)
    mtg = ((R + 127) // 128 + E) * (I // 128)
    mtd = ((R + 127) // 128 + E) * (H // 128)
    off = up(off + 16 * mtg, 256)
    off = up(off + 16 * mtd, 256)
    views["h"] = workspace[off:off + 2 * R * I].view(torch.bfloat16).view(R, I)
    return views


def dbf_workspace(m: int, r: int, n: int, B: int, device=None) -> torch.Tensor:
    """A zeroed workspace for dbf_apply (the grid-barrier words start at zero)."""
    nbytes = _lib.call("dbf_workspace_size", m, r, n, B)
    if nbytes == 0:
        raise ValueError("invalid DBF sizes")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


def dbf_apply(a: torch.Tensor, B1: torch.Tensor, mid: torch.Tensor, B2: torch.Tensor, b: torch.Tensor,
              x: torch.Tensor, y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """y [B, m] = a * (U @ (mid * (V @ (b * x)))) with U = B1 [m, r/32], V = B2 [r, n/32] sign words."""
    m = a.shape[0]
    r = mid.shape[0]
    n = b.shape[0]
    B = x.shape[0]
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if workspace is None:
        workspace = dbf_workspace(m, r, n, B, x.device)
    if y is None:
        y = torch.empty((B, m), dtype=torch.float32, device=x.device)
    st = _lib.call("dbf_apply", _ptr(a), _ptr(B1), _ptr(mid), _ptr(B2), _ptr(b), m, r, n, _ptr(x), B,
                   _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream, x))
    _lib.check(st, "dbf_apply")
    return y


def dbf_apply_noalloc(a: torch.Tensor, B1: torch.Tensor, mid: torch.Tensor, B2: torch.Tensor, b: torch.Tensor,
                      x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
    """dbf_apply without a workspace (the library's static scratch); y must be given."""
    m, r, n, B = a.shape[0], mid.shape[0], b.shape[0], x.shape[0]
    st = _lib.call("dbf_apply_noalloc", _ptr(a), _ptr(B1), _ptr(mid), _ptr(B2), _ptr(b), m, r, n, _ptr(x), B,
                   _ptr(y), _stream(stream, x))
    _lib.check(st, "dbf_apply_noalloc")
    return y
