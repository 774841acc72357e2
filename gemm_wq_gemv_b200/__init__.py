"""Python binding of ``libwq.so`` (the C ABI declared in ``include/wq.h``).

Argument marshalling only: every step of the product runs in the library's
sm_100a kernels.  Tensors must already live on the current CUDA device; calls
are enqueued on ``torch.cuda.current_stream()``.  There is no CPU path: if the
library is missing or the device is not an sm_100 GPU, the calls raise.

Entry points (same names as the C ABI, without the ``wq_`` prefix):

* ``pack_kmajor(codes_kn, bits) -> (w_q, w_lo)``
* ``unpack_kmajor(w_q, w_lo, K, bits) -> codes_kn``
* ``gemv(x, w_q, w_lo, scales, zeros, bits, group_size, out=None, pdl=False,
  inputs_ready=False, bias=None) -> y``
* ``gemm(x, w_q, w_lo, scales, zeros, bits, group_size, out=None, pdl=False,
  workspace=None, inputs_ready=False, bias=None) -> y``
* ``gemm_workspace_size(M, K, N, bits, group_size) -> bytes``
* ``matmul(...)``: same arguments as ``gemm``; ``wq_gemv`` or ``wq_gemm`` by M
* ``gemm_noalloc(x, w_q, w_lo, scales, zeros, bits, group_size, out) -> out``
* ``selftest_wait_timeout(limit_ns) -> status`` (the bounded-wait failure path)
* ``from_gptqmodel(qweight, qzeros, bits, group_size, K, dtype) -> (w_q, w_lo, zeros)``
  and ``gptqmodel_quantized_matmul(x, qweight, qzeros, scales, bits, group_size)``
  (the GPTQModel packed format)
* ``mse_search(w, bits, group_size, maxshrink=0.2, grid=100, norm=2.4,
  patience=None, symmetric=False) -> dict`` (per-group s, z of the MSE observer)

x, scales, zeros, bias and the output are all ``torch.float16`` or all
``torch.bfloat16`` (the type of x decides; bfloat16 sets ``WQ_FLAG_BF16``).
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

_PKG = Path(__file__).resolve().parent
# WQ_LIB=checked loads the checked build (libwq_checked.so, see build.py) instead
LIB_PATH = _PKG / ("libwq_checked.so" if os.environ.get("WQ_LIB") == "checked" else "libwq.so")

STATUS = {
    0: "WQ_OK",
    1: "WQ_ERR_INVALID_ARG",
    2: "WQ_ERR_UNSUPPORTED",
    3: "WQ_ERR_ALIGNMENT",
    4: "WQ_ERR_CODE_RANGE",
    5: "WQ_ERR_TIMEOUT",
    6: "WQ_ERR_CUDA",
    7: "WQ_ERR_SCRATCH_LIMIT",
    8: "WQ_ERR_CHECK",
    9: "WQ_ERR_NOT_POSITIVE_DEFINITE",
}
WQ_FLAG_PDL = 1
WQ_FLAG_PDL_INPUTS_READY = 2
WQ_FLAG_BF16 = 4

_lib = None


class WQError(RuntimeError):
    """A call into libwq.so returned a status other than WQ_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{fn}: {self.name} ({describe(status)})")


def lib() -> ctypes.CDLL:
    """Load ``libwq.so`` (built in-tree by ``python -m gemm_wq_gemv_b200.build``)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gemm_wq_gemv_b200.build` (needs nvcc)")
        L = ctypes.CDLL(str(LIB_PATH))
        p, i, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        L.wq_abi_version.restype = i
        L.wq_status_string.argtypes = [i]
        L.wq_status_string.restype = ctypes.c_char_p
        L.wq_pack_kmajor.argtypes = [p, i, i, i, p, p, p, p]
        L.wq_unpack_kmajor.argtypes = [p, p, i, i, i, p, p]
        L.wq_gemv.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, u, p]
        L.wq_gemm.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, u, p, ctypes.c_size_t, p]
        L.wq_gemm_workspace_size.argtypes = [i, i, i, i, i]
        L.wq_gemm_workspace_size.restype = ctypes.c_size_t
        L.wq_gemm_noalloc.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, u, p]
        L.wq_matmul.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, u, p, ctypes.c_size_t, p]
        L.wq_matmul.restype = i
        L.wq_matmul_uses_gemv.argtypes = [i, i, i, i, i]
        L.wq_matmul_uses_gemv.restype = i
        L.wq_matmul_workspace_size.argtypes = [i, i, i, i, i]
        L.wq_matmul_workspace_size.restype = ctypes.c_size_t
        L.wq_gemm_noalloc.restype = i
        L.wq_device_status.argtypes = [i]
        L.wq_selftest_wait_timeout.argtypes = [ctypes.c_uint64, p]
        L.wq_gptqmodel_convert.argtypes = [p, p, i, i, i, i, p, p, p, u, p]
        L.wq_gptqmodel_convert.restype = i
        L.wq_mse_search.argtypes = [p, i, i, i, i, i, i, i, ctypes.c_float, i, p, p, p, p, p, ctypes.c_size_t, p]
        L.wq_mse_search.restype = i
        L.wq_gemv_plan_create.argtypes = [p, p, p, p, p, i, i, i, i, i, u, ctypes.POINTER(p)]
        L.wq_gemv_plan_create.restype = i
        L.wq_gemv_plan_run.argtypes = [p, p, p, p]
        L.wq_gemv_plan_run.restype = i
        L.wq_gemv_plan_destroy.argtypes = [p]
        L.wq_gemv_plan_destroy.restype = None
        L.wq_checked_build.restype = i
        L.wq_gptq_workspace_size.argtypes = [i, i]
        L.wq_gptq_workspace_size.restype = ctypes.c_size_t
        L.wq_gptq_quantize.argtypes = [p, p, p, p, i, i, i, i, i, ctypes.c_float, p, p, p, p, ctypes.c_size_t, p]
        L.wq_gptq_quantize.restype = i
        for f in ("wq_pack_kmajor", "wq_unpack_kmajor", "wq_gemv", "wq_gemm", "wq_device_status",
                  "wq_selftest_wait_timeout"):
            getattr(L, f).restype = i
        _lib = L
    return _lib


def describe(status: int) -> str:
    return lib().wq_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise WQError(fn, status)


def _torch():
    import torch
    return torch


def _stream():
    torch = _torch()
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:  # the handle without building a Stream object per call
        return raw(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, ndim=2):
    try:  # the common case in one expression; the messages below only on failure
        if t.is_cuda and t.dtype == dtype and t.dim() == ndim and t.is_contiguous():
            return
    except AttributeError:
        pass
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def words_shape(K: int, N: int, bits: int):
    """Shapes of the packed planes for a (K, N) code matrix: (w_q, w_lo or None)."""
    if bits == 3:
        return (K // 16, N), (K // 32, N)
    return (K // (32 // bits), N), None


_BITS = (1, 2, 3, 4, 8)
_EPS = {1: 32, 2: 16, 3: 16, 4: 8, 8: 4}  # codes per word of the main plane


def _same_device(ref, **tensors):
    d = ref.device
    for name, t in tensors.items():
        if t is not None and t.device != d:
            raise ValueError(f"{name} is on {t.device}, x on {ref.device}: all tensors must share one device")


def _check_planes(w_q, w_lo, K: int, bits: int):
    """w_q (and w_lo) must have the packed shape of a (K, N) code matrix, N = w_q.shape[1].

    The library sizes its copies from K, N and bits, so a plane of another shape
    would be read out of its bounds; a bit width it does not take is left to the
    C call, which rejects it."""
    eps = _EPS.get(bits)
    if eps is None:
        return
    N = w_q.shape[1]
    if w_q.shape != (K // eps, N):
        raise ValueError(f"w_q has shape {tuple(w_q.shape)}; K={K}, {bits}-bit words need {(K // eps, N)}")
    if bits == 3:
        if w_lo is None:
            raise ValueError("3-bit words need the lo plane w_lo")
        if w_lo.shape != (K // 32, N):
            raise ValueError(f"w_lo has shape {tuple(w_lo.shape)}; K={K} 3-bit needs {(K // 32, N)}")
    elif w_lo is not None:
        raise ValueError(f"w_lo must be None for {bits}-bit words")


def _check_product(x, w_q, w_lo, scales, zeros, bias, out, bits: int, group_size: int):
    """Every tensor of a product has the shape its K, N, M, bits and group size
    imply, and sits on x's device.  Raises ValueError before any C call.
    Shapes the C rules reject anyway (a K that is not a multiple of the word
    width, a group size that does not divide K) are left to the C call, which
    names the rule.  (Runs on every call: kept to plain shape comparisons.)"""
    M, K = x.shape
    N = w_q.shape[1]
    d = x.get_device()
    if (d < 0 or w_q.get_device() != d or scales.get_device() != d or zeros.get_device() != d
            or (w_lo is not None and w_lo.get_device() != d) or (bias is not None and bias.get_device() != d)
            or (out is not None and out.get_device() != d)):
        _same_device(x, w_q=w_q, w_lo=w_lo, scales=scales, zeros=zeros, bias=bias, out=out)
    _check_planes(w_q, w_lo, K, bits)
    G = K if group_size == -1 else group_size
    if G > 0 and K % G == 0:
        sz = (K // G, N)
        if scales.shape != sz:
            raise ValueError(f"scales has shape {tuple(scales.shape)}; K={K}, group size {group_size} "
                             f"and N={N} need {sz}")
        if zeros.shape != sz:
            raise ValueError(f"zeros has shape {tuple(zeros.shape)}; K={K}, group size {group_size} "
                             f"and N={N} need {sz}")
    if bias is not None and bias.shape != (N,):
        raise ValueError(f"bias has shape {tuple(bias.shape)}; N={N} needs ({N},)")
    if out is not None and out.shape != (M, N):
        raise ValueError(f"out has shape {tuple(out.shape)}; M={M}, N={N} need {(M, N)}")


def pack_kmajor(codes_kn, bits: int, check_range: bool = True):
    """(K, N) uint8 codes -> (w_q, w_lo) int32 words (w_lo is None unless bits == 3).

    With ``check_range`` the call counts codes that do not fit ``bits`` bits on
    the device, waits for the stream, and raises WQ_ERR_CODE_RANGE if any.
    """
    torch = _torch()
    _need(codes_kn, torch.uint8, "codes_kn")
    K, N = codes_kn.shape
    hs, ls = words_shape(K, N, bits)
    dev = codes_kn.device
    w_q = torch.empty(hs, dtype=torch.int32, device=dev)
    w_lo = torch.empty(ls, dtype=torch.int32, device=dev) if ls else None
    bad = torch.zeros(1, dtype=torch.int32, device=dev) if check_range else None
    _check("wq_pack_kmajor", lib().wq_pack_kmajor(_ptr(codes_kn), K, N, bits, _ptr(w_q),
                                                  _ptr(w_lo), _ptr(bad), _stream()))
    if check_range and int(bad.item()) != 0:
        raise WQError("wq_pack_kmajor", 4)
    return w_q, w_lo


def unpack_kmajor(w_q, w_lo, K: int, bits: int):
    torch = _torch()
    _need(w_q, torch.int32, "w_q")
    if w_lo is not None:
        _need(w_lo, torch.int32, "w_lo")
    _same_device(w_q, w_lo=w_lo)
    _check_planes(w_q, w_lo, K, bits)
    N = w_q.shape[1]
    out = torch.empty((K, N), dtype=torch.uint8, device=w_q.device)
    _check("wq_unpack_kmajor", lib().wq_unpack_kmajor(_ptr(w_q), _ptr(w_lo), K, N, bits,
                                                      _ptr(out), _stream()))
    return out


def _elem_type(x):
    """float16 or bfloat16: the type of x, which scales, zeros, bias and y share."""
    torch = _torch()
    dt = getattr(x, "dtype", None)
    if dt is torch.float16 or dt is torch.bfloat16:
        return dt
    if isinstance(x, torch.Tensor):
        raise TypeError(f"x must be torch.float16 or torch.bfloat16, got {dt}")
    raise TypeError("x must be a torch.Tensor")


def _product(fn, x, w_q, w_lo, scales, zeros, bits, group_size, out, pdl, workspace=False,
             inputs_ready=False, bias=None):
    torch = _torch()
    dt = _elem_type(x)
    _need(x, dt, "x")
    _need(w_q, torch.int32, "w_q")
    if w_lo is not None:
        _need(w_lo, torch.int32, "w_lo")
    _need(scales, dt, "scales")
    _need(zeros, dt, "zeros")
    if bias is not None:
        _need(bias, dt, "bias", ndim=1)
    if out is not None:
        _need(out, dt, "out")
    _check_product(x, w_q, w_lo, scales, zeros, bias, out, bits, group_size)
    M, K = x.shape
    N = w_q.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=x.device)
    flags = ((WQ_FLAG_PDL if pdl else 0) | (WQ_FLAG_PDL_INPUTS_READY if inputs_ready else 0)
             | (WQ_FLAG_BF16 if dt is torch.bfloat16 else 0))
    args = [_ptr(x), _ptr(w_q), _ptr(w_lo), _ptr(scales), _ptr(zeros), _ptr(bias), _ptr(out),
            M, K, N, bits, group_size, flags]
    if workspace is not False:  # wq_gemm: (workspace, bytes)
        if workspace is None:
            key = (fn, x.device.index, M, K, N, bits, group_size)
            need = _ws_sizes.get(key)
            if need is None:  # wq_matmul's size is wq_gemm's on that route, else 0
                query = lib().wq_matmul_workspace_size if fn == "wq_matmul" else lib().wq_gemm_workspace_size
                need = _ws_sizes[key] = int(query(M, K, N, bits, group_size))
            workspace = _cached_workspace(x.device, need)
        args += [_ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size()]
    st = getattr(lib(), fn)(*args, _stream())
    _check(fn, st)
    return out


def gemv(x, w_q, w_lo, scales, zeros, bits: int, group_size: int, out=None, pdl: bool = False,
         inputs_ready: bool = False, bias=None):
    """y (M, N) = x (M, K) @ dequant(w_q), 1 <= M <= 16 (``wq_gemv``), in the type of x.

    ``pdl``: WQ_FLAG_PDL; ``inputs_ready``: WQ_FLAG_PDL_INPUTS_READY (the previous
    kernel on the stream writes none of this call's inputs); ``bias``: optional (N,)
    tensor of x's type added to every row of the output."""
    return _product("wq_gemv", x, w_q, w_lo, scales, zeros, bits, group_size, out, pdl,
                    inputs_ready=inputs_ready, bias=bias)


class GemvPlan:
    """A decode product with its weights bound once (``wq_gemv_plan``): the
    dashq_kernel.py page's TritonQuantLinear, as a prepared launch.

    ``plan = GemvPlan(w_q, w_lo, scales, zeros, bits, group_size, M, bias=None,
    pdl=False, inputs_ready=False)`` checks the weights as ``gemv`` would for an
    ``(M, K)`` x of the scales' type and records the kernel, its launch shape
    and the weight descriptors; ``plan(x, out=None)`` is then ``gemv(x, ...)``
    with the same bits, for a CUDA tensor x of shape (M, K) on the same device,
    at the cost of one launch.  The plan holds references to the weight
    tensors, which must not be resized or moved (their contents may change)."""

    def __init__(self, w_q, w_lo, scales, zeros, bits: int, group_size: int, M: int, bias=None,
                 pdl: bool = False, inputs_ready: bool = False):
        torch = _torch()
        dt = _elem_type(scales)
        if bits not in _BITS:
            raise ValueError(f"bits must be one of {_BITS}, got {bits}")
        K = w_q.shape[0] * _EPS[bits]  # word rows x codes per word
        x_meta = torch.empty((M, K), dtype=dt, device=w_q.device)
        for t, name in ((w_q, "w_q"), (scales, "scales"), (zeros, "zeros")):
            _need(t, torch.int32 if name == "w_q" else dt, name)
        if w_lo is not None:
            _need(w_lo, torch.int32, "w_lo")
        if bias is not None:
            _need(bias, dt, "bias", ndim=1)
        _check_product(x_meta, w_q, w_lo, scales, zeros, bias, None, bits, group_size)
        N = w_q.shape[1]
        flags = ((WQ_FLAG_PDL if pdl else 0) | (WQ_FLAG_PDL_INPUTS_READY if inputs_ready else 0)
                 | (WQ_FLAG_BF16 if dt is torch.bfloat16 else 0))
        self._lib = lib()
        h = ctypes.c_void_p()
        with torch.cuda.device(w_q.device):
            st = self._lib.wq_gemv_plan_create(_ptr(w_q), _ptr(w_lo), _ptr(scales), _ptr(zeros), _ptr(bias),
                                               M, K, N, bits, group_size, flags, ctypes.byref(h))
        _check("wq_gemv_plan_create", st)
        self._h = h.value
        self._keep = (w_q, w_lo, scales, zeros, bias)
        self.dtype, self.device, self.M, self.K, self.N = dt, w_q.device, M, K, N
        self._dev = w_q.get_device()
        self._xshape, self._yshape = (M, K), (M, N)
        self._run = self._lib.wq_gemv_plan_run

    def __call__(self, x, out=None):
        if not (getattr(x, "is_cuda", False) and x.dtype is self.dtype and x.shape == self._xshape
                and x.is_contiguous() and x.get_device() == self._dev):
            raise ValueError(f"x must be a contiguous {self.dtype} CUDA tensor of shape {self._xshape} "
                             f"on {self.device}")
        if out is None:
            out = _torch().empty(self._yshape, dtype=self.dtype, device=x.device)
        elif not (getattr(out, "is_cuda", False) and out.dtype is self.dtype and out.shape == self._yshape
                  and out.is_contiguous() and out.get_device() == self._dev):
            raise ValueError(f"out must be a contiguous {self.dtype} CUDA tensor of shape {self._yshape} "
                             f"on {self.device}")
        st = self._run(self._h, x.data_ptr(), out.data_ptr(), _stream())
        if st != 0:
            raise WQError("wq_gemv_plan_run", st)
        return out

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h:
            self._lib.wq_gemv_plan_destroy(h)


def gemm_workspace_size(M: int, K: int, N: int, bits: int, group_size: int) -> int:
    """Bytes of split-K workspace ``wq_gemm`` uses for this shape on the current device."""
    return int(lib().wq_gemm_workspace_size(M, K, N, bits, group_size))


_workspaces = {}
_ws_sizes = {}


def _cached_workspace(device, nbytes: int):
    """A workspace of at least ``nbytes`` for calls on the current stream of ``device``.

    One buffer per (device, stream): calls on one stream run one after another,
    so they may share it; calls on different streams get their own.  It only
    grows.  Allocated inside a CUDA graph capture it comes from the graph's
    pool and stays valid while cached, like any tensor the capture returns.  A
    captured graph keeps the buffer's address: graphs replayed at the same time
    on different streams must be captured with workspaces of their own
    (``workspace=``).
    """
    if nbytes == 0:
        return None
    torch = _torch()
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def gemm(x, w_q, w_lo, scales, zeros, bits: int, group_size: int, out=None, pdl: bool = False,
         workspace=None, inputs_ready: bool = False, bias=None):
    """y (M, N) = x (M, K) @ dequant(w_q), any M >= 1 (``wq_gemm``), in the type of x.

    ``workspace``: a CUDA uint8 tensor of at least ``gemm_workspace_size(...)``
    bytes for splitting K over a cluster; by default one cached per stream.
    """
    if workspace is not None:
        torch = _torch()
        _need(workspace, torch.uint8, "workspace", ndim=1)
        _same_device(x, workspace=workspace)
    return _product("wq_gemm", x, w_q, w_lo, scales, zeros, bits, group_size, out, pdl, workspace,
                    inputs_ready=inputs_ready, bias=bias)


def device_status(reset: bool = False) -> int:
    """``wq_device_status``: 0, 5 (WQ_ERR_TIMEOUT) if a kernel gave up a bounded
    wait, or 8 (WQ_ERR_CHECK) if a bounds check of the checked build fired."""
    return int(lib().wq_device_status(1 if reset else 0))


def checked_build() -> bool:
    """Whether the loaded library is the checked build (``WQ_LIB=checked``)."""
    return bool(lib().wq_checked_build())


def gemm_noalloc(x, w_q, w_lo, scales, zeros, bits: int, group_size: int, out, pdl: bool = False,
                 bias=None):
    """``wq_gemm_noalloc``: the product into the caller's ``out`` with the
    library's fixed split-K scratch; neither the call nor this wrapper
    allocates device memory."""
    _need(out, _elem_type(x), "out")
    return _product("wq_gemm_noalloc", x, w_q, w_lo, scales, zeros, bits, group_size, out, pdl,
                    bias=bias)


def selftest_wait_timeout(limit_ns: int = 1_000_000) -> int:
    """``wq_selftest_wait_timeout``: run the bounded-wait failure path on purpose
    (a wait on a barrier nothing completes) on the current stream; returns the
    status, 5 (WQ_ERR_TIMEOUT) when the wait gave up as it should."""
    return int(lib().wq_selftest_wait_timeout(int(limit_ns), _stream()))


def matmul(x, w_q, w_lo, scales, zeros, bits: int, group_size: int, out=None, pdl: bool = False,
           workspace=None, inputs_ready: bool = False, bias=None):
    """``wq_matmul``: the product for any M, on ``wq_gemv`` or ``wq_gemm`` by the
    library's measured M crossover (``uses_gemv`` tells which)."""
    if workspace is not None:
        torch = _torch()
        _need(workspace, torch.uint8, "workspace", ndim=1)
        _same_device(x, workspace=workspace)
    return _product("wq_matmul", x, w_q, w_lo, scales, zeros, bits, group_size, out, pdl, workspace,
                    inputs_ready=inputs_ready, bias=bias)


def uses_gemv(M: int, K: int, N: int, bits: int, group_size: int) -> bool:
    return bool(lib().wq_matmul_uses_gemv(M, K, N, bits, group_size))


def mse_search(w, bits: int, group_size: int, maxshrink: float = 0.2, grid: int = 100, norm: float = 2.4,
               patience=None, symmetric: bool = False):
    """``wq_mse_search``: the MSE-observer search of each group's scale and zero
    point over ``int(maxshrink * grid)`` shrink candidates (as the page counts
    them), on the current stream.

    ``w``: (rows, cols) float32 CUDA tensor, groups of ``group_size`` values
    along a row.  ``patience``: None evaluates every candidate.  Returns a dict
    of (rows, cols // group_size) tensors ``step`` (int32), ``scale``,
    ``zero`` and ``err`` (float32); with ``symmetric`` the zero points are 0
    (signed codes)."""
    torch = _torch()
    _need(w, torch.float32, "w")
    rows, cols = w.shape
    steps = int(maxshrink * grid)
    if group_size < 1 or cols % group_size != 0:
        raise ValueError(f"cols={cols} is not a multiple of group_size={group_size}")
    shape = (rows, cols // group_size)
    out = {k: torch.empty(shape, dtype=torch.float32, device=w.device) for k in ("scale", "zero", "err")}
    out["step"] = torch.empty(shape, dtype=torch.int32, device=w.device)
    pat = 0 if patience is None else int(patience)
    if patience is not None and pat < 1:
        raise ValueError("patience must be at least 1 (None evaluates every candidate)")
    ws = torch.empty(1, dtype=torch.int32, device=w.device) if pat else None
    st = lib().wq_mse_search(_ptr(w), rows, cols, group_size, bits, 1 if symmetric else 0, steps, grid,
                             float(norm), pat, _ptr(out["scale"]), _ptr(out["zero"]), _ptr(out["step"]),
                             _ptr(out["err"]), _ptr(ws), 4 if ws is not None else 0, _stream())
    _check("wq_mse_search", st)
    return out


def gptq_quantize(W, H, scale, zero, group_size: int, bits: int, blocksize: int = 128,
                  percdamp: float = 0.01, want_q: bool = True, want_codes: bool = True):
    """``wq_gptq_quantize``: GPTQ block quantisation of ``W`` (rows, cols) with
    the Hessian ``H`` (cols, cols), on the current stream, in fp32.

    ``scale`` / ``zero``: (rows, ceil(cols / group_size)) float32, the zero
    points on the signed scale (0 for symmetric arguments).  Returns a dict:
    ``Q`` (rows, cols) float32, the fake-quantised W; ``codes`` (cols, rows)
    uint8, ``q + 2**(bits-1)``, the K-major codes ``pack_kmajor`` takes;
    ``losses`` (rows,) float32.  A Hessian that is not positive definite shows
    as ``device_status() == 9`` and NaN outputs."""
    torch = _torch()
    _need(W, torch.float32, "W")
    _need(H, torch.float32, "H")
    _need(scale, torch.float32, "scale")
    _need(zero, torch.float32, "zero")
    _same_device(W, H=H, scale=scale, zero=zero)
    rows, cols = W.shape
    if tuple(H.shape) != (cols, cols):
        raise ValueError(f"H has shape {tuple(H.shape)}, expected {(cols, cols)}")
    if group_size < 1:
        raise ValueError("group_size must be at least 1")
    ng = -(-cols // group_size)
    for name, t in (("scale", scale), ("zero", zero)):
        if tuple(t.shape) != (rows, ng):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {(rows, ng)}")
    dev = W.device
    out = {"losses": torch.empty(rows, dtype=torch.float32, device=dev)}
    out["Q"] = torch.empty((rows, cols), dtype=torch.float32, device=dev) if want_q else None
    out["codes"] = torch.empty((cols, rows), dtype=torch.uint8, device=dev) if want_codes else None
    nbytes = lib().wq_gptq_workspace_size(rows, cols)
    if nbytes == 0:
        raise ValueError(f"unsupported shape ({rows}, {cols})")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = lib().wq_gptq_quantize(_ptr(W), _ptr(H), _ptr(scale), _ptr(zero), rows, cols, group_size, bits,
                                blocksize, float(percdamp), _ptr(out["Q"]), _ptr(out["codes"]),
                                _ptr(out["losses"]), _ptr(ws), nbytes, _stream())
    _check("wq_gptq_quantize", st)
    out["workspace"] = ws  # kept alive until the caller drops the result
    return out


_GQ_V = {2: 16, 3: 10, 4: 8, 8: 4}


def from_gptqmodel(qweight, qzeros, bits: int, group_size: int, K: int, dtype=None):
    """``wq_gptqmodel_convert``: GPTQModel (qweight, qzeros) -> this library's
    (w_q, w_lo, zeros).  For 2, 4 and 8 bits w_q is ``qweight`` itself (the same
    K-major words); 3-bit words (10 per int32) become the two planes.  ``zeros``
    has the type ``dtype`` (float16 by default, or bfloat16)."""
    torch = _torch()
    dtype = torch.float16 if dtype is None else dtype
    if dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("zeros are float16 or bfloat16")
    if bits not in _GQ_V:
        raise ValueError(f"the GPTQModel format takes 2, 3, 4 or 8 bits, not {bits}")
    _need(qweight, torch.int32, "qweight")
    _need(qzeros, torch.int32, "qzeros")
    _same_device(qweight, qzeros=qzeros)
    V = _GQ_V[bits]
    N = qweight.shape[1]
    G = K if group_size == -1 else group_size
    if tuple(qweight.shape) != ((K + V - 1) // V, N):
        raise ValueError(f"qweight has shape {tuple(qweight.shape)}; K={K}, {bits}-bit needs {((K + V - 1) // V, N)}")
    if G < 1 or K % G != 0:
        raise ValueError(f"group size {group_size} does not divide K={K}")
    if tuple(qzeros.shape) != (K // G, (N + V - 1) // V):
        raise ValueError(f"qzeros has shape {tuple(qzeros.shape)}; needs {(K // G, (N + V - 1) // V)}")
    dev = qweight.device
    zeros = torch.empty((K // G, N), dtype=dtype, device=dev)
    if bits == 3:
        hs, ls = words_shape(K, N, 3)
        w_q = torch.empty(hs, dtype=torch.int32, device=dev)
        w_lo = torch.empty(ls, dtype=torch.int32, device=dev)
    else:
        w_q, w_lo = qweight, None
    flags = WQ_FLAG_BF16 if dtype is torch.bfloat16 else 0
    st = lib().wq_gptqmodel_convert(_ptr(qweight), _ptr(qzeros), K, N, bits, group_size,
                                    _ptr(w_q) if bits == 3 else None, _ptr(w_lo), _ptr(zeros), flags, _stream())
    _check("wq_gptqmodel_convert", st)
    return w_q, w_lo, zeros


def gptqmodel_quantized_matmul(x, qweight, qzeros, scales, bits: int, group_size: int, out=None):
    """The README's ``gptqmodel_quantized_matmul``: y = x @ dequantize(qweight)
    with GPTQModel operands, through ``from_gptqmodel`` and ``matmul``."""
    w_q, w_lo, zeros = from_gptqmodel(qweight, qzeros, bits, group_size, x.shape[1], dtype=_elem_type(x))
    return matmul(x, w_q, w_lo, scales, zeros, bits, group_size, out=out)
