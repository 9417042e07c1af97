"""Thin ctypes binding of libmosaicq (include/mosaicq.h).

Argument marshalling only: every step of the decomposition, packing and
product runs inside the library (host C++ for packing, CUDA kernels for the
product). PyTorch supplies device memory and streams. There is no fallback:
if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmosaicq.so")

OK, INVALID_ARG, UNSUPPORTED, OUT_OF_MEMORY, CUDA, DEVICE_TIMEOUT = range(6)
PATH_AUTO, PATH_DECODE, PATH_PREFILL = range(3)
UNFUSED_NOALLOC_MAX_OUTPUTS = 2 * 1024 * 1024  # MQ_UNFUSED_NOALLOC_MAX_OUTPUTS
_PATHS = {"auto": PATH_AUTO, "decode": PATH_DECODE, "prefill": PATH_PREFILL}


class MQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


class _PackOpts(ctypes.Structure):
    _fields_ = [("group_size", ctypes.c_int32), ("residual_density", ctypes.c_double),
                ("residual_blocks", ctypes.c_int32), ("block_fraction", ctypes.c_double),
                ("channel_weight", ctypes.c_void_p)]


class _Decomp(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("s", ctypes.c_void_p), ("z", ctypes.c_void_p),
                ("row_ptr", ctypes.c_void_p), ("col", ctypes.c_void_p),
                ("qr", ctypes.c_void_p), ("sr", ctypes.c_void_p)]


class _HostPacked(ctypes.Structure):
    _fields_ = [("qweight", ctypes.c_void_p), ("sz", ctypes.c_void_p),
                ("row_ptr", ctypes.c_void_p), ("col", ctypes.c_void_p),
                ("val", ctypes.c_void_p), ("rscale", ctypes.c_void_p)]


class _Info(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("nnz", ctypes.c_int64),
                ("group_size", ctypes.c_int32), ("device", ctypes.c_int32),
                ("device_bytes", ctypes.c_int64), ("max_row_nnz", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmosaicq.so is not built ({LIB_PATH}); run "
                          "`python -m bit_gemm_w4_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "mq_pack": ([vp, i64, i64, ctypes.POINTER(_PackOpts), vp, ctypes.POINTER(vp)], st),
        "mq_linear": ([vp, vp, i64, vp, vp], st),
        "mq_linear_path": ([vp, vp, i64, vp, vp, ctypes.c_int], st),
        "mq_linear_prefetch": ([vp, vp, i64, vp, vp, vp], st),
        "mq_linear_unfused": ([vp, vp, i64, vp, vp, ctypes.c_size_t, vp], st),
        "mq_linear_unfused_noalloc": ([vp, vp, i64, vp, vp], st),
        "mq_quantize_activations": ([vp, i64, i64, vp, vp, vp], st),
        "mq_selftest_bounded_wait": ([i64, ctypes.POINTER(ctypes.c_int32)], st),
        "mq_read_probe": ([vp, i64, vp, vp], st),
        "mq_w4a4_workspace_bytes": ([vp, i64], i64),
        "mq_linear_w4a4": ([vp, vp, i64, vp, vp, ctypes.c_size_t, vp], st),
        "mq_free": ([vp], None),
        "mq_residual_nnz": ([i64, i64, ctypes.POINTER(_PackOpts), ctypes.POINTER(i64)], st),
        "mq_pack_host": ([vp, i64, i64, ctypes.POINTER(_PackOpts), ctypes.POINTER(_HostPacked)], st),
        "mq_prefill_lists_host": ([i64, i64, vp, vp, vp, vp, vp], st),
        "mq_wide_lists_host": ([i64, i64, vp, vp, vp, vp, vp, vp, ctypes.POINTER(i64)], st),
        "mq_tile_lists_host": ([i64, i64, vp, vp, vp, vp, vp], st),
        "mq_pack_decomposed": ([ctypes.POINTER(_Decomp), vp, ctypes.POINTER(vp)], st),
        "mq_get_info": ([vp, ctypes.POINTER(_Info)], st),
        "mq_export": ([vp, ctypes.POINTER(_HostPacked)], st),
        "mq_export_blocks": ([vp, vp, vp, vp, ctypes.POINTER(i64)], st),
        "mq_block_tiles_host": ([ctypes.POINTER(_Decomp), vp, vp, vp, ctypes.POINTER(i64)], st),
        "mq_device_error": ([vp, vp, ctypes.POINTER(ctypes.c_int32)], st),
        "mq_strerror": ([st], ctypes.c_char_p),
        "mq_last_error": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def lib():
    return _lib


def _check(status: int, where: str):
    if status != OK:
        detail = _lib.mq_last_error().decode() or _lib.mq_strerror(status).decode()
        raise MQError(status, where, detail)


def _opts(rho: float, group: int = 128, block_fraction=None, channel_weight=None):
    """Pack options: row mode (rho) unless block_fraction is given, which
    selects block mode. Returns (options, kept) where kept holds the arrays
    the options point at for the duration of the call."""
    if block_fraction is None:
        return _PackOpts(group, float(rho), 0, 0.0, None), None
    h = None
    if channel_weight is not None:
        h = np.ascontiguousarray(channel_weight, dtype=np.float32)
    return _PackOpts(group, 0.0, 1, float(block_fraction), None if h is None else h.ctypes.data), h


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data if a.size else 0


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def residual_nnz(N: int, K: int, rho: float, group: int = 128, *, block_fraction=None) -> int:
    out = ctypes.c_int64()
    o, _ = _opts(rho, group, block_fraction)
    _check(_lib.mq_residual_nnz(N, K, ctypes.byref(o), ctypes.byref(out)), "mq_residual_nnz")
    return out.value


def _alloc_packed(N: int, K: int, nnz: int):
    arrs = dict(qweight=np.zeros((N, K // 8), np.uint32), sz=np.zeros((N, K // 128), np.uint32),
                row_ptr=np.zeros(N + 1, np.int32), col=np.zeros(nnz, np.uint16),
                val=np.zeros((nnz + 1) // 2, np.uint8), rscale=np.zeros(N, np.uint16))
    hp = _HostPacked(*(_ptr(arrs[k]) for k in
                       ("qweight", "sz", "row_ptr", "col", "val", "rscale")))
    return arrs, hp


def pack_host(W: np.ndarray, rho: float, group: int = 128, *, block_fraction=None,
              channel_weight=None) -> dict:
    """Decompose and pack on the host (no CUDA call). Returns the packed arrays.
    block_fraction selects block mode (see mq_pack_opts)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    nnz = residual_nnz(N, K, rho, group, block_fraction=block_fraction)
    arrs, hp = _alloc_packed(N, K, nnz)
    o, keep = _opts(rho, group, block_fraction, channel_weight)
    _check(_lib.mq_pack_host(_ptr(W), N, K, ctypes.byref(o), ctypes.byref(hp)), "mq_pack_host")
    del keep
    return arrs


def prefill_lists_host(N: int, K: int, packed: dict):
    """The prefill kernel's residual lists of a host pack (pack_host's arrays):
    (ptr int32 [ceil(N/128) * K/64 * 4 + 1], ent uint32 [nnz]); no CUDA call."""
    row_ptr = np.ascontiguousarray(packed["row_ptr"], np.int32)
    col = np.ascontiguousarray(packed["col"], np.uint16)
    val = np.ascontiguousarray(packed["val"], np.uint8)
    nnz = int(row_ptr[-1])
    ptr = np.zeros(((N + 127) // 128) * (K // 64) * 4 + 1, np.int32)
    ent = np.zeros(max(nnz, 1), np.uint32)
    _check(_lib.mq_prefill_lists_host(N, K, _ptr(row_ptr), _ptr(col), _ptr(val), _ptr(ptr), _ptr(ent)),
           "mq_prefill_lists_host")
    return ptr, ent[:nnz]


def wide_lists_host(N: int, K: int, packed: dict):
    """The wide decode kernel's residual lists of a host pack: (ptr int32,
    off uint16 [slices, 136], ent uint16 [nnz], longest slice); no CUDA call."""
    row_ptr = np.ascontiguousarray(packed["row_ptr"], np.int32)
    col = np.ascontiguousarray(packed["col"], np.uint16)
    val = np.ascontiguousarray(packed["val"], np.uint8)
    nnz = int(row_ptr[-1])
    slices = ((N + 127) // 128) * ((K + 255) // 256)
    ptr = np.zeros(slices + 1, np.int32)
    off = np.zeros((slices, 136), np.uint16)
    ent = np.zeros(max(nnz, 1), np.uint16)
    mx = ctypes.c_int64(0)
    _check(_lib.mq_wide_lists_host(N, K, _ptr(row_ptr), _ptr(col), _ptr(val), _ptr(ptr), _ptr(off),
                                   _ptr(ent), ctypes.byref(mx)), "mq_wide_lists_host")
    return ptr, off, ent[:nnz], int(mx.value)


def tile_lists_host(N: int, K: int, packed: dict):
    """The tall-layer decode kernel's residual lists of a host pack: (ptr
    int32 [ceil(N/16) * K/128 + 1], ent uint16 [nnz]); no CUDA call."""
    row_ptr = np.ascontiguousarray(packed["row_ptr"], np.int32)
    col = np.ascontiguousarray(packed["col"], np.uint16)
    val = np.ascontiguousarray(packed["val"], np.uint8)
    nnz = int(row_ptr[-1])
    ptr = np.zeros(((N + 15) // 16) * (K // 128) + 1, np.int32)
    ent = np.zeros(max(nnz, 1), np.uint16)
    _check(_lib.mq_tile_lists_host(N, K, _ptr(row_ptr), _ptr(col), _ptr(val), _ptr(ptr), _ptr(ent)),
           "mq_tile_lists_host")
    return ptr, ent[:nnz]


def selftest_bounded_wait(limit_cycles: int = 1 << 20) -> list:
    """Run the bounded-wait self-test on the current device (synchronous):
    [completed phase seen, stuck wait returned, later wait returned, error
    code]; [1, 0, 0, 2] when the bounded wait works."""
    out = (ctypes.c_int32 * 4)()
    _check(_lib.mq_selftest_bounded_wait(int(limit_cycles), out), "mq_selftest_bounded_wait")
    return list(out)


def _decomp_struct(d: dict, keep: dict) -> "_Decomp":
    return _Decomp(int(d["N"]), int(d["K"]),
                   *(_ptr(keep[k]) for k in ("q", "s", "z", "row_ptr", "col", "qr", "sr")))


def block_tiles_host(d: dict) -> dict:
    """The library's host-side block tiles of a decomposition given as arrays
    (as for Weight.pack_decomposed); MQError with UNSUPPORTED when the
    residual is not made of whole 16 x 64 blocks."""
    keep = dict(
        q=np.ascontiguousarray(d["q"], np.uint8),
        s=np.ascontiguousarray(np.asarray(d["s"], np.float16).view(np.uint16)),
        z=np.ascontiguousarray(np.asarray(d["z"], np.float16).view(np.uint16)),
        row_ptr=np.ascontiguousarray(d["row_ptr"], np.int64),
        col=np.ascontiguousarray(d["col"], np.int32),
        qr=np.ascontiguousarray(d["qr"], np.int8),
        sr=np.ascontiguousarray(np.asarray(d["sr"], np.float16).view(np.uint16)))
    dc = _decomp_struct(d, keep)
    n = ctypes.c_int64()
    _check(_lib.mq_block_tiles_host(ctypes.byref(dc), None, None, None, ctypes.byref(n)),
           "mq_block_tiles_host")
    N = int(d["N"])
    out = dict(blk_ptr=np.zeros(N // 16 + 1, np.int32), blk_col=np.zeros(max(n.value, 1), np.uint16),
               blk_q=np.zeros((max(n.value, 1), 16, 8), np.uint32))
    _check(_lib.mq_block_tiles_host(ctypes.byref(dc), _ptr(out["blk_ptr"]), _ptr(out["blk_col"]),
                                    _ptr(out["blk_q"]), ctypes.byref(n)), "mq_block_tiles_host")
    out["blk_col"] = out["blk_col"][:n.value]
    out["blk_q"] = out["blk_q"][:n.value]
    return out


def read_probe(buf_ptr: int, nbytes: int, sink_ptr: int, *, stream=None) -> None:
    """One launch of the library's streaming-read probe (mq_read_probe) over
    nbytes of device memory at buf_ptr; sink_ptr is a 4-byte device word."""
    _check(_lib.mq_read_probe(ctypes.c_void_p(buf_ptr), int(nbytes), ctypes.c_void_p(sink_ptr),
                              _stream(stream)), "mq_read_probe")


def quantize_activations(X, *, stream=None):
    """Per-token int4 codes (int8 [M, K]) and fp32 scales [M] of bf16 X on
    its device (the W4A4 quantization stage)."""
    import torch
    X = X.contiguous()
    M, K = X.shape
    codes = torch.empty((M, K), dtype=torch.int8, device=X.device)
    scales = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(_lib.mq_quantize_activations(X.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(),
                                        _stream(stream)), "mq_quantize_activations")
    return codes, scales


class Weight:
    """A packed weight on the current CUDA device (owns its device buffers)."""

    def __init__(self, handle: int):
        self._h = handle

    @classmethod
    def pack(cls, W: np.ndarray, rho: float = 0.0, group: int = 128, stream=None, *,
             block_fraction=None, channel_weight=None) -> "Weight":
        """Decompose, pack and upload fp32 W [N, K]. Row mode keeps k_n =
        floor(rho*K + 0.5) residual entries per row; block_fraction selects
        block mode (16x64 blocks ranked by the channel-weighted squared error,
        channel_weight = K diagonal-Hessian weights or None for all ones)."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        h = ctypes.c_void_p()
        o, keep = _opts(rho, group, block_fraction, channel_weight)
        _check(_lib.mq_pack(_ptr(W), N, K, ctypes.byref(o), _stream(stream), ctypes.byref(h)),
               "mq_pack")
        del keep
        return cls(h.value)

    @classmethod
    def pack_decomposed(cls, d: dict, stream=None) -> "Weight":
        """Pack a decomposition given as arrays (q u8 [N,K], s/z fp16 [N,G],
        row_ptr, col, qr, sr fp16 [N])."""
        N, K = int(d["N"]), int(d["K"])
        keep = dict(
            q=np.ascontiguousarray(d["q"], np.uint8),
            s=np.ascontiguousarray(np.asarray(d["s"], np.float16).view(np.uint16)),
            z=np.ascontiguousarray(np.asarray(d["z"], np.float16).view(np.uint16)),
            row_ptr=np.ascontiguousarray(d["row_ptr"], np.int64),
            col=np.ascontiguousarray(d["col"], np.int32),
            qr=np.ascontiguousarray(d["qr"], np.int8),
            sr=np.ascontiguousarray(np.asarray(d["sr"], np.float16).view(np.uint16)))
        dc = _decomp_struct(d, keep)
        h = ctypes.c_void_p()
        _check(_lib.mq_pack_decomposed(ctypes.byref(dc), _stream(stream), ctypes.byref(h)),
               "mq_pack_decomposed")
        return cls(h.value)

    @property
    def handle(self) -> int:
        return self._h

    def info(self) -> dict:
        i = _Info()
        _check(_lib.mq_get_info(self._h, ctypes.byref(i)), "mq_get_info")
        return {f: getattr(i, f) for f, _ in _Info._fields_}

    def linear(self, X, Y=None, *, stream=None, path: str = "auto"):
        """Y = X @ W_hat^T for bf16 X [M, K] on the packing device."""
        import torch
        info = self.info()
        if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != info["K"]:
            raise ValueError("X must be a bf16 [M, K] tensor")
        X = X.contiguous()
        if Y is None:
            Y = torch.empty((X.shape[0], info["N"]), dtype=torch.bfloat16, device=X.device)
        self.linear_raw(X.data_ptr(), X.shape[0], Y.data_ptr(), stream=stream, path=path)
        return Y

    def linear_raw(self, x_ptr: int, M: int, y_ptr: int, *, stream=None, path: str = "auto",
                   next_weight: "Weight | None" = None):
        """mq_linear on raw device pointers; with next_weight (decode only),
        mq_linear_prefetch: that weight is brought into L2 meanwhile."""
        if next_weight is not None and path == "auto":
            _check(_lib.mq_linear_prefetch(self._h, x_ptr, M, y_ptr, next_weight._h,
                                           _stream(stream)), "mq_linear_prefetch")
            return
        _check(_lib.mq_linear_path(self._h, x_ptr, M, y_ptr, _stream(stream), _PATHS[path]),
               "mq_linear")

    def linear_unfused(self, X, Y=None, workspace=None, *, stream=None):
        """The split comparison path: dense kernel into an fp32 workspace,
        then a separate residual kernel (caller-owned workspace of M*N fp32)."""
        import torch
        info = self.info()
        X = X.contiguous()
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, info["N"]), dtype=torch.bfloat16, device=X.device)
        if workspace is None:
            workspace = torch.empty((M, info["N"]), dtype=torch.float32, device=X.device)
        _check(_lib.mq_linear_unfused(self._h, X.data_ptr(), M, Y.data_ptr(),
                                      workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)), "mq_linear_unfused")
        return Y

    def linear_w4a4(self, X, Y=None, workspace=None, *, stream=None):
        """The W4A4 variant: per-token int4 activation codes in a
        caller-owned workspace (mq_w4a4_workspace_bytes), then the fused
        int4 x int4 pass (decode kernels for M <= 16, the tcgen05 prefill
        kernel above, which needs K % 256 == 0)."""
        import torch
        info = self.info()
        X = X.contiguous()
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, info["N"]), dtype=torch.bfloat16, device=X.device)
        if workspace is None:
            nbytes = max(16, int(_lib.mq_w4a4_workspace_bytes(self._h, M)))
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=X.device)
        _check(_lib.mq_linear_w4a4(self._h, X.data_ptr(), M, Y.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "mq_linear_w4a4")
        return Y

    def linear_unfused_noalloc(self, X, Y=None, *, stream=None):
        """The split comparison path with the library's built-in scratch (no
        workspace argument and no device allocation by the library)."""
        import torch
        info = self.info()
        X = X.contiguous()
        if Y is None:
            Y = torch.empty((X.shape[0], info["N"]), dtype=torch.bfloat16, device=X.device)
        _check(_lib.mq_linear_unfused_noalloc(self._h, X.data_ptr(), X.shape[0], Y.data_ptr(),
                                              _stream(stream)), "mq_linear_unfused_noalloc")
        return Y

    def export_blocks(self) -> dict:
        """The device copy of the block tiles (blk_ptr, blk_col, blk_q);
        MQError with UNSUPPORTED when the residual is not block-structured."""
        n = ctypes.c_int64()
        _check(_lib.mq_export_blocks(self._h, None, None, None, ctypes.byref(n)), "mq_export_blocks")
        N = self.info()["N"]
        out = dict(blk_ptr=np.zeros(N // 16 + 1, np.int32), blk_col=np.zeros(max(n.value, 1), np.uint16),
                   blk_q=np.zeros((max(n.value, 1), 16, 8), np.uint32))
        _check(_lib.mq_export_blocks(self._h, _ptr(out["blk_ptr"]), _ptr(out["blk_col"]),
                                     _ptr(out["blk_q"]), ctypes.byref(n)), "mq_export_blocks")
        out["blk_col"] = out["blk_col"][:n.value]
        out["blk_q"] = out["blk_q"][:n.value]
        return out

    def export(self) -> dict:
        info = self.info()
        arrs, hp = _alloc_packed(info["N"], info["K"], info["nnz"])
        _check(_lib.mq_export(self._h, ctypes.byref(hp)), "mq_export")
        return arrs

    def device_error(self, stream=None) -> int:
        code = ctypes.c_int32()
        st = _lib.mq_device_error(self._h, _stream(stream), ctypes.byref(code))
        if st not in (OK, DEVICE_TIMEOUT):
            _check(st, "mq_device_error")
        return code.value

    def free(self):
        if self._h:
            _lib.mq_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass
