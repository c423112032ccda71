"""Python binding of libfp4fqt.so (the C ABI declared in include/fp4.h).

Argument marshalling only: every step of the quantizers, GEMMs and the
linear layer runs in the library's CUDA kernels.  PyTorch supplies device
memory and the current CUDA stream.  There is no fallback: if the library is
missing or cannot be loaded, every call raises.

The function names mirror the C entry points: ``fp4_quantize``,
``fp4_gemm``, ``fqt_linear_fwd``, ``fqt_linear_bwd``.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp4fqt.so")

NVFP4, MXFP4 = 0, 1
RTN, SR, QUEST = 0, 1, 2
BLOCK_1D, BLOCK_2D = 0, 1
OUT_BF16, OUT_F32 = 0, 1
RHT_FPROP, RHT_DGRAD, RHT_WGRAD = 1, 2, 4

STATUS = {0: "FP4_OK", 1: "FP4_ERR_NULL", 2: "FP4_ERR_SHAPE", 3: "FP4_ERR_ALIGN",
          4: "FP4_ERR_FORMAT", 5: "FP4_ERR_WORKSPACE", 6: "FP4_ERR_CUDA",
          7: "FP4_ERR_NONFINITE", 8: "FP4_ERR_TIMEOUT", 9: "FP4_ERR_UNSUPPORTED"}

# Every symbol include/fp4.h declares.
EXPORTS = ("fp4_qtensor_sizes", "fp4_qparams_default", "fp4_workspace_bytes", "fp4_quantize",
           "fp4_gemm", "fqt_linear_cfg_default", "fqt_linear_fwd", "fqt_linear_bwd",
           "fp4_read_device_status", "fp4_clear_device_status", "fp4_status_str",
           "fp4_abi_version", "fp4_kernel_launches", "fp4_gemm_noalloc", "fp4_mma_rate",
           "fp4_quant_noise", "fp4_gemm_quant", "fp4_gemm_quant_ex", "fp4_allreduce_sum_f32")


class Fp4Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class QTensorC(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("scales_mma", C.c_void_p),
                ("amax", C.c_void_p), ("s_dec", C.c_void_p), ("rows", C.c_int64),
                ("cols", C.c_int64), ("fmt", C.c_int32), ("block", C.c_int32)]


class QParamsC(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("block", C.c_int32), ("round", C.c_int32),
                ("round_t", C.c_int32), ("rht_n", C.c_int32), ("rht_n_t", C.c_int32),
                ("rht_seed", C.c_uint64), ("sr_seed", C.c_uint64), ("sr_stream", C.c_uint32),
                ("sr_stream_t", C.c_uint32), ("amax_in", C.c_void_p), ("amax_in_t", C.c_void_p)]


class LinearCfgC(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("w_block", C.c_int32), ("round_fwd", C.c_int32),
                ("round_bwd", C.c_int32), ("round_x_t", C.c_int32), ("rht_mask", C.c_int32),
                ("rht_n", C.c_int32), ("out_dtype", C.c_int32), ("seed", C.c_uint64)]


class SavedC(C.Structure):
    _fields_ = [("xq", QTensorC), ("xq_t", QTensorC), ("wq", QTensorC), ("wq_t", QTensorC),
                ("dyq", QTensorC), ("dyq_t", QTensorC)]


_lib = None


def load() -> C.CDLL:
    """Load the in-tree CUDA library; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m fp4_fully_quantized_b200.build`")
    L = C.CDLL(LIB_PATH)
    vp, i64, i32, sz = C.c_void_p, C.c_int64, C.c_int32, C.c_size_t
    L.fp4_qtensor_sizes.restype = None
    L.fp4_qtensor_sizes.argtypes = [i64, i64, i32, i32, C.POINTER(sz), C.POINTER(sz), C.POINTER(sz)]
    L.fp4_qparams_default.restype = None
    L.fp4_qparams_default.argtypes = [C.POINTER(QParamsC)]
    L.fp4_workspace_bytes.restype = sz
    L.fp4_workspace_bytes.argtypes = [i64, i64, i64]
    L.fp4_quantize.restype = i32
    L.fp4_quantize.argtypes = [vp, i64, i64, i64, C.POINTER(QParamsC), C.POINTER(QTensorC),
                               C.POINTER(QTensorC), vp, sz, vp]
    L.fp4_gemm.restype = i32
    L.fp4_gemm.argtypes = [C.POINTER(QTensorC), C.POINTER(QTensorC), C.c_float, vp, i64, i32, vp,
                           vp, sz, vp]
    L.fqt_linear_cfg_default.restype = None
    L.fqt_linear_cfg_default.argtypes = [C.POINTER(LinearCfgC), i32]
    L.fqt_linear_fwd.restype = i32
    L.fqt_linear_fwd.argtypes = [C.POINTER(LinearCfgC), i64, i64, i64, vp, vp, vp,
                                 C.POINTER(SavedC), vp, sz, vp]
    L.fqt_linear_bwd.restype = i32
    L.fqt_linear_bwd.argtypes = [C.POINTER(LinearCfgC), i64, i64, i64, vp, C.POINTER(SavedC), vp,
                                 vp, vp, sz, vp]
    L.fp4_read_device_status.restype = i32
    L.fp4_read_device_status.argtypes = [vp, vp]
    L.fp4_clear_device_status.restype = i32
    L.fp4_clear_device_status.argtypes = [vp, vp]
    L.fp4_status_str.restype = C.c_char_p
    L.fp4_status_str.argtypes = [i32]
    L.fp4_abi_version.restype = i32
    L.fp4_abi_version.argtypes = []
    L.fp4_kernel_launches.restype = C.c_uint64
    L.fp4_kernel_launches.argtypes = []
    L.fp4_mma_rate.restype = i32
    L.fp4_mma_rate.argtypes = [i32, i32, C.POINTER(C.c_float), vp, sz, vp]
    L.fp4_gemm_quant.restype = i32
    L.fp4_gemm_quant.argtypes = [C.POINTER(QTensorC), C.POINTER(QTensorC), C.c_float, vp,
                                 C.POINTER(QTensorC), vp, vp, sz, vp]
    L.fp4_gemm_quant_ex.restype = i32
    L.fp4_gemm_quant_ex.argtypes = [C.POINTER(QTensorC), C.POINTER(QTensorC), C.c_float, vp, i32,
                                    C.c_uint64, C.c_uint32, C.POINTER(QTensorC), vp, i64, vp, vp,
                                    sz, vp]
    L.fp4_allreduce_sum_f32.restype = i32
    L.fp4_allreduce_sum_f32.argtypes = [vp, vp, i64, vp]
    L.fp4_quant_noise.restype = i32
    L.fp4_quant_noise.argtypes = [vp, i64, i64, i64, C.POINTER(QTensorC), vp, vp, sz, vp]
    L.fp4_gemm_noalloc.restype = i32
    L.fp4_gemm_noalloc.argtypes = [C.POINTER(QTensorC), C.POINTER(QTensorC), C.c_float, vp, i64,
                                   i32, vp, vp]
    _lib = L
    return L


def kernel_launches() -> int:
    """Kernels this library has enqueued in this process so far."""
    return int(load().fp4_kernel_launches())


def _check(code: int, where: str):
    if code != 0:
        raise Fp4Error(code, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def qtensor_sizes(rows: int, cols: int, fmt: int = NVFP4, block: int = BLOCK_1D):
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    load().fp4_qtensor_sizes(rows, cols, fmt, block, C.byref(a), C.byref(b), C.byref(c))
    return a.value, b.value, c.value


@dataclass
class QTensor:
    """Device buffers of one quantized operand of logical shape [rows, cols]."""
    rows: int
    cols: int
    fmt: int
    block: int
    codes: torch.Tensor
    scales: torch.Tensor | None
    scales_mma: torch.Tensor | None
    amax: torch.Tensor
    s_dec: torch.Tensor
    _c: QTensorC = field(default=None, repr=False)

    @staticmethod
    def empty(rows: int, cols: int, fmt: int = NVFP4, block: int = BLOCK_1D, device="cuda",
              logical_scales: bool = True, mma_scales: bool = True) -> "QTensor":
        nc, ns, nm = qtensor_sizes(rows, cols, fmt, block)
        dev = torch.device(device)
        codes = torch.empty(max(nc, 16), dtype=torch.uint8, device=dev)[:nc]
        scales = torch.empty(max(ns, 16), dtype=torch.uint8, device=dev)[:ns] if logical_scales else None
        mma = torch.zeros(max(nm, 16), dtype=torch.uint8, device=dev)[:nm] if mma_scales else None
        scal = torch.zeros(2, dtype=torch.float32, device=dev)
        q = QTensor(rows, cols, fmt, block, codes, scales, mma, scal[0:1], scal[1:2])
        q._c = QTensorC(_ptr(codes), _ptr(scales), _ptr(mma), _ptr(q.amax), _ptr(q.s_dec),
                        rows, cols, fmt, block)
        return q

    @property
    def c(self) -> QTensorC:
        return self._c

    def codes_2d(self) -> torch.Tensor:
        return self.codes.view(self.rows, self.cols // 2)

    def scales_2d(self) -> torch.Tensor:
        if self.block == BLOCK_2D:
            return self.scales.view(self.rows // 16, self.cols // 16)
        return self.scales.view(self.rows, self.cols // (32 if self.fmt == MXFP4 else 16))


class Workspace:
    """Caller-owned device workspace; its first 256 bytes are the status block."""

    def __init__(self, M: int = 128, N: int = 128, K: int = 64, device="cuda"):
        n = load().fp4_workspace_bytes(M, N, K)
        self.buf = torch.zeros(n, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return C.c_void_p(self.buf.data_ptr())

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def status(self, stream=None) -> int:
        return load().fp4_read_device_status(self.ptr, _stream(stream))

    def clear(self, stream=None):
        _check(load().fp4_clear_device_status(self.ptr, _stream(stream)), "fp4_clear_device_status")


def fp4_quantize(x: torch.Tensor, out: QTensor | None = None, out_t: QTensor | None = None,
                 fmt: int = NVFP4, block: int = BLOCK_1D, round: int = RTN, round_t: int = RTN,
                 rht_n: int = 0, rht_n_t: int = 0, rht_seed: int = 0, sr_seed: int = 0,
                 sr_stream: int = 0, sr_stream_t: int = 0, amax_in: torch.Tensor | None = None,
                 amax_in_t: torch.Tensor | None = None, ws: Workspace | None = None, stream=None):
    """Quantize a BF16 [rows, cols] CUDA tensor into `out` and/or `out_t` (x^T)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    assert x.stride(1) == 1
    p = QParamsC(fmt, block, round, round_t, rht_n, rht_n_t, rht_seed, sr_seed, sr_stream,
                 sr_stream_t, _ptr(amax_in), _ptr(amax_in_t))
    code = load().fp4_quantize(_ptr(x), x.shape[0], x.shape[1], x.stride(0), C.byref(p),
                               C.byref(out.c) if out is not None else None,
                               C.byref(out_t.c) if out_t is not None else None,
                               ws.ptr if ws is not None else None,
                               ws.nbytes if ws is not None else 0, _stream(stream))
    _check(code, "fp4_quantize")


def fp4_gemm(a: QTensor, b: QTensor, out: torch.Tensor, alpha: float = 1.0,
             c_amax: torch.Tensor | None = None, ws: Workspace | None = None, stream=None):
    """out[M, N] = alpha * s_dec(a) * s_dec(b) * a_hat @ b_hat^T (FP32 accumulation)."""
    assert out.dtype in (torch.bfloat16, torch.float32) and out.is_cuda and out.stride(1) == 1
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    if ws is None:
        ws = Workspace(a.rows, b.rows, a.cols, device=out.device)
    code = load().fp4_gemm(C.byref(a.c), C.byref(b.c), float(alpha), _ptr(out), out.stride(0), od,
                           _ptr(c_amax), ws.ptr, ws.nbytes, _stream(stream))
    _check(code, "fp4_gemm")


def fp4_gemm_noalloc(a: QTensor, b: QTensor, out: torch.Tensor, alpha: float = 1.0,
                     c_amax: torch.Tensor | None = None, stream=None):
    """fp4_gemm without a workspace: for callers that cannot allocate device
    memory.  Its scratch is a small array held by the library on each device;
    calls that overlap on the GPU share it and race."""
    assert out.dtype in (torch.bfloat16, torch.float32) and out.is_cuda and out.stride(1) == 1
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    code = load().fp4_gemm_noalloc(C.byref(a.c), C.byref(b.c), float(alpha), _ptr(out),
                                   out.stride(0), od, _ptr(c_amax), _stream(stream))
    _check(code, "fp4_gemm_noalloc")


def mma_rate(variant: int = 0, iters: int = 20000, stream=None) -> float:
    """Achieved TFLOP/s of back-to-back block-scaled NVFP4 MMAs (see fp4.h)."""
    ws = Workspace()
    out = C.c_float()
    _check(load().fp4_mma_rate(variant, iters, C.byref(out), ws.ptr, ws.nbytes, _stream(stream)),
           "fp4_mma_rate")
    return float(out.value)


def fp4_gemm_quant(a: QTensor, b: QTensor, out: QTensor, amax_in: torch.Tensor, alpha: float = 1.0,
                   c_amax: torch.Tensor | None = None, ws: Workspace | None = None, stream=None):
    """out = NVFP4 1x16 RTN of (alpha * s_dec(a) * s_dec(b) * a_hat @ b_hat^T), encoded in
    the GEMM epilogue with the supplied tensor amax (device float32 tensor)."""
    if ws is None:
        ws = Workspace(a.rows, b.rows, a.cols, device=amax_in.device)
    code = load().fp4_gemm_quant(C.byref(a.c), C.byref(b.c), float(alpha), _ptr(amax_in),
                                 C.byref(out.c), _ptr(c_amax), ws.ptr, ws.nbytes, _stream(stream))
    _check(code, "fp4_gemm_quant")


def fp4_gemm_quant_ex(a: QTensor, b: QTensor, out: QTensor, amax_in: torch.Tensor,
                      round: int = RTN, sr_seed: int = 0, sr_stream: int = 0,
                      c_bf16: torch.Tensor | None = None, alpha: float = 1.0,
                      c_amax: torch.Tensor | None = None, ws: Workspace | None = None, stream=None):
    """fp4_gemm_quant with RTN or SR encoding and an optional BF16 copy of the
    FP32 result (c_bf16, [M, >= N] BF16 CUDA tensor)."""
    if ws is None:
        ws = Workspace(a.rows, b.rows, a.cols, device=amax_in.device)
    if c_bf16 is not None:
        assert c_bf16.dtype == torch.bfloat16 and c_bf16.is_cuda and c_bf16.stride(1) == 1
    code = load().fp4_gemm_quant_ex(C.byref(a.c), C.byref(b.c), float(alpha), _ptr(amax_in),
                                    int(round), int(sr_seed), int(sr_stream), C.byref(out.c),
                                    _ptr(c_bf16), c_bf16.stride(0) if c_bf16 is not None else 0,
                                    _ptr(c_amax), ws.ptr, ws.nbytes, _stream(stream))
    _check(code, "fp4_gemm_quant_ex")


def fp4_quant_noise(x: torch.Tensor, q: QTensor, sums: torch.Tensor, ws: Workspace | None = None,
                    stream=None):
    """sums[0] = sum x^2, sums[1] = sum (deq(q) - x)^2 (float64 CUDA tensor of 2)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda and x.stride(1) == 1
    assert sums.dtype == torch.float64 and sums.numel() >= 2 and sums.is_cuda
    code = load().fp4_quant_noise(_ptr(x), x.shape[0], x.shape[1], x.stride(0), C.byref(q.c),
                                  _ptr(sums), ws.ptr if ws is not None else None,
                                  ws.nbytes if ws is not None else 0, _stream(stream))
    _check(code, "fp4_quant_noise")


class NcclComm:
    """An NCCL communicator for fp4_allreduce_sum_f32 (plumbing only): made
    with the process's NCCL, its unique id passed from rank 0 to the others
    through the torch.distributed process group `group` (any backend)."""

    def __init__(self, rank: int, world: int, group=None):
        import torch.distributed as dist
        self._nccl = C.CDLL("libnccl.so.2", mode=os.RTLD_NOLOAD | os.RTLD_LAZY) \
            if _nccl_loaded() else C.CDLL("libnccl.so.2")
        uid = _NcclUniqueId()
        if rank == 0 and self._nccl.ncclGetUniqueId(C.byref(uid)) != 0:
            raise RuntimeError("ncclGetUniqueId failed")
        if world > 1:
            box = [bytes(uid.internal)]
            dist.broadcast_object_list(box, src=0, group=group)
            C.memmove(C.byref(uid), box[0], 128)
        self.comm = C.c_void_p()
        self._nccl.ncclCommInitRank.argtypes = [C.POINTER(C.c_void_p), C.c_int, _NcclUniqueId, C.c_int]
        if self._nccl.ncclCommInitRank(C.byref(self.comm), world, uid, rank) != 0:
            raise RuntimeError("ncclCommInitRank failed")

    def destroy(self):
        if self.comm:
            self._nccl.ncclCommDestroy(self.comm)
            self.comm = C.c_void_p()


class _NcclUniqueId(C.Structure):
    """ncclUniqueId: 128 opaque bytes, passed to ncclCommInitRank by value."""
    _fields_ = [("internal", C.c_char * 128)]


def _nccl_loaded() -> bool:
    try:
        C.CDLL("libnccl.so.2", mode=os.RTLD_NOLOAD | os.RTLD_LAZY)
        return True
    except OSError:
        return False


def fp4_allreduce_sum_f32(comm: NcclComm, buf: torch.Tensor, stream=None):
    """buf (FP32 CUDA tensor) <- its sum over the communicator's ranks."""
    assert buf.dtype == torch.float32 and buf.is_cuda and buf.is_contiguous()
    _check(load().fp4_allreduce_sum_f32(comm.comm, _ptr(buf), buf.numel(), _stream(stream)),
           "fp4_allreduce_sum_f32")


def linear_cfg(fmt: int = NVFP4, **overrides) -> LinearCfgC:
    cfg = LinearCfgC()
    load().fqt_linear_cfg_default(C.byref(cfg), fmt)
    for k, v in overrides.items():
        setattr(cfg, k, v)
    return cfg


@dataclass
class Saved:
    """Quantized operands of one linear layer (M tokens, N out, K in)."""
    xq: QTensor
    xq_t: QTensor
    wq: QTensor
    wq_t: QTensor
    dyq: QTensor
    dyq_t: QTensor
    _c: SavedC = field(default=None, repr=False)

    @staticmethod
    def empty(M: int, N: int, K: int, cfg: LinearCfgC, device="cuda",
              logical_scales: bool = False) -> "Saved":
        f, wb = cfg.fmt, cfg.w_block
        mk = lambda r, c, b=BLOCK_1D: QTensor.empty(r, c, f, b, device, logical_scales, True)
        s = Saved(mk(M, K), mk(K, M), mk(N, K, wb), mk(K, N, wb), mk(M, N), mk(N, M))
        s._c = SavedC(s.xq.c, s.xq_t.c, s.wq.c, s.wq_t.c, s.dyq.c, s.dyq_t.c)
        return s


def fqt_linear_fwd(cfg: LinearCfgC, x: torch.Tensor, w: torch.Tensor, y: torch.Tensor,
                   saved: Saved, ws: Workspace, stream=None):
    M, K = x.shape
    N = w.shape[0]
    assert x.is_contiguous() and w.is_contiguous() and y.is_contiguous()
    code = load().fqt_linear_fwd(C.byref(cfg), M, N, K, _ptr(x), _ptr(w), _ptr(y),
                                 C.byref(saved._c), ws.ptr, ws.nbytes, _stream(stream))
    _check(code, "fqt_linear_fwd")


def fqt_linear_bwd(cfg: LinearCfgC, dy: torch.Tensor, saved: Saved, dx: torch.Tensor,
                   dw: torch.Tensor, ws: Workspace, stream=None):
    M, N = dy.shape
    K = dx.shape[1]
    assert dy.is_contiguous() and dx.is_contiguous() and dw.is_contiguous()
    assert dw.dtype == torch.float32
    code = load().fqt_linear_bwd(C.byref(cfg), M, N, K, _ptr(dy), C.byref(saved._c), _ptr(dx),
                                 _ptr(dw), ws.ptr, ws.nbytes, _stream(stream))
    _check(code, "fqt_linear_bwd")
