"""Python binding of libtq (argument marshalling only).

Every function here forwards to the C function of the same name in
``libtq.so`` (declared in include/tq.h); all arithmetic runs in the library's
CUDA kernels.  PyTorch is used for device memory and streams only.  There is
no fallback: if the library is missing or the device is not a B200 the calls
raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

(TQ_OK, TQ_ERR_SHAPE, TQ_ERR_ALIGN, TQ_ERR_NULL, TQ_ERR_ARCH, TQ_ERR_WORKSPACE, TQ_ERR_CUDA, TQ_ERR_TIMEOUT,
 TQ_ERR_SCRATCH, TQ_ERR_VALUE) = range(10)
TQ_ENCODE_MAX_REFITS = 16
TQ_F32, TQ_F16 = 0, 1
OPS = ("q", "k", "v", "o", "gate", "up", "down")

EXPORTS = ("tq_pack_info", "tq_decode", "tq_rht", "tq_gemv_workspace", "tq_gemv", "tq_gemm_workspace", "tq_gemm",
           "tq_workspace_init", "tq_stack_phase_seed", "tq_layer_phase_workspace", "tq_layer_stack_workspace",
           "tq_layer_phase", "tq_layer_stack", "tq_status_string", "tq_last_cuda_error", "tq_gemv_noalloc",
           "tq_layer_stack_buffers", "tq_layer_stack_outputs", "tq_encode", "tq_ldlq_workspace", "tq_ldlq_encode",
           "tq_layer_stack_ex", "tq_workspace_status", "tq_gemm_ex")
TQ_STATUS_OFFSET = 65532
TQ_GEMV_MAX_K = 53760


class TqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().tq_status_string(status).decode()
        if status == TQ_ERR_CUDA:
            msg += f" (cudaError {_lib().tq_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


class tq_weight_t(ctypes.Structure):
    _fields_ = [("codes_d", ctypes.c_void_p), ("scales_d", ctypes.c_void_p), ("codebook_d", ctypes.c_void_p),
                ("n", ctypes.c_int32), ("k", ctypes.c_int32)]


class tq_pack_info_t(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("k", ctypes.c_int32), ("group", ctypes.c_int32), ("block", ctypes.c_int32),
                ("rht_block", ctypes.c_int32), ("n_states", ctypes.c_int32), ("code_bytes", ctypes.c_int64),
                ("scale_bytes", ctypes.c_int64), ("codebook_bytes", ctypes.c_int64), ("packed_bytes", ctypes.c_int64),
                ("bits_per_weight", ctypes.c_double)]


class tq_layer_t(ctypes.Structure):
    _fields_ = [(op, tq_weight_t) for op in OPS]


class tq_stack_options_t(ctypes.Structure):
    _fields_ = [("spin_limit", ctypes.c_uint32), ("test_skip_arrive", ctypes.c_int32)]


_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtq.so not built ({LIB_PATH}); run decode_matmul_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
        W = ctypes.POINTER(tq_weight_t)
        LY = ctypes.POINTER(tq_layer_t)
        szp = ctypes.POINTER(ctypes.c_size_t)
        sig = {
            "tq_pack_info": ([i32, i32, ctypes.POINTER(tq_pack_info_t)], ctypes.c_int),
            "tq_decode": ([W, vp, vp], ctypes.c_int),
            "tq_rht": ([vp, i32, i32, u64, vp, i32, vp], ctypes.c_int),
            "tq_gemv_workspace": ([i32, i32, szp], ctypes.c_int),
            "tq_gemv": ([W, vp, vp, vp, sz, vp], ctypes.c_int),
            "tq_gemv_noalloc": ([W, vp, vp, vp], ctypes.c_int),
            "tq_gemm_workspace": ([i32, i32, i32, szp], ctypes.c_int),
            "tq_gemm": ([W, vp, i32, vp, vp, sz, vp], ctypes.c_int),
            "tq_gemm_ex": ([W, vp, i32, vp, vp, sz, ctypes.POINTER(tq_stack_options_t), vp], ctypes.c_int),
            "tq_workspace_init": ([vp, sz, vp], ctypes.c_int),
            "tq_stack_phase_seed": ([u64, i32, i32], u64),
            "tq_layer_phase_workspace": ([LY, i32, i32, szp], ctypes.c_int),
            "tq_layer_stack_workspace": ([LY, i32, i32, szp], ctypes.c_int),
            "tq_layer_phase": ([LY, i32, vp, i32, u64, vp, vp, vp, sz, vp], ctypes.c_int),
            "tq_layer_stack": ([LY, i32, vp, i32, u64, vp, vp, sz, vp], ctypes.c_int),
            "tq_layer_stack_ex": ([LY, i32, vp, i32, u64, vp, vp, sz, ctypes.POINTER(tq_stack_options_t), vp],
                                  ctypes.c_int),
            "tq_workspace_status": ([vp, ctypes.POINTER(ctypes.c_int32), vp], ctypes.c_int),
            "tq_layer_stack_buffers": ([LY, i32, i32, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "tq_layer_stack_outputs": ([LY, i32, i32, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "tq_encode": ([vp, i32, i32, vp, ctypes.c_float, i32, vp, vp, vp, vp], ctypes.c_int),
            "tq_ldlq_workspace": ([i32, i32, szp], ctypes.c_int),
            "tq_ldlq_encode": ([vp, i32, i32, vp, vp, ctypes.c_float, i32, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "tq_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "tq_last_cuda_error": ([], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _ = i64
        _L = L
    return _L


def lib():
    """The loaded libtq (ctypes.CDLL)."""
    return _lib()


def _ok(st: int, where: str):
    if st != TQ_OK:
        raise TqError(st, where)


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ---- device-side containers ----------------------------------------------------

class DeviceWeight:
    """Caller-owned device copy of one trellis-coded weight (torch tensors)."""

    def __init__(self, codes, scales, codebook, n: int, k: int):
        self.codes, self.scales, self.codebook, self.n, self.k = codes, scales, codebook, n, k

    @classmethod
    def from_host(cls, codes: np.ndarray, scales: np.ndarray, codebook, n: int, k: int, device="cuda"):
        import torch
        c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).to(device)
        s = torch.from_numpy(np.ascontiguousarray(scales, dtype=np.uint16).view(np.int16)).to(device)
        if isinstance(codebook, np.ndarray):
            codebook = torch.from_numpy(np.ascontiguousarray(codebook, dtype=np.uint16).view(np.int16)).to(device)
        return cls(c, s, codebook, n, k)

    def struct(self) -> tq_weight_t:
        return tq_weight_t(self.codes.data_ptr(), self.scales.data_ptr(), self.codebook.data_ptr(), self.n, self.k)


def layer_struct(weights: dict) -> tq_layer_t:
    return tq_layer_t(*[weights[op].struct() for op in OPS])


# ---- the ABI ---------------------------------------------------------------------

def tq_pack_info(n: int, k: int) -> dict:
    out = tq_pack_info_t()
    _ok(_lib().tq_pack_info(n, k, ctypes.byref(out)), "tq_pack_info")
    return {f: getattr(out, f) for f, _ in tq_pack_info_t._fields_}


def tq_decode(w: DeviceWeight, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((w.n, w.k), dtype=torch.int16, device=w.codes.device)
    ws = w.struct()
    _ok(_lib().tq_decode(ctypes.byref(ws), _ptr(out), _stream(stream)), "tq_decode")
    return out


def tq_rht(x_bf16, seed: int, out_dtype: int = TQ_F32, out=None, stream=None):
    """x_bf16: int16 (bf16 bits) or bfloat16 tensor [m][k] on the device."""
    import torch
    m, k = x_bf16.shape
    if out is None:
        out = torch.empty((m, k), dtype=torch.float32 if out_dtype == TQ_F32 else torch.float16, device=x_bf16.device)
    _ok(_lib().tq_rht(_ptr(x_bf16), m, k, seed, _ptr(out), out_dtype, _stream(stream)), "tq_rht")
    return out


def tq_gemv_workspace(n: int, k: int) -> int:
    b = ctypes.c_size_t()
    _ok(_lib().tq_gemv_workspace(n, k, ctypes.byref(b)), "tq_gemv_workspace")
    return b.value


def tq_gemm_workspace(n: int, k: int, m: int) -> int:
    b = ctypes.c_size_t()
    _ok(_lib().tq_gemm_workspace(n, k, m, ctypes.byref(b)), "tq_gemm_workspace")
    return b.value


def workspace(nbytes: int, device="cuda", stream=None):
    """A zeroed device workspace of at least nbytes (16-byte aligned)."""
    import torch
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _ok(_lib().tq_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "tq_workspace_init")
    return ws


def tq_gemv(w: DeviceWeight, x_rot, y=None, ws=None, stream=None):
    import torch
    if y is None:
        y = torch.empty(w.n, dtype=torch.float32, device=x_rot.device)
    if ws is None:
        ws = workspace(tq_gemv_workspace(w.n, w.k), x_rot.device, stream)
    s = w.struct()
    _ok(_lib().tq_gemv(ctypes.byref(s), _ptr(x_rot), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)), "tq_gemv")
    return y


def tq_gemv_noalloc(w: DeviceWeight, x_rot, y, stream=None):
    """Batch-1 GEMV with the library's built-in scratch (no workspace); y must
    be given, so this call allocates nothing."""
    s = w.struct()
    _ok(_lib().tq_gemv_noalloc(ctypes.byref(s), _ptr(x_rot), _ptr(y), _stream(stream)), "tq_gemv_noalloc")
    return y


def tq_gemm(w: DeviceWeight, x_rot_f16, y=None, ws=None, stream=None):
    import torch
    m = x_rot_f16.shape[0]
    if y is None:
        y = torch.empty((m, w.n), dtype=torch.float32, device=x_rot_f16.device)
    if ws is None:
        ws = workspace(tq_gemm_workspace(w.n, w.k, m), x_rot_f16.device, stream)
    s = w.struct()
    _ok(_lib().tq_gemm(ctypes.byref(s), _ptr(x_rot_f16), m, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
        "tq_gemm")
    return y


def tq_gemm_ex(w: DeviceWeight, x_rot_f16, y, ws, spin_limit: int = 0, test_skip_arrive: int = -1, stream=None):
    """tq_gemm with options: the tcgen05 kernel's poll limit (0 = the default)
    and its timeout test hook (a thread block whose MMA wait runs out; -1 =
    off).  Both act from 33 tokens on."""
    opt = tq_stack_options_t(spin_limit, test_skip_arrive)
    s = w.struct()
    _ok(_lib().tq_gemm_ex(ctypes.byref(s), _ptr(x_rot_f16), x_rot_f16.shape[0], _ptr(y), _ptr(ws), ws.numel(),
                          ctypes.byref(opt), _stream(stream)), "tq_gemm_ex")
    return y


def tq_stack_phase_seed(seed: int, layer: int, phase: int) -> int:
    return int(_lib().tq_stack_phase_seed(seed, layer, phase))


def tq_layer_phase_workspace(layer: tq_layer_t, phase: int, m: int) -> int:
    b = ctypes.c_size_t()
    _ok(_lib().tq_layer_phase_workspace(ctypes.byref(layer), phase, m, ctypes.byref(b)), "tq_layer_phase_workspace")
    return b.value


def tq_layer_stack_workspace(layers, m: int) -> int:
    arr = (tq_layer_t * len(layers))(*layers)
    b = ctypes.c_size_t()
    _ok(_lib().tq_layer_stack_workspace(arr, len(layers), m, ctypes.byref(b)), "tq_layer_stack_workspace")
    return b.value


def tq_layer_phase(layer: tq_layer_t, phase: int, x_bf16, phase_seed: int, y, handoff, ws, stream=None):
    m = x_bf16.shape[0]
    _ok(_lib().tq_layer_phase(ctypes.byref(layer), phase, _ptr(x_bf16), m, phase_seed, _ptr(y), _ptr(handoff),
                              _ptr(ws), ws.numel(), _stream(stream)), "tq_layer_phase")


def tq_layer_stack_buffers(layers, m: int):
    """Workspace byte offsets of the last layer's q, o, gate handoffs, its
    input h and the last phase's fp32 y."""
    arr = (tq_layer_t * len(layers))(*layers)
    out = (ctypes.c_size_t * 5)()
    _ok(_lib().tq_layer_stack_buffers(arr, len(layers), m, out), "tq_layer_stack_buffers")
    return list(out)


def tq_layer_stack_outputs(layers, m: int):
    """Workspace byte offsets of the fp32 outputs of the last layer's four
    phases (equal offsets when m > 16: only the last phase's survive)."""
    arr = (tq_layer_t * len(layers))(*layers)
    out = (ctypes.c_size_t * 4)()
    _ok(_lib().tq_layer_stack_outputs(arr, len(layers), m, out), "tq_layer_stack_outputs")
    return list(out)


class StackArgs:
    """Pre-marshalled arguments of tq_layer_stack (so a timed loop only calls C)."""

    def __init__(self, layers, m: int):
        self.n_layers = len(layers)
        self.arr = (tq_layer_t * len(layers))(*layers)
        self.m = m


def tq_layer_stack(args: StackArgs, h_in, seed: int, h_out, ws, stream=None):
    _ok(_lib().tq_layer_stack(args.arr, args.n_layers, _ptr(h_in), args.m, seed, _ptr(h_out), _ptr(ws), ws.numel(),
                              _stream(stream)), "tq_layer_stack")


def tq_layer_stack_ex(args: StackArgs, h_in, seed: int, h_out, ws, spin_limit: int = 0, test_skip_arrive: int = -1,
                      stream=None):
    """tq_layer_stack with options: the bounded waits' poll limit (0 = the
    default) and the timeout test hook (a thread block that skips its arrive
    at the first grid barrier; -1 = off)."""
    opt = tq_stack_options_t(spin_limit, test_skip_arrive)
    _ok(_lib().tq_layer_stack_ex(args.arr, args.n_layers, _ptr(h_in), args.m, seed, _ptr(h_out), _ptr(ws),
                                 ws.numel(), ctypes.byref(opt), _stream(stream)), "tq_layer_stack_ex")


def tq_workspace_status(ws, stream=None) -> int:
    """The workspace's device status word (TQ_OK or TQ_ERR_TIMEOUT) once the
    stream has reached this call (synchronises the stream)."""
    v = ctypes.c_int32()
    _ok(_lib().tq_workspace_status(_ptr(ws), ctypes.byref(v), _stream(stream)), "tq_workspace_status")
    return v.value


def tq_encode(w_rot, codebook, gain: float, refits: int = 1, codes=None, scales=None, err=None, want_err=True,
              stream=None):
    """Trellis-encode rotated weights w_rot (fp32 [n][k] on the device).
    codebook: int16 (fp16 bits) tensor [8*256*4] on the device.  Returns
    (codes uint8 [n][k/4], scales int16 fp16 bits [n][k/256], err fp32
    [n][k/256] or None)."""
    import torch
    n, k = w_rot.shape
    dev = w_rot.device
    if codes is None:
        codes = torch.empty((n, k // 4), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((n, k // 256), dtype=torch.int16, device=dev)
    if err is None and want_err:
        err = torch.empty((n, k // 256), dtype=torch.float32, device=dev)
    _ok(_lib().tq_encode(_ptr(w_rot), n, k, _ptr(codebook), float(gain), int(refits), _ptr(codes), _ptr(scales),
                         _ptr(err), _stream(stream)), "tq_encode")
    return codes, scales, err


def tq_ldlq_workspace(n: int, k: int) -> int:
    b = ctypes.c_size_t()
    _ok(_lib().tq_ldlq_workspace(n, k, ctypes.byref(b)), "tq_ldlq_workspace")
    return b.value


def tq_ldlq_encode(w_rot, u, codebook, gain: float, refits: int = 1, codes=None, scales=None, err=None,
                   want_err=True, ws=None, stream=None):
    """Block LDLQ encoding of rotated weights w_rot (fp32 [n][k], device) with
    the Hessian factor u (fp32 [k][k], device).  Returns (codes, scales, err)
    as tq_encode."""
    import torch
    n, k = w_rot.shape
    dev = w_rot.device
    if codes is None:
        codes = torch.empty((n, k // 4), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((n, k // 256), dtype=torch.int16, device=dev)
    if err is None and want_err:
        err = torch.empty((n, k // 256), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(tq_ldlq_workspace(n, k), dtype=torch.uint8, device=dev)
    _ok(_lib().tq_ldlq_encode(_ptr(w_rot), n, k, _ptr(u), _ptr(codebook), float(gain), int(refits), _ptr(codes),
                              _ptr(scales), _ptr(err), _ptr(ws), ws.numel(), _stream(stream)), "tq_ldlq_encode")
    return codes, scales, err
