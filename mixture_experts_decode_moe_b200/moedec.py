"""Python binding of libmoedec (argument marshalling only).

Every function here forwards to the C ABI declared in include/moedec.h with
the same name; all computation runs in the library's CUDA kernels. Tensors
are torch CUDA tensors (PyTorch only provides device memory and streams).
Importing this module raises if libmoedec.so has not been built: there is no
fallback path.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoedec.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoedec.so is not built ({LIB_PATH}); run "
                      "`python -m mixture_experts_decode_moe_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(5)
MOE_W_BF16, MOE_W_INT4_G64 = 0, 1
MOE_EXPERT_SWIGLU, MOE_EXPERT_LINEAR = 0, 1
MOE_LAYOUT_PLANAR, MOE_LAYOUT_CHANNEL_MAJOR = 0, 1
MOE_STACK_PRE_RMSNORM = 1
MOE_INJECT_BARRIER_EXTRA_ARRIVAL = 1
MOE_RECOVERY_RANK = 32
MOE_STATIC_SCRATCH_BYTES = 256 * 1024

EXPORTS = [
    "moe_abi_version", "moe_status_string", "moe_workspace_bytes", "moe_workspace_init",
    "moe_get_status", "moe_route_topk", "moe_expert_forward", "moe_layer_forward",
    "moe_stack_forward", "moe_channel_topk_forward", "moe_touched_experts",
    "moe_layer_forward_static", "moe_channel_stack_forward", "moe_reader_build", "moe_reader_screen",
    "moe_workspace_set_wait_budget", "moe_workspace_set_inject", "moe_recovery_scratch_bytes",
    "moe_recovery_build", "moe_channel_recover", "moe_reader_codes_coordinate_major",
    "moe_reader_screen_partial",
]


class LayerDesc(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("E", ctypes.c_int32), ("I", ctypes.c_int32), ("k", ctypes.c_int32),
        ("kind", ctypes.c_int32), ("wtype", ctypes.c_int32), ("layout", ctypes.c_int32),
        ("I_shared", ctypes.c_int32),
        ("router", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("up", ctypes.c_void_p),
        ("down_t", ctypes.c_void_p), ("gate_s", ctypes.c_void_p), ("up_s", ctypes.c_void_p),
        ("down_s", ctypes.c_void_p), ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
        ("sh_down_t", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_lib.moe_abi_version.restype = ctypes.c_int
_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_status_string.argtypes = [ctypes.c_int]
_lib.moe_workspace_bytes.restype = _S
_lib.moe_workspace_bytes.argtypes = [ctypes.POINTER(LayerDesc), _I]
_lib.moe_workspace_init.argtypes = [_P, _S, _P]
_lib.moe_get_status.argtypes = [_P, _P]
_lib.moe_route_topk.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _S, _P]
_lib.moe_expert_forward.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _P, _S, _P]
_lib.moe_layer_forward.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _P, _P, _S, _P]
_lib.moe_stack_forward.argtypes = [ctypes.POINTER(LayerDesc), _I, _P, _I, ctypes.c_uint32, _P, _P, _P, _P, _P, _P, _S, _P]
_lib.moe_channel_topk_forward.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _I, _P, _P, _P,
                                          _P, _P, _P, _S, _P]
_lib.moe_touched_experts.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _P]
class SketchDesc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("dnorm", ctypes.c_void_p)]


_lib.moe_channel_stack_forward.argtypes = [ctypes.POINTER(LayerDesc), _I, _P, ctypes.c_uint32, _P,
                                           ctypes.POINTER(SketchDesc), _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _S,
                                           _P]
_lib.moe_layer_forward_static.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _P, _P, _P]
_lib.moe_reader_build.argtypes = [ctypes.POINTER(LayerDesc), _P, _P, _P, _P, _P, _P]
_lib.moe_reader_screen.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]
_lib.moe_reader_codes_coordinate_major.argtypes = [ctypes.POINTER(LayerDesc), _P, _P, _P]
_lib.moe_reader_screen_partial.argtypes = [ctypes.POINTER(LayerDesc), _P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                                           _P]
_lib.moe_recovery_scratch_bytes.argtypes = [ctypes.POINTER(LayerDesc)]
_lib.moe_recovery_build.argtypes = [ctypes.POINTER(LayerDesc), _P, _P, _P, _S, _P]
_lib.moe_channel_recover.argtypes = [ctypes.POINTER(LayerDesc), _I, _P, _P, _P, _P, _I, _P, _P, _P, _P]
_lib.moe_workspace_set_wait_budget.argtypes = [_P, ctypes.c_ulonglong, _P]
_lib.moe_workspace_set_inject.argtypes = [_P, ctypes.c_uint32, _P]
for _f in EXPORTS[3:]:
    getattr(_lib, _f).restype = ctypes.c_int
_lib.moe_recovery_scratch_bytes.restype = _S


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")
        self.status = status


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def moe_abi_version() -> int:
    return _lib.moe_abi_version()


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def make_desc(H, E, I, k, *, kind=MOE_EXPERT_SWIGLU, wtype=MOE_W_BF16, layout=MOE_LAYOUT_PLANAR,
              router=None, gate=None, up=None, down_t=None, gate_s=None, up_s=None, down_s=None,
              sh_gate=None, sh_up=None, sh_down_t=None) -> LayerDesc:
    """Build a descriptor from tensors (None for absent pieces)."""
    I_shared = 0 if sh_gate is None else int(sh_gate.shape[0])
    d = LayerDesc(H, E, I, k, kind, wtype, layout, I_shared)
    for name, t in (("router", router), ("gate", gate), ("up", up), ("down_t", down_t),
                    ("gate_s", gate_s), ("up_s", up_s), ("down_s", down_s), ("sh_gate", sh_gate),
                    ("sh_up", sh_up), ("sh_down_t", sh_down_t)):
        setattr(d, name, None if t is None else t.data_ptr())
    return d


def moe_workspace_bytes(desc: LayerDesc, B: int) -> int:
    return int(_lib.moe_workspace_bytes(ctypes.byref(desc), B))


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def alloc_workspace(desc: LayerDesc, B: int, device="cuda") -> torch.Tensor:
    """Allocate (through torch) and clear a workspace for `desc` at batch B."""
    n = moe_workspace_bytes(desc, B)
    if n == 0:
        raise MoeError(MOE_ERR_INVALID, "moe_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


def moe_get_status(ws: torch.Tensor, stream=None) -> int:
    return int(_lib.moe_get_status(_ptr(ws), _stream(stream)))


def moe_workspace_set_wait_budget(ws: torch.Tensor, cycles: int, stream=None):
    _check(_lib.moe_workspace_set_wait_budget(_ptr(ws), cycles, _stream(stream)), "moe_workspace_set_wait_budget")


def moe_workspace_set_inject(ws: torch.Tensor, flags: int, stream=None):
    _check(_lib.moe_workspace_set_inject(_ptr(ws), flags, _stream(stream)), "moe_workspace_set_inject")


def moe_route_topk(x, router, k, ids, w, margin=None, ws=None, stream=None):
    B, H = x.shape
    E = router.shape[0]
    _check(_lib.moe_route_topk(_ptr(x), _ptr(router), B, H, E, k, _ptr(ids), _ptr(w), _ptr(margin),
                               _ptr(ws), ws.numel(), _stream(stream)), "moe_route_topk")


def moe_expert_forward(desc, x, ids, w, y, ws, stream=None):
    _check(_lib.moe_expert_forward(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(y),
                                   _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_forward")


def moe_layer_forward(desc, x, y, ws, x_next=None, ids_out=None, w_out=None, stream=None):
    _check(_lib.moe_layer_forward(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(y), _ptr(x_next),
                                  _ptr(ids_out), _ptr(w_out), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_layer_forward")


def moe_stack_forward(descs, x, x_out, ws, x_hist=None, y_hist=None, ids_hist=None, w_hist=None,
                      flags=0, stream=None):
    arr = (LayerDesc * len(descs))(*descs)
    _check(_lib.moe_stack_forward(arr, len(descs), _ptr(x), x.shape[0], flags, _ptr(x_out), _ptr(x_hist),
                                  _ptr(y_hist), _ptr(ids_hist), _ptr(w_hist), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_stack_forward")


def moe_channel_topk_forward(desc, x, ids, w, scores, keep, y, sectors, ws, kept=None, union_count=None,
                             union_sectors=None, stream=None):
    _check(_lib.moe_channel_topk_forward(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(ids), _ptr(w),
                                         _ptr(scores), keep, _ptr(y), _ptr(kept), _ptr(sectors),
                                         _ptr(union_count), _ptr(union_sectors), _ptr(ws), ws.numel(),
                                         _stream(stream)), "moe_channel_topk_forward")


def make_sketch(codes, scales, dnorm) -> SketchDesc:
    """One layer's channel-screen sketch (moe_reader_build's buffers)."""
    return SketchDesc(codes.data_ptr(), scales.data_ptr(), dnorm.data_ptr())


def moe_channel_stack_forward(descs, x, scores, keep, x_out, sectors, ws, x_hist=None, y_hist=None, ids_hist=None,
                              w_hist=None, kept_hist=None, flags=0, sketches=None, signs=None, stream=None):
    """scores [L, E, I] given, or scores=None with sketches (one make_sketch()
    per layer) and signs: the kernel screens every layer itself."""
    arr = (LayerDesc * len(descs))(*descs)
    sk = None if sketches is None else (SketchDesc * len(sketches))(*sketches)
    _check(_lib.moe_channel_stack_forward(arr, len(descs), _ptr(x), flags, _ptr(scores), sk, _ptr(signs), keep,
                                          _ptr(x_out),
                                          _ptr(x_hist), _ptr(y_hist), _ptr(ids_hist), _ptr(w_hist),
                                          _ptr(kept_hist), _ptr(sectors), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_channel_stack_forward")


def moe_touched_experts(ids, E, count, bitmap=None, offsets=None, pairs=None, stream=None):
    B, k = ids.shape
    _check(_lib.moe_touched_experts(_ptr(ids), B, k, E, _ptr(count), _ptr(bitmap), _ptr(offsets),
                                    _ptr(pairs), _stream(stream)), "moe_touched_experts")


def moe_layer_forward_static(desc, x, y, x_next=None, ids_out=None, w_out=None, status_out=None, stream=None):
    """moe_layer_forward without a caller workspace: the library's fixed scratch
    array is used instead (see include/moedec.h for who needs this and the
    rules on sharing it)."""
    _check(_lib.moe_layer_forward_static(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(y), _ptr(x_next),
                                         _ptr(ids_out), _ptr(w_out), _ptr(status_out), _stream(stream)),
           "moe_layer_forward_static")


def reader_sketch_shapes(desc: LayerDesc) -> dict:
    """Shapes of the channel screen's sketch buffers for one layer."""
    n = desc.E * desc.I
    return {"codes": (n, 2, desc.H // 16), "scales": (n, 2, desc.H // 128), "rho": (n, 2, desc.H // 128),
            "dnorm": (n,)}


def moe_reader_build(desc, signs, codes, scales, rho, dnorm, stream=None):
    _check(_lib.moe_reader_build(ctypes.byref(desc), _ptr(signs), _ptr(codes), _ptr(scales), _ptr(rho),
                                 _ptr(dnorm), _stream(stream)), "moe_reader_build")


def moe_reader_screen(desc, x, ids, w, signs, codes, scales, dnorm, scores, est=None, stream=None):
    _check(_lib.moe_reader_screen(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(signs),
                                  _ptr(codes), _ptr(scales), _ptr(dnorm), _ptr(scores), _ptr(est),
                                  _stream(stream)), "moe_reader_screen")


def moe_recovery_build(desc, U, coeffs, stream=None):
    """Load-time recovery map of one channel-major layer: U [H, 32] fp32 and
    coeffs [E*I, 32] (fp16 bit patterns, any 2-byte dtype). The build's
    scratch is allocated through torch and released when the call returns
    (stream-ordered by torch's allocator)."""
    n = int(_lib.moe_recovery_scratch_bytes(ctypes.byref(desc)))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_recovery_scratch_bytes")
    scratch = torch.empty(n, dtype=torch.uint8, device=U.device)
    _check(_lib.moe_recovery_build(ctypes.byref(desc), _ptr(U), _ptr(coeffs), _ptr(scratch), n, _stream(stream)),
           "moe_recovery_build")
    return scratch


def moe_channel_recover(desc, ids, w, est, kept, keep, U, coeffs, y, stream=None):
    _check(_lib.moe_channel_recover(ctypes.byref(desc), ids.shape[0], _ptr(ids), _ptr(w), _ptr(est), _ptr(kept),
                                    keep, _ptr(U), _ptr(coeffs), _ptr(y), _stream(stream)), "moe_channel_recover")


def reader_cmaj_shape(desc: LayerDesc) -> tuple:
    """Shape of the coordinate-major code buffer of one layer."""
    return (desc.E, 2, desc.H, desc.I // 16)


def moe_reader_codes_coordinate_major(desc, codes, codes_cmaj, stream=None):
    _check(_lib.moe_reader_codes_coordinate_major(ctypes.byref(desc), _ptr(codes), _ptr(codes_cmaj),
                                                  _stream(stream)), "moe_reader_codes_coordinate_major")


def moe_reader_screen_partial(desc, x, ids, w, signs, codes_cmaj, scales, dnorm, m, scores, est=None, stream=None):
    _check(_lib.moe_reader_screen_partial(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(signs),
                                          _ptr(codes_cmaj), _ptr(scales), _ptr(dnorm), m, _ptr(scores), _ptr(est),
                                          _stream(stream)), "moe_reader_screen_partial")
