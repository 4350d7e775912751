"""ctypes binding of libeta.so: the C ABI declared in include/eta.h, one Python
function per entry point with the same name.  Argument marshalling only: torch
tensors are turned into device pointers, and every non-OK status raises.

The library must be built (python -m long_context_decoding_eta_b200.build); there
is no fallback of any kind when it is missing.  With ETA_CHECKED=1 in the
environment the range-checked build (libeta_checked.so, `build --checked`) is
loaded instead: same entry points, same outputs, every computed global index
checked on the device (include/eta.h, ETA_DEVSTAT_BOUNDS).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(
    _HERE, "libeta_checked.so" if os.environ.get("ETA_CHECKED") == "1" else "libeta.so")

ETA_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported shape",
                3: "workspace missing or too small", 4: "CUDA error",
                5: "device wait timed out", 6: "non-finite query",
                7: "out-of-range index (checked build)"}
BOUND = {"exact": 0, "prob": 1, "prob_dim": 2}
CENT = {"f32": 0, "bf16": 1}
PRUNE = {"skip": 0, "floor": 1}
TAIL_BLOCK = -1
DEVSTAT_TIMEOUT, DEVSTAT_NONFINITE_Q, DEVSTAT_BAD_BLOCK, DEVSTAT_BAD_LENGTH = 1, 2, 4, 8
DEVSTAT_BOUNDS = 0x10

EXPORTS = ("eta_build_block_meta", "eta_predict_tau", "eta_screen_workspace_size",
           "eta_screen", "eta_decode_workspace_size", "eta_decode", "eta_dense_decode",
           "eta_calibrate_const_tau", "eta_status_from_device", "eta_status_string",
           "eta_set_decode_engine", "eta_get_decode_engine", "eta_decode_static",
           "eta_decode_static_max_workspace", "eta_selftest_wait_timeout", "eta_prefill",
           "eta_decode_step_workspace_size", "eta_decode_step", "eta_lse_merge",
           "eta_append_and_predict_tau", "eta_screen_launches", "eta_decode_launches",
           "eta_set_prefill_kernel", "eta_get_prefill_kernel", "eta_prefill_kernel_for",
           "eta_build_checked", "eta_selftest_bounds", "eta_set_screen_engine",
           "eta_get_screen_engine")
ENGINE = {"auto": 0, "tcgen05": 1, "fma": 2}
PREFILL_KERNEL = {"auto": 0, "one_tile": 1, "two_tile": 2}


class EtaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code} ({STATUS_NAMES.get(code, '?')})")
        self.code = code


class Dims(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("d", C.c_int32),
                ("blk", C.c_int32), ("T_max", C.c_int32)]

    @classmethod
    def of(cls, B, Hq, Hkv, d, blk, T_max):
        return cls(int(B), int(Hq), int(Hkv), int(d), int(blk), int(T_max))

    def __repr__(self):
        return (f"Dims(B={self.B}, Hq={self.Hq}, Hkv={self.Hkv}, d={self.d}, blk={self.blk}, "
                f"T_max={self.T_max})")


_lib: Optional[C.CDLL] = None
P = C.c_void_p
I32 = C.c_int32
F32 = C.c_float
DIMS = C.POINTER(Dims)


def lib() -> C.CDLL:
    """Loads libeta.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m long_context_decoding_eta_b200.build`")
    L = C.CDLL(LIB_PATH)
    L.eta_build_block_meta.argtypes = [DIMS, P, P, P, I32, I32, I32, P, P, P, P, P, P, P]
    L.eta_predict_tau.argtypes = [DIMS, P, P, P, P, P, P, P]
    L.eta_screen_workspace_size.argtypes = [DIMS]
    L.eta_screen_workspace_size.restype = C.c_size_t
    L.eta_screen_launches.argtypes = [DIMS, I32]
    L.eta_screen_launches.restype = I32
    L.eta_decode_launches.argtypes = [DIMS]
    L.eta_decode_launches.restype = I32
    L.eta_screen.argtypes = [DIMS, P, P, I32, P, P, P, P, P, I32, F32, F32, P, P, P, P, P, P,
                             C.c_size_t, P, P]
    L.eta_decode_workspace_size.argtypes = [DIMS]
    L.eta_decode_workspace_size.restype = C.c_size_t
    L.eta_decode.argtypes = [DIMS, P, P, P, P, P, P, P, F32, F32, I32, P, P, P, P, P,
                             C.c_size_t, P, P]
    L.eta_dense_decode.argtypes = [DIMS, P, P, P, P, F32, P, P, P, C.c_size_t, P, P]
    L.eta_calibrate_const_tau.argtypes = [P, P, I32, I32, I32, F32, P]
    L.eta_status_from_device.argtypes = [I32]
    L.eta_status_string.argtypes = [I32]
    L.eta_status_string.restype = C.c_char_p
    L.eta_decode_static.argtypes = [DIMS, P, P, P, P, P, P, P, F32, F32, I32, P, P, P, P, P,
                                    P]
    L.eta_decode_static.restype = I32
    L.eta_decode_static_max_workspace.argtypes = []
    L.eta_decode_static_max_workspace.restype = C.c_size_t
    L.eta_prefill.argtypes = [DIMS, P, P, P, P, P, F32, F32, P, P, P, P]
    L.eta_prefill.restype = I32
    L.eta_decode_step_workspace_size.argtypes = [DIMS]
    L.eta_decode_step_workspace_size.restype = C.c_size_t
    L.eta_decode_step.argtypes = [DIMS, P, P, P, P, P, P, P, I32, I32, P, P, P, P, P, I32, F32,
                                  F32, F32, P, P, P, P, P, P, P, P, C.c_size_t, P, P]
    L.eta_decode_step.restype = I32
    L.eta_append_and_predict_tau.argtypes = [DIMS, P, P, P, I32, P, P, P, P, P, P, P, P, P, P,
                                             P, P, P]
    L.eta_append_and_predict_tau.restype = I32
    L.eta_lse_merge.argtypes = [I32, I32, I32, P, P, P, P, P]
    L.eta_lse_merge.restype = I32
    L.eta_selftest_wait_timeout.argtypes = [C.c_uint32, P, P, P]
    L.eta_selftest_wait_timeout.restype = I32
    L.eta_set_decode_engine.argtypes = [I32]
    L.eta_set_decode_engine.restype = I32
    L.eta_get_decode_engine.argtypes = []
    L.eta_get_decode_engine.restype = I32
    L.eta_set_prefill_kernel.argtypes = [I32]
    L.eta_set_prefill_kernel.restype = I32
    L.eta_get_prefill_kernel.argtypes = []
    L.eta_get_prefill_kernel.restype = I32
    L.eta_prefill_kernel_for.argtypes = [DIMS, F32]
    L.eta_prefill_kernel_for.restype = I32
    L.eta_set_screen_engine.argtypes = [I32]
    L.eta_set_screen_engine.restype = I32
    L.eta_get_screen_engine.argtypes = []
    L.eta_get_screen_engine.restype = I32
    L.eta_build_checked.argtypes = []
    L.eta_build_checked.restype = I32
    L.eta_selftest_bounds.argtypes = [C.c_int64, C.c_int64, P, P]
    L.eta_selftest_bounds.restype = I32
    for name in ("eta_build_block_meta", "eta_predict_tau", "eta_screen", "eta_decode",
                 "eta_dense_decode", "eta_calibrate_const_tau", "eta_status_from_device"):
        getattr(L, name).restype = I32
    _lib = L
    return L


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream) -> Optional[C.c_void_p]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _check(fn: str, code: int):
    if code != ETA_OK:
        raise EtaError(fn, code)


def _cent_format(cent) -> int:
    return CENT["bf16"] if cent.dtype == torch.bfloat16 else CENT["f32"]


def eta_build_block_meta(dims: Dims, K, V, lengths, blk_begin, blk_end, cent, rmax, var, cnt,
                         vsum=None, stream=None, vardim=None):
    """cent: fp32 or bf16 tensor [B, Hkv, d, NB]; its dtype selects the format."""
    _check("eta_build_block_meta", lib().eta_build_block_meta(
        C.byref(dims), _p(K), _p(V), _p(lengths), int(blk_begin), int(blk_end),
        _cent_format(cent), _p(cent), _p(rmax), _p(var), _p(cnt), _p(vsum), _p(vardim),
        _stream(stream)))


def eta_predict_tau(dims: Dims, q, W, bias, tau_const, tau, dev_status=None, stream=None):
    _check("eta_predict_tau", lib().eta_predict_tau(
        C.byref(dims), _p(q), _p(W), _p(bias), _p(tau_const), _p(tau), _p(dev_status),
        _stream(stream)))


def eta_append_and_predict_tau(dims: Dims, K, V, lengths, cent, rmax, var, cnt, vsum, vardim, q,
                               W, bias, tau_const, tau, dev_status=None, stream=None):
    """Tail-block metadata refresh and thresholds in one launch (see include/eta.h)."""
    _check("eta_append_and_predict_tau", lib().eta_append_and_predict_tau(
        C.byref(dims), _p(K), _p(V), _p(lengths), _cent_format(cent), _p(cent), _p(rmax),
        _p(var), _p(cnt), _p(vsum), _p(vardim), _p(q), _p(W), _p(bias), _p(tau_const), _p(tau),
        _p(dev_status), _stream(stream)))


def eta_screen_workspace_size(dims: Dims) -> int:
    return int(lib().eta_screen_workspace_size(C.byref(dims)))


def eta_decode_launches(dims: Dims) -> int:
    n = int(lib().eta_decode_launches(C.byref(dims)))
    if n < 0:
        raise EtaError("eta_decode_launches", 1)
    return n


def eta_screen_launches(dims: Dims, cent_format: str = "f32") -> int:
    n = int(lib().eta_screen_launches(C.byref(dims), CENT[cent_format]))
    if n < 0:
        raise EtaError("eta_screen_launches", 1)
    return n


def eta_screen(dims: Dims, q, tau, cent, rmax, var, cnt, bound, z, scale, head_mask,
               union_idx, union_cnt, bounds_out, head_cnt, ws, dev_status=None, stream=None,
               vardim=None):
    _check("eta_screen", lib().eta_screen(
        C.byref(dims), _p(q), _p(tau), _cent_format(cent), _p(cent), _p(rmax), _p(var),
        _p(vardim), _p(cnt),
        BOUND[bound] if isinstance(bound, str) else int(bound), float(z), float(scale),
        _p(head_mask), _p(union_idx), _p(union_cnt), _p(bounds_out), _p(head_cnt), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _p(dev_status), _stream(stream)))


def eta_decode_workspace_size(dims: Dims) -> int:
    return int(lib().eta_decode_workspace_size(C.byref(dims)))


def eta_decode(dims: Dims, q, tau, K, V, lengths, union_idx, union_cnt, T, scale, prune,
               vsum, cnt, o, lse, ws, dev_status=None, stream=None):
    _check("eta_decode", lib().eta_decode(
        C.byref(dims), _p(q), _p(tau), _p(K), _p(V), _p(lengths), _p(union_idx),
        _p(union_cnt), float(T), float(scale),
        PRUNE[prune] if isinstance(prune, str) else int(prune), _p(vsum), _p(cnt), _p(o),
        _p(lse), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _p(dev_status),
        _stream(stream)))


def eta_decode_static(dims: Dims, q, tau, K, V, lengths, union_idx, union_cnt, T, scale,
                      prune, vsum, cnt, o, lse, dev_status=None, stream=None):
    """eta_decode without a workspace argument: the library's fixed device scratch
    is used instead (for callers that cannot allocate device memory)."""
    _check("eta_decode_static", lib().eta_decode_static(
        C.byref(dims), _p(q), _p(tau), _p(K), _p(V), _p(lengths), _p(union_idx),
        _p(union_cnt), float(T), float(scale),
        PRUNE[prune] if isinstance(prune, str) else int(prune), _p(vsum), _p(cnt), _p(o),
        _p(lse), _p(dev_status), _stream(stream)))


def eta_decode_step_workspace_size(dims: Dims) -> int:
    return int(lib().eta_decode_step_workspace_size(C.byref(dims)))


def eta_decode_step(dims: Dims, q, W, bias, tau_const, K, V, lengths, update_tail, cent, rmax,
                    var, vardim, cnt, bound, z, T, scale, tau, head_mask, union_idx, union_cnt,
                    head_cnt, o, lse, ws, dev_status=None, stream=None):
    """The whole decode step in one launch (see include/eta.h).  `ws` must be
    zero-filled before its first use."""
    _check("eta_decode_step", lib().eta_decode_step(
        C.byref(dims), _p(q), _p(W), _p(bias), _p(tau_const), _p(K), _p(V), _p(lengths),
        1 if update_tail else 0, _cent_format(cent), _p(cent), _p(rmax), _p(var), _p(vardim),
        _p(cnt), BOUND[bound] if isinstance(bound, str) else int(bound), float(z), float(T),
        float(scale), _p(tau), _p(head_mask), _p(union_idx), _p(union_cnt), _p(head_cnt),
        _p(o), _p(lse), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _p(dev_status), _stream(stream)))


def eta_lse_merge(o_parts, lse_parts, o, lse, stream=None):
    """o_parts fp32 [P, ..., d], lse_parts fp32 [P, ...] -> o [..., d], lse [...]
    (see include/eta.h)."""
    n_parts, d = int(o_parts.shape[0]), int(o_parts.shape[-1])
    n_rows = int(lse_parts.numel() // n_parts)
    _check("eta_lse_merge", lib().eta_lse_merge(
        n_parts, n_rows, d, _p(o_parts), _p(lse_parts), _p(o), _p(lse), _stream(stream)))


def eta_decode_static_max_workspace() -> int:
    return int(lib().eta_decode_static_max_workspace())


def eta_dense_decode(dims: Dims, q, K, V, lengths, scale, o, lse, ws, dev_status=None,
                     stream=None):
    _check("eta_dense_decode", lib().eta_dense_decode(
        C.byref(dims), _p(q), _p(K), _p(V), _p(lengths), float(scale), _p(o), _p(lse), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _p(dev_status), _stream(stream)))


def eta_calibrate_const_tau(bounds: torch.Tensor, valid: torch.Tensor, density: float):
    """Host call: bounds fp32 [n_q, Hq, NB] and valid bool/uint8 of the same shape
    (CPU tensors).  Returns tau fp32 [Hq] (CPU)."""
    b = bounds.detach().to("cpu", torch.float32).contiguous()
    v = valid.detach().to("cpu", torch.uint8).contiguous()
    n_q, Hq, NB = b.shape
    out = torch.empty(Hq, dtype=torch.float32)
    _check("eta_calibrate_const_tau", lib().eta_calibrate_const_tau(
        _p(b), _p(v), n_q, Hq, NB, float(density), _p(out)))
    return out


def eta_status_from_device(word: int) -> int:
    return int(lib().eta_status_from_device(int(word)))


def eta_status_string(code: int) -> str:
    return lib().eta_status_string(int(code)).decode()


def eta_set_decode_engine(engine) -> None:
    """engine: "auto" | "tcgen05" | "fma" (or the integer value)."""
    _check("eta_set_decode_engine", lib().eta_set_decode_engine(
        ENGINE[engine] if isinstance(engine, str) else int(engine)))


def eta_get_decode_engine() -> str:
    v = int(lib().eta_get_decode_engine())
    return {k: n for n, k in ENGINE.items()}.get(v, str(v))


def eta_set_screen_engine(engine) -> None:
    """engine: "auto" | "tcgen05" | "fma" (or the integer value)."""
    _check("eta_set_screen_engine", lib().eta_set_screen_engine(
        ENGINE[engine] if isinstance(engine, str) else int(engine)))


def eta_get_screen_engine() -> str:
    v = int(lib().eta_get_screen_engine())
    return {k: n for n, k in ENGINE.items()}.get(v, str(v))


def eta_set_prefill_kernel(kernel) -> None:
    """kernel: "auto" | "one_tile" | "two_tile" (or the integer value)."""
    _check("eta_set_prefill_kernel", lib().eta_set_prefill_kernel(
        PREFILL_KERNEL[kernel] if isinstance(kernel, str) else int(kernel)))


def eta_get_prefill_kernel() -> str:
    v = int(lib().eta_get_prefill_kernel())
    return {k: n for n, k in PREFILL_KERNEL.items()}.get(v, str(v))


def eta_prefill_kernel_for(dims: Dims, T: float) -> str:
    """The kernel eta_prefill would launch for these dims and gate T ("one_tile" or
    "two_tile"); raises EtaError(INVALID_ARG) for dims or T that eta_prefill refuses."""
    v = int(lib().eta_prefill_kernel_for(C.byref(dims), float(T)))
    if v < 0:
        raise EtaError("eta_prefill_kernel_for", 1)
    return {k: n for n, k in PREFILL_KERNEL.items()}[v]


def eta_build_checked() -> bool:
    """True when the loaded library is the range-checked build."""
    return bool(lib().eta_build_checked())


def eta_selftest_bounds(index: int, extent: int, dev_status, stream=None) -> None:
    """Runs the checked build's range check on (index, extent) (see include/eta.h)."""
    _check("eta_selftest_bounds", lib().eta_selftest_bounds(
        int(index), int(extent), _p(dev_status), _stream(stream)))


def eta_selftest_wait_timeout(wait_limit: int, never_set, dev_status, stream=None) -> None:
    """Runs the bounded-wait diagnostic kernel (see include/eta.h)."""
    _check("eta_selftest_wait_timeout", lib().eta_selftest_wait_timeout(
        int(wait_limit), _p(never_set), _p(dev_status), _stream(stream)))


def eta_prefill(dims: Dims, Q, tau, K, V, lengths, T, scale, O, lse, dev_status=None,
                stream=None) -> None:
    """Dense gated causal prefill attention (see include/eta.h)."""
    _check("eta_prefill", lib().eta_prefill(
        C.byref(dims), _p(Q), _p(tau), _p(K), _p(V), _p(lengths), float(T), float(scale), _p(O),
        _p(lse), _p(dev_status), _stream(stream)))
