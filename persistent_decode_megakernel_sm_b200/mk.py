"""Thin ctypes binding of libmk.so (include/mk.h): argument marshalling only.

Every step of the decode path runs in the CUDA library.  There is no CPU
fallback: importing this module fails loudly when libmk.so is missing or
cannot be loaded.  Device buffers are passed as torch CUDA tensors (their
data_ptr) or raw integers; streams as torch.cuda.Stream or raw handles.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK, MK_ERR_INVALID, MK_ERR_OOM, MK_ERR_CUDA, MK_ERR_DEVICE_TIMEOUT, MK_ERR_DEVICE_BOUNDS, MK_ERR_STATE = range(7)
STATUS_NAMES = {0: "MK_OK", 1: "MK_ERR_INVALID", 2: "MK_ERR_OOM", 3: "MK_ERR_CUDA", 4: "MK_ERR_DEVICE_TIMEOUT",
                5: "MK_ERR_DEVICE_BOUNDS", 6: "MK_ERR_STATE"}

# Every symbol include/mk.h declares.
EXPORTS = ("mk_create", "mk_init_random", "mk_load_weights", "mk_kv_create", "mk_kv_fill_random", "mk_kv_copy_out",
           "mk_kv_copy_in", "mk_kv_bytes", "mk_decode_step", "mk_decode_step_noalloc", "mk_verify", "mk_prefill",
           "mk_spec_generate", "mk_decode_step_multikernel",
           "mk_set_router_trace", "mk_set_trace", "mk_sync_status", "mk_reset", "mk_launch_info", "mk_weight_bytes",
           "mk_debug_inject_stall", "mk_last_error", "mk_kv_destroy", "mk_destroy")


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class mk_model_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn",
                                              "vocab")] + \
               [("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float)] + \
               [(n, ctypes.c_int32) for n in ("n_routed", "n_shared", "top_k", "expert_ffn", "kv_lora_rank",
                                              "rope_dim", "expert_fp8", "max_batch", "max_ctx")]


class mk_synth_params(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("w_sigma", ctypes.c_float), ("router_sigma", ctypes.c_float),
                ("gain_sigma", ctypes.c_float), ("fp8_block_base", ctypes.c_float)]


class mk_spec_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("launches", "proposed", "accepted", "emitted")]


# int32_t draft(void* user, const int32_t* history, int32_t n_history, int32_t* proposals, int32_t max_k)
DRAFT_FN = ctypes.CFUNCTYPE(ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                            ctypes.POINTER(ctypes.c_int32), ctypes.c_int32)


class mk_tensor_src(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("layer", ctypes.c_int32), ("expert", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("data", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("on_device", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmk.so not built ({LIB_PATH}); run `python persistent_decode_megakernel_sm_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    st = ctypes.c_int
    sig = {
        "mk_create": ([ctypes.POINTER(mk_model_desc), ctypes.c_int, ctypes.POINTER(vp)], st),
        "mk_init_random": ([vp, ctypes.POINTER(mk_synth_params)], st),
        "mk_load_weights": ([vp, ctypes.POINTER(mk_tensor_src), ctypes.c_int], st),
        "mk_kv_create": ([vp, ctypes.c_int, ctypes.c_int, ctypes.POINTER(vp)], st),
        "mk_kv_fill_random": ([vp, ctypes.c_uint64, ctypes.c_float, i32], st),
        "mk_kv_copy_out": ([vp, vp], st),
        "mk_kv_copy_in": ([vp, vp], st),
        "mk_kv_bytes": ([vp], i64),
        "mk_decode_step": ([vp, vp, vp, ctypes.c_int, vp, vp, vp, vp], st),
        "mk_decode_step_noalloc": ([vp, vp, vp, ctypes.c_int, vp, vp, vp, vp], st),
        "mk_decode_step_multikernel": ([vp, vp, vp, ctypes.c_int, vp, vp, vp, vp], st),
        "mk_verify": ([vp, vp, ctypes.c_int, i32, vp, vp, vp, vp, vp], st),
        "mk_prefill": ([vp, vp, ctypes.c_int, ctypes.c_int, i32, vp, vp, vp], st),
        "mk_spec_generate": ([vp, vp, i32, i32, i32, DRAFT_FN, vp, ctypes.POINTER(i32), ctypes.POINTER(mk_spec_stats),
                              vp], st),
        "mk_set_router_trace": ([vp, vp, vp], st),
        "mk_set_trace": ([vp, vp, i32], st),
        "mk_sync_status": ([vp], st),
        "mk_reset": ([vp], st),
        "mk_launch_info": ([vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)], st),
        "mk_weight_bytes": ([vp], i64),
        "mk_debug_inject_stall": ([vp, i64], st),
        "mk_last_error": ([vp], ctypes.c_char_p),
        "mk_kv_destroy": ([vp], None),
        "mk_destroy": ([vp], None),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(h, code: int):
    if code != MK_OK:
        msg = lib.mk_last_error(h).decode()  # with h = None: why mk_create failed
        raise MkError(code, msg)


# ---------------------------------------------------------------------------
# the C ABI, one function each
# ---------------------------------------------------------------------------

def mk_create(desc: mk_model_desc, device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(None, lib.mk_create(ctypes.byref(desc), device, ctypes.byref(h)))
    return h.value


def mk_init_random(h: int, seed: int, w_sigma: float, router_sigma: float, gain_sigma: float,
                   fp8_block_base: float) -> None:
    p = mk_synth_params(seed, w_sigma, router_sigma, gain_sigma, fp8_block_base)
    _check(h, lib.mk_init_random(h, ctypes.byref(p)))


def mk_load_weights(h: int, tensors) -> None:
    arr = (mk_tensor_src * len(tensors))(*tensors)
    _check(h, lib.mk_load_weights(h, arr, len(tensors)))


def mk_kv_create(h: int, max_seqs: int, max_ctx: int) -> int:
    kv = ctypes.c_void_p()
    _check(h, lib.mk_kv_create(h, max_seqs, max_ctx, ctypes.byref(kv)))
    return kv.value


def mk_kv_fill_random(h: int, kv: int, seed: int, sigma: float, length: int) -> None:
    _check(h, lib.mk_kv_fill_random(kv, seed, sigma, length))


def mk_kv_copy_out(h: int, kv: int, dst) -> None:
    _check(h, lib.mk_kv_copy_out(kv, _ptr(dst)))


def mk_kv_copy_in(h: int, kv: int, src) -> None:
    _check(h, lib.mk_kv_copy_in(kv, _ptr(src)))


def mk_kv_bytes(kv: int) -> int:
    return lib.mk_kv_bytes(kv)


def mk_decode_step(h: int, tokens, positions, B: int, kv: int, logits_out, argmax_out, stream=None) -> None:
    _check(h, lib.mk_decode_step(h, _ptr(tokens), _ptr(positions), B, kv, _ptr(logits_out), _ptr(argmax_out),
                                 _stream(stream)))


def mk_decode_step_noalloc(h: int, tokens, positions, B: int, kv: int, logits_out, argmax_out, stream=None) -> None:
    """mk_decode_step with every scratch buffer in the library's static
    device array: no device allocation in the call (include/mk.h)."""
    _check(h, lib.mk_decode_step_noalloc(h, _ptr(tokens), _ptr(positions), B, kv, _ptr(logits_out), _ptr(argmax_out),
                                         _stream(stream)))


def mk_decode_step_multikernel(h: int, tokens, positions, B: int, kv: int, logits_out, argmax_out,
                               stream=None) -> None:
    """The decode step as one kernel per phase in a CUDA graph (include/mk.h)."""
    _check(h, lib.mk_decode_step_multikernel(h, _ptr(tokens), _ptr(positions), B, kv, _ptr(logits_out),
                                             _ptr(argmax_out), _stream(stream)))


def mk_verify(h: int, tokens8, n_prop: int, position: int, kv: int, logits_out, argmax_out, accepted_out,
              stream=None) -> None:
    _check(h, lib.mk_verify(h, _ptr(tokens8), n_prop, position, kv, _ptr(logits_out), _ptr(argmax_out),
                            _ptr(accepted_out), _stream(stream)))


def mk_prefill(h: int, tokens, n: int, seq: int, start: int, kv: int, argmax_last=None, stream=None) -> None:
    _check(h, lib.mk_prefill(h, _ptr(tokens), n, seq, start, kv, _ptr(argmax_last), _stream(stream)))


def mk_spec_generate(h: int, kv: int, anchor: int, position: int, n_out: int, draft, stream=None):
    """draft(history: list[int], max_k: int) -> list[int] of proposals.
    Returns (emitted tokens, stats dict)."""
    def _cb(user, hist, n, props, max_k):
        out = draft([hist[i] for i in range(n)], int(max_k))
        k = min(len(out), int(max_k))
        for i in range(k):
            props[i] = int(out[i])
        return k
    cb = DRAFT_FN(_cb)
    out = (ctypes.c_int32 * n_out)()
    stats = mk_spec_stats()
    _check(h, lib.mk_spec_generate(h, kv, anchor, position, n_out, cb, None, out, ctypes.byref(stats), _stream(stream)))
    return list(out), {n: getattr(stats, n) for n, _ in mk_spec_stats._fields_}


def mk_set_router_trace(h: int, idx_dev, w_dev) -> None:
    _check(h, lib.mk_set_router_trace(h, _ptr(idx_dev), _ptr(w_dev)))


def mk_set_trace(h: int, trace_dev, max_tasks_per_cta: int) -> None:
    _check(h, lib.mk_set_trace(h, _ptr(trace_dev), max_tasks_per_cta))


def mk_sync_status(h: int) -> int:
    return lib.mk_sync_status(h)


def mk_reset(h: int) -> None:
    _check(h, lib.mk_reset(h))


def mk_launch_info(h: int):
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(h, lib.mk_launch_info(h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def mk_weight_bytes(h: int) -> int:
    return lib.mk_weight_bytes(h)


def mk_debug_inject_stall(h: int, timeout_ns: int) -> None:
    _check(h, lib.mk_debug_inject_stall(h, timeout_ns))


def mk_last_error(h: int) -> str:
    return lib.mk_last_error(h).decode()


def mk_kv_destroy(kv: int) -> None:
    lib.mk_kv_destroy(kv)


def mk_destroy(h: int) -> None:
    lib.mk_destroy(h)
