"""Thin ctypes binding of libws (include/ws.h): the same entry points, argument
marshalling only.  Every step of the unit step runs in the library's kernels;
there is no Python or CPU fallback: if the library is missing, loading fails
with an error that says how to build it.

Tensor arguments may be torch tensors (CUDA, contiguous, bfloat16 / int16 /
uint16 storage) or raw device addresses (int).  ``stream`` defaults to torch's
current stream.  Each call returns the library's status code; with
``check=True`` (the default) a non-zero status raises :class:`WsError`.
"""
from __future__ import annotations

import ctypes as C
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
# WS_LIBRARY=debug loads the build with device index checks (libws_debug.so).
LIB_PATH = os.path.join(HERE, "libws_debug.so" if os.environ.get("WS_LIBRARY") == "debug" else "libws.so")
SYNTH_PATH = os.path.join(HERE, "libws_synth.so")
HEADER = os.path.join(ROOT, "include", "ws.h")

WS_OK = 0
WS_ERR_ARG = -1
WS_ERR_ALIGN = -2
WS_ERR_OOM = -3
WS_ERR_UNIT_ORDER = -4
WS_ERR_EVICTED = -5
WS_ERR_NOT_READY = -6
WS_ERR_CUDA = -7
WS_ERR_DEVICE_TIMEOUT = -8
WS_ERR_UNSUPPORTED = -9
WS_ERR_DEVICE_CHECK = -10
WS_SEG_COND = 0
WS_SEG_LATENT = 1


class ws_cache_config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("n_heads", C.c_int32), ("head_dim", C.c_int32),
                ("n_video", C.c_int32), ("n_audio", C.c_int32), ("n_cond", C.c_int32),
                ("history_units", C.c_int32)]


class ws_cache_info(C.Structure):
    _fields_ = [("slots", C.c_int32), ("tokens_per_unit", C.c_int32), ("n_query", C.c_int32),
                ("newest_unit", C.c_int64), ("cache_bytes", C.c_uint64), ("workspace_bytes", C.c_uint64),
                ("n_sessions", C.c_int32)]


class ws_profile(C.Structure):
    _fields_ = [("attention_launches", C.c_int64), ("attention_ms", C.c_double),
                ("combine_launches", C.c_int64), ("combine_ms", C.c_double),
                ("latent_write_launches", C.c_int64), ("latent_write_ms", C.c_double),
                ("last_n_split", C.c_int32), ("last_ctas", C.c_int32), ("last_keys", C.c_int64),
                ("last_kernel", C.c_int32)]


class ws_unit_io(C.Structure):
    _fields_ = [("n_steps", C.c_int32), ("out_per_call", C.c_int32), ("dt", C.c_float), ("n_latent", C.c_int64),
                ("cond_k", C.c_void_p), ("cond_v", C.c_void_p), ("q", C.c_void_p), ("k_new", C.c_void_p),
                ("v_new", C.c_void_p), ("out", C.c_void_p), ("x", C.c_void_p), ("vel", C.c_void_p),
                ("commit_k", C.c_void_p), ("commit_v", C.c_void_p), ("session", C.c_int32)]


class ws_unit_graph_stats(C.Structure):
    _fields_ = [("launches", C.c_int64), ("instantiations", C.c_int64), ("updates", C.c_int64),
                ("nodes", C.c_int64), ("record_ms", C.c_double)]


class WsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib = None
_synth = None
_P = C.c_void_p


def _declare(lib):
    i32, i64 = C.c_int32, C.c_int64
    sig = {
        "ws_cache_create": (C.c_int, [C.POINTER(_P), C.POINTER(ws_cache_config), _P]),
        "ws_cache_destroy": (C.c_int, [_P]),
        "ws_cache_append": (C.c_int, [_P, i64, C.c_int, _P, _P, _P]),
        "ws_unit_attention": (C.c_int, [_P, C.c_int, i64, _P, _P, _P, _P, _P]),
        "ws_prefill_attention": (C.c_int, [_P, C.c_int, i64, i32, _P, _P, _P, _P, _P]),
        "ws_flow_step": (C.c_int, [_P, _P, C.c_float, i64, _P]),
        "ws_cache_read": (C.c_int, [_P, C.c_int, i64, C.c_int, _P, _P, _P]),
        "ws_cache_slot_table": (C.c_int, [_P, C.POINTER(i64)]),
        "ws_cache_get_info": (C.c_int, [_P, C.POINTER(ws_cache_info)]),
        "ws_cache_set_splits": (C.c_int, [_P, C.c_int]),
        "ws_sync": (C.c_int, [_P, _P]),
        "ws_status_string": (C.c_char_p, [C.c_int]),
        "ws_profile_enable": (C.c_int, [_P, C.c_int]),
        "ws_profile_read": (C.c_int, [_P, C.POINTER(ws_profile)]),
        "ws_plan_visible": (C.c_int, [C.POINTER(ws_cache_config), C.POINTER(i64), C.POINTER(C.c_uint8), C.c_int,
                                      i64, C.POINTER(i32), C.POINTER(i32), i32, C.POINTER(i32)]),
        "ws_attention_noalloc": (C.c_int, [_P, _P, _P, i32, i32, i32, i32, _P]),
        "ws_attention_noalloc_sync": (C.c_int, [_P]),
        "ws_debug_inject_stall": (C.c_int, [_P, C.c_int]),
        "ws_unit_graph_create": (C.c_int, [C.POINTER(_P), _P, C.POINTER(ws_unit_io)]),
        "ws_unit_graph_launch": (C.c_int, [_P, i64, _P]),
        "ws_unit_graph_get_stats": (C.c_int, [_P, C.POINTER(ws_unit_graph_stats)]),
        "ws_unit_graph_destroy": (C.c_int, [_P]),
        "ws_pool_create": (C.c_int, [C.POINTER(_P), C.POINTER(ws_cache_config), i32, _P]),
        "ws_session_append": (C.c_int, [_P, i32, i64, C.c_int, _P, _P, _P]),
        "ws_session_read": (C.c_int, [_P, i32, C.c_int, i64, C.c_int, _P, _P, _P]),
        "ws_session_slot_table": (C.c_int, [_P, i32, C.POINTER(i64)]),
        "ws_session_reset": (C.c_int, [_P, i32]),
        "ws_session_attention": (C.c_int, [_P, C.c_int, i32, C.POINTER(i32), C.POINTER(i64), _P, _P, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args


def lib():
    """The loaded libws.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_serving_ws_b200.build`"
                               + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
        _lib = C.CDLL(LIB_PATH)
        _declare(_lib)
    return _lib


def synth_lib():
    global _synth
    if _synth is None:
        if not os.path.exists(SYNTH_PATH):
            raise RuntimeError(f"{SYNTH_PATH} is missing: build it with `python -m kv_cache_serving_ws_b200.build`")
        _synth = C.CDLL(SYNTH_PATH)
        _synth.ws_synth_fill_normal_bf16.restype = C.c_int
        _synth.ws_synth_fill_normal_bf16.argtypes = [_P, C.c_int64, C.c_uint64, C.c_int64, _P, _P, C.c_int32, _P]
    return _synth


def header_symbols(path: str = HEADER) -> list[str]:
    """Names of the functions declared in a C header of this package."""
    text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*[\s\*]+(ws_[a-z0-9_]+)\s*\(", text, re.M)))


# ---------------------------------------------------------------- marshalling

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor or a device address")
    if not t.is_cuda:
        raise ValueError("tensor must be in CUDA device memory")
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected 16-bit bf16 storage, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _done(st: int, where: str, check: bool):
    if check and st != WS_OK:
        raise WsError(st, where)
    return st


def make_config(n_layers, n_heads, head_dim, n_video, n_audio, n_cond, history_units) -> ws_cache_config:
    return ws_cache_config(n_layers, n_heads, head_dim, n_video, n_audio, n_cond, history_units)


def status_string(status: int) -> str:
    return lib().ws_status_string(status).decode()


ws_status_string = status_string


def ws_cache_create(cfg: ws_cache_config, stream=None, check=True):
    """Returns (status, handle)."""
    h = _P()
    st = lib().ws_cache_create(C.byref(h), C.byref(cfg), _stream(stream))
    _done(st, "ws_cache_create", check)
    return st, h


def ws_cache_destroy(h, check=True):
    return _done(lib().ws_cache_destroy(h), "ws_cache_destroy", check)


def ws_cache_append(h, unit, seg, k_slice, v_slice, stream=None, check=True):
    return _done(lib().ws_cache_append(h, unit, seg, _ptr(k_slice), _ptr(v_slice), _stream(stream)),
                 "ws_cache_append", check)


def ws_unit_attention(h, layer, unit, q, k_new, v_new, out, stream=None, check=True):
    return _done(lib().ws_unit_attention(h, layer, unit, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                         _stream(stream)), "ws_unit_attention", check)


def ws_prefill_attention(h, layer, unit_first, n_units, q, k_new, v_new, out, stream=None, check=True):
    return _done(lib().ws_prefill_attention(h, layer, unit_first, n_units, _ptr(q), _ptr(k_new), _ptr(v_new),
                                            _ptr(out), _stream(stream)), "ws_prefill_attention", check)


def ws_flow_step(x, v, dt, n=None, stream=None, check=True):
    if n is None:
        n = x.numel()
    return _done(lib().ws_flow_step(_ptr(x), _ptr(v), float(dt), int(n), _stream(stream)), "ws_flow_step", check)


def ws_cache_read(h, layer, unit, seg, k_out, v_out, stream=None, check=True):
    return _done(lib().ws_cache_read(h, layer, unit, seg, _ptr(k_out), _ptr(v_out), _stream(stream)),
                 "ws_cache_read", check)


def ws_cache_slot_table(h) -> list[int]:
    info = ws_cache_get_info(h)
    buf = (C.c_int64 * info["slots"])()
    _done(lib().ws_cache_slot_table(h, buf), "ws_cache_slot_table", True)
    return list(buf)


def ws_cache_get_info(h) -> dict:
    info = ws_cache_info()
    _done(lib().ws_cache_get_info(h, C.byref(info)), "ws_cache_get_info", True)
    return {k: getattr(info, k) for k, _ in ws_cache_info._fields_}


def ws_cache_set_splits(h, n_split, check=True):
    return _done(lib().ws_cache_set_splits(h, n_split), "ws_cache_set_splits", check)


def ws_sync(h, stream=None, check=True):
    return _done(lib().ws_sync(h, _stream(stream)), "ws_sync", check)


def ws_debug_inject_stall(h, tile, check=True):
    """Test hook: leave out one V load per CTA so the kernel's bounded wait runs out (-1 = off).
    With h = None it applies to ws_attention_noalloc calls."""
    return _done(lib().ws_debug_inject_stall(h, tile), "ws_debug_inject_stall", check)


def ws_profile_enable(h, enable=True, check=True):
    return _done(lib().ws_profile_enable(h, 1 if enable else 0), "ws_profile_enable", check)


def ws_profile_read(h) -> dict:
    p = ws_profile()
    _done(lib().ws_profile_read(h, C.byref(p)), "ws_profile_read", True)
    return {k: getattr(p, k) for k, _ in ws_profile._fields_}


def ws_plan_visible(cfg: ws_cache_config, slot_unit, latent_ready, layer, unit, max_runs=192):
    """Returns (status, [(row_begin, rows), ...]); touches no GPU."""
    n = len(slot_unit)
    su = (C.c_int64 * n)(*slot_unit)
    lr = (C.c_uint8 * len(latent_ready))(*[1 if x else 0 for x in latent_ready])
    rb = (C.c_int32 * max(1, max_runs))()
    rw = (C.c_int32 * max(1, max_runs))()
    nr = C.c_int32(0)
    st = lib().ws_plan_visible(C.byref(cfg), su, lr, layer, unit, rb, rw, max_runs, C.byref(nr))
    return st, [(rb[i], rw[i]) for i in range(nr.value)] if st == WS_OK else []


def ws_attention_noalloc(q, kv, out, n_query, n_keys, n_heads, head_dim, stream=None, check=True):
    """Attention over caller-owned K/V planes kv [2][H][Nk][D]; no device allocation."""
    return _done(lib().ws_attention_noalloc(_ptr(q), _ptr(kv), _ptr(out), n_query, n_keys, n_heads, head_dim,
                                            _stream(stream)), "ws_attention_noalloc", check)


def ws_attention_noalloc_sync(stream=None, check=True):
    """Wait for the stream; WS_ERR_DEVICE_TIMEOUT if the last no-alloc call's bounded wait ran out."""
    return _done(lib().ws_attention_noalloc_sync(_stream(stream)), "ws_attention_noalloc_sync", check)


def ws_pool_create(cfg: ws_cache_config, n_sessions: int, stream=None, check=True):
    h = _P()
    st = lib().ws_pool_create(C.byref(h), C.byref(cfg), int(n_sessions), _stream(stream))
    _done(st, "ws_pool_create", check)
    return st, h


def ws_session_append(h, session, unit, seg, k_slice, v_slice, stream=None, check=True):
    return _done(lib().ws_session_append(h, int(session), int(unit), int(seg), _ptr(k_slice), _ptr(v_slice),
                                         _stream(stream)), "ws_session_append", check)


def ws_session_read(h, session, layer, unit, seg, k_out, v_out, stream=None, check=True):
    return _done(lib().ws_session_read(h, int(session), int(layer), int(unit), int(seg), _ptr(k_out), _ptr(v_out),
                                       _stream(stream)), "ws_session_read", check)


def ws_session_slot_table(h, session) -> list[int]:
    info = ws_cache_get_info(h)
    buf = (C.c_int64 * info["slots"])()
    _done(lib().ws_session_slot_table(h, int(session), buf), "ws_session_slot_table", True)
    return list(buf)


def ws_session_reset(h, session, check=True):
    return _done(lib().ws_session_reset(h, int(session)), "ws_session_reset", check)


def ws_session_attention(h, layer, sessions, units, q, k_new, v_new, out, stream=None, check=True):
    n = len(sessions)
    if len(units) != n:
        raise ValueError("sessions and units differ in length")
    s_arr = (C.c_int32 * max(1, n))(*[int(s) for s in sessions])
    u_arr = (C.c_int64 * max(1, n))(*[int(u) for u in units])
    st = lib().ws_session_attention(h, int(layer), n, s_arr, u_arr, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                    _stream(stream))
    return _done(st, "ws_session_attention", check)


def ws_unit_graph_create(h, n_steps, dt, cond_k, cond_v, q, k_new, v_new, out, x, vel, commit_k, commit_v,
                         out_per_call=True, n_latent=None, session=0, check=True):
    """Unit program over cache h; the tensors must stay alive (and in place) while it exists."""
    io = ws_unit_io(int(n_steps), 1 if out_per_call else 0, float(dt), int(x.numel() if n_latent is None else n_latent),
                    _ptr(cond_k), _ptr(cond_v), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(x), _ptr(vel),
                    _ptr(commit_k), _ptr(commit_v), int(session))
    g = _P()
    st = lib().ws_unit_graph_create(C.byref(g), h, C.byref(io))
    _done(st, "ws_unit_graph_create", check)
    return st, g


def ws_unit_graph_launch(g, unit, stream=None, check=True):
    return _done(lib().ws_unit_graph_launch(g, int(unit), _stream(stream)), "ws_unit_graph_launch", check)


def ws_unit_graph_get_stats(g) -> dict:
    st = ws_unit_graph_stats()
    _done(lib().ws_unit_graph_get_stats(g, C.byref(st)), "ws_unit_graph_get_stats", True)
    return {k: getattr(st, k) for k, _ in ws_unit_graph_stats._fields_}


def ws_unit_graph_destroy(g, check=True):
    return _done(lib().ws_unit_graph_destroy(g), "ws_unit_graph_destroy", check)


def synth_fill(dst, key: int, index0: int = 0, stream=None):
    """Fill a CUDA bf16 tensor with the seeded generator's values (device twin of synth.normal_tensor)."""
    import torch

    from . import synth
    thr, vals = synth.normal_table()
    dev = dst.device
    cache = getattr(synth_fill, "_tables", {})
    if dev not in cache:
        cache[dev] = (torch.from_numpy(thr.view("int64").copy()).to(dev), torch.from_numpy(vals.view("int16").copy()).to(dev))
        synth_fill._tables = cache
    t_thr, t_val = cache[dev]
    st = synth_lib().ws_synth_fill_normal_bf16(_ptr(dst), dst.numel(), C.c_uint64(key), index0, t_thr.data_ptr(),
                                               t_val.data_ptr(), len(thr), _stream(stream))
    if st != 0:
        raise RuntimeError(f"ws_synth_fill_normal_bf16 failed ({st})")
