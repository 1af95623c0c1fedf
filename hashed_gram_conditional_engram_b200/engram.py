"""Python binding of libengram_b200.so (argument marshalling only).

Every function here has the name of the C entry point it calls and passes raw
device pointers (``tensor.data_ptr()``) and the current CUDA stream through
ctypes; all arithmetic happens in the library's kernels.  PyTorch is used only
to own device memory and streams.  The library must be built
(``python -m hashed_gram_conditional_engram_b200.build``); importing a
function without it raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libengram_b200.so")

MAX_HEADS = 32
F32, BF16 = 0, 1
WS_VOCAB, WS_FORWARD, WS_BACKWARD, WS_TABLE_GRAD = 0, 1, 2, 3
WS_HOSTCACHE_RANK, WS_HOSTCACHE_GATHER = 4, 5
SAVE_KV = 1  # EngramCfg.flags
# formulation variants (fp32 and bf16 layers)
CONV_DILATED, CONV_PRENORM, CONV_PER_BRANCH, NORM_SCALES = 2, 4, 8, 16
STATUS_BAD_ID, STATUS_BAD_INDEX, STATUS_TIMEOUT = 1, 2, 4
# test only: the call's bounded device-side waits run out (see engram.h)
TEST_STALL = 1 << 30

ERRORS = {
    -1: "ENGRAM_ERR_INVALID_ARG",
    -2: "ENGRAM_ERR_MISALIGNED",
    -3: "ENGRAM_ERR_WORKSPACE",
    -4: "ENGRAM_ERR_UNSUPPORTED",
    -5: "ENGRAM_ERR_CUDA",
    -6: "ENGRAM_ERR_TIMEOUT",
    -7: "ENGRAM_ERR_TOO_LARGE",
}
NOALLOC_MAX_ITEMS = 131072

EXPORTED = (
    "engram_workspace_size", "engram_saved_size", "engram_build_vocab_proj",
    "engram_hash_indices", "engram_gather", "engram_forward", "engram_decode_step",
    "engram_backward",
    "engram_table_grad", "engram_table_grad_noalloc", "engram_forward_hosttable",
    "engram_get_status",
    "engram_device_sm_count", "engram_table_rows", "engram_param_floats",
    "engram_hostcache_rank", "engram_hostcache_fill", "engram_forward_hostcache",
)


class EngramError(RuntimeError):
    def __init__(self, fn: str, rc: int):
        super().__init__(f"{fn} returned {rc} ({ERRORS.get(rc, 'unknown')})")
        self.rc = rc


class EngramCfg(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int32), ("D_h", ctypes.c_int32), ("d_model", ctypes.c_int32),
        ("n_branch", ctypes.c_int32), ("V_raw", ctypes.c_int32), ("V_c", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32),
        ("rows", ctypes.c_int64 * MAX_HEADS),
        ("mult", (ctypes.c_uint64 * 3) * MAX_HEADS),
    ]

    @property
    def J(self) -> int:
        return 2 * self.K

    @property
    def E(self) -> int:
        return 2 * self.K * self.D_h


def make_cfg(K: int, D_h: int, d_model: int, n_branch: int, V_raw: int, V_c: int, dtype: int,
             rows: Sequence[int], mult, flags: int = 0) -> EngramCfg:
    c = EngramCfg()
    c.K, c.D_h, c.d_model, c.n_branch = K, D_h, d_model, n_branch
    c.V_raw, c.V_c, c.dtype, c.flags = V_raw, V_c, dtype, flags
    mult = np.asarray(mult, dtype=np.uint64)
    for j in range(2 * K):
        c.rows[j] = int(rows[j])
        for i in range(3):
            c.mult[j][i] = int(mult[j, i])
    return c


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run "
                           "python -m hashed_gram_conditional_engram_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(EngramCfg)
    sig = {
        "engram_workspace_size": (sz, [cfgp, i32, i64]),
        "engram_saved_size": (sz, [cfgp, i64]),
        "engram_build_vocab_proj": (ctypes.c_int, [P, i32, P, ctypes.POINTER(i32), P, sz, P]),
        "engram_hash_indices": (ctypes.c_int, [cfgp, P, P, i32, i32, P, P, P]),
        "engram_gather": (ctypes.c_int, [cfgp, P, P, i64, P, P]),
        "engram_forward": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, P, i32, i32, P, sz, P]),
        "engram_decode_step": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, i32, P,
                                              sz, P]),
        "engram_backward": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                           i32, i32, P, sz, P]),
        "engram_table_grad": (ctypes.c_int, [cfgp, P, P, i64, P, P, P, P, sz, P]),
        "engram_table_grad_noalloc": (ctypes.c_int, [cfgp, P, P, i64, P, P, P, P]),
        "engram_forward_hosttable": (ctypes.c_int, [cfgp, P, P, i64, P, P, P]),
        "engram_get_status": (ctypes.c_int, [P]),
        "engram_device_sm_count": (ctypes.c_int, []),
        "engram_table_rows": (ctypes.c_int64, [cfgp]),
        "engram_param_floats": (ctypes.c_int64, [cfgp]),
        "engram_hostcache_rank": (ctypes.c_int, [cfgp, P, i64, i64, P, P, P, sz, P]),
        "engram_hostcache_fill": (ctypes.c_int, [cfgp, P, P, i64, P, P, P]),
        "engram_forward_hostcache": (ctypes.c_int, [cfgp, P, P, P, P, i64, P, P, P, sz, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _p(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int) -> int:
    if rc < 0:
        raise EngramError(fn, rc)
    return rc


def engram_workspace_size(cfg: Optional[EngramCfg], call: int, n: int) -> int:
    return lib().engram_workspace_size(ctypes.byref(cfg) if cfg is not None else None, call, n)


def engram_saved_size(cfg: EngramCfg, n_tok: int) -> int:
    return lib().engram_saved_size(ctypes.byref(cfg), n_tok)


def engram_build_vocab_proj(keys, V: int, proj, ws, ws_bytes: int, stream=None) -> int:
    vc = ctypes.c_int32(0)
    _check("engram_build_vocab_proj",
           lib().engram_build_vocab_proj(_p(keys), V, _p(proj), ctypes.byref(vc), _p(ws), ws_bytes,
                                         _s(stream)))
    return vc.value


def engram_hash_indices(cfg: EngramCfg, proj, ids, B: int, T: int, ngram_state, idx,
                        stream=None) -> None:
    _check("engram_hash_indices",
           lib().engram_hash_indices(ctypes.byref(cfg), _p(proj), _p(ids), B, T, _p(ngram_state),
                                     _p(idx), _s(stream)))


def engram_gather(cfg: EngramCfg, idx, table, n_tok: int, e, stream=None) -> None:
    _check("engram_gather",
           lib().engram_gather(ctypes.byref(cfg), _p(idx), _p(table), n_tok, _p(e), _s(stream)))


def engram_forward(cfg: EngramCfg, idx, table, e, h, Wk, Wv, conv_w, conv_state, out, saved,
                   B: int, T: int, ws, ws_bytes: int, stream=None) -> None:
    _check("engram_forward",
           lib().engram_forward(ctypes.byref(cfg), _p(idx), _p(table), _p(e), _p(h), _p(Wk),
                                _p(Wv), _p(conv_w), _p(conv_state), _p(out), _p(saved), B, T,
                                _p(ws), ws_bytes, _s(stream)))


def engram_decode_step(cfg: EngramCfg, proj, ids, ngram_state, idx, table, e, h, Wk, Wv,
                       conv_w, conv_state, out, B: int, ws, ws_bytes: int, stream=None) -> None:
    _check("engram_decode_step",
           lib().engram_decode_step(ctypes.byref(cfg), _p(proj), _p(ids), _p(ngram_state),
                                    _p(idx), _p(table), _p(e), _p(h), _p(Wk), _p(Wv),
                                    _p(conv_w), _p(conv_state), _p(out), B, _p(ws), ws_bytes,
                                    _s(stream)))


def engram_backward(cfg: EngramCfg, idx, e, h, Wk, Wv, conv_w, saved, dout, dh, dWk, dWv,
                    dconv_w, de, dtab_keys, dtab_rows, n_unique, B: int, T: int, ws,
                    ws_bytes: int, stream=None) -> None:
    _check("engram_backward",
           lib().engram_backward(ctypes.byref(cfg), _p(idx), _p(e), _p(h), _p(Wk), _p(Wv),
                                 _p(conv_w), _p(saved), _p(dout), _p(dh), _p(dWk), _p(dWv),
                                 _p(dconv_w), _p(de), _p(dtab_keys), _p(dtab_rows), _p(n_unique),
                                 B, T, _p(ws), ws_bytes, _s(stream)))


def engram_table_grad(cfg: EngramCfg, idx, de, n_tok: int, dtab_keys, dtab_rows, n_unique, ws,
                      ws_bytes: int, stream=None) -> None:
    _check("engram_table_grad",
           lib().engram_table_grad(ctypes.byref(cfg), _p(idx), _p(de), n_tok, _p(dtab_keys),
                                   _p(dtab_rows), _p(n_unique), _p(ws), ws_bytes, _s(stream)))


def engram_table_grad_noalloc(cfg: EngramCfg, idx, de, n_tok: int, dtab_keys, dtab_rows, n_unique,
                              stream=None) -> None:
    """engram_table_grad on the library's built-in scratch array: allocates
    nothing; n_tok * J must not exceed NOALLOC_MAX_ITEMS."""
    _check("engram_table_grad_noalloc",
           lib().engram_table_grad_noalloc(ctypes.byref(cfg), _p(idx), _p(de), n_tok,
                                           _p(dtab_keys), _p(dtab_rows), _p(n_unique),
                                           _s(stream)))


def engram_forward_hosttable(cfg: EngramCfg, idx, host_table, n_tok: int, e, side_stream=None,
                             done_event=None) -> None:
    ev = None
    if isinstance(done_event, int):
        ev = done_event
    elif done_event is not None:
        # a torch.cuda.Event creates its CUDA event on first record only
        if done_event.cuda_event == 0:
            done_event.record(side_stream)
        ev = done_event.cuda_event
    _check("engram_forward_hosttable",
           lib().engram_forward_hosttable(ctypes.byref(cfg), _p(idx), _p(host_table), n_tok, _p(e),
                                          _s(side_stream), ev))


def _event_handle(done_event, side_stream):
    if done_event is None or isinstance(done_event, int):
        return done_event
    # a torch.cuda.Event creates its CUDA event on first record only
    if done_event.cuda_event == 0:
        done_event.record(side_stream)
    return done_event.cuda_event


def engram_param_floats(cfg: EngramCfg) -> int:
    return int(lib().engram_param_floats(ctypes.byref(cfg)))


def engram_table_rows(cfg: EngramCfg) -> int:
    return int(lib().engram_table_rows(ctypes.byref(cfg)))


def engram_hostcache_rank(cfg: EngramCfg, idx, n_tok: int, C: int, rows_out, n_out, ws,
                          ws_bytes: int, stream=None) -> None:
    _check("engram_hostcache_rank",
           lib().engram_hostcache_rank(ctypes.byref(cfg), _p(idx), n_tok, C, _p(rows_out),
                                       _p(n_out), _p(ws), ws_bytes, _s(stream)))


def engram_hostcache_fill(cfg: EngramCfg, host_table, rows, C: int, cache, map_, stream=None):
    _check("engram_hostcache_fill",
           lib().engram_hostcache_fill(ctypes.byref(cfg), _p(host_table), _p(rows), C, _p(cache),
                                       _p(map_), _s(stream)))


def engram_forward_hostcache(cfg: EngramCfg, idx, host_table, cache, map_, n_tok: int, e, n_miss,
                             ws, ws_bytes: int, side_stream=None, done_event=None) -> None:
    _check("engram_forward_hostcache",
           lib().engram_forward_hostcache(ctypes.byref(cfg), _p(idx), _p(host_table), _p(cache),
                                          _p(map_), n_tok, _p(e), _p(n_miss), _p(ws), ws_bytes,
                                          _s(side_stream), _event_handle(done_event, side_stream)))


def engram_get_status(stream=None) -> int:
    return _check("engram_get_status", lib().engram_get_status(_s(stream)))


def engram_device_sm_count() -> int:
    return _check("engram_device_sm_count", lib().engram_device_sm_count())
