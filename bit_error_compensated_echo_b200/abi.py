"""ctypes binding of the C ABI in include/echo.h and include/echo_rank.h --
same names, argument marshalling only.

Every function here forwards to the function of the same name in
libecho_b200.so and raises ``EchoError`` (carrying the status code) when it
returns anything but ECHO_OK.  Pointers are passed as Python ints (device
or host addresses), streams as cudaStream_t handles (ints; 0 is the legacy
default stream).  Importing this module loads the library and fails loudly
if it has not been built, or was built from headers of another ABI version
(ABI_VERSION): there is no other implementation to fall back on.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libecho_b200.so")
ABI_VERSION = 5            # ECHO_ABI_VERSION of the headers these bindings follow

ECHO_MAX_RANKS = 8

STATUS = {
    0: "ECHO_OK", 1: "ECHO_ERR_INVALID_ARG", 2: "ECHO_ERR_SHAPE",
    3: "ECHO_ERR_ALIGNMENT", 4: "ECHO_ERR_UNSUPPORTED", 5: "ECHO_ERR_OOM",
    6: "ECHO_ERR_CUDA", 7: "ECHO_ERR_TIMEOUT",
}
ECHO_OK, ECHO_ERR_INVALID_ARG, ECHO_ERR_SHAPE, ECHO_ERR_ALIGNMENT = 0, 1, 2, 3
ECHO_ERR_UNSUPPORTED, ECHO_ERR_OOM, ECHO_ERR_CUDA, ECHO_ERR_TIMEOUT = 4, 5, 6, 7

ECHO_FIXUP_EXIT, ECHO_FIXUP_SIDE, ECHO_FIXUP_DEFERRED = 0, 1, 2
FIXUP_MODES = {"exit": ECHO_FIXUP_EXIT, "side": ECHO_FIXUP_SIDE,
               "deferred": ECHO_FIXUP_DEFERRED}


class EchoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, STATUS.get(status, "status %d" % status)))


class echo_config(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int32), ("G", ctypes.c_int32), ("N", ctypes.c_int64),
                ("compensate", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("beta_fast", ctypes.c_float), ("beta_slow", ctypes.c_float),
                ("device", ctypes.c_int32), ("fixup", ctypes.c_int32),
                ("bits", ctypes.c_int32)]


class echo_debug_view(ctypes.Structure):
    _fields_ = [("m_fast", ctypes.c_void_p), ("m_slow", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("rcodes", ctypes.c_void_p), ("rscales", ctypes.c_void_p),
                ("e_req", ctypes.c_void_p), ("fixup_pending", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("guard", ctypes.c_void_p),
                ("guard_bytes", ctypes.c_int64)]


class echo_rank_window_layout(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t),
                ("recv_codes", ctypes.c_size_t), ("recv_scales", ctypes.c_size_t),
                ("red_codes", ctypes.c_size_t), ("red_scales", ctypes.c_size_t),
                ("guard", ctypes.c_size_t), ("guard_bytes", ctypes.c_size_t)]


class echo_ipc_handle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_uint8 * 64)]


class echo_profile(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_int64), ("entry_ms", ctypes.c_double),
                ("reduce_ms", ctypes.c_double), ("exit_ms", ctypes.c_double),
                ("fixup_ms", ctypes.c_double), ("launches", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libecho_b200.so is not built (%s); run "
            "`python -m bit_error_compensated_echo_b200.build` -- the CUDA "
            "library is the only implementation of this path" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, st = ctypes.c_void_p, ctypes.c_int
    sig = {
        "echo_config_default": (None, [ctypes.POINTER(echo_config)]),
        "echo_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(echo_config)]),
        "echo_plan_create": (st, [ctypes.POINTER(vp), ctypes.POINTER(echo_config)]),
        "echo_plan_destroy": (st, [vp]),
        "echo_allreduce": (st, [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp]),
        "echo_allreduce_host": (st, [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp]),
        "echo_reduce_scatter": (st, [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp]),
        "echo_reset_state": (st, [vp, vp]),
        "echo_get_state": (st, [vp, vp, vp, vp]),
        "echo_set_state": (st, [vp, vp, vp, vp]),
        "echo_debug_view_get": (st, [vp, ctypes.POINTER(echo_debug_view)]),
        "echo_profile_enable": (st, [vp, ctypes.c_int32]),
        "echo_profile_read": (st, [vp, ctypes.POINTER(echo_profile), ctypes.c_int32]),
        "echo_launches_per_call": (ctypes.c_int32, [vp]),
        "echo_plan_set_bits": (st, [vp, ctypes.c_int32]),
        "echo_status_string": (ctypes.c_char_p, [st]),
        "echo_abi_version": (ctypes.c_int32, []),
        "echo_device_error_get": (st, [ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                       ctypes.c_int32]),
        "echo_selftest_wait_limit": (st, [ctypes.c_int32]),
        "echo_allreduce_noalloc": (st, [ctypes.POINTER(echo_config), ctypes.POINTER(vp),
                                        ctypes.POINTER(vp), vp, vp, vp]),
        # include/echo_rank.h
        "echo_rank_exchange_bytes": (st, [ctypes.POINTER(echo_config),
                                          ctypes.POINTER(ctypes.c_size_t),
                                          ctypes.POINTER(ctypes.c_size_t)]),
        "echo_rank_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(echo_config)]),
        "echo_rank_plan_create": (st, [ctypes.POINTER(vp), ctypes.POINTER(echo_config),
                                       ctypes.c_int32]),
        "echo_rank_plan_destroy": (st, [vp]),
        "echo_rank_entry": (st, [vp, vp, vp, vp, vp]),
        "echo_rank_reduce": (st, [vp, vp, vp, vp, vp, vp, vp]),
        "echo_rank_exit": (st, [vp, vp, vp, vp, vp]),
        "echo_rank_reduce_scatter": (st, [vp, vp, vp, vp, vp, vp]),
        "echo_rank_reset_state": (st, [vp, vp]),
        "echo_rank_get_state": (st, [vp, vp, vp, vp]),
        "echo_rank_set_state": (st, [vp, vp, vp, vp]),
        "echo_rank_launches_per_call": (ctypes.c_int32, [vp]),
        "echo_rank_plan_set_bits": (st, [vp, ctypes.c_int32]),
        "echo_rank_window": (st, [vp, ctypes.POINTER(echo_rank_window_layout)]),
        "echo_rank_entry_peers": (st, [vp, vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp]),
        "echo_rank_exit_peers": (st, [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp]),
        "echo_ipc_handle_get": (st, [vp, ctypes.POINTER(echo_ipc_handle)]),
        "echo_ipc_open": (st, [ctypes.POINTER(echo_ipc_handle), ctypes.c_int32,
                               ctypes.POINTER(vp)]),
        "echo_ipc_close": (st, [vp, ctypes.c_int32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if L.echo_abi_version() != ABI_VERSION:
        raise ImportError(
            "%s has ABI version %d, these bindings expect %d; rebuild it with "
            "`python -m bit_error_compensated_echo_b200.build`"
            % (LIB_PATH, L.echo_abi_version(), ABI_VERSION))
    return L


lib = _load()


def _check(status: int, where: str):
    if status != ECHO_OK:
        raise EchoError(status, where)


def _ptr_array(ptrs: Sequence[int]):
    arr = (ctypes.c_void_p * max(1, len(ptrs)))()
    for i, p in enumerate(ptrs):
        arr[i] = p
    return arr


def echo_config_default() -> echo_config:
    cfg = echo_config()
    lib.echo_config_default(ctypes.byref(cfg))
    return cfg


def echo_workspace_bytes(cfg: echo_config) -> int:
    return int(lib.echo_workspace_bytes(ctypes.byref(cfg)))


def echo_plan_create(cfg: echo_config) -> int:
    h = ctypes.c_void_p()
    _check(lib.echo_plan_create(ctypes.byref(h), ctypes.byref(cfg)), "echo_plan_create")
    return h.value


def echo_plan_destroy(plan: int) -> None:
    _check(lib.echo_plan_destroy(plan), "echo_plan_destroy")


def echo_allreduce(plan: int, in_device: Sequence[int], out_device: Sequence[int],
                   stream: int = 0, side_stream: int = 0) -> None:
    _check(lib.echo_allreduce(plan, _ptr_array(in_device), _ptr_array(out_device),
                              stream or None, side_stream or None), "echo_allreduce")


def echo_reduce_scatter(plan: int, in_device: Sequence[int], out_device: Sequence[int],
                        stream: int = 0, side_stream: int = 0) -> None:
    _check(lib.echo_reduce_scatter(plan, _ptr_array(in_device), _ptr_array(out_device),
                                   stream or None, side_stream or None), "echo_reduce_scatter")


def echo_allreduce_host(plan: int, in_host: Sequence[int], out_host: Sequence[int],
                        stream: int = 0) -> None:
    _check(lib.echo_allreduce_host(plan, _ptr_array(in_host), _ptr_array(out_host),
                                   stream or None), "echo_allreduce_host")


def echo_reset_state(plan: int, stream: int = 0) -> None:
    _check(lib.echo_reset_state(plan, stream or None), "echo_reset_state")


def echo_get_state(plan: int, m_fast_device: int, m_slow_device: int, stream: int = 0) -> None:
    _check(lib.echo_get_state(plan, m_fast_device, m_slow_device, stream or None),
           "echo_get_state")


def echo_set_state(plan: int, m_fast_device: int, m_slow_device: int, stream: int = 0) -> None:
    _check(lib.echo_set_state(plan, m_fast_device, m_slow_device, stream or None),
           "echo_set_state")


def echo_debug_view_get(plan: int) -> echo_debug_view:
    v = echo_debug_view()
    _check(lib.echo_debug_view_get(plan, ctypes.byref(v)), "echo_debug_view_get")
    return v


def echo_profile_enable(plan: int, on: bool) -> None:
    _check(lib.echo_profile_enable(plan, int(bool(on))), "echo_profile_enable")


def echo_profile_read(plan: int, reset: bool = False) -> echo_profile:
    p = echo_profile()
    _check(lib.echo_profile_read(plan, ctypes.byref(p), int(bool(reset))), "echo_profile_read")
    return p


def echo_plan_set_bits(plan: int, bits: int) -> None:
    _check(lib.echo_plan_set_bits(plan, int(bits)), "echo_plan_set_bits")


def echo_launches_per_call(plan: int) -> int:
    return int(lib.echo_launches_per_call(plan))


def echo_status_string(status: int) -> str:
    return lib.echo_status_string(status).decode()


ECHO_DEVERR_WAIT_TIMEOUT = 1


def echo_device_error_get(device: int, clear: bool = False) -> int:
    """The library's device error word on `device` (ECHO_DEVERR_* bits),
    cleared afterwards if `clear`.  The C call returns ECHO_ERR_TIMEOUT when
    a wait ran out; here that is the returned flags, not an exception."""
    flags = ctypes.c_int32()
    rc = lib.echo_device_error_get(device, ctypes.byref(flags), int(bool(clear)))
    if rc != ECHO_ERR_TIMEOUT:
        _check(rc, "echo_device_error_get")
    return int(flags.value)


def echo_selftest_wait_limit(device: int) -> None:
    """Run the bounded-wait self-test on `device` (about one second)."""
    _check(lib.echo_selftest_wait_limit(device), "echo_selftest_wait_limit")


def echo_abi_version() -> int:
    return int(lib.echo_abi_version())


ECHO_NOALLOC_MAX_SCRATCH_BYTES = 80 << 20


def echo_allreduce_noalloc(cfg: echo_config, in_device: Sequence[int],
                           out_device: Sequence[int], m_fast_device: int, m_slow_device: int,
                           stream: int = 0) -> None:
    """The allocation-free call: no plan, caller-owned state, scratch in the
    library's fixed device array (see include/echo.h)."""
    _check(lib.echo_allreduce_noalloc(ctypes.byref(cfg), _ptr_array(in_device),
                                      _ptr_array(out_device), m_fast_device or None,
                                      m_slow_device or None, stream or None),
           "echo_allreduce_noalloc")


# ---------------------------------------------------------------- include/echo_rank.h

def echo_rank_exchange_bytes(cfg: echo_config) -> tuple[int, int]:
    """(code bytes, scale bytes) of one chunk: C*bits/8 and 4*C/G."""
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.echo_rank_exchange_bytes(ctypes.byref(cfg), ctypes.byref(cb), ctypes.byref(sb)),
           "echo_rank_exchange_bytes")
    return int(cb.value), int(sb.value)


def echo_rank_workspace_bytes(cfg: echo_config) -> int:
    return int(lib.echo_rank_workspace_bytes(ctypes.byref(cfg)))


def echo_rank_plan_create(cfg: echo_config, rank: int) -> int:
    h = ctypes.c_void_p()
    _check(lib.echo_rank_plan_create(ctypes.byref(h), ctypes.byref(cfg), int(rank)),
           "echo_rank_plan_create")
    return h.value


def echo_rank_plan_destroy(plan: int) -> None:
    _check(lib.echo_rank_plan_destroy(plan), "echo_rank_plan_destroy")


def echo_rank_entry(plan: int, x_device: int, send_codes_device: int, send_scales_device: int,
                    stream: int = 0) -> None:
    _check(lib.echo_rank_entry(plan, x_device, send_codes_device, send_scales_device,
                               stream or None), "echo_rank_entry")


def echo_rank_reduce(plan: int, recv_codes_device: int, recv_scales_device: int,
                     red_codes_device: int, red_scales_device: int, stream: int = 0,
                     side_stream: int = 0) -> None:
    _check(lib.echo_rank_reduce(plan, recv_codes_device, recv_scales_device, red_codes_device,
                                red_scales_device, stream or None, side_stream or None),
           "echo_rank_reduce")


def echo_rank_exit(plan: int, all_codes_device: int, all_scales_device: int, out_device: int,
                   stream: int = 0) -> None:
    _check(lib.echo_rank_exit(plan, all_codes_device, all_scales_device, out_device,
                              stream or None), "echo_rank_exit")


def echo_rank_window(plan: int) -> dict:
    """The plan's window (allocated on first use): base, bytes and the byte
    offsets recv_codes, recv_scales, red_codes, red_scales."""
    L = echo_rank_window_layout()
    _check(lib.echo_rank_window(plan, ctypes.byref(L)), "echo_rank_window")
    return {"base": int(L.base or 0), "bytes": int(L.bytes), "recv_codes": int(L.recv_codes),
            "recv_scales": int(L.recv_scales), "red_codes": int(L.red_codes),
            "red_scales": int(L.red_scales), "guard": int(L.guard),
            "guard_bytes": int(L.guard_bytes)}


def echo_rank_entry_peers(plan: int, x_device: int, recv_codes_peers: Sequence[int],
                          recv_scales_peers: Sequence[int], stream: int = 0) -> None:
    _check(lib.echo_rank_entry_peers(plan, x_device, _ptr_array(recv_codes_peers),
                                     _ptr_array(recv_scales_peers), stream or None),
           "echo_rank_entry_peers")


def echo_rank_exit_peers(plan: int, red_codes_peers: Sequence[int],
                         red_scales_peers: Sequence[int], out_device: int,
                         stream: int = 0) -> None:
    _check(lib.echo_rank_exit_peers(plan, _ptr_array(red_codes_peers),
                                    _ptr_array(red_scales_peers), out_device, stream or None),
           "echo_rank_exit_peers")


def echo_ipc_handle_get(device_ptr: int) -> bytes:
    """The 64-byte CUDA IPC handle of the allocation holding device_ptr."""
    h = echo_ipc_handle()
    _check(lib.echo_ipc_handle_get(device_ptr, ctypes.byref(h)), "echo_ipc_handle_get")
    return bytes(h.bytes)


def echo_ipc_open(handle: bytes, device: int) -> int:
    """Map another process's allocation (its handle) into this one; returns
    the base address."""
    h = echo_ipc_handle()
    ctypes.memmove(h.bytes, handle, 64)
    out = ctypes.c_void_p()
    _check(lib.echo_ipc_open(ctypes.byref(h), device, ctypes.byref(out)), "echo_ipc_open")
    return int(out.value)


def echo_ipc_close(ptr: int, device: int) -> None:
    _check(lib.echo_ipc_close(ptr, device), "echo_ipc_close")


def echo_rank_reduce_scatter(plan: int, recv_codes_device: int, recv_scales_device: int,
                             out_device: int, stream: int = 0, side_stream: int = 0) -> None:
    _check(lib.echo_rank_reduce_scatter(plan, recv_codes_device, recv_scales_device, out_device,
                                        stream or None, side_stream or None),
           "echo_rank_reduce_scatter")


def echo_rank_reset_state(plan: int, stream: int = 0) -> None:
    _check(lib.echo_rank_reset_state(plan, stream or None), "echo_rank_reset_state")


def echo_rank_get_state(plan: int, m_fast_device: int, m_slow_device: int,
                        stream: int = 0) -> None:
    _check(lib.echo_rank_get_state(plan, m_fast_device, m_slow_device, stream or None),
           "echo_rank_get_state")


def echo_rank_set_state(plan: int, m_fast_device: int, m_slow_device: int,
                        stream: int = 0) -> None:
    _check(lib.echo_rank_set_state(plan, m_fast_device, m_slow_device, stream or None),
           "echo_rank_set_state")


def echo_rank_launches_per_call(plan: int) -> int:
    return int(lib.echo_rank_launches_per_call(plan))


def echo_rank_plan_set_bits(plan: int, bits: int) -> None:
    _check(lib.echo_rank_plan_set_bits(plan, int(bits)), "echo_rank_plan_set_bits")
