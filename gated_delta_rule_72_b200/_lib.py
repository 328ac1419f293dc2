"""ctypes binding of libgdn.so: the C-ABI functions under their own names.

Argument marshalling only; every step of the scan runs in the library's
CUDA kernels.  There is no fallback: if libgdn.so has not been built, the
first call raises.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_F32 = 0
GDN_BF16 = 1

STATUS = {
    0: "GDN_OK", -1: "GDN_ERR_NULL", -2: "GDN_ERR_SHAPE", -3: "GDN_ERR_DTYPE",
    -4: "GDN_ERR_ALIGN", -5: "GDN_ERR_UNSUPPORTED", -6: "GDN_ERR_WORKSPACE", -7: "GDN_ERR_CUDA",
}

# name -> (restype, argtypes)
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "gdn_scan_causal": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "gdn_scan_bidir": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "gdn_scan_bidir_states": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                   _P, _Z, _P]),
    "gdn_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "gdn_step_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "gdn_vda_scan": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P,
                          _Z, _P]),
    "gdn_vda_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "gdn_readout_gate": (_I, [_P, _I, _P, _I, _P, ctypes.c_float, _P, _I, _I, _I, _I, _I, _P]),
    "gdn_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_version": (ctypes.c_char_p, []),
    "gdn_launch_count": (ctypes.c_ulonglong, []),
    "gdn_device_timeouts": (_I, [ctypes.POINTER(ctypes.c_uint)]),
    "gdn_set_kernel_timing": (None, [_I]),
    "gdn_set_short_call_tokens": (_I, [_I]),
    "gdn_set_chain_segments": (_I, [_I]),
    "gdn_read_kernel_timing": (_I, [ctypes.c_char_p, _I, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(_I), _I]),
}

_lib = None


class GDNError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (fn, STATUS.get(status, status),
                                                 gdn_status_string(status)))


def load(path: str = LIB_PATH):
    """Load libgdn.so (once).  Raises if it is missing: there is no CPU path."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError("libgdn.so is not built (%s); run `python -m gated_delta_rule_72_b200.build` "
                               "or __graft_entry__.build()" % path)
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def gdn_scan_causal(q, k, v, alpha, beta, state_in, state_out, o, B, T, H, dk, dv, dt, o_dt,
                    workspace, ws_bytes, stream):
    return load().gdn_scan_causal(q, k, v, alpha, beta, state_in, state_out, o, B, T, H, dk, dv,
                                  dt, o_dt, workspace, ws_bytes, stream)


def gdn_scan_bidir(q, k, v, alpha, beta, o, B, T, H, dk, dv, dt, o_dt, workspace, ws_bytes,
                   stream):
    return load().gdn_scan_bidir(q, k, v, alpha, beta, o, B, T, H, dk, dv, dt, o_dt, workspace,
                                 ws_bytes, stream)


def gdn_scan_bidir_states(q, k, v, alpha, beta, state_in, state_in_bwd, state_out, state_out_bwd, o,
                          B, T, H, dk, dv, dt, o_dt, workspace, ws_bytes, stream):
    return load().gdn_scan_bidir_states(q, k, v, alpha, beta, state_in, state_in_bwd, state_out,
                                        state_out_bwd, o, B, T, H, dk, dv, dt, o_dt, workspace,
                                        ws_bytes, stream)


def gdn_step(q, k, v, alpha, beta, state, o, B, T, H, dk, dv, dt, o_dt, workspace, ws_bytes,
             stream):
    return load().gdn_step(q, k, v, alpha, beta, state, o, B, T, H, dk, dv, dt, o_dt, workspace,
                           ws_bytes, stream)


def gdn_step_noalloc(q, k, v, alpha, beta, state, o, B, T, H, dk, dv, dt, o_dt, stream):
    return load().gdn_step_noalloc(q, k, v, alpha, beta, state, o, B, T, H, dk, dv, dt, o_dt,
                                   stream)


GDN_NOALLOC_SCRATCH_BYTES = 64 << 20


def gdn_workspace_size(B, T, H, dk, dv, dt, o_dt, bidir):
    return load().gdn_workspace_size(B, T, H, dk, dv, dt, o_dt, bidir)


def gdn_status_string(status):
    return load().gdn_status_string(status).decode()


def gdn_version():
    return load().gdn_version().decode()


def gdn_device_timeouts():
    """Bounded device-side waits that gave up on the current device (0 = none)."""
    c = ctypes.c_uint(0)
    st = load().gdn_device_timeouts(ctypes.byref(c))
    if st != 0:
        raise GDNError("gdn_device_timeouts", st)
    return int(c.value)


def gdn_launch_count():
    return int(load().gdn_launch_count())


def gdn_vda_scan(q, k, v, alpha_frame, beta, state_in, state_in_bwd, state_out, state_out_bwd, o, B, F, U, H,
                 dk, dv, bidir, dt, o_dt, workspace, ws_bytes, stream):
    return load().gdn_vda_scan(q, k, v, alpha_frame, beta, state_in, state_in_bwd, state_out, state_out_bwd, o,
                               B, F, U, H, dk, dv, bidir, dt, o_dt, workspace, ws_bytes, stream)


def gdn_vda_workspace_size(B, F, U, H, dk, dv, bidir):
    return int(load().gdn_vda_workspace_size(B, F, U, H, dk, dv, int(bool(bidir))))


def gdn_readout_gate(o, o_dt, z, z_dt, gamma, eps, y, y_dt, B, T, H, dv, stream):
    return load().gdn_readout_gate(o, o_dt, z, z_dt, gamma, eps, y, y_dt, B, T, H, dv, stream)


def gdn_set_kernel_timing(on):
    load().gdn_set_kernel_timing(int(bool(on)))


def gdn_set_short_call_tokens(max_t):
    """Causal calls of at most max_t tokens (at most 64) run token by token;
    max_t < 0 restores the automatic choice.  Returns the previous setting
    (-1 for automatic)."""
    return int(load().gdn_set_short_call_tokens(int(max_t)))


def gdn_set_chain_segments(g):
    """Segments per chunk walk of the tensor-core path (sequence
    parallelism); g < 1 restores the automatic choice.  Returns the previous
    setting (-1 for automatic)."""
    return int(load().gdn_set_chain_segments(int(g)))


def gdn_read_kernel_timing(max_kernels=16, name_len=64):
    """{kernel name: (total device ms, launches)} since the previous read."""
    names = ctypes.create_string_buffer(max_kernels * name_len)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (_I * max_kernels)()
    n = load().gdn_read_kernel_timing(names, name_len, ms, cnt, max_kernels)
    if n < 0:
        raise GDNError("gdn_read_kernel_timing", n)
    raw = names.raw
    out = {}
    for i in range(n):
        nm = raw[i * name_len:(i + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(cnt[i]))
    return out
