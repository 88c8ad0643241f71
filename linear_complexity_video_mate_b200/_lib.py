"""ctypes declarations of the C ABI in include/mate.h (argument marshalling only)."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmate.so")

(MATE_OK, MATE_ERR_ARG, MATE_ERR_SHAPE, MATE_ERR_WORKSPACE, MATE_ERR_CUDA, MATE_ERR_TIMEOUT, MATE_ERR_UNSUPPORTED,
 MATE_ERR_TOO_LARGE) = range(8)
MATE_SSD_NOALLOC_SCRATCH_BYTES = 64 << 20
MATE_BF16, MATE_F32 = 0, 1

# every symbol include/mate.h declares
EXPORTS = (
    "mate_status_str", "mate_check_config", "mate_workspace_bytes", "mate_ssd_workspace_bytes", "rms_permute",
    "rms_unpermute", "review_pool", "ssd_scan_bidir", "tesa_forward", "mate_forward", "mate_forward_host",
    "mate_forward_host_workspace_bytes", "mate_device_status", "mate_last_launch_count", "mate_project_bf16",
    "ssd_scan_bidir_noalloc", "mate_trace_start", "mate_trace_stop", "mate_trace_read", "mate_kernel_name",
    "mate_scan_locality", "ssd_scan_bidir_pd", "mate_ssd_pd_workspace_bytes", "ssd_scan_bidir_backward",
    "mate_ssd_backward_workspace_bytes", "mate_selftest_wait_timeout", "mate_forward_host_pipelined",
    "mate_packed_weights_bytes", "mate_pack_weights", "mate_dit_workspace_bytes", "mate_dit_block_forward",
    "mate_forward_host_flush", "mate_tesa_backward_workspace_bytes", "tesa_backward",
)

_CONFIG_FIELDS = ("B", "T", "H", "W", "d", "nh", "P", "N", "Q", "R", "th", "tp", "wt", "wh", "ww", "st", "sh", "sw")


class CConfig(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int) for f in _CONFIG_FIELDS] + [("dtype", ctypes.c_int), ("mamba_extras", ctypes.c_int)]


class CWeights(ctypes.Structure):
    _fields_ = [("W_in", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
                ("D", ctypes.c_void_p), ("W_out", ctypes.c_void_p), ("W_qkv", ctypes.c_void_p),
                ("W_o", ctypes.c_void_p), ("dt_bias_b", ctypes.c_void_p), ("A_log_b", ctypes.c_void_p),
                ("D_b", ctypes.c_void_p), ("W_z", ctypes.c_void_p), ("conv_w", ctypes.c_void_p),
                ("conv_b", ctypes.c_void_p), ("norm_w", ctypes.c_void_p), ("packed", ctypes.c_void_p)]


class CDitWeights(ctypes.Structure):
    _fields_ = [("W_ada", ctypes.c_void_p), ("b_ada", ctypes.c_void_p), ("W1", ctypes.c_void_p),
                ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


class CTraceRecord(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("ms", ctypes.c_float)]


class MateError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


_lib = None


def load():
    """Load libmate.so from the package directory; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmate.so is not built ({LIB_PATH}); run linear_complexity_video_mate_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    cfgp, wp = ctypes.POINTER(CConfig), ctypes.POINTER(CWeights)
    sigs = {
        "mate_status_str": (ctypes.c_char_p, [ci]),
        "mate_check_config": (ci, [cfgp]),
        "mate_workspace_bytes": (sz, [cfgp]),
        "mate_ssd_workspace_bytes": (sz, [cfgp, ci]),
        "mate_ssd_pd_workspace_bytes": (sz, [cfgp, ci]),
        "mate_ssd_backward_workspace_bytes": (sz, [cfgp, ci]),
        "mate_selftest_wait_timeout": (ci, [ctypes.c_uint, vp]),
        "ssd_scan_bidir_backward": (ci, [vp] * 7 + [ci] + [vp] * 8 + [cfgp, vp, sz, vp]),
        "rms_permute": (ci, [vp, vp, ci, cfgp, vp]),
        "rms_unpermute": (ci, [vp, vp, ci, cfgp, vp]),
        "review_pool": (ci, [vp, vp, ci, cfgp, vp]),
        "ssd_scan_bidir": (ci, [vp, vp, vp, vp, vp, vp, vp, ci, vp, cfgp, vp, sz, vp]),
        "ssd_scan_bidir_noalloc": (ci, [vp, vp, vp, vp, vp, vp, vp, ci, vp, cfgp, vp]),
        "ssd_scan_bidir_pd": (ci, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, cfgp, vp, sz, vp]),
        "mate_trace_start": (ci, [ci]),
        "mate_trace_stop": (ci, []),
        "mate_trace_read": (ci, [ctypes.POINTER(CTraceRecord), ci]),
        "mate_kernel_name": (ctypes.c_char_p, [ci]),
        "mate_scan_locality": (ci, [ci, ci, ci, ci, vp, vp]),
        "tesa_forward": (ci, [vp, vp, ci, cfgp, vp]),
        "mate_forward": (ci, [vp, wp, ci, vp, cfgp, vp, sz, vp]),
        "mate_forward_host": (ci, [vp, wp, ci, vp, cfgp, vp, sz, vp]),
        "mate_forward_host_pipelined": (ci, [vp, wp, ci, vp, cfgp, vp, sz, vp]),
        "mate_packed_weights_bytes": (sz, [cfgp]),
        "mate_forward_host_flush": (ci, [vp]),
        "mate_tesa_backward_workspace_bytes": (sz, [cfgp]),
        "tesa_backward": (ci, [vp, vp, vp, vp, ci, cfgp, vp, sz, vp]),
        "mate_pack_weights": (ci, [wp, cfgp, vp, sz, vp]),
        "mate_dit_workspace_bytes": (sz, [cfgp]),
        "mate_dit_block_forward": (ci, [vp, vp, ci, ctypes.POINTER(CDitWeights), wp, ci, vp, cfgp, vp, sz, vp]),
        "mate_forward_host_workspace_bytes": (sz, [cfgp]),
        "mate_device_status": (ci, [vp, ctypes.POINTER(ctypes.c_uint)]),
        "mate_last_launch_count": (ci, []),
        "mate_project_bf16": (ci, [vp, ci, ctypes.c_longlong, ci, vp, ci, ci, vp, ci, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load().mate_status_str(int(status)).decode()


def check(status: int, where: str):
    if status != MATE_OK:
        raise MateError(status, where)


def make_config(cfg, mamba_extras: bool = False) -> CConfig:
    """C config from any object with the block's shape attributes (e.g. mate_inputs.MateConfig);
    mamba_extras adds the convolution, gate and gated norm of a full Mamba2 block."""
    c = CConfig()
    for f in _CONFIG_FIELDS:
        setattr(c, f, int(getattr(cfg, f)))
    c.dtype = MATE_BF16 if cfg.dtype == "bf16" else MATE_F32
    c.mamba_extras = 1 if mamba_extras else 0
    return c
