"""ctypes binding of the C ABI in include/sparse_attn.h (argument marshalling only).

Every computation happens in ``libsparse_attn.so``. This module only mirrors
the C structs, loads the library and passes pointers and sizes through. If
the library is missing it raises; there is no other implementation to fall
back to.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_attn.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE = 0, 1, 2, 3
SA_ERR_CUDA, SA_ERR_DEVICE_TIMEOUT, SA_ERR_DEVICE_BOUNDS = 4, 5, 6

SA_MASK_TOPK, SA_MASK_STA, SA_MASK_SPATIOTEMPORAL = 1, 2, 3
SA_MASK_SPADE, SA_MASK_FG, SA_MASK_EXPLICIT = 4, 5, 6

SA_LAYOUT_IDENTITY, SA_LAYOUT_FRAME_MAJOR, SA_LAYOUT_TILE = 0, 1, 2
SA_SUMMARIZER_MEAN, SA_SUMMARIZER_MAX, SA_SUMMARIZER_MIN = 0, 1, 2

SA_EXPORT_BLOCK_BITS, SA_EXPORT_HEAD_INFO, SA_EXPORT_FG_BITS, SA_EXPORT_FG_TAU = 1, 2, 3, 4
SA_EXPORT_FG_TILE_KEYS = 5

EXPORTED = ("sparse_attn_workspace_size", "sparse_attn_build_mask", "sparse_attn_forward",
            "sparse_attn_permute", "sparse_attn_attend",
            "sparse_attn_export_bytes", "sparse_attn_mask_export", "sparse_attn_status",
            "sparse_attn_build_mask_static", "sparse_attn_status_static",
            "sparse_attn_selftest_wait_timeout",
            "sparse_attn_profile_heads", "sparse_attn_sta_window_search",
            "sparse_attn_profile_workspace_size",
            "sparse_attn_build_mask_fg_cached", "sparse_attn_quantize_e4m3",
            "sparse_attn_permute_fp8", "sparse_attn_attend_fp8",
            "sparse_attn_forward_host", "sparse_attn_strerror")

SA_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


class Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("T", ctypes.c_int),
                ("H", ctypes.c_int), ("W", ctypes.c_int), ("head_dim", ctypes.c_int)]


class Policy(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("block", ctypes.c_int), ("tile", ctypes.c_int * 3),
                ("topk", ctypes.c_int), ("keep_diagonal", ctypes.c_int),
                ("window", ctypes.c_int * 3), ("head_is_temporal", ctypes.POINTER(ctypes.c_int8)),
                ("sink_tokens", ctypes.c_int), ("frame_radius", ctypes.c_int),
                ("n_candidates", ctypes.c_int), ("candidates", (ctypes.c_int * 3) * 4),
                ("top_p", ctypes.c_float), ("fg_group", ctypes.c_int),
                ("fg_keep_fraction", ctypes.c_float), ("explicit_layout", ctypes.c_int),
                ("explicit_bits", ctypes.c_void_p), ("summarizer", ctypes.c_int),
                ("head_windows", ctypes.POINTER(ctypes.c_int))]


class HeadInfo(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("candidate", ctypes.c_int32),
                ("bt", ctypes.c_int32), ("bh", ctypes.c_int32), ("bw", ctypes.c_int32),
                ("nt", ctypes.c_int32), ("nh", ctypes.c_int32), ("nw", ctypes.c_int32),
                ("nb", ctypes.c_int32), ("kept", ctypes.c_int32),
                ("sics_total", ctypes.c_float * 4), ("window", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class SparseAttnError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {strerror(code)} (status {code})")
        self.code = code


_LIB = None


def lib():
    """The loaded native library. Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python sparse_attention_video_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        P, PP = ctypes.POINTER(Problem), ctypes.POINTER(Policy)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L.sparse_attn_workspace_size.argtypes = [P, PP, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.sparse_attn_build_mask.argtypes = [P, PP, vp, vp, vp, vp, vp]
        L.sparse_attn_forward.argtypes = [P, PP, vp, vp, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_forward_host.argtypes = [P, PP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_permute.argtypes = [P, PP, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_attend.argtypes = [P, PP, vp, vp, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_export_bytes.argtypes = [P, PP, ctypes.c_int, ctypes.POINTER(sz)]
        L.sparse_attn_mask_export.argtypes = [P, PP, vp, ctypes.c_int, vp, sz, vp]
        L.sparse_attn_status.argtypes = [vp, vp, ctypes.c_int]
        L.sparse_attn_build_mask_static.argtypes = [P, PP, vp, vp, vp, vp]
        L.sparse_attn_status_static.argtypes = [vp, ctypes.c_int]
        L.sparse_attn_selftest_wait_timeout.argtypes = [vp, vp]
        L.sparse_attn_profile_heads.argtypes = [P, PP, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp,
                                                vp, vp]
        L.sparse_attn_profile_workspace_size.argtypes = [P, ctypes.c_int, ctypes.POINTER(sz)]
        L.sparse_attn_sta_window_search.argtypes = [P, PP, vp, vp, vp, vp, ctypes.c_int, vp,
                                                    ctypes.c_int, vp, vp, vp, vp, vp]
        L.sparse_attn_build_mask_fg_cached.argtypes = [P, PP, vp, vp, vp, ctypes.c_float, vp, vp,
                                                       vp]
        L.sparse_attn_quantize_e4m3.argtypes = [vp, ctypes.c_longlong, ctypes.c_int, vp, vp, vp]
        L.sparse_attn_permute_fp8.argtypes = [P, PP, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_attend_fp8.argtypes = [P, PP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_strerror.argtypes = [ctypes.c_int]
        L.sparse_attn_strerror.restype = ctypes.c_char_p
        for name in EXPORTED:
            if name != "sparse_attn_strerror":
                getattr(L, name).restype = ctypes.c_int
        _LIB = L
    return _LIB


def strerror(code):
    return lib().sparse_attn_strerror(int(code)).decode()


def _check(code, where):
    if code != SA_OK:
        raise SparseAttnError(code, where)


def workspace_size(problem, policy):
    m, s = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().sparse_attn_workspace_size(ctypes.byref(problem), ctypes.byref(policy),
                                            ctypes.byref(m), ctypes.byref(s)),
           "sparse_attn_workspace_size")
    return m.value, s.value


def build_mask(problem, policy, q, k, mask_ws, scratch_ws, stream=0):
    _check(lib().sparse_attn_build_mask(ctypes.byref(problem), ctypes.byref(policy), q, k,
                                        mask_ws, scratch_ws, stream),
           "sparse_attn_build_mask")


def forward(problem, policy, q, k, v, mask_ws, scratch_ws, o, lse, stream=0):
    _check(lib().sparse_attn_forward(ctypes.byref(problem), ctypes.byref(policy), q, k, v,
                                     mask_ws, scratch_ws, o, lse, stream),
           "sparse_attn_forward")


def forward_host(problem, policy, q_host, k_host, v_host, o_host, lse_host, qkv_dev, o_dev,
                 lse_dev, mask_ws, scratch_ws, stream=0):
    _check(lib().sparse_attn_forward_host(ctypes.byref(problem), ctypes.byref(policy), q_host,
                                          k_host, v_host, o_host, lse_host, qkv_dev, o_dev,
                                          lse_dev, mask_ws, scratch_ws, stream),
           "sparse_attn_forward_host")


def permute(problem, policy, q, k, v, mask_ws, scratch_ws, stream=0):
    _check(lib().sparse_attn_permute(ctypes.byref(problem), ctypes.byref(policy), q, k, v,
                                     mask_ws, scratch_ws, stream),
           "sparse_attn_permute")


def attend(problem, policy, q, k, v, mask_ws, scratch_ws, o, lse, stream=0):
    _check(lib().sparse_attn_attend(ctypes.byref(problem), ctypes.byref(policy), q, k, v,
                                    mask_ws, scratch_ws, o, lse, stream),
           "sparse_attn_attend")


def profile_workspace_size(problem, n_rows):
    n = ctypes.c_size_t()
    _check(lib().sparse_attn_profile_workspace_size(ctypes.byref(problem), int(n_rows),
                                                    ctypes.byref(n)),
           "sparse_attn_profile_workspace_size")
    return n.value


def profile_heads(problem, policy, q, k, v, rows, n_rows, row_err, mse, is_temporal,
                  scratch_ws=None, stream=0):
    _check(lib().sparse_attn_profile_heads(ctypes.byref(problem), ctypes.byref(policy), q, k, v,
                                           rows, n_rows, row_err, mse, is_temporal, scratch_ws,
                                           stream),
           "sparse_attn_profile_heads")


def sta_window_search(problem, policy, q, k, v, rows, n_rows, candidates, n_candidates, row_err,
                      mse, choice, scratch_ws=None, stream=0):
    _check(lib().sparse_attn_sta_window_search(ctypes.byref(problem), ctypes.byref(policy), q, k,
                                               v, rows, n_rows, candidates, n_candidates, row_err,
                                               mse, choice, scratch_ws, stream),
           "sparse_attn_sta_window_search")


def build_mask_fg_cached(problem, policy, q, k, lse, tau, mask_ws, scratch_ws, stream=0):
    _check(lib().sparse_attn_build_mask_fg_cached(ctypes.byref(problem), ctypes.byref(policy), q,
                                                  k, lse, float(tau), mask_ws, scratch_ws, stream),
           "sparse_attn_build_mask_fg_cached")


def quantize_e4m3(x, n_elems, n_tensors, codes, inv, stream=0):
    _check(lib().sparse_attn_quantize_e4m3(x, n_elems, n_tensors, codes, inv, stream),
           "sparse_attn_quantize_e4m3")


def permute_fp8(problem, policy, q8, k8, v8, mask_ws, scratch_ws, stream=0):
    _check(lib().sparse_attn_permute_fp8(ctypes.byref(problem), ctypes.byref(policy), q8, k8, v8,
                                         mask_ws, scratch_ws, stream),
           "sparse_attn_permute_fp8")


def attend_fp8(problem, policy, q8, k8, v8, q_inv, k_inv, v_inv, mask_ws, scratch_ws, o, lse,
               stream=0):
    _check(lib().sparse_attn_attend_fp8(ctypes.byref(problem), ctypes.byref(policy), q8, k8, v8,
                                        q_inv, k_inv, v_inv, mask_ws, scratch_ws, o, lse, stream),
           "sparse_attn_attend_fp8")


def export_bytes(problem, policy, what):
    n = ctypes.c_size_t()
    _check(lib().sparse_attn_export_bytes(ctypes.byref(problem), ctypes.byref(policy), what,
                                          ctypes.byref(n)), "sparse_attn_export_bytes")
    return n.value


def mask_export(problem, policy, mask_ws, what, host_ptr, nbytes, stream=0):
    _check(lib().sparse_attn_mask_export(ctypes.byref(problem), ctypes.byref(policy), mask_ws,
                                         what, host_ptr, nbytes, stream),
           "sparse_attn_mask_export")


def build_mask_static(problem, policy, q, k, mask_ws, stream=0):
    """sparse_attn_build_mask with the library's static scratch array."""
    _check(lib().sparse_attn_build_mask_static(ctypes.byref(problem), ctypes.byref(policy), q, k,
                                               mask_ws, stream),
           "sparse_attn_build_mask_static")


def status_static(stream=0, clear=False):
    """Status word of the static-scratch mask build (sparse_attn_status_static)."""
    return lib().sparse_attn_status_static(stream, 1 if clear else 0)


def status(scratch_ws, stream=0, clear=False):
    return lib().sparse_attn_status(scratch_ws, stream, 1 if clear else 0)
