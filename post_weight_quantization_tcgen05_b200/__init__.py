"""Python binding of libhq.so: GPTQ int4 weight quantisation and the Bf16TrilDiagF32 codec
on NVIDIA B200 (sm_100a).

Argument marshalling only: every function checks tensor dtypes, shapes and devices, turns
them into raw pointers and sizes, and calls the C entry point of the same name (declared in
include/hq.h and include/hq_debug.h).  Every step of the computation runs in the library's
CUDA kernels.  Importing this package fails loudly when libhq.so has not been built
(``python post_weight_quantization_tcgen05_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os

import torch

# HQ_LIBRARY=libhq_bounds.so selects the bounds-checking build of the same library (hq_debug.h);
# no other name is accepted.
_LIB_NAME = os.environ.get("HQ_LIBRARY", "libhq.so")
if _LIB_NAME not in ("libhq.so", "libhq_bounds.so"):
    raise ImportError(f"HQ_LIBRARY must be libhq.so or libhq_bounds.so, not {_LIB_NAME!r}")
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)

HQ_OK = 0
HQ_ERR_INVALID = 1
HQ_ERR_UNSUPPORTED = 2
HQ_ERR_NOT_PD = 3
HQ_ERR_TIMEOUT = 4
HQ_ERR_CUDA = 5
HQ_ERR_WORKSPACE = 6
HQ_F32 = 0
HQ_BF16 = 1
# groups N * (K / group) that hq_rtn_quantize_noalloc's fixed scratch holds (hq.h)
HQ_RTN_NOALLOC_MAX_GROUPS = 1048576

_DTYPE = {torch.float32: HQ_F32, torch.bfloat16: HQ_BF16}


class HQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_NAME} not found at {_LIB_PATH}; build it with "
                      "`python post_weight_quantization_tcgen05_b200/build.py`")

lib = ctypes.CDLL(_LIB_PATH)

_vp, _i64, _int, _f, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_dbl = ctypes.c_double

_SIGS = {
    "hq_status_string": (ctypes.c_char_p, [_int]),
    "hq_abi_version": (_int, []),
    "hq_hessian_accumulate": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp]),
    "hq_imatrix": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "hq_gptq_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "hq_gptq_quantize": (_int, [_vp, _int, _i64, _i64, _vp, _i64, _f, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hq_rtn_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "hq_rtn_quantize": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hq_rtn_quantize_noalloc": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "hq_qerr_terms": (_int, [_vp, _vp, _vp]),
    "hq_qerr_from_terms": (_int, [_vp, _vp, _vp]),
    "hq_gptq_factor_bytes": (_sz, [_i64]),
    "hq_gptq_factor_workspace_bytes": (_sz, [_i64]),
    "hq_gptq_sweep_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "hq_gptq_factorize": (_int, [_vp, _i64, _f, _vp, _sz, _vp, _sz, _vp]),
    "hq_gptq_sweep": (_int, [_vp, _int, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hq_tril32_count": (_sz, [_i64]),
    "hq_hessian_pack_lower": (_int, [_vp, _i64, _vp, _vp]),
    "hq_hessian_unpack_lower": (_int, [_vp, _i64, _vp, _vp]),
    "hq_hadamard_rotate_weights": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp]),
    "hq_hadamard_rotate_hessian": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "hq_psd_workspace_bytes": (_sz, [_i64]),
    "hq_hessian_project_psd": (_int, [_vp, _i64, _int, _vp, _sz, _vp]),
    "hq_bf16tril_bytes": (_sz, [_i64]),
    "hq_hessian_pack_bf16tril": (_int, [_vp, _i64, _vp, _vp]),
    "hq_hessian_unpack_bf16tril": (_int, [_vp, _i64, _vp, _vp]),
    "hq_debug_factor": (_int, [_vp, _i64, _f, _vp, _vp, _sz, _vp]),
    "hq_debug_gptq_quantize_impl": (_int, [_vp, _int, _i64, _i64, _vp, _i64, _f, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                           _int, _vp]),
    "hq_debug_hessian_accumulate_impl": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _int, _vp]),
    "hq_debug_hessian_accumulate_timeout": (_int, [_vp, _vp, _i64, _i64, _vp, _i64, _int, _vp]),
    "hq_debug_launch_count": (ctypes.c_uint64, []),
    "hq_debug_bounds_status": (_int, [_vp, _vp]),
    "hq_debug_bounds_selftest": (_int, [_vp]),
    "hq_debug_rcp_f64": (_int, [_vp, _vp, _i64, _vp]),
    "hq_debug_upd_gemm": (_int, [_vp, _i64, _int, _int, _int, _vp, _vp, _i64, _vp, _vp, _i64, _vp]),
    "hq_debug_fp64_mma_rate": (ctypes.c_double, [_vp, _i64, _vp]),
    "hq_debug_timing_start": (_int, [_int]),
    "hq_debug_timing_serialize": (_int, [_int]),
    "hq_debug_timing_stop": (_int, []),
    "hq_debug_timing_read": (_int, [_int, _vp, _vp, _vp]),
    "hq_debug_f64_gemm": (_int, [_vp, _i64, _int, _int, _int, _vp, _i64, _vp, _i64, _dbl, _dbl, _int, _int, _vp,
                                 _i64, _vp]),
    "hq_debug_i8x_scratch_bytes": (_sz, [_int, _int, _int]),
    "hq_debug_i8x_gemm": (_int, [_vp, _i64, _int, _int, _int, _vp, _i64, _vp, _i64, _dbl, _dbl, _int, _int, _vp,
                                 _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def status_string(status: int) -> str:
    return lib.hq_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != HQ_OK:
        raise HQError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype(t) -> int:
    if t.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DTYPE[t.dtype]


# --------------------------------------------------------------------------- entry points

def hq_abi_version() -> int:
    return lib.hq_abi_version()


def hq_debug_launch_count() -> int:
    return int(lib.hq_debug_launch_count())


def hq_debug_bounds_status():
    """(enabled, violation): whether this is the bounds-checking build, and the first recorded
    failing index check (0 if none; cleared by the call)."""
    en, v = ctypes.c_int(), ctypes.c_int()
    _check(lib.hq_debug_bounds_status(ctypes.byref(en), ctypes.byref(v)), "hq_debug_bounds_status")
    return bool(en.value), int(v.value)


def hq_debug_bounds_selftest(stream=None) -> None:
    """Launch one index check that fails by construction (bounds-checking build only)."""
    _check(lib.hq_debug_bounds_selftest(_stream(stream)), "hq_debug_bounds_selftest")


def bounds_file_tag(name: str) -> int:
    """The tag the bounds-checking build records for source file `name` (bits 16-30)."""
    h = 0
    for c in name.encode():
        h = (h * 31 + c) & 0x7FFF
    return h | 1


def hq_hessian_accumulate(H, X, dev_status=None, stream=None) -> None:
    """H (fp32 [K, K]) += X^T X on the lower triangle; X [T, K] bf16 or fp32."""
    T, K = X.shape
    if H.dtype != torch.float32 or tuple(H.shape) != (K, K):
        raise ValueError("H must be fp32 [K, K]")
    _check(lib.hq_hessian_accumulate(_ptr(H), _ptr(X), _dtype(X), T, K, _ptr(dev_status), _stream(stream)),
           "hq_hessian_accumulate")


def hq_debug_hessian_accumulate_impl(H, X, impl: int, dev_status=None, stream=None) -> None:
    T, K = X.shape
    _check(lib.hq_debug_hessian_accumulate_impl(_ptr(H), _ptr(X), _dtype(X), T, K, _ptr(dev_status), int(impl),
                                                _stream(stream)), "hq_debug_hessian_accumulate_impl")


def hq_debug_hessian_accumulate_timeout(H, X, dev_status, wait_limit_cycles: int, withhold_stage: int = -1,
                                        stream=None) -> None:
    """The tensor-core SYRK with a runtime wait limit and, for the test of its timeout path, one
    operand stage the MMA issuer never releases (hq_debug.h)."""
    if X.dtype != torch.bfloat16:
        raise ValueError("the tensor-core SYRK takes bf16 X")
    T, K = X.shape
    st = lib.hq_debug_hessian_accumulate_timeout(_ptr(H), _ptr(X), T, K, _ptr(dev_status), int(wait_limit_cycles),
                                                 int(withhold_stage), _stream(stream))
    _check(st, "hq_debug_hessian_accumulate_timeout")


def hq_imatrix(H, tokens: int, imp, stream=None) -> None:
    K = H.shape[0]
    _check(lib.hq_imatrix(_ptr(H), K, int(tokens), _ptr(imp), _stream(stream)), "hq_imatrix")


def hq_gptq_workspace_bytes(N: int, K: int, group: int) -> int:
    return int(lib.hq_gptq_workspace_bytes(N, K, group))


def hq_rtn_workspace_bytes(N: int, K: int, group: int) -> int:
    return int(lib.hq_rtn_workspace_bytes(N, K, group))


def hq_gptq_quantize(W, H, group: int, damp: float, codes, scales, workspace, imp=None, want_qerr: bool = True,
                     qerr_dev=None, stream=None):
    """GPTQ int4 of W [N, K] against the undamped fp32 H; returns qerr (host) if requested."""
    N, K = W.shape
    q = ctypes.c_double(float("nan"))
    st = lib.hq_gptq_quantize(_ptr(W), _dtype(W), N, K, _ptr(H), int(group), float(damp), _ptr(imp), _ptr(codes),
                              _ptr(scales), ctypes.byref(q) if want_qerr else None, _ptr(qerr_dev), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hq_gptq_quantize")
    return q.value if want_qerr else None


def hq_gptq_factor_bytes(K: int) -> int:
    return int(lib.hq_gptq_factor_bytes(K))


def hq_gptq_factor_workspace_bytes(K: int) -> int:
    return int(lib.hq_gptq_factor_workspace_bytes(K))


def hq_gptq_sweep_workspace_bytes(N: int, K: int, group: int) -> int:
    return int(lib.hq_gptq_sweep_workspace_bytes(N, K, group))


def hq_gptq_factorize(H, damp: float, factor, workspace, stream=None) -> None:
    """Damping and factorisation of the undamped fp32 H [K, K] into the factor buffer (uint8)."""
    K = H.shape[0]
    st = lib.hq_gptq_factorize(_ptr(H), K, float(damp), _ptr(factor), factor.numel() * factor.element_size(),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hq_gptq_factorize")


def hq_gptq_sweep(W, factor, group: int, codes, scales, workspace, imp=None, want_qerr: bool = True, qerr_dev=None,
                  stream=None):
    """The GPTQ sweep of W [N, K] against a factor buffer; returns qerr (host) if requested."""
    N, K = W.shape
    q = ctypes.c_double(float("nan"))
    st = lib.hq_gptq_sweep(_ptr(W), _dtype(W), N, K, _ptr(factor), int(group), _ptr(imp), _ptr(codes), _ptr(scales),
                           ctypes.byref(q) if want_qerr else None, _ptr(qerr_dev), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hq_gptq_sweep")
    return q.value if want_qerr else None


def hq_qerr_from_terms(terms_dev, qerr_dev, stream=None) -> None:
    _check(lib.hq_qerr_from_terms(_ptr(terms_dev), _ptr(qerr_dev), _stream(stream)), "hq_qerr_from_terms")


def hq_tril32_count(K: int) -> int:
    return int(lib.hq_tril32_count(K))


def _need_f32(*ts) -> None:
    for t in ts:
        if t.dtype != torch.float32:
            raise ValueError("expected an fp32 tensor")


def hq_hessian_pack_lower(H, packed, stream=None) -> None:
    _need_f32(H, packed)
    K = H.shape[0]
    _check(lib.hq_hessian_pack_lower(_ptr(H), K, _ptr(packed), _stream(stream)), "hq_hessian_pack_lower")


def hq_hessian_unpack_lower(packed, K: int, H, stream=None) -> None:
    _need_f32(H, packed)
    _check(lib.hq_hessian_unpack_lower(_ptr(packed), K, _ptr(H), _stream(stream)), "hq_hessian_unpack_lower")


def hq_debug_gptq_quantize_impl(W, H, group: int, damp: float, codes, scales, workspace, update_impl: int, imp=None,
                                want_qerr: bool = True, qerr_dev=None, stream=None):
    N, K = W.shape
    q = ctypes.c_double(float("nan"))
    st = lib.hq_debug_gptq_quantize_impl(_ptr(W), _dtype(W), N, K, _ptr(H), int(group), float(damp), _ptr(imp),
                                         _ptr(codes), _ptr(scales), ctypes.byref(q) if want_qerr else None,
                                         _ptr(qerr_dev), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         int(update_impl), _stream(stream))
    _check(st, "hq_debug_gptq_quantize_impl")
    return q.value if want_qerr else None


def hq_rtn_quantize(W, group: int, codes, scales, workspace, imp=None, want_qerr: bool = True, qerr_dev=None,
                    stream=None):
    N, K = W.shape
    q = ctypes.c_double(float("nan"))
    st = lib.hq_rtn_quantize(_ptr(W), _dtype(W), N, K, int(group), _ptr(imp), _ptr(codes), _ptr(scales),
                             ctypes.byref(q) if want_qerr else None, _ptr(qerr_dev), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hq_rtn_quantize")
    return q.value if want_qerr else None


def hq_rtn_quantize_noalloc(W, group: int, codes, scales, imp=None, want_qerr: bool = True, qerr_dev=None,
                            stream=None):
    """hq_rtn_quantize with the library's own fixed scratch instead of a workspace."""
    N, K = W.shape
    q = ctypes.c_double(float("nan"))
    st = lib.hq_rtn_quantize_noalloc(_ptr(W), _dtype(W), N, K, int(group), _ptr(imp), _ptr(codes), _ptr(scales),
                                     ctypes.byref(q) if want_qerr else None, _ptr(qerr_dev), _stream(stream))
    _check(st, "hq_rtn_quantize_noalloc")
    return q.value if want_qerr else None


def hq_psd_workspace_bytes(K: int) -> int:
    return int(lib.hq_psd_workspace_bytes(int(K)))


def hq_hessian_project_psd(H, workspace=None, steps: int = 40, stream=None) -> None:
    """H (fp32 [K, K], symmetric, device) <- its projection onto the PSD cone, in place."""
    K = H.shape[0]
    if workspace is None:
        workspace = alloc_workspace(hq_psd_workspace_bytes(K), H.device)
    _check(lib.hq_hessian_project_psd(_ptr(H), K, int(steps), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "hq_hessian_project_psd")


def hq_hadamard_rotate_weights(W, signs, block: int, W_out, stream=None) -> None:
    """W_out (fp32 [N, K]) = W R, R = diag(signs) blockdiag(Hadamard_block / sqrt(block))."""
    N, K = W.shape
    _check(lib.hq_hadamard_rotate_weights(_ptr(W), _dtype(W), N, K, int(block), _ptr(signs), _ptr(W_out),
                                          _stream(stream)), "hq_hadamard_rotate_weights")


def hq_hadamard_rotate_hessian(H, signs, block: int, H_out, stream=None) -> None:
    """H_out (fp32 [K, K]) = R^T H R, H read from its lower triangle."""
    K = H.shape[0]
    _check(lib.hq_hadamard_rotate_hessian(_ptr(H), K, int(block), _ptr(signs), _ptr(H_out), _stream(stream)),
           "hq_hadamard_rotate_hessian")


def hq_qerr_terms(workspace, terms_dev, stream=None) -> None:
    """terms_dev (fp64 [2], device) <- the qerr numerator and denominator sums of the last
    quantisation that used `workspace`."""
    _check(lib.hq_qerr_terms(_ptr(workspace), _ptr(terms_dev), _stream(stream)), "hq_qerr_terms")


def hq_debug_factor(H, damp: float, Ut_out, workspace, stream=None) -> None:
    K = H.shape[0]
    _check(lib.hq_debug_factor(_ptr(H), K, float(damp), _ptr(Ut_out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "hq_debug_factor")


def hq_debug_fp64_mma_rate(stream=None) -> float:
    """Measured fp64 MMA rate (TFLOP/s) of a kernel that does nothing else."""
    scratch = torch.empty(296 * 256, dtype=torch.float64, device="cuda")
    r = lib.hq_debug_fp64_mma_rate(_ptr(scratch), scratch.numel() * 8, _stream(stream))
    if r < 0:
        raise HQError(HQ_ERR_CUDA, "hq_debug_fp64_mma_rate")
    return float(r)


TIMING_CLASSES = {"f64_gemm_128": 0, "f64_gemm_64": 1, "leaf": 2, "sweep": 3, "tf32_gemm": 4, "syrk": 5,
                  "i8x_gemm": 6, "i8x_slice": 7}


def hq_debug_timing_start(classes) -> None:
    """Start event timing of the named kernel classes (see TIMING_CLASSES)."""
    mask = 0
    for c in classes:
        mask |= 1 << TIMING_CLASSES[c]
    _check(lib.hq_debug_timing_start(mask), "hq_debug_timing_start")


def hq_debug_timing_serialize(on: bool) -> None:
    """Run the factorisation's second-stream work on the caller's stream (on) or not (off)."""
    _check(lib.hq_debug_timing_serialize(1 if on else 0), "hq_debug_timing_serialize")


def hq_debug_timing_stop() -> None:
    _check(lib.hq_debug_timing_stop(), "hq_debug_timing_stop")


def hq_debug_timing_read(cls: str):
    """(total ms, total work, launches) recorded for one kernel class."""
    ms, work, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_int64()
    _check(lib.hq_debug_timing_read(TIMING_CLASSES[cls], ctypes.byref(ms), ctypes.byref(work), ctypes.byref(n)),
           "hq_debug_timing_read")
    return ms.value, work.value, n.value


def hq_debug_upd_gemm(C, A_hi, A_lo, B_hi, B_lo, stream=None) -> None:
    """C -= (A_hi + A_lo) (B_hi + B_lo)^T by the lazy-update kernel (3xTF32)."""
    M, Kred = A_hi.shape
    N = B_hi.shape[0]
    _check(lib.hq_debug_upd_gemm(_ptr(C), C.stride(0), M, N, Kred, _ptr(A_hi), _ptr(A_lo), A_hi.stride(0),
                                 _ptr(B_hi), _ptr(B_lo), B_hi.stride(0), _stream(stream)), "hq_debug_upd_gemm")


def hq_debug_rcp_f64(d, out, stream=None) -> None:
    """out = 1 / d (fp64) by the factorisation leaf's pivot reciprocal."""
    _check(lib.hq_debug_rcp_f64(_ptr(d), _ptr(out), d.numel(), _stream(stream)), "hq_debug_rcp_f64")


def hq_debug_f64_gemm(C, A, B, alpha=1.0, beta=0.0, lower=False, tri=0, scratch=None, stream=None) -> None:
    """C = beta C + alpha A B^T (fp64 row-major views, fp64 tensor cores); tri declares a triangular operand."""
    M, Kred = A.shape
    N = B.shape[0]
    _check(lib.hq_debug_f64_gemm(_ptr(C), C.stride(0), M, N, Kred, _ptr(A), A.stride(0), _ptr(B), B.stride(0),
                                 float(alpha), float(beta), int(bool(lower)), int(tri), _ptr(scratch),
                                 0 if scratch is None else scratch.numel(), _stream(stream)), "hq_debug_f64_gemm")


def hq_debug_i8x_gemm(C, A, B, alpha=1.0, beta=0.0, lower=False, tri=0, scratch=None, stream=None) -> None:
    """C = beta C + alpha A B^T (fp64) through the int8-sliced tensor-core GEMM (hq_debug.h)."""
    M, Kred = A.shape
    N = B.shape[0]
    need = lib.hq_debug_i8x_scratch_bytes(M, N, Kred)
    if scratch is None:
        scratch = alloc_workspace(need, C.device)
    st = lib.hq_debug_i8x_gemm(_ptr(C), C.shape[1], M, N, Kred, _ptr(A), A.shape[1], _ptr(B), B.shape[1],
                               float(alpha), float(beta), int(bool(lower)), int(tri), _ptr(scratch),
                               scratch.numel() * scratch.element_size(), _stream(stream))
    _check(st, "hq_debug_i8x_gemm")


def hq_bf16tril_bytes(K: int) -> int:
    return int(lib.hq_bf16tril_bytes(K))


def hq_hessian_pack_bf16tril(H, out, stream=None) -> None:
    K = H.shape[0]
    _check(lib.hq_hessian_pack_bf16tril(_ptr(H), K, _ptr(out), _stream(stream)), "hq_hessian_pack_bf16tril")


def hq_hessian_unpack_bf16tril(inp, K: int, H_full, stream=None) -> None:
    _check(lib.hq_hessian_unpack_bf16tril(_ptr(inp), K, _ptr(H_full), _stream(stream)), "hq_hessian_unpack_bf16tril")


# --------------------------------------------------------------------------- allocation helpers

def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A uint8 device buffer of nbytes (torch's caching allocator returns 512-byte aligned blocks)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def gptq_outputs(N: int, K: int, group: int, device="cuda"):
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((N, K // group), dtype=torch.float32, device=device)
    return codes, scales
