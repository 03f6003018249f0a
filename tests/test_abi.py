"""The C ABI without a GPU: libhq.so loads, exports every function include/*.h declares,
and refuses invalid arguments before launching anything.  Size queries are checked against
the page formulas."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in ("hq.h", "hq_debug.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(hq_[a-z0-9_]+)\s*\(", src, re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


def test_every_declared_symbol_is_exported(hq):
    names = _declared_functions()
    assert len(names) >= 14
    for n in sorted(names):
        assert hasattr(hq.lib, n), n
        assert n in hq._SIGS, f"binding lacks {n}"


def test_version_and_status_strings(hq):
    assert hq.hq_abi_version() == 1
    assert hq.status_string(0) == "HQ_OK"
    assert hq.status_string(3) == "HQ_ERR_NOT_PD"
    assert hq.status_string(99) == "HQ_ERR_UNKNOWN"


def test_bf16tril_bytes_matches_page_formula(hq):
    import oracle
    for K in (1, 2, 3, 128, 5120, 6144, 17408):
        assert hq.hq_bf16tril_bytes(K) == oracle.bf16tril_bytes(K)
    assert hq.hq_bf16tril_bytes(0) == 0


def test_workspace_queries(hq):
    assert hq.hq_gptq_workspace_bytes(64, 128, 32) > 0
    assert hq.hq_gptq_workspace_bytes(64, 100, 32) == 0      # K not a multiple of 128
    assert hq.hq_gptq_workspace_bytes(64, 128, 48) == 0      # group not a multiple of 32
    assert hq.hq_gptq_workspace_bytes(0, 128, 32) == 0
    assert hq.hq_gptq_workspace_bytes(64, 384, 96) == 0      # 96 straddles 128-column blocks
    big = hq.hq_gptq_workspace_bytes(5120, 17408, 128)
    assert big >= 2 * 17408 * 17408 * 4 + 5120 * 17408 * 4
    assert hq.hq_rtn_workspace_bytes(64, 128, 32) > 0
    assert hq.hq_rtn_workspace_bytes(64, 128, 3) == 0


def test_invalid_arguments_refused_before_launch(hq):
    L = hq.lib
    fake = ctypes.c_void_p(256)  # never dereferenced: refusals happen on the host
    # NULL pointers
    assert L.hq_hessian_accumulate(None, fake, 1, 8, 8, None, None) == hq.HQ_ERR_INVALID
    assert L.hq_hessian_accumulate(fake, None, 1, 8, 8, None, None) == hq.HQ_ERR_INVALID
    # bad dtype, bad sizes
    assert L.hq_hessian_accumulate(fake, fake, 7, 8, 8, None, None) == hq.HQ_ERR_INVALID
    assert L.hq_hessian_accumulate(fake, fake, 1, -1, 8, None, None) == hq.HQ_ERR_INVALID
    assert L.hq_hessian_accumulate(fake, fake, 1, 8, 0, None, None) == hq.HQ_ERR_INVALID
    # T == 0 is a no-op that launches nothing
    assert L.hq_hessian_accumulate(fake, None, 1, 0, 8, None, None) == hq.HQ_OK
    args = dict(W=fake, dt=1, N=64, K=128, H=fake, group=32, damp=0.01, imp=None, codes=fake, scales=fake,
                qo=None, qd=None, ws=ctypes.c_void_p(1 << 20), wsb=1 << 40, s=None)

    def gq(**kw):
        a = dict(args, **kw)
        return L.hq_gptq_quantize(a["W"], a["dt"], a["N"], a["K"], a["H"], a["group"], a["damp"], a["imp"],
                                  a["codes"], a["scales"], a["qo"], a["qd"], a["ws"], a["wsb"], a["s"])

    assert gq(W=None) == hq.HQ_ERR_INVALID
    assert gq(dt=5) == hq.HQ_ERR_INVALID
    assert gq(damp=0.0) == hq.HQ_ERR_INVALID
    assert gq(damp=float("nan")) == hq.HQ_ERR_INVALID
    assert gq(group=48) == hq.HQ_ERR_INVALID            # does not divide K
    assert gq(K=100, group=50) == hq.HQ_ERR_UNSUPPORTED  # K not a multiple of 128
    assert gq(K=384, group=96) == hq.HQ_ERR_UNSUPPORTED
    assert gq(ws=None) == hq.HQ_ERR_WORKSPACE
    assert gq(wsb=16) == hq.HQ_ERR_WORKSPACE
    assert gq(ws=ctypes.c_void_p((1 << 20) + 8)) == hq.HQ_ERR_WORKSPACE  # misaligned
    assert L.hq_rtn_quantize(fake, 1, 64, 128, 3, None, fake, fake, None, None, fake, 1 << 30, None) == hq.HQ_ERR_INVALID
    assert L.hq_rtn_quantize(fake, 1, 64, 128, 32, None, fake, fake, None, None, None, 1 << 30, None) == hq.HQ_ERR_WORKSPACE
    assert L.hq_hessian_pack_bf16tril(fake, 0, fake, None) == hq.HQ_ERR_INVALID
    assert L.hq_hessian_pack_bf16tril(fake, 8, ctypes.c_void_p(258), None) == hq.HQ_ERR_INVALID  # out not 16-B aligned
    assert L.hq_hessian_unpack_bf16tril(None, 8, fake, None) == hq.HQ_ERR_INVALID
    assert L.hq_imatrix(fake, 8, 0, fake, None) == hq.HQ_ERR_INVALID
    assert L.hq_qerr_terms(None, fake, None) == hq.HQ_ERR_INVALID
    assert L.hq_qerr_terms(fake, None, None) == hq.HQ_ERR_INVALID


def test_header_constants_match_the_binding(hq):
    """#define constants of hq.h that the binding repeats."""
    src = open(os.path.join(ROOT, "include", "hq.h")).read()
    m = re.search(r"#define\s+HQ_RTN_NOALLOC_MAX_GROUPS\s+(\d+)", src)
    assert m and int(m.group(1)) == hq.HQ_RTN_NOALLOC_MAX_GROUPS
    # refused on the host: one group more than the scratch holds, before anything is launched
    fake = ctypes.c_void_p(256)
    over = hq.HQ_RTN_NOALLOC_MAX_GROUPS // 2 + 1
    assert hq.lib.hq_rtn_quantize_noalloc(fake, 0, over, 64, 32, None, fake, fake, None, None, None) == \
        hq.HQ_ERR_UNSUPPORTED


def test_bounds_build_exports_the_same_symbols():
    """libhq_bounds.so (the HQ_DEBUG_BOUNDS build) is built beside libhq.so and exports every
    declared function too."""
    path = os.path.join(ROOT, "post_weight_quantization_tcgen05_b200", "libhq_bounds.so")
    if not os.path.exists(path):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "hq_build", os.path.join(ROOT, "post_weight_quantization_tcgen05_b200", "build.py"))
        b = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(b)
        b.build(bounds=True)
    blib = ctypes.CDLL(path)
    for n in sorted(_declared_functions()):
        assert hasattr(blib, n), n


def test_regular_build_reports_no_bounds_checks(hq):
    """In libhq.so the checks compile away: the status says so and the self-test is refused
    without launching anything."""
    assert hq.hq_debug_bounds_status() == (False, 0)
    with pytest.raises(hq.HQError) as e:
        hq.hq_debug_bounds_selftest(stream=0)
    assert e.value.status == hq.HQ_ERR_UNSUPPORTED


def test_bounds_file_tag_matches_the_device_side_hash(hq):
    """The tag the binding computes for a file name follows the same hash as the device macro
    (31-multiplier rolling hash of the bytes, 15 bits, low bit set): fixed values."""
    def ref(name):
        h = 0
        for c in name.encode():
            h = (h * 31 + c) % 32768
        return h | 1
    for n in ("api.cu", "gptq.cu", "syrk.cu", "codec.cu", "factor.cu"):
        assert hq.bounds_file_tag(n) == ref(n)
        assert 1 <= hq.bounds_file_tag(n) < 32768


def test_i8x_scratch_sizes_keep_256_byte_alignment(hq):
    """The int8-sliced GEMM's scratch size is a multiple of 256 bytes (the factorisation places
    one scratch per stream back to back, and the product requires a 256-byte aligned base)."""
    for M, N, K in ((64, 64, 32), (1280, 1280, 1280), (2560, 2560, 2560), (8704, 8704, 8704), (1000, 600, 300)):
        assert hq.lib.hq_debug_i8x_scratch_bytes(M, N, K) % 256 == 0


def test_i8x_scratch_covers_whole_tile_blocks(hq):
    """The slices are stored in whole tile blocks (A rows in blocks of 128, B rows in blocks of
    64, the contraction in 32-byte chunks, 7 slices), and every pipeline stage of the product is
    one bulk copy of a whole block; the scratch therefore holds the padded blocks of both
    operands plus the row exponents, so that the last block's copies stay inside it."""
    def up(x, m):
        return (x + m - 1) // m * m
    for M, N, K in ((1, 1, 1), (64, 64, 32), (129, 65, 33), (1000, 600, 300), (2560, 1280, 2560)):
        kp = up(K, 32)
        need = up(7 * up(M, 128) * kp, 256) + up(7 * up(N, 64) * kp, 256) + up(4 * M, 256) + up(4 * N, 256)
        assert hq.lib.hq_debug_i8x_scratch_bytes(M, N, K) >= need, (M, N, K)
