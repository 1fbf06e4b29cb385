"""CPU-side checks of the C ABI: the library builds and loads without a GPU, exports every
function include/mxattn.h declares, and rejects bad arguments on the host before any CUDA call."""
import os
import re

import pytest

from mxfp4_microscaled_bit_quantize_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxattn.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 0x100000  # aligned non-null address; never dereferenced by the host-side checks


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxattn_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n


def test_status_strings_and_version(lib):
    assert lib.mxattn_version() >= 100
    assert lib.mxattn_status_string(0) == b"ok"
    assert lib.mxattn_status_string(5) == b"device pipeline timeout"
    assert lib.mxattn_status_string(99) == b"unknown status"


def test_quantize_argument_checks(lib):
    q = lib.mxattn_quantize
    assert q(None, 0, 10, 10, 0, 1, None, None, None) == OK          # empty: no-op
    assert q(None, 1, 10, 10, 0, 1, None, None, None) == INVALID
    assert q(FAKE, 1, 10, 10, 0, 7, FAKE, FAKE, None) == INVALID        # bad mode
    assert q(FAKE, 1, 10, 10, 2, 1, FAKE, FAKE, None) == INVALID        # bad transpose flag
    assert q(FAKE + 1, 1, 10, 10, 0, 1, FAKE, FAKE, None) == INVALID    # misaligned x
    assert q(FAKE, 1, 10, 10, 0, 1, FAKE + 8, FAKE, None) == INVALID    # misaligned codes
    assert q(FAKE, -1, 10, 10, 0, 1, FAKE, FAKE, None) == INVALID
    assert q(FAKE, 70000, 32, 32, 1, 1, FAKE, FAKE, None) == UNSUPPORTED
    assert q(FAKE, 1 << 20, 1 << 20, 1024, 0, 1, FAKE, FAKE, None) == UNSUPPORTED


def _ws_mirror(B, Hq, Hkv, N, d):
    up = lambda x, a: -(-x // a) * a  # noqa: E731
    npad = up(N, 128)
    t = npad // 128
    off = 1024
    qk_atoms = d // 64 if d >= 128 else 1
    for nbytes in (B * Hq * npad * d // 2, B * Hq * t * qk_atoms * 512, B * Hkv * npad * d // 2,
                   B * Hkv * t * qk_atoms * 512, B * Hkv * d * npad // 2, B * Hkv * t * 1024):
        off = up(off + nbytes, 1024)
    return off


@pytest.mark.parametrize("shape", [(1, 2, 2, 256, 64), (1, 40, 40, 32760, 128), (4, 32, 8, 8192, 128),
                                   (1, 24, 24, 76800, 128), (2, 3, 1, 1, 64)])
def test_workspace_size(lib, shape):
    assert lib.mxattn_forward_workspace_size(*shape) == _ws_mirror(*shape)


def test_workspace_size_rejects_bad_shapes(lib):
    ws = lib.mxattn_forward_workspace_size
    assert ws(1, 2, 2, 256, 96) == 0
    assert ws(1, 3, 2, 256, 64) == 0
    assert ws(1, 2, 2, 0, 64) == 0


def _host_ws_mirror(B, Hq, Hkv, N, d, out_bytes):
    """Three device slots, each holding one chunk of KV heads: bf16 Q, K, V, the output and the
    chunk's own attention workspace. A chunk covers about 512 attention CTAs (whole KV heads)."""
    up = lambda x, a: -(-x // a) * a  # noqa: E731
    group, units, n_qt = Hq // Hkv, B * Hkv, -(-N // 128)
    cg = min(max(-(-512 // (group * n_qt)), 1), units)
    hd = N * d
    slot = (up(cg * group * hd * 2, 1024) + 2 * up(cg * hd * 2, 1024) + up(cg * group * hd * out_bytes, 1024)
            + up(_ws_mirror(1, cg * group, cg, N, d), 1024))
    return 1024 + 3 * slot


@pytest.mark.parametrize("shape", [(1, 2, 2, 256, 64), (1, 40, 40, 32760, 128), (4, 32, 8, 8192, 128),
                                   (1, 24, 24, 76800, 128), (2, 3, 1, 1, 64)])
def test_host_workspace_size(lib, shape):
    hw = lib.mxattn_forward_host_workspace_size
    assert hw(*shape, 0) == _host_ws_mirror(*shape, 4)
    assert hw(*shape, 1) == _host_ws_mirror(*shape, 2)
    assert hw(*shape, 2) == 0                                   # no such output type
    # a fraction of what mxattn_forward holds on the device (bf16 Q, K, V, fp32 output, workspace)
    B, Hq, Hkv, N, d = shape
    if Hkv >= 8:
        resident = (2 * B * (Hq + 2 * Hkv) + 4 * B * Hq) * N * d + lib.mxattn_forward_workspace_size(*shape)
        assert hw(*shape, 0) < resident / 4


def test_host_forward_argument_checks(lib):
    f = lib.mxattn_forward_host
    good = lib.mxattn_forward_host_workspace_size(1, 2, 2, 256, 64, 0)

    def call(q=FAKE, out=FAKE, Hq=2, d=64, mode=1, od=0, wsb=good):
        return f(q, FAKE, FAKE, out, 1, Hq, 2, 256, d, 0, mode, 1, od, FAKE, wsb, None)

    assert call(q=None) == INVALID
    assert call(out=None) == INVALID
    assert call(Hq=3) == INVALID
    assert call(mode=3) == INVALID
    assert call(od=5) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(wsb=good - 1) == WORKSPACE


def test_forward_argument_checks(lib):
    f = lib.mxattn_forward
    good = lib.mxattn_forward_workspace_size(1, 2, 2, 256, 64)
    args = lambda **kw: dict(dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, Hq=2, Hkv=2, N=256, d=64,  # noqa: E731
                                  causal=0, mode=1, pnq=1, od=0, ws=FAKE, wsb=good, st=None), **kw)

    def call(**kw):
        a = args(**kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["causal"],
                 a["mode"], a["pnq"], a["od"], a["ws"], a["wsb"], a["st"])

    assert call(d=96) == UNSUPPORTED
    assert call(Hq=3) == INVALID
    assert call(N=0) == INVALID
    assert call(mode=3) == INVALID
    assert call(od=5) == INVALID
    assert call(q=None) == INVALID
    assert call(q=FAKE + 2) == INVALID
    assert call(ws=FAKE + 16) == INVALID
    assert call(wsb=good - 1) == WORKSPACE
    # the P~ rule: conventional, PNQ or exp-free; the exp-free rule needs power-of-two scales
    assert call(pnq=3) == INVALID
    assert call(pnq=-1) == INVALID
    assert call(pnq=2, mode=2) == UNSUPPORTED
    assert call(pnq=2, wsb=good - 1) == WORKSPACE      # accepted up to the workspace check


def test_forward_quantized_argument_checks(lib):
    f = lib.mxattn_forward_quantized
    good = lib.mxattn_forward_workspace_size(1, 2, 2, 256, 64)
    ops = [FAKE] * 6

    def call(ops=ops, out=FAKE, d=64, mode=1, wsb=good):
        return f(*ops, out, 1, 2, 2, 256, d, 0, mode, 1, 0, FAKE, wsb, None)

    assert call(ops=[None] + ops[1:]) == INVALID
    assert call(out=None) == INVALID
    assert call(ops=[FAKE + 8] + ops[1:]) == INVALID                  # codes must be 16-byte aligned
    assert call(ops=ops[:4] + [FAKE + 4, FAKE]) == INVALID
    assert call(ops=[FAKE, FAKE + 1] + ops[2:], wsb=good - 1) == WORKSPACE   # scales: any alignment
    assert call(d=96) == UNSUPPORTED
    assert call(mode=3) == INVALID


def _gemm_ws_mirror(M, N, K):
    up = lambda x, a: -(-x // a) * a  # noqa: E731
    kst = -(-K // 256)
    off = 1024
    for rows in (-(-M // 128), 2 * -(-N // 256)):
        off = up(off + rows * 2 * kst * 512, 1024)
    return off


def test_gemm_workspace_and_argument_checks(lib):
    ws = lib.mxattn_gemm_workspace_size
    for shape in [(1, 8, 32), (300, 520, 992), (16384, 16384, 8192)]:
        assert ws(*shape) == _gemm_ws_mirror(*shape)
    assert ws(4, 8, 48) == 0          # K % 32 != 0
    assert ws(4, 12, 64) == 0         # N % 8 != 0
    g = lib.mxattn_gemm
    good = ws(256, 256, 512)
    ok = dict(a=FAKE, sa=FAKE, b=FAKE, sb=FAKE, c=FAKE, M=256, N=256, K=512, od=0, w=FAKE, wb=good)

    def call(**kw):
        x = dict(ok, **kw)
        return g(x["a"], x["sa"], x["b"], x["sb"], x["c"], x["M"], x["N"], x["K"], x["od"], x["w"], x["wb"], None)

    assert call(a=None) == INVALID
    assert call(b=FAKE + 8) == INVALID
    assert call(c=FAKE + 4) == INVALID
    assert call(od=3) == INVALID
    assert call(K=100) == UNSUPPORTED
    assert call(N=250) == UNSUPPORTED
    assert call(wb=good - 1) == WORKSPACE


def test_nvfp4_argument_checks(lib):
    q = lib.mxattn_quantize_nvfp4
    assert q(None, 0, 16, None, None, None) == OK                   # empty: no-op
    assert q(None, 4, 16, FAKE, FAKE, None) == INVALID
    assert q(FAKE + 1, 4, 16, FAKE, FAKE, None) == INVALID           # misaligned x
    assert q(FAKE, 4, 16, FAKE + 4, FAKE, None) == INVALID           # misaligned codes
    ws = lib.mxattn_gemm_nvfp4_workspace_size
    assert ws(4, 12, 64) == 0 and ws(4, 8, 48) == 0
    assert ws(300, 520, 992) > lib.mxattn_gemm_workspace_size(300, 520, 992)   # twice the scale atoms
    g = lib.mxattn_gemm_nvfp4
    good = ws(256, 256, 512)
    assert g(None, FAKE, FAKE, FAKE, FAKE, 256, 256, 512, 0, FAKE, good, None) == INVALID
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 256, 250, 512, 0, FAKE, good, None) == UNSUPPORTED
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 256, 256, 512, 0, FAKE, good - 1, None) == WORKSPACE


def test_debug_argument_checks(lib):
    good = lib.mxattn_forward_workspace_size(1, 2, 2, 256, 64)
    r = lib.mxattn_forward_debug(FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 1, 1, 0, FAKE, good, None,
                                 5, 0, 16, FAKE, FAKE)   # head index out of range
    assert r == INVALID
    r = lib.mxattn_forward_debug(FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 1, 1, 0, FAKE, good, None,
                                 0, 10, 5, FAKE, FAKE)   # empty row range
    assert r == INVALID


def test_kv_tile_constant_agrees():
    """P~ codes depend on the online-softmax tile width; the binding and the oracle's default
    must use the width the library declares."""
    from mxfp4_microscaled_bit_quantize_b200 import api
    from oracle import attention as oa
    m = re.search(r"#define\s+MXATTN_KV_TILE\s+(\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == api.KV_TILE == oa.KV_TILE
