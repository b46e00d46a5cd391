"""The C-ABI library: it loads, exports every call include/fa.h declares, and
rejects bad arguments on the host before touching the GPU (no compute calls)."""
import ctypes
import math
import os
import re

import pytest

import io_aware_exact_32_b200 as fa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fa.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from io_aware_exact_32_b200 import build
    build.build()
    return fa.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_decode_splitkv", "fa_decode_workspace_size",
              "fa_quantize_fp8", "fa_fwd_fp8", "fa_fwd_ext", "fa_bwd_ext", "fa_get_device_error", "fa_status_string",
              "fa_version"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_only_declared_symbols_are_exported():
    out = os.popen(f"nm -D --defined-only {fa.lib_path}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported == set(declared_functions())


def test_status_strings(L):
    for code in range(7):
        assert len(fa.fa_status_string(code)) > 0
    assert fa.fa_version() == 100


NULL = ctypes.c_void_p(0)
A16 = ctypes.c_void_p(0x10000)      # fake, aligned, never dereferenced
MIS = ctypes.c_void_p(0x10008)      # fake, misaligned


def fwd(L, q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=1, Nq=128, Nk=128, d=64, scale=0.125, causal=0):
    return L.fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, NULL)


def test_fwd_validation(L):
    assert fwd(L, d=96) == 2
    assert fwd(L, d=32) == 2
    assert fwd(L, B=-1) == 1
    assert fwd(L, Nq=-5) == 1
    assert fwd(L, scale=0.0) == 1
    assert fwd(L, scale=float("nan")) == 1
    assert fwd(L, scale=-1.0) == 1
    assert fwd(L, Nq=(1 << 24) + 1) == 2
    assert fwd(L, q=NULL) == 1
    assert fwd(L, lse=NULL) == 1
    assert fwd(L, k=MIS) == 3
    assert fwd(L, o=MIS) == 3
    # empty problems are no-ops that launch nothing
    assert fwd(L, B=0) == 0
    assert fwd(L, H=0, q=NULL) == 0
    assert fwd(L, Nq=0, q=NULL, o=NULL, lse=NULL) == 0


def bwd(L, ws=A16, ws_bytes=1 << 30, d=64, Nq=128, Nk=128, mis=None, null=None):
    args = [A16] * 9
    if mis is not None:
        args[mis] = MIS
    if null is not None:
        args[null] = NULL
    return L.fa_bwd(*args, ws, ws_bytes, 1, 1, Nq, Nk, d, 0.125, 0, NULL)


def test_bwd_validation(L):
    assert bwd(L, d=80) == 2
    assert bwd(L, null=4) == 1          # dO
    assert bwd(L, null=5) == 1          # lse
    assert bwd(L, mis=7) == 3           # dk
    assert bwd(L, ws=NULL) == 4
    assert bwd(L, ws_bytes=16) == 4
    assert bwd(L, ws=ctypes.c_void_p(0x10010)) == 3   # workspace must be 256-byte aligned
    assert L.fa_bwd_workspace_size(2, 8, 1024, 64) == 2 * 8 * 1024 * 4 + 2 * 8 * 1024 * 64 * 4
    assert L.fa_bwd_workspace_size(1, 1, 3, 128) == 256 + 3 * 128 * 4 + (256 - (3 * 128 * 4) % 256) % 256
    assert L.fa_bwd_workspace_size(1, 1, 8, 96) == 0


def dec(L, Lmax=8192, d=128, S=0, ws_bytes=1 << 30, seq=A16, q=A16, ws=A16):
    return L.fa_decode_splitkv(q, A16, A16, seq, Lmax, A16, A16, 2, 4, d, 0.088, S, ws, ws_bytes, NULL)


def test_decode_validation(L):
    assert dec(L, d=256) == 2
    assert dec(L, Lmax=0) == 1
    assert dec(L, S=257) == 2
    assert dec(L, S=-1) == 1
    assert dec(L, seq=NULL) == 1
    assert dec(L, seq=ctypes.c_void_p(0x10002)) == 3
    assert dec(L, q=MIS) == 3
    assert dec(L, ws_bytes=8) == 4
    n = L.fa_decode_workspace_size(2, 4, 8192, 128, 0)
    assert n >= 2 * 4 * 8 * (128 + 2) * 4
    assert L.fa_decode_workspace_size(2, 4, 8192, 128, 3) == 2 * 4 * 3 * 128 * 4 + 256
    assert L.fa_decode_workspace_size(2, 4, 0, 128, 0) == 0


def test_binding_rejects_bad_tensors():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 1, 4, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        fa.fa_fwd(q, q, q, q, torch.zeros(1, 1, 4), causal=False)


def test_fp8_validation(L):
    def fwd8(d=128, q=A16, dq=A16, dv=A16, o=A16, Nq=128, Nk=128, B=1):
        return L.fa_fwd_fp8(q, A16, A16, dq, A16, dv, o, A16, B, 1, Nq, Nk, d, 0.088, 1, NULL)

    assert fwd8(d=64) == 2
    assert fwd8(d=96) == 2
    assert fwd8(q=NULL) == 1
    assert fwd8(dq=NULL) == 1
    assert fwd8(dv=NULL) == 1
    assert fwd8(o=MIS) == 3
    assert fwd8(dq=ctypes.c_void_p(0x10002)) == 3
    assert fwd8(B=0) == 0
    assert fwd8(Nq=0, q=NULL, o=NULL) == 0

    def quant(d=128, x=A16, x8=A16, ds=A16, signs=NULL, N=64, B=1):
        return L.fa_quantize_fp8(x, signs, x8, ds, B, 1, N, d, 1, NULL)

    assert quant(d=32) == 2
    assert quant(N=-1) == 1
    assert quant(ds=NULL) == 1
    assert quant(x=NULL) == 1
    assert quant(x8=MIS) == 3
    assert quant(ds=ctypes.c_void_p(0x10001)) == 3
    assert quant(signs=ctypes.c_void_p(0x10002)) == 3
    assert quant(B=0) == 0


def test_ext_validation(L):
    def fwdx(p=0.1, bias=A16, bB=1, bH=1, Nk=128, B=2, d=64):
        return L.fa_fwd_ext(A16, A16, A16, bias, bB, bH, A16, A16, B, 2, 128, Nk, d, 0.125, 1, p, 7, 0, NULL)

    assert fwdx(p=1.0) == 1
    assert fwdx(p=-0.1) == 1
    assert fwdx(p=float("nan")) == 1
    assert fwdx(Nk=130) == 2            # a bias needs Nk % 8 == 0
    assert fwdx(bB=3) == 1
    assert fwdx(bH=0) == 1
    assert fwdx(bias=ctypes.c_void_p(0x10008)) == 3
    assert fwdx(d=96) == 2
    assert fwdx(B=0) == 0

    def bwdx(p=0.1, bias=A16, ws=A16):
        args = [A16] * 6 + [bias, 1, 1] + [A16] * 3
        return L.fa_bwd_ext(*args, ws, 1 << 30, 1, 1, 128, 128, 64, 0.125, 0, p, 7, 0, NULL)

    assert bwdx(p=1.5) == 1
    assert bwdx(bias=ctypes.c_void_p(0x10004)) == 3
    assert bwdx(ws=NULL) == 4


def test_binding_rejects_host_tensors_and_bad_shapes():
    """Host tensors never reach the C ABI (its kernels take device pointers), and shape errors of the
    bias / FP8 arguments are caught in Python."""
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    o = torch.zeros_like(q)
    lse = torch.zeros(1, 2, 16)
    for call in (lambda: fa.fa_fwd(q, q, q, o, lse, causal=False),
                 lambda: fa.fa_fwd_ext(q, q, q, o, lse, None, False),
                 lambda: fa.quantize_fp8(q, None, True),
                 lambda: fa.fa_fwd_fp8(q.to(torch.uint8), q.to(torch.uint8), q.to(torch.uint8),
                                       torch.zeros(1, 2), torch.zeros(1, 2), torch.zeros(1, 2), o, lse, False)):
        with pytest.raises(ValueError, match="CUDA"):
            call()
    with pytest.raises(ValueError, match="bias"):
        fa._bias_dims(torch.zeros(1, 3, 16, 16, dtype=torch.bfloat16), 1, 2, 16, 16, q.device)
    with pytest.raises(ValueError, match="bias"):
        fa._bias_dims(torch.zeros(1, 2, 16, 8, dtype=torch.bfloat16), 1, 2, 16, 16, q.device)


def test_binding_argument_counts_match_the_header(L):
    """Each ctypes signature in the binding has as many arguments as the C declaration in include/fa.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(([^)]*)\)\s*;", text)
    assert len(decls) == len(declared_functions())
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        fn = getattr(L, name)
        assert fn.argtypes is not None, f"{name}: no argtypes in the binding"
        assert len(fn.argtypes) == n, f"{name}: binding has {len(fn.argtypes)} arguments, header {n}"


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "io_aware_exact_32_b200")
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".inc")):
                src = open(os.path.join(root, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, flags=re.M), f
                assert "oracle/" not in src, f


class _FakeTensor:
    """Shape, device and pointer of a tensor, without memory (never dereferenced: the library is faked)."""

    def __init__(self, shape, device):
        self.shape = tuple(shape)
        self.device = device

    def data_ptr(self):
        return 0x10000

    def numel(self):
        return math.prod(self.shape)


def test_binding_makes_the_tensors_device_current(monkeypatch):
    """Each C-ABI call runs with the tensors' device current (the library resolves the SM count, its
    shared-memory opt-in, its scratch and the default stream from the current device)."""
    torch = pytest.importorskip("torch")
    current = ["cuda:0"]
    calls = []

    class Guard:
        def __init__(self, dev):
            self.dev = dev

        def __enter__(self):
            self.prev = current[0]
            current[0] = str(self.dev)

        def __exit__(self, *exc):
            current[0] = self.prev

    class FakeLib:
        def __getattr__(self, name):
            def call(*args):
                calls.append((name, current[0]))
                return 0
            return call

    monkeypatch.setattr(fa, "_on_device", Guard)
    monkeypatch.setattr(fa, "lib", lambda: FakeLib())
    monkeypatch.setattr(fa, "_need", lambda *a, **k: None)
    monkeypatch.setattr(fa, "_stream_ptr", lambda s, d=None: ctypes.c_void_p(0))
    dev = torch.device("cuda", 1)
    t = _FakeTensor((1, 2, 128, 64), dev)
    lse = _FakeTensor((1, 2, 128), dev)
    fa.fa_fwd(t, t, t, t, lse, causal=True)
    fa.fa_bwd(t, t, t, t, t, lse, t, t, t, _FakeTensor((1 << 20,), dev), causal=True)
    fa.fa_fwd_ext(t, t, t, t, lse, None, True)
    one = _FakeTensor((1, 2, 1, 64), dev)
    fa.fa_decode_splitkv(one, t, t, _FakeTensor((1,), dev), one, None, _FakeTensor((1 << 20,), dev))
    assert [n for n, _ in calls] == ["fa_fwd", "fa_bwd", "fa_fwd_ext", "fa_decode_splitkv"]
    assert all(d == "cuda:1" for _, d in calls), calls
    assert current[0] == "cuda:0"


def test_binding_refuses_a_stream_of_another_device():
    torch = pytest.importorskip("torch")

    class Stream:
        device = torch.device("cuda", 1)
        cuda_stream = 0

    with pytest.raises(ValueError, match="stream"):
        fa._stream_ptr(Stream(), torch.device("cuda", 0))
    assert fa._stream_ptr(Stream(), torch.device("cuda", 1)).value in (None, 0)


def test_bwd_without_query_rows_needs_only_dk_dv(L):
    """Nq == 0, Nk > 0: the only outputs are dK = dV = 0, so q, o, dO, lse, dq and the workspace may be
    NULL.  Validation accepts the call; with no GPU in this process the zeroing memset itself fails
    (FA_ERR_CUDA).  Skipped where a GPU exists: the fake pointers would reach a device memset there
    (the GPU half is tests/test_parity_bwd.py::test_no_query_rows_gives_zero_dk_dv)."""
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("fake pointers must not reach a device")
    st = L.fa_bwd(NULL, A16, A16, NULL, NULL, NULL, NULL, A16, A16, NULL, 0, 1, 2, 0, 128, 64, 0.125, 1, NULL)
    assert st == 5, fa.fa_status_string(st)
    assert L.fa_bwd(NULL, NULL, A16, NULL, NULL, NULL, NULL, A16, A16, NULL, 0, 1, 2, 0, 128, 64, 0.125, 1,
                    NULL) == 1   # k is still needed


def test_wait_limit_hook_without_a_device(L):
    """The test hook copies to device constant memory; with no GPU that copy fails cleanly."""
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("changes the device's wait limit; covered by tests/test_bounded_wait.py")
    assert L.fa_debug_set_wait_limit(0) == 5
