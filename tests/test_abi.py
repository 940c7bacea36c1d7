"""The C-ABI library: it loads, exports every symbol include/gptq.h declares, and
rejects bad arguments on the host before launching anything.  No compute calls."""
import ctypes
import os
import re

import pytest
import torch

from post_weight_quantization_20_b200 import gptq as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")

no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                            reason="passes fake device pointers; only run without a GPU")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = G.load_library()
    names = declared_functions()
    assert len(names) == 13, names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(G.EXPORTS) == names


def test_last_error_starts_empty():
    assert G.gptq_last_error() == ""


def test_status_strings():
    assert G.gptq_status_string(0) == "GPTQ_OK"
    assert G.gptq_status_string(G.GPTQ_ERR_NOT_PD) == "GPTQ_ERR_NOT_PD"
    assert G.status_names(G.GPTQ_ERR_NOT_PD | G.GPTQ_ERR_NONFINITE) == "GPTQ_ERR_NOT_PD|GPTQ_ERR_NONFINITE"


def test_workspace_sizes():
    cfg = G.make_config(4, 128)
    a = G.gptq_workspace_size(G.GPTQ_OP_PREPARE, 0, 768, cfg)
    b = G.gptq_workspace_size(G.GPTQ_OP_PREPARE, 0, 3072, cfg)
    assert a > 2 * 768 * 768 * 4 and b > a and a % 256 == 0
    q = G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, 3072, 768, cfg)
    assert q >= 3072 * 768 * 5
    assert G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, 10, 0, cfg) == 0
    assert G.gptq_workspace_size(99, 10, 10, cfg) == 0
    bad = G.make_config(5, 128)
    assert G.gptq_workspace_size(G.GPTQ_OP_PREPARE, 0, 10, bad) == 0


def _raw(name, *args):
    return getattr(G.load_library(), name)(*args)


def test_pack_rejects_bad_bits_and_nulls():
    assert _raw("gptq_pack", None, 4, 4, 5, None, None) == G.GPTQ_ERR_INVALID_ARG
    assert _raw("gptq_pack", None, 4, 4, 4, None, None) == G.GPTQ_ERR_INVALID_ARG
    assert _raw("gptq_pack", None, -1, 4, 4, None, None) == G.GPTQ_ERR_INVALID_ARG
    # empty input is a valid no-op
    assert _raw("gptq_pack", None, 0, 7, 4, None, None) == G.GPTQ_OK


def test_hessian_rejects_bad_arguments():
    n = ctypes.c_int64(0)
    f = G.load_library().gptq_hessian_accumulate
    assert f(None, ctypes.byref(n), None, 1, 10, 8, 8, None, None) == G.GPTQ_ERR_INVALID_ARG
    neg = ctypes.c_int64(-3)
    assert f(ctypes.c_void_p(256), ctypes.byref(neg), None, 1, 10, 8, 8, None, None) == G.GPTQ_ERR_INVALID_ARG
    # m == 0 is a no-op that touches nothing
    assert f(ctypes.c_void_p(256), ctypes.byref(n), None, 1, 0, 8, 8, None, None) == G.GPTQ_OK
    assert n.value == 0


@no_gpu
def test_hessian_rejects_bad_dtype_and_stride():
    n = ctypes.c_int64(0)
    f = G.load_library().gptq_hessian_accumulate
    fake = ctypes.c_void_p(4096)
    assert f(fake, ctypes.byref(n), fake, 7, 10, 8, 8, None, None) == G.GPTQ_ERR_INVALID_ARG
    assert f(fake, ctypes.byref(n), fake, 1, 10, 8, 4, None, None) == G.GPTQ_ERR_INVALID_ARG


@no_gpu
def test_prepare_and_quantize_validation():
    lib = G.load_library()
    fake = ctypes.c_void_p(4096)
    cfg = G.make_config(4, 128)
    ws_need = G.gptq_workspace_size(G.GPTQ_OP_PREPARE, 0, 64, cfg)
    assert lib.gptq_prepare(fake, 64, ctypes.byref(cfg), fake, fake, fake, ws_need - 1, None,
                            None) == G.GPTQ_ERR_WORKSPACE
    assert lib.gptq_prepare(fake, 64, ctypes.byref(cfg), fake, fake, ctypes.c_void_p(4100),
                            ws_need, None, None) == G.GPTQ_ERR_INVALID_ARG  # unaligned ws
    assert lib.gptq_prepare(fake, 64, None, fake, fake, fake, ws_need, None,
                            None) == G.GPTQ_ERR_INVALID_ARG
    q = G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, 8, 64, cfg)
    for g, B, want in [(96, 128, G.GPTQ_ERR_UNSUPPORTED), (256, 128, G.GPTQ_ERR_UNSUPPORTED),
                       (64, 48, G.GPTQ_ERR_UNSUPPORTED)]:
        c = G.make_config(4, g, block_size=B)
        assert lib.gptq_quantize_layer(fake, 1, 8, 64, 64, fake, fake, ctypes.byref(c), fake, fake,
                                       fake, fake, fake, fake, q, None, None) == want
    c = G.make_config(4, 64)
    assert lib.gptq_quantize_layer(fake, 1, 8, 64, 32, fake, fake, ctypes.byref(c), fake, fake,
                                   fake, fake, fake, fake, q, None, None) == G.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_quantize_layer(fake, 1, 8, 64, 64, fake, fake, ctypes.byref(c), fake, fake,
                                   fake, fake, fake, fake, q - 1, None, None) == G.GPTQ_ERR_WORKSPACE
    bad = G.make_config(4, 64, damp=float("nan"))
    assert lib.gptq_quantize_layer(fake, 1, 8, 64, 64, fake, fake, ctypes.byref(bad), fake, fake,
                                   fake, fake, fake, fake, q, None, None) == G.GPTQ_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    H = torch.zeros(4, 4)
    X = torch.zeros(8, 4)
    with pytest.raises(ValueError):
        G.gptq_hessian_accumulate(H, 0, X)


def test_selftest_rejects_bad_arguments_before_launching():
    lib = G.load_library()
    # a NULL status word, or an unknown self-test, is refused on the host
    assert lib.gptq_selftest_timeout(G.GPTQ_SELFTEST_MBARRIER, None, None) == G.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_selftest_timeout(7, ctypes.c_void_p(4096), None) == G.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_selftest_timeout(-1, ctypes.c_void_p(4096), None) == G.GPTQ_ERR_INVALID_ARG


def test_binding_helpers_refuse_host_tensors_and_mixed_groups():
    cfg = G.make_config(4, 128)
    with pytest.raises(ValueError):
        G.gptq_selftest_timeout(G.GPTQ_SELFTEST_MBARRIER, torch.zeros(1, dtype=torch.int32))
    assert G.quantize_layers_shared([], torch.zeros(4, 4), cfg) == []
    with pytest.raises(ValueError):
        G.quantize_layers_shared([torch.zeros(2, 4), torch.zeros(2, 5)], torch.zeros(8, 4), cfg)


def test_binding_checks_buffer_shapes_before_calling_the_library():
    # the C ABI cannot see buffer sizes, so the binding refuses a buffer that does not
    # hold what the call reads or writes (checked before the device check, on CPU)
    cfg = G.make_config(4, 64)
    R, C = 8, 128
    W = torch.zeros(R, C, dtype=torch.float16)
    U = torch.zeros(C, C)
    perm = torch.zeros(C, dtype=torch.int32)
    ok = dict(codes=torch.zeros(R, C, dtype=torch.uint8), scales=torch.zeros(R, 2),
              zeros=torch.zeros(R, 2), g_idx=torch.zeros(C, dtype=torch.int32),
              losses=torch.zeros(C), ws=torch.zeros(16, dtype=torch.uint8))

    def quantize(**over):
        a = dict(ok, **over)
        G.gptq_quantize_layer(W, U, perm, cfg, a["codes"], a["scales"], a["zeros"], a["g_idx"],
                              a["losses"], a["ws"])

    for name, bad in (("codes", torch.zeros(R, C - 1, dtype=torch.uint8)),
                      ("codes", torch.zeros(R, C, dtype=torch.int32)),
                      ("scales", torch.zeros(R, 1)),          # g = 64 gives 2 groups
                      ("zeros", torch.zeros(R, 2, dtype=torch.float64)),
                      ("g_idx", torch.zeros(C - 1, dtype=torch.int32)),
                      ("losses", torch.zeros(C + 1)),
                      ("codes", torch.zeros(C, R, dtype=torch.uint8).t()),   # not contiguous
                      ("ws", torch.zeros(4, dtype=torch.float32))):
        with pytest.raises(ValueError, match=name):
            quantize(**{name: bad})
    with pytest.raises(ValueError, match="device tensors"):
        quantize()                          # shapes fine: refused as host tensors
    with pytest.raises(ValueError, match="U"):
        G.gptq_quantize_layer(W, torch.zeros(C, C - 1), perm, cfg, *ok.values())
    with pytest.raises(ValueError, match="perm"):
        G.gptq_prepare(U, cfg, torch.zeros(C, C), torch.zeros(C, dtype=torch.int64), ok["ws"])
    with pytest.raises(ValueError, match="H"):
        G.gptq_hessian_accumulate(torch.zeros(C, C + 1), 0, torch.zeros(4, C))
    with pytest.raises(ValueError, match="packed"):
        G.gptq_pack(ok["codes"], 3, torch.zeros(R, C * 3 // 32 - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="status"):
        G.gptq_selftest_timeout(G.GPTQ_SELFTEST_MBARRIER, torch.zeros(1, dtype=torch.int64))
    # rows = 0: nothing is written through codes, scales or zeros, so empty ones pass
    # the shape check (and fail only the device check here)
    with pytest.raises(ValueError, match="device tensors"):
        G.gptq_quantize_layer(torch.zeros(0, C, dtype=torch.float16), U, perm, cfg,
                              torch.zeros(0, dtype=torch.uint8), torch.zeros(0), torch.zeros(0),
                              ok["g_idx"], ok["losses"], ok["ws"])


def test_header_compiles_as_c99_and_the_library_links(tmp_path):
    # a plain C caller: no C++ in the header, the library links without torch, and the
    # calls that need no device answer before anything is launched
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    G.load_library()                                  # builds nothing; the .so must exist
    libdir = os.path.dirname(G.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    src = os.path.join(ROOT, "tests", "c_abi_check.c")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), src, "-o", str(exe),
                        "-L", libdir, "-lgptq", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr


class _FakeLib:
    """Stands in for libgptq: records the calls, returns GPTQ_OK, computes nothing."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("gptq_"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append(name)
            if name == "gptq_workspace_size":
                return 4096
            if name == "gptq_hessian_accumulate":
                n = args[1]._obj
                n.value += int(args[4])
            return 0
        return call


@pytest.mark.parametrize("rows,cols,group,act", [(8, 128, 128, False), (5, 96, 32, True),
                                                  (3, 40, 0, False), (0, 64, 64, False)])
def test_layer_helpers_pass_the_buffer_checks(monkeypatch, rows, cols, group, act):
    # the one-layer helpers allocate every buffer themselves; with the device and the
    # library faked out on CPU, every buffer they pass must satisfy the wrappers' checks
    fake = _FakeLib()
    monkeypatch.setattr(G, "load_library", lambda *a: fake)
    monkeypatch.setattr(G, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(G, "_stream", lambda s: None)
    cfg = G.make_config(4, group, act_order=act)
    W = torch.zeros(rows, cols, dtype=torch.float16)
    X = torch.zeros(50, cols, dtype=torch.float16)
    r = G.quantize_layer(W, X, cfg, chunk_tokens=20)
    assert r.n_tokens == 50 and r.packed.shape == (rows, G.packed_words(cols, 4))
    assert fake.calls.count("gptq_hessian_accumulate") == 3
    assert fake.calls[-2:] == ["gptq_quantize_layer", "gptq_pack"]
    shared = G.quantize_layers_shared([W, torch.zeros(rows + 2, cols, dtype=torch.bfloat16)], X, cfg)
    assert [x.codes.shape for x in shared] == [(rows, cols), (rows + 2, cols)]
    rtn = G.quantize_rtn(W, cfg)
    assert rtn.scales.shape == (rows, G.n_groups(cols, group))


class _PivotFakeLib(_FakeLib):
    """gptq_prepare reports a non-positive pivot while damp < `needs`; the Hessian can
    report non-finite data instead."""

    def __init__(self, needs, nonfinite=False):
        super().__init__()
        self.needs, self.nonfinite, self.damps = needs, nonfinite, []

    def __getattr__(self, name):
        base = super().__getattr__(name)
        if name not in ("gptq_prepare", "gptq_hessian_accumulate"):
            return base

        def call(*args):
            r = base(*args)
            if name == "gptq_prepare":
                damp = args[2]._obj.damp
                self.damps.append(round(damp, 6))
                if damp < self.needs:
                    ctypes.c_int32.from_address(args[7].value).value |= G.GPTQ_ERR_NOT_PD
            elif self.nonfinite:
                ctypes.c_int32.from_address(args[7].value).value |= G.GPTQ_ERR_NONFINITE
            return r
        return call


def _run_retry(monkeypatch, fake, **kw):
    monkeypatch.setattr(G, "load_library", lambda *a: fake)
    monkeypatch.setattr(G, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(G, "_stream", lambda s: None)
    W = torch.zeros(4, 64, dtype=torch.float16)
    X = torch.zeros(10, 64, dtype=torch.float16)
    return G.quantize_layer(W, X, G.make_config(4, 64, damp=0.01), **kw)


def test_damping_retry_refactors_until_the_pivots_are_positive(monkeypatch):
    # a near-singular Hessian is stabilised by a larger damp_percent (e.g. 0.1)
    fake = _PivotFakeLib(needs=0.1)
    r = _run_retry(monkeypatch, fake, damp_retry=(0.05, 0.1, 0.5))
    assert fake.damps == [0.01, 0.05, 0.1] and r.damp == pytest.approx(0.1)
    fake = _PivotFakeLib(needs=0.0)                       # no retry needed
    r = _run_retry(monkeypatch, fake, damp_retry=(0.1,))
    assert fake.damps == [0.01] and r.damp == pytest.approx(0.01)


def test_damping_retry_gives_up_and_leaves_other_conditions_alone(monkeypatch):
    fake = _PivotFakeLib(needs=1.0)                       # every value too small
    with pytest.raises(G.GPTQError) as e:
        _run_retry(monkeypatch, fake, damp_retry=(0.1,))
    assert e.value.code == G.GPTQ_ERR_NOT_PD and fake.damps == [0.01, 0.1]
    fake = _PivotFakeLib(needs=0.1)                       # no retry values: no retry
    with pytest.raises(G.GPTQError):
        _run_retry(monkeypatch, fake)
    assert fake.damps == [0.01]
    fake = _PivotFakeLib(needs=0.1, nonfinite=True)       # non-finite data is not retried
    with pytest.raises(G.GPTQError) as e:
        _run_retry(monkeypatch, fake, damp_retry=(0.1,))
    assert e.value.code & G.GPTQ_ERR_NONFINITE and fake.damps == [0.01]


def test_guarded_buffers_detect_writes_past_either_end():
    # the helper the GPU canary test uses, checked on CPU
    from tests.guards import MARGIN, Guarded
    g = Guarded((3, 5), torch.float32, "cpu")
    assert g.t.is_contiguous() and g.t.data_ptr() % 256 == g.raw.data_ptr() % 256
    g.t.fill_(1.0)                                     # writes inside the view only
    assert g.intact()
    g.raw[MARGIN + g.nbytes] = 0                       # one byte past the end
    assert not g.intact()
    h = Guarded((7,), torch.uint8, "cpu", fill=torch.arange(7, dtype=torch.uint8))
    assert h.t.tolist() == list(range(7)) and h.intact()
    h.raw[MARGIN - 1] = 1                              # one byte before the start
    assert not h.intact()
