"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/ssd.h declares, and rejects bad arguments with a
status and a message before it touches the device."""
import ctypes
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_12_b200 import build

    build.build()
    from selective_state_space_12_b200 import _lib

    return _lib.load()


def _header_functions(name):
    text = open(os.path.join(ROOT, "include", name), encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_entry_point(lib):
    declared = _header_functions("ssd.h")
    assert "ssd_forward" in declared and "ssd_step" in declared
    for name in declared:
        assert hasattr(lib, name), name
    nm = subprocess.run(["nm", "-D", "--defined-only",
                         os.path.join(ROOT, "selective_state_space_12_b200", "libssd.so")],
                        capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssd_\w+)", nm))
    assert set(declared) <= exported


def test_binding_covers_the_header(lib):
    from selective_state_space_12_b200 import _lib

    assert set(_header_functions("ssd.h")) == set(_lib.exported_symbols())


def test_abi_version(lib):
    assert lib.ssd_abi_version() == 2


def _dims(**kw):
    from selective_state_space_12_b200 import _lib

    d = dict(batch=2, seqlen=64, nheads=4, headdim=64, dstate=128, ngroups=2, dtype=1, reserved=0)
    d.update(kw)
    return _lib.Dims(**d)


def _fwd(lib, dims, chunk=64, x=0x1000, dt=0x2000, A=0x3000, B=0x4000, C=0x5000, D=None,
         h0=None, y=0x6000, hf=None, ws=0x100000, ws_bytes=1 << 40):
    d = ctypes.byref(dims) if dims is not None else None
    return lib.ssd_forward(x, dt, A, B, C, D, h0, chunk, y, hf, d, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(headdim=72), 2), (dict(headdim=144), 2), (dict(dstate=24), 2), (dict(dstate=512), 2),
    (dict(nheads=5, ngroups=2), 1), (dict(batch=0), 1), (dict(seqlen=-1), 1), (dict(dtype=7), 1),
    (dict(reserved=1), 1), (dict(ngroups=0), 1),
])
def test_forward_rejects_bad_sizes(lib, kw, status):
    assert _fwd(lib, _dims(**kw)) == status
    assert lib.ssd_last_error()


def test_forward_rejects_null_dims_and_bad_chunk(lib):
    assert _fwd(lib, None) == 1
    for chunk in (0, 8, 48, 512):
        assert _fwd(lib, _dims(), chunk=chunk) == 2
        assert b"chunk" in lib.ssd_last_error()


def test_forward_rejects_null_and_misaligned_pointers(lib):
    assert _fwd(lib, _dims(), x=None) == 1
    assert _fwd(lib, _dims(), A=None) == 1
    assert _fwd(lib, _dims(), x=0x1008) == 1
    assert b"x is not 16-byte aligned" in lib.ssd_last_error()
    assert _fwd(lib, _dims(), h0=0x7004) == 1
    assert _fwd(lib, _dims(), y=0x1000) == 1  # y aliases x
    # fp32 I/O always takes the CUDA-core path, which needs a workspace, so
    # these two are rejected on every device
    assert _fwd(lib, _dims(dtype=0), ws_bytes=16) == 1
    assert b"workspace" in lib.ssd_last_error()
    assert _fwd(lib, _dims(dtype=0), ws=0x100010) == 1


def _bwd(lib, **kw):
    a = dict(x=0x1000, dt=0x2000, A=0x3000, B=0x4000, C=0x5000, D=None, h0=None, dy=0x6000,
             dhf=None, dx=0x7000, ddt=0x8000, dA=0x9000, dB=0xa000, dC=0xb000, dD=0xc000,
             dh0=None)
    a.update(kw)
    return lib.ssd_backward(*a.values(), ctypes.byref(_dims()), 0x100000, 1 << 40, None)


@pytest.mark.parametrize("name", ["x", "B", "C", "dy", "dx", "dB", "dC"])
def test_backward_rejects_tensors_not_16_byte_aligned(lib, name):
    # the tensor-core kernels read these as tiles and write dx, dB, dC in
    # 16-byte vectors: a pointer aligned only to its element is refused
    # before anything is launched
    assert _bwd(lib, **{name: 0x20004}) == 1
    assert f"{name} is not 16-byte aligned".encode() in lib.ssd_last_error()
    assert _bwd(lib, ddt=0x8001) == 1


def test_workspace_size_is_zero_for_bad_sizes(lib):
    assert lib.ssd_forward_workspace_size(ctypes.byref(_dims(headdim=72)), 64) == 0
    assert lib.ssd_forward_workspace_size(ctypes.byref(_dims()), 48) == 0
    assert lib.ssd_forward_workspace_size(ctypes.byref(_dims()), 64) > 0


def test_step_rejects_bad_arguments(lib):
    d = ctypes.byref(_dims())
    ok = dict(h=0x1000, x=0x2000, dt=0x3000, A=0x4000, B=0x5000, C=0x6000, D=None, y=0x7000)

    def step(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.ssd_step(a["h"], a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["y"],
                            d, None)

    assert step(h=None) == 1
    assert step(h=0x1004) == 1
    assert step(B=0x5008) == 1
    assert step(y=0x1000) == 1
    assert lib.ssd_step(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None, 0x7000,
                        ctypes.byref(_dims(dstate=20)), None) == 2


def _opts(**kw):
    from selective_state_space_12_b200 import _lib

    o = _lib.Options()
    for k, v in kw.items():
        if k == "reserved":
            o.reserved[0] = v
        else:
            setattr(o, k, v)
    return o


@pytest.mark.parametrize("kw", [dict(discretization=2), dict(discretization=-1),
                                dict(reserved=1), dict(dt_bias=0x3002),
                                dict(dt_min=-0.1, dt_max=1.0), dict(dt_min=2.0, dt_max=1.0),
                                dict(dt_max=float("nan"))])
def test_options_are_validated_before_any_launch(lib, kw):
    o = ctypes.byref(_opts(**kw))
    assert lib.ssd_forward_ex(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, None, None, 64, 0x6000,
                              None, ctypes.byref(_dims()), o, 0x100000, 1 << 40, None) == 1
    assert b"options" in lib.ssd_last_error()
    assert lib.ssd_step_ex(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None, 0x7000,
                           ctypes.byref(_dims()), o, None) == 1


def test_ex_entry_points_validate_sizes_like_the_plain_ones(lib):
    o = ctypes.byref(_opts(dt_softplus=1, discretization=1))
    assert lib.ssd_forward_ex(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, None, None, 64, 0x6000,
                              None, ctypes.byref(_dims(headdim=72)), o, 0x100000, 1 << 40,
                              None) == 2
    assert lib.ssd_step_ex(None, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None, 0x7000,
                           ctypes.byref(_dims()), o, None) == 1


def test_state_and_chain_validate_arguments(lib):
    d = ctypes.byref(_dims())
    ok = dict(x=0x1000, dt=0x2000, A=0x3000, B=0x4000, so=0x5000, do=0x6000)

    def state(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.ssd_forward_state(a["x"], a["dt"], a["A"], a["B"], 64, a["so"], a["do"], d,
                                     None, 0x100000, 1 << 40, None)

    assert state(so=None) == 1
    assert state(so=0x5008) == 1
    assert state(A=None) == 1
    assert lib.ssd_forward_state(0x1000, 0x2000, 0x3000, 0x4000, 48, 0x5000, 0x6000, d, None,
                                 0x100000, 1 << 40, None) == 2
    assert lib.ssd_forward_state_workspace_size(ctypes.byref(_dims(headdim=72)), 64) == 0
    chain = lib.ssd_state_chain
    assert chain(0x1000, 0x2000, 2, 2, None, 0x3000, None, d, None) == 1  # part out of range
    assert chain(0x1000, 0x2000, 0, 0, None, 0x3000, None, d, None) == 1  # no pieces
    assert chain(0x1000, 0x2000, 2, 1, None, None, None, d, None) == 1    # no output
    assert chain(0x1008, 0x2000, 2, 1, None, 0x3000, None, d, None) == 1  # misaligned


def test_selective_scan_validates_arguments(lib):
    def scan(dims, B=0x4000, opts=None):
        return lib.ssd_selective_scan(0x1000, 0x2000, 0x3000, B, 0x5000, None, None, 0x6000,
                                      None, ctypes.byref(dims), opts, None)

    ok = dict(headdim=1, dstate=16, nheads=64, ngroups=1)
    assert scan(_dims(**dict(ok, headdim=64))) == 1       # one channel per head
    assert scan(_dims(**dict(ok, dstate=12))) == 2        # dstate 4, 8, 16
    assert scan(_dims(**dict(ok, dstate=32))) == 2
    assert scan(_dims(**dict(ok, nheads=63, ngroups=2))) == 1
    assert scan(_dims(**ok), B=0x4002) == 1               # B rows read 4 at a time
    assert scan(_dims(**ok), opts=ctypes.byref(_opts(discretization=3))) == 1
    assert lib.ssd_selective_scan(0x1000, 0x2000, None, 0x4000, 0x5000, None, None, 0x6000,
                                  None, ctypes.byref(_dims(**ok)), None, None) == 1


def test_package_import_does_not_need_the_library():
    # the binding loads libssd lazily; importing never falls back to anything
    import selective_state_space_12_b200 as pkg

    assert callable(pkg.ssd_forward) and callable(pkg.ssd_step)


def test_header_is_plain_c_and_links(tmp_path):
    """include/ssd.h compiles as strict C99 and a C program links against
    libssd and calls it (no CUDA types cross the boundary)."""
    import shutil
    import subprocess

    from tests.conftest import ROOT

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "ssd.h"\n'
        "int main(void) {\n"
        "    ssd_dims d = {0};\n"
        "    ssd_options o = {0};\n"
        "    d.batch = 1; d.seqlen = 8; d.nheads = 2; d.headdim = 64; d.dstate = 128;\n"
        "    d.ngroups = 1; d.dtype = SSD_BF16;\n"
        "    (void)o;\n"
        "    if (ssd_abi_version() != SSD_ABI_VERSION) return 1;\n"
        "    /* a NULL input is rejected before anything is enqueued */\n"
        "    if (ssd_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 64, NULL, NULL,\n"
        "                    &d, NULL, 0, NULL) != SSD_ERR_INVALID_ARG) return 2;\n"
        "    if (ssd_last_error() == NULL || ssd_last_error()[0] == 0) return 3;\n"
        "    return 0;\n"
        "}\n")
    lib_dir = os.path.join(ROOT, "selective_state_space_12_b200")
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I" + os.path.join(ROOT, "include"), str(src), "-L" + lib_dir, "-lssd",
                        "-Wl,-rpath," + lib_dir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_binding_refuses_host_tensors():
    """No CPU fallback: every entry point of the binding refuses host tensors
    before anything runs."""
    torch = pytest.importorskip("torch")
    import selective_state_space_12_b200 as ssd

    bf = torch.bfloat16
    x = torch.zeros(1, 8, 2, 64, dtype=bf)
    dt = torch.ones(1, 8, 2, dtype=bf)
    A = -torch.ones(2)
    B = torch.zeros(1, 8, 1, 128, dtype=bf)
    calls = [
        lambda: ssd.ssd_forward(x, dt, A, B, B),
        lambda: ssd.ssd_forward_ex(x, dt, A, B, B, dt_softplus=True),
        lambda: ssd.ssd_step(torch.zeros(1, 2, 64, 128), x[:, 0], dt[:, 0], A, B[:, 0], B[:, 0]),
        lambda: ssd.ssd_backward(x, dt, A, B, B, None, None, x),
        lambda: ssd.ssd_selective_scan(torch.zeros(1, 8, 16, dtype=bf),
                                       torch.zeros(1, 8, 16, dtype=bf), -torch.ones(16, 16),
                                       torch.zeros(1, 8, 1, 16, dtype=bf),
                                       torch.zeros(1, 8, 1, 16, dtype=bf)),
    ]
    for call in calls:
        with pytest.raises((ValueError, RuntimeError), match="(?i)cuda"):
            call()


def test_make_options_fills_the_struct():
    pytest.importorskip("torch")
    from selective_state_space_12_b200 import _lib, make_options

    o = make_options(dt_softplus=True, dt_limit=(1e-3, 0.1), zoh=True)
    assert o.dt_softplus == 1 and o.discretization == _lib.SSD_DISC_ZOH
    assert abs(o.dt_min - 1e-3) < 1e-9 and abs(o.dt_max - 0.1) < 1e-7
    assert not o.dt_bias and list(o.reserved) == [0, 0, 0, 0]
    p = make_options()  # the plain layer
    assert (p.dt_softplus, p.discretization, p.dt_min, p.dt_max) == (0, _lib.SSD_DISC_EULER, 0.0, 0.0)
