"""CPU checks of the C ABI: the library loads, exports every symbol include/eot.h declares,
and rejects bad arguments on the host before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_ge", os.path.join(ROOT, "__graft_entry__.py"))
    ge = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(ge)
    ge._build_lib()
    from entropic_ot_attention_b200 import _abi
    return _abi


def _declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"^\s*(?:[\w\*]+\s+)+\**(eot_\w+)\s*\(", src, re.M))
    return sorted(names)


def test_every_declared_symbol_is_exported(abi):
    names = _declared_symbols()
    assert "eot_sinkhorn_fwd" in names and "eot_sinkhorn_bwd" in names
    for n in names:
        assert hasattr(abi.lib, n), n
    assert set(abi.EXPORTED) <= set(names)


def test_struct_layout_matches_header(abi):
    # 14 four-byte fields, no padding
    assert ctypes.sizeof(abi.eot_problem) == 14 * 4
    assert abi.eot_abi_version() == 1


def _prob(abi, **kw):
    p = abi.eot_problem()
    base = dict(B=1, H=2, L=256, d=64, W=32, T=3, R=2, dtype=abi.EOT_BF16, scale=0.0, dustbin=0,
                dustbin_index=-1, dustbin_mass=0.0, dustbin_self=1, impl=abi.EOT_IMPL_AUTO)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(L=200), 1),                   # not a multiple of 128
    (dict(d=0), 1),
    (dict(d=136), 1),
    (dict(d=12), 1),
    (dict(W=-2), 1),
    (dict(T=-1), 1),
    (dict(R=9), 1),
    (dict(R=-1), 1),
    (dict(dtype=7), 1),
    (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1),
    (dict(dustbin=1, dustbin_index=256, dustbin_mass=0.1), 1),
    (dict(dustbin=1, dustbin_index=100, dustbin_mass=1.0), 1),
    (dict(dustbin=1, dustbin_index=100, dustbin_mass=-0.1), 1),
    (dict(dustbin=2), 1),
    (dict(impl=5), 1),
    (dict(dtype=0, impl=2), 2),         # tensor-core kernels are bf16 only
    (dict(d=32, impl=2), 2),            # tensor-core kernels need d in {64, 128}
    (dict(B=300, H=300), 2),            # too many units for the grid
    (dict(B=0), 0),                     # empty problem is valid
])
def test_validation(abi, kw, status):
    assert abi.eot_validate(_prob(abi, **kw)) == status


def test_workspace_query(abi):
    p = _prob(abi)
    fw = abi.eot_workspace_bytes(p, False)
    bw = abi.eot_workspace_bytes(p, True)
    assert fw > 0 and bw > fw
    assert abi.eot_workspace_bytes(_prob(abi, L=200), False) == 0
    assert abi.eot_workspace_bytes(_prob(abi, B=0), True) == 0
    # more tail steps keep more staircase and modifier vectors (R = 3 and 4 both leave the
    # modifiers unfolded: 2 R > 5)
    p3, p4 = _prob(abi, R=3), _prob(abi, R=4)
    assert abi.eot_workspace_bytes(p4, True) > abi.eot_workspace_bytes(p3, True)


def test_host_errors_launch_nothing(abi):
    p = _prob(abi)
    lib = abi.lib
    # null tensors: rejected before any CUDA call
    st = lib.eot_sinkhorn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, None, 0, None)
    assert st == abi.EOT_ERR_INVALID_ARGUMENT
    # too-small workspace (fake non-null, 256-aligned addresses; nothing is dereferenced)
    fake = 1 << 20
    st = lib.eot_sinkhorn_fwd(ctypes.byref(p), fake, fake, fake, None, fake, fake, fake, fake, 16, None)
    assert st == abi.EOT_ERR_WORKSPACE_TOO_SMALL
    st = lib.eot_sinkhorn_fwd(ctypes.byref(p), fake, fake, fake, None, fake, fake, fake, fake + 8, 1 << 30, None)
    assert st == abi.EOT_ERR_INVALID_ARGUMENT     # misaligned workspace
    st = lib.eot_sinkhorn_bwd(ctypes.byref(p), fake, fake, fake, None, fake, fake, None, fake, fake, fake,
                              fake, 1 << 30, None)
    assert st == abi.EOT_ERR_INVALID_ARGUMENT     # null dO
    bad = _prob(abi, L=100)
    st = lib.eot_sinkhorn_bwd(ctypes.byref(bad), fake, fake, fake, None, fake, fake, fake, fake, fake, fake,
                              fake, 1 << 30, None)
    assert st == abi.EOT_ERR_INVALID_ARGUMENT
    assert lib.eot_sinkhorn_fwd(None, None, None, None, None, None, None, None, None, 0, None) == 1


def test_half_step_host_errors_launch_nothing(abi):
    lib, fake = abi.lib, 1 << 20
    p = _prob(abi)
    ws_bytes = abi.eot_workspace_bytes(p, False)
    assert lib.eot_band_half_step(ctypes.byref(p), None, fake, fake, fake, fake, fake, ws_bytes, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT                                  # null X
    assert lib.eot_band_half_step(ctypes.byref(p), fake, fake, fake, fake, fake, fake, ws_bytes - 1, None) \
        == abi.EOT_ERR_WORKSPACE_TOO_SMALL
    assert lib.eot_band_half_step(ctypes.byref(p), fake, fake, fake, fake, fake, fake + 8, ws_bytes, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT                                  # misaligned workspace
    db = _prob(abi, dustbin=1, dustbin_index=5, dustbin_mass=0.1)
    assert lib.eot_band_half_step(ctypes.byref(db), fake, fake, fake, fake, fake, fake, 1 << 30, None) \
        == abi.EOT_ERR_UNSUPPORTED                                       # the dustbin needs every position
    bad = _prob(abi, L=100)
    assert lib.eot_band_half_step(ctypes.byref(bad), fake, fake, fake, fake, fake, fake, 1 << 30, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT
    empty = _prob(abi, H=0)
    assert lib.eot_band_half_step(ctypes.byref(empty), None, None, None, None, None, None, 0, None) == abi.EOT_OK
    # the output of given potentials: no dustbin, no null pointer
    o = lib.eot_band_output
    assert o(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake, fake, ws_bytes, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT
    assert o(ctypes.byref(db), fake, fake, fake, fake, fake, fake, fake, fake, 1 << 30, None) == abi.EOT_ERR_UNSUPPORTED
    assert o(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, 16, None) \
        == abi.EOT_ERR_WORKSPACE_TOO_SMALL
    # the dustbin form: a dustbin problem and an own range inside [0, D] are required
    f = lib.eot_band_half_step_dustbin
    assert f(ctypes.byref(p), fake, fake, fake, fake, fake, 0, 128, fake, fake, 1 << 30, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT                                  # no dustbin
    for lo, hi in ((-1, 5), (3, 2), (0, 6)):
        assert f(ctypes.byref(db), fake, fake, fake, fake, fake, lo, hi, fake, fake, 1 << 30, None) \
            == abi.EOT_ERR_INVALID_ARGUMENT
    assert f(ctypes.byref(db), fake, fake, fake, fake, fake, 0, 5, None, fake, 1 << 30, None) \
        == abi.EOT_ERR_INVALID_ARGUMENT                                  # null partial
    assert f(ctypes.byref(db), fake, fake, fake, fake, fake, 0, 5, fake, fake, 16, None) \
        == abi.EOT_ERR_WORKSPACE_TOO_SMALL


def test_empty_problem_is_a_noop(abi):
    p = _prob(abi, B=0)
    assert abi.lib.eot_sinkhorn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, None, 0, None) == 0


def test_status_strings(abi):
    for s in range(7):
        assert abi.eot_status_string(s)
    assert "unknown" in abi.eot_status_string(99)


def test_static_scratch_size_matches_header(abi):
    """The size the library was built with equals the header's EOT_STATIC_SCRATCH_BYTES."""
    src = open(os.path.join(ROOT, "include", "eot.h")).read()
    m = re.search(r"#define\s+EOT_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", src)
    assert m, "EOT_STATIC_SCRATCH_BYTES not found in the header"
    want = int(m.group(1)) * int(m.group(2)) * int(m.group(3))
    assert abi.lib.eot_static_scratch_bytes() == want == abi.EOT_STATIC_SCRATCH_BYTES


def test_nvtx_build_flag_compiles(tmp_path):
    """The NVTX ranges around the passes (EOT_NVTX=1 builds) compile for sm_100a."""
    import subprocess
    src = os.path.join(ROOT, "entropic_ot_attention_b200", "csrc", "api.cu")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    res = subprocess.run([nvcc, "-DEOT_NVTX", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                          "-I", os.path.join(ROOT, "include"), "-c", src, "-o", str(tmp_path / "api_nvtx.o")],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
