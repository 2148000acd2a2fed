"""Host-side checks of the C ABI (no GPU needed).

* the shared library loads and exports every function include/retention.h declares;
* invalid arguments are rejected with the documented status before anything is
  launched (these calls never reach the CUDA runtime, so they run on the CPU).
"""
import ctypes
import os
import re
import tempfile

import pytest

from retnet_retention_chunkwise_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retention.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(retention_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    return _abi.load()


def test_header_and_binding_agree():
    assert _declared() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_only_abi_symbols_are_exported():
    # built with -fvisibility=hidden: the dynamic symbol table holds the C ABI
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    ours = sorted({ln.split()[-1] for ln in out.splitlines() if ln.split()[-1].startswith("retention_")})
    assert ours == _declared()


def test_status_strings_and_version(lib):
    names = [lib.retention_status_str(i).decode() for i in range(6)]
    assert names == ["RET_OK", "RET_EINVAL", "RET_EUNSUPPORTED", "RET_ECUDA", "RET_ETIMEOUT", "RET_EBOUNDS"]
    assert lib.retention_status_str(99).decode() == "RET_UNKNOWN"
    assert lib.retention_abi_version() == 104


def _g(*vals):
    return (ctypes.c_float * len(vals))(*vals)


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first

# The validation tests pass made-up device addresses that the library must
# refuse before any launch.  Were a check ever to regress on a machine with a
# GPU, the call would launch kernels on those addresses and fault the device,
# so these tests run only where no CUDA device is visible.
try:
    import torch as _torch
    _DEVICE_VISIBLE = _torch.cuda.is_available()
except Exception:  # pragma: no cover
    _DEVICE_VISIBLE = False
NO_DEVICE = pytest.mark.skipif(_DEVICE_VISIBLE, reason="made-up device addresses: host-only validation test")


@pytest.mark.parametrize("gamma", [-0.01, 1.0001, float("nan"), float("inf")])
@NO_DEVICE
def test_bad_gamma_is_einval(lib, gamma):
    s = _abi.RetShape(1, 1, 8, 64, 128)
    assert lib.retention_parallel(FAKE, FAKE, FAKE, _g(gamma), FAKE, s, _abi.RET_BF16, None) == _abi.RET_EINVAL
    assert lib.retention_chunkwise(FAKE, FAKE, FAKE, _g(gamma), FAKE, None, None, 64, s, _abi.RET_BF16,
                                   None, 0, None) == _abi.RET_EINVAL
    assert lib.retention_recurrent_step(FAKE, FAKE, FAKE, _g(gamma), FAKE, FAKE, s, _abi.RET_BF16,
                                        None) == _abi.RET_EINVAL


@NO_DEVICE
def test_null_gamma_and_pointers_are_einval(lib):
    s = _abi.RetShape(1, 1, 8, 64, 128)
    assert lib.retention_parallel(FAKE, FAKE, FAKE, None, FAKE, s, _abi.RET_BF16, None) == _abi.RET_EINVAL
    assert lib.retention_parallel(None, FAKE, FAKE, _g(0.5), FAKE, s, _abi.RET_BF16, None) == _abi.RET_EINVAL
    assert lib.retention_chunkwise(FAKE, None, FAKE, _g(0.5), FAKE, None, None, 64, s, _abi.RET_BF16,
                                   None, 0, None) == _abi.RET_EINVAL
    assert lib.retention_recurrent_step(FAKE, FAKE, FAKE, _g(0.5), FAKE, None, s, _abi.RET_BF16,
                                        None) == _abi.RET_EINVAL


@pytest.mark.parametrize("shape", [(0, 1, 8, 64, 128), (1, 0, 8, 64, 128), (1, 1, -1, 64, 128),
                                   (1, 1, 8, 0, 128), (1, 1, 8, 64, 0)])
@NO_DEVICE
def test_bad_shapes_are_einval(lib, shape):
    s = _abi.RetShape(*shape)
    g = _g(*([0.5] * max(shape[1], 1)))
    assert lib.retention_chunkwise(FAKE, FAKE, FAKE, g, FAKE, None, None, 64, s, _abi.RET_BF16,
                                   None, 0, None) == _abi.RET_EINVAL


@NO_DEVICE
def test_too_many_heads_is_unsupported(lib):
    H = _abi.RET_MAX_HEADS + 1
    s = _abi.RetShape(1, H, 8, 64, 128)
    assert lib.retention_parallel(FAKE, FAKE, FAKE, _g(*([0.5] * H)), FAKE, s, _abi.RET_BF16,
                                  None) == _abi.RET_EUNSUPPORTED


@NO_DEVICE
def test_misaligned_pointers_are_einval(lib):
    s = _abi.RetShape(1, 1, 8, 64, 128)
    odd = ctypes.c_void_p(0x10008)
    assert lib.retention_parallel(odd, FAKE, FAKE, _g(0.5), FAKE, s, _abi.RET_BF16, None) == _abi.RET_EINVAL
    assert lib.retention_chunkwise(FAKE, FAKE, FAKE, _g(0.5), FAKE, None, None, 64, s, _abi.RET_BF16,
                                   ctypes.c_void_p(0x10010), 1 << 20, None) == _abi.RET_EINVAL


@pytest.mark.parametrize("chunk,dk,dv", [(8, 64, 128), (24, 64, 128), (272, 64, 128), (144, 256, 128),
                                         (256, 256, 512), (64, 96, 128), (64, 64, 192), (64, 512, 128)])
@NO_DEVICE
def test_unsupported_bf16_shapes(lib, chunk, dk, dv):
    s = _abi.RetShape(1, 1, 256, dk, dv)
    assert lib.retention_chunkwise(FAKE, FAKE, FAKE, _g(0.5), FAKE, None, None, chunk, s, _abi.RET_BF16,
                                   None, 0, None) == _abi.RET_EUNSUPPORTED


@NO_DEVICE
def test_zero_chunk_is_einval(lib):
    s = _abi.RetShape(1, 1, 8, 64, 128)
    assert lib.retention_chunkwise(FAKE, FAKE, FAKE, _g(0.5), FAKE, None, None, 0, s, _abi.RET_F32,
                                   None, 0, None) == _abi.RET_EINVAL


def test_empty_parallel_call_is_a_noop(lib):
    s = _abi.RetShape(2, 2, 0, 64, 128)
    assert lib.retention_parallel(None, None, None, _g(0.5, 0.9), None, s, _abi.RET_BF16, None) == _abi.RET_OK


def test_workspace_query(lib):
    few_heads = _abi.RetShape(1, 2, 8192, 64, 128)
    many_heads = _abi.RetShape(4, 8, 8192, 256, 512)
    assert lib.retention_chunkwise_workspace_bytes(64, many_heads, _abi.RET_BF16) == 0
    n = lib.retention_chunkwise_workspace_bytes(64, few_heads, _abi.RET_BF16)
    assert n > 0 and n % (2 * 64 * 128 * 4) == 0
    assert lib.retention_chunkwise_workspace_bytes(64, few_heads, _abi.RET_F32) == 0
    # blocks of up to 256 rows for dk <= 128; none beyond 128 for dk = 256
    assert lib.retention_chunkwise_workspace_bytes(256, few_heads, _abi.RET_BF16) > 0
    assert lib.retention_chunkwise_workspace_bytes(256, _abi.RetShape(1, 2, 8192, 256, 128), _abi.RET_BF16) == 0


@NO_DEVICE
def test_host_entry_validation(lib):
    s = _abi.RetShape(1, 2, 256, 64, 128)
    g = _g(0.5, 0.9)
    args = lambda qh, dev: (qh, FAKE, FAKE, g, FAKE, dev, FAKE, FAKE, FAKE, None, None, 64, s,  # noqa: E731
                            _abi.RET_BF16, None, 0, 0, None)
    assert lib.retention_chunkwise_host(*args(None, FAKE)) == _abi.RET_EINVAL      # host q missing
    assert lib.retention_chunkwise_host(*args(FAKE, None)) == _abi.RET_EINVAL      # device q missing
    bad = _abi.RetShape(1, 2, 256, 96, 128)
    assert lib.retention_chunkwise_host(FAKE, FAKE, FAKE, g, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 64, bad,
                                        _abi.RET_BF16, None, 0, 0, None) == _abi.RET_EUNSUPPORTED
    assert lib.retention_chunkwise_host(FAKE, FAKE, FAKE, _g(0.5, 1.5), FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                        64, s, _abi.RET_BF16, None, 0, 0, None) == _abi.RET_EINVAL


def test_host_entry_workspace_query(lib):
    # groups are 4 heads of one batch row here (8 groups over B*H = 32 rows)
    s = _abi.RetShape(4, 8, 8192, 128, 256)
    n = lib.retention_chunkwise_host_workspace_bytes(128, s, _abi.RET_BF16, 8)
    assert n == lib.retention_chunkwise_workspace_bytes(128, _abi.RetShape(1, 4, 8192, 128, 256), _abi.RET_BF16)
    assert n > 0


@NO_DEVICE
def test_parallel_backward_validation(lib):
    s = _abi.RetShape(1, 2, 64, 64, 128)
    g = _g(0.5, 0.9)
    # the anti-causal sums read the inputs in place: no workspace
    assert lib.retention_parallel_backward_workspace_bytes(s, _abi.RET_F32) == 0
    assert lib.retention_parallel_backward_workspace_bytes(s, _abi.RET_BF16) == 0
    call = lambda dt=_abi.RET_F32, shape=s, dy=FAKE, gam=g: lib.retention_parallel_backward(  # noqa: E731
        FAKE, FAKE, FAKE, gam, dy, FAKE, FAKE, FAKE, shape, dt, None, 0, None)
    assert call(dy=None) == _abi.RET_EINVAL
    assert call(gam=_g(0.5, 1.5)) == _abi.RET_EINVAL
    assert call(_abi.RET_BF16, _abi.RetShape(1, 2, 64, 96, 128)) == _abi.RET_EUNSUPPORTED


@NO_DEVICE
def test_chunkwise_backward_state_validation(lib):
    # every case below returns before any launch
    s = _abi.RetShape(1, 2, 64, 64, 128)
    g = _g(0.5, 0.9)
    base = lib.retention_chunkwise_backward_workspace_bytes(64, s, _abi.RET_F32)
    need = lib.retention_chunkwise_backward_state_workspace_bytes(64, s, _abi.RET_F32)
    assert need == base + 3 * ((2 * 64 * 128 * 4 + 255) // 256 * 256)
    # bf16 on a long sequence: the split scratch of the chunkwise calls
    long = _abi.RetShape(1, 2, 8192, 128, 128)
    assert lib.retention_chunkwise_backward_workspace_bytes(128, long, _abi.RET_BF16) > 0
    ws = ctypes.c_void_p(0x100000)

    def call(nbytes, s0=FAKE, dso=FAKE, ds0=FAKE, chunk=64, dt=_abi.RET_F32, shape=s, dy=FAKE, w=ws):
        return lib.retention_chunkwise_backward_state(FAKE, FAKE, FAKE, g, dy, s0, dso, FAKE, FAKE, FAKE, ds0,
                                                      chunk, shape, dt, w, nbytes, None)

    assert call(need - 1) == _abi.RET_EINVAL                       # states need their three regions
    assert call(base, s0=None, dso=None) == _abi.RET_EINVAL        # dstate_in alone needs them too
    assert call(need, ds0=ctypes.c_void_p(0x1008)) == _abi.RET_EINVAL  # misaligned state
    assert call(need, s0=ctypes.c_void_p(0x1004)) == _abi.RET_EINVAL
    assert call(need, dy=None) == _abi.RET_EINVAL
    assert call(need, chunk=0) == _abi.RET_EINVAL
    assert call(need, w=ctypes.c_void_p(0x100010)) == _abi.RET_EINVAL  # workspace not 256-byte aligned
    assert call(need, dt=_abi.RET_F32, shape=_abi.RetShape(1, 2, 64, 64, 512)) == _abi.RET_EUNSUPPORTED
    assert lib.retention_chunkwise_backward_state(FAKE, FAKE, FAKE, _g(1.5, 0.9), FAKE, FAKE, FAKE, FAKE, FAKE,
                                                  FAKE, FAKE, 64, s, _abi.RET_F32, ws, need,
                                                  None) == _abi.RET_EINVAL  # gamma outside [0, 1]


@NO_DEVICE
def test_groupnorm_gated_validation(lib):
    s = _abi.RetShape(1, 2, 8, 1, 128)
    call = lambda gate, act, y=FAKE: lib.retention_groupnorm_gated(  # noqa: E731
        y, gate, FAKE, 1e-5, None, None, act, s, _abi.RET_BF16, None)
    assert call(FAKE, 3) == _abi.RET_EINVAL       # unknown activation
    assert call(FAKE, -1) == _abi.RET_EINVAL
    assert call(ctypes.c_void_p(0x10008), 1) == _abi.RET_EINVAL  # gate not 16-byte aligned (dv % 128 == 0)
    assert call(FAKE, 1, y=None) == _abi.RET_EINVAL
    assert lib.retention_groupnorm_gated(FAKE, FAKE, FAKE, -1.0, None, None, 1, s, _abi.RET_BF16,
                                         None) == _abi.RET_EINVAL  # eps < 0
    assert lib.retention_groupnorm_gated(FAKE, FAKE, FAKE, 1e-5, None, None, 1, _abi.RetShape(1, 2, 8, 1, 2048),
                                         _abi.RET_BF16, None) == _abi.RET_EUNSUPPORTED


@NO_DEVICE
def test_chunkwise_state_and_fold_validation(lib):
    # every case below returns before any launch
    s = _abi.RetShape(1, 2, 256, 128, 128)
    g = _g(0.5, 0.9)
    need = lib.retention_chunkwise_state_workspace_bytes(64, s, _abi.RET_BF16)
    assert need >= 2 * 2 * 128 * 128 * 4                      # at least two states per (b, h)
    assert lib.retention_chunkwise_state_workspace_bytes(64, s, _abi.RET_F32) == 0
    assert lib.retention_chunkwise_state_workspace_bytes(64, _abi.RetShape(1, 2, 256, 96, 128), _abi.RET_BF16) == 0
    ws = ctypes.c_void_p(0x100000)
    call = lambda out=FAKE, s_in=None, chunk=64, shape=s, dt=_abi.RET_BF16, w=ws, nb=need: (  # noqa: E731
        lib.retention_chunkwise_state(FAKE, FAKE, g, s_in, out, chunk, shape, dt, w, nb, None))
    assert call(out=None) == _abi.RET_EINVAL                   # state_out is required
    assert call(out=ctypes.c_void_p(0x10004)) == _abi.RET_EINVAL
    assert call(s_in=ctypes.c_void_p(0x10008)) == _abi.RET_EINVAL
    assert call(chunk=0) == _abi.RET_EINVAL
    assert call(w=ctypes.c_void_p(0x100040)) == _abi.RET_EINVAL  # workspace not 256-byte aligned
    assert call(shape=_abi.RetShape(1, 2, 256, 96, 128)) == _abi.RET_EUNSUPPORTED
    assert call(dt=_abi.RET_F32, chunk=256) == _abi.RET_EUNSUPPORTED
    # fold
    lens = (ctypes.c_int * 3)(10, 20, 30)
    fold = lambda parts=FAKE, ln=lens, n=3, out=FAKE: lib.retention_state_fold(  # noqa: E731
        parts, ln, n, g, None, out, s, None)
    assert fold(n=257) == _abi.RET_EINVAL                      # at most 256 parts
    assert fold(n=-1) == _abi.RET_EINVAL
    assert fold(parts=None) == _abi.RET_EINVAL
    assert fold(ln=None) == _abi.RET_EINVAL
    assert fold(ln=(ctypes.c_int * 3)(10, -1, 30)) == _abi.RET_EINVAL
    assert fold(out=None) == _abi.RET_EINVAL
    assert fold(parts=ctypes.c_void_p(0x10004)) == _abi.RET_EINVAL


@NO_DEVICE
def test_state_fold_rejects_out_inside_parts(lib):
    s = _abi.RetShape(1, 2, 0, 16, 16)
    lens = (ctypes.c_int * 2)(5, 7)
    per = 2 * 16 * 16 * 4
    parts = 0x100000
    for out in (parts, parts + per, parts + per - 16, parts - per + 16):
        assert lib.retention_state_fold(ctypes.c_void_p(parts), lens, 2, _g(0.5, 0.9), None, ctypes.c_void_p(out), s,
                                        None) == _abi.RET_EINVAL, hex(out)


def test_plain_c_caller():
    # the header compiles as C99 and the library links and answers from C
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.join(root, "retnet_retention_chunkwise_b200")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "c_caller")
        subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                        os.path.join(root, "tests", "c_caller.c"), "-o", exe, "-L", libdir, "-lretention",
                        f"-Wl,-rpath,{libdir}"], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("ok ")


@NO_DEVICE
def test_chunkwise_gn_gated_validation(lib):
    s = _abi.RetShape(1, 2, 64, 128, 128)
    g = _g(0.5, 0.9)
    call = lambda gate, act, eps=1e-5, y=ctypes.c_void_p(0x20000): lib.retention_chunkwise_gn_gated(  # noqa: E731
        FAKE, FAKE, FAKE, g, y, None, None, 64, s, _abi.RET_BF16, eps, None, None, gate, act, None, 0, None)
    assert call(FAKE, 5) == _abi.RET_EINVAL                       # unknown activation
    assert call(FAKE, 1, eps=-1.0) == _abi.RET_EINVAL             # eps < 0
    assert call(ctypes.c_void_p(0x10008), 1) == _abi.RET_EINVAL   # gate not 16-byte aligned
    assert call(ctypes.c_void_p(0x20000), 1) == _abi.RET_EINVAL   # gate is y
    # a gate that shares any byte with y (y is 2*64*128 bf16 = 0x8000 bytes at 0x20000)
    assert call(ctypes.c_void_p(0x20010), 1) == _abi.RET_EINVAL   # a few rows into y
    assert call(ctypes.c_void_p(0x27ff0), 1) == _abi.RET_EINVAL   # its last 16 bytes
    assert call(ctypes.c_void_p(0x18010), 1) == _abi.RET_EINVAL   # ends inside y


def test_missing_library_fails_loudly():
    # no fallback: without the built library the binding raises, naming the build step
    with pytest.raises(ImportError, match="build"):
        _abi.load("/nonexistent/libretention.so")


def test_calls_fail_without_cuda_tensors():
    # the binding never computes on the host: CPU tensors are refused
    import torch

    import retnet_retention_chunkwise_b200 as ret
    q = torch.zeros((1, 1, 4, 64), dtype=torch.bfloat16)
    v = torch.zeros((1, 1, 4, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ret.chunkwise(q, q, v, torch.tensor([0.5]), 64)
    with pytest.raises(ValueError, match="CUDA"):
        ret.parallel(q, q, v, torch.tensor([0.5]))
    with pytest.raises(ValueError, match="CUDA"):
        ret.chunkwise_state(q, v, torch.tensor([0.5]), 64)
