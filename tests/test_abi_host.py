"""The C-ABI library on the host, without a GPU: it loads, exports every
function include/mamba_scan.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

from selective_state_space_20_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mamba_scan.h")


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(mamba_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_abi():
    assert declared_functions() == sorted(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"
    out = os.popen(f"nm -D --defined-only {build.LIB}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), f"{name} missing from dynamic symbol table"


def _prototypes():
    """{name: [parameter type strings]} parsed from the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\*?\s*(mamba_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.M | re.S):
        params = [p.strip() for p in m.group(2).replace("\n", " ").split(",")]
        protos[m.group(1)] = [] if params == ["void"] else params
    return protos


def test_binding_argtypes_match_the_header(lib):
    """Every declared function has ctypes argtypes of the header's arity and
    kind: pointers as void pointers (the binding passes c_void_p for every
    buffer), int64_t, int, size_t and the stream as a pointer."""
    import ctypes as C
    protos = _prototypes()
    assert sorted(protos) == sorted(binding.EXPORTED)
    for name, params in protos.items():
        fn = getattr(lib, name)
        types = fn.argtypes or []
        assert len(types) == len(params), (name, len(types), len(params))
        for p, t in zip(params, types):
            if "*" in p or p.startswith("cudaStream_t"):
                want = (C.c_void_p, C.POINTER(binding.Tuning), C.POINTER(binding.ScanStrides))
                assert t in want, (name, p, t)
            elif p.startswith("int64_t"):
                assert t is C.c_int64, (name, p, t)
            elif p.startswith("size_t"):
                assert t is C.c_size_t, (name, p, t)
            elif p.startswith("int "):
                assert t is C.c_int, (name, p, t)
            else:
                raise AssertionError((name, p))


def test_library_is_built_for_sm100a_only():
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings_and_version(lib):
    for code in list(binding.STATUS_NAMES) + [12345]:
        s = lib.mamba_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.mamba_abi_version() >> 16 == 1


def _scan(lib, ptrs=None, batch=2, dim=4, L=8, N=16, dtype=1, softplus=1, last=None, tuning=None):
    P = ptrs or {}
    get = lambda k, default=0x10000: P.get(k, default)  # noqa: E731
    args = [get("u", 0x100000), get("delta", 0x200000), get("A", 0x300000), get("B", 0x400000),
            get("C", 0x500000), get("D", None), get("z", None), get("bias", None), softplus,
            get("out", 0x600000), last, batch, dim, L, N, dtype]
    args = [ctypes.c_void_p(a) if isinstance(a, int) and i not in (8, 11, 12, 13, 14, 15) else a
            for i, a in enumerate(args)]
    if tuning is not None:
        return lib.mamba_scan_fwd_tuned(*args, ctypes.byref(tuning), None)
    return lib.mamba_scan_fwd(*args, None)


def test_null_pointers_rejected(lib):
    for key in ("u", "delta", "A", "B", "C", "out"):
        assert _scan(lib, {key: None}) == -1, key


def test_bad_sizes_rejected(lib):
    assert _scan(lib, batch=0) == -2
    assert _scan(lib, dim=-3) == -2
    assert _scan(lib, L=0) == -2
    assert _scan(lib, N=0) == -2
    assert _scan(lib, N=65) == -3
    assert _scan(lib, dtype=7) == -3
    assert _scan(lib, batch=1 << 40, dim=1 << 20) == -2


def test_overlap_rejected(lib):
    # out shifted into u by one element: partial overlap
    assert _scan(lib, {"u": 0x100000, "out": 0x100002}) == -7
    # out overlapping B
    assert _scan(lib, {"B": 0x600000, "out": 0x600000}) == -7
    # last_state overlapping out
    assert _scan(lib, {"out": 0x600000}, last=ctypes.c_void_p(0x600010)) == -7


def test_initial_state_validation(lib):
    vp = ctypes.c_void_p
    tun = binding.Tuning(0, 0, 0, 0)

    def init(h0, last=None):
        args = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), None, None,
                None, 1, h0, vp(0x600000), last, 2, 4, 8, 16, 1]
        return lib.mamba_scan_fwd_init(*args, ctypes.byref(tun), None, 0, None)

    assert init(None) == -1                                   # h0 is required
    assert init(vp(0x600000 + 4)) == -7                       # h0 inside out
    assert init(vp(0x700000), last=vp(0x700000 + 16)) == -7   # partly overlaps last_state


def test_bad_tuning_rejected(lib):
    assert _scan(lib, tuning=binding.Tuning(3, 0, 0, 0)) == -3
    assert _scan(lib, tuning=binding.Tuning(0, 100, 0, 0)) == -3
    assert _scan(lib, tuning=binding.Tuning(0, 0, 7, 0)) == -3
    assert _scan(lib, tuning=binding.Tuning(0, 0, 0, -5)) == -3


def test_state_update_validation(lib):
    su = lib.mamba_state_update
    vp = ctypes.c_void_p
    ok = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), vp(0x600000),
          None, None, None, 1, vp(0x700000), 4, 8, 16, 1, None]
    bad = list(ok)
    bad[0] = None
    assert su(*bad) == -1
    bad = list(ok)
    bad[11] = 0
    assert su(*bad) == -2
    bad = list(ok)
    bad[13] = 100
    assert su(*bad) == -3
    bad = list(ok)
    bad[10] = vp(0x100000 + 8)  # out inside the state
    assert su(*bad) == -7


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        binding.mamba_scan_fwd(x, x, torch.zeros(2, 16), torch.zeros(1, 16, 8), torch.zeros(1, 16, 8))


def test_conv1d_validation(lib):
    vp = ctypes.c_void_p
    cf = lib.mamba_conv1d_fwd
    # x, weight, bias, silu, out, batch, dim, L, width, stride, dtype, stream
    ok = [vp(0x100000), vp(0x200000), None, 1, vp(0x800000), 2, 4, 64, 4, 0, 1, None]

    def call(**kw):
        a = list(ok)
        names = ["x", "w", "bias", "silu", "out", "batch", "dim", "L", "width", "stride", "dtype"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return cf(*a)
    assert call(x=None) == -1 and call(w=None) == -1 and call(out=None) == -1
    assert call(batch=0) == -2 and call(L=-1) == -2
    assert call(width=0) == -3 and call(width=5) == -3 and call(dtype=3) == -3
    assert call(stride=4 * 64 - 1) == -2  # rows of one batch row would overlap the next
    assert call(out=vp(0x100000 + 64)) == -7  # out inside x
    cu = lib.mamba_conv1d_update
    # state, x, weight, bias, silu, out, batch, dim, width, stride, dtype, stream
    okc = [vp(0x100000), vp(0x200000), vp(0x300000), None, 1, vp(0x400000), 2, 4, 4, 0, 1, None]
    bad = list(okc)
    bad[0] = None
    assert cu(*bad) == -1  # width 4 needs a state
    bad = list(okc)
    bad[0], bad[8] = None, 1
    assert cu(*bad) != -1  # width 1 keeps no state (fails later only for want of a device)
    bad = list(okc)
    bad[8] = 9
    assert cu(*bad) == -3
    bad = list(okc)
    bad[5] = vp(0x100000 + 4)  # out inside the state
    assert cu(*bad) == -7


def test_scan_bwd_validation(lib):
    vp = ctypes.c_void_p
    assert lib.mamba_scan_bwd_workspace_size(2, 40, 100, 16) > 0
    assert lib.mamba_scan_bwd_workspace_size(2, 40, 100, 17) == 0
    ws_n = lib.mamba_scan_bwd_workspace_size(2, 8, 64, 16)
    P = [vp(0x100000 * (i + 1)) for i in range(20)]
    # u delta A B C D z bias sp dout dlast du ddelta dA dB dC dD dz dbias b d L N act ws wsb stream
    ok = [P[0], P[1], P[2], P[3], P[4], None, None, None, 1, P[5], None, P[6], P[7], P[8], P[9], P[10],
          None, None, None, 2, 8, 64, 16, 1, P[11], ws_n, None]

    def call(**kw):
        a = list(ok)
        idx = {"u": 0, "z": 6, "dout": 9, "du": 11, "dz": 17, "N": 22, "ws": 24, "wsb": 25, "dB": 14}
        for k, v in kw.items():
            a[idx[k]] = v
        return lib.mamba_scan_bwd(*a)
    assert call(u=None) == -1 and call(dout=None) == -1 and call(du=None) == -1
    assert call(z=P[12]) == -1  # a gate needs dz
    assert call(N=32) == -3
    assert call(ws=None) == -8 and call(wsb=ws_n - 1) == -8 and call(ws=vp(0x1000008)) == -8
    assert call(dB=vp(0x400000 + 64)) == -7  # dB inside B

    # the initial-state form: h0 after the softplus flag, dh0 after dbias
    def call_init(h0, dh0):
        a = ok[:9] + [h0] + ok[9:19] + [dh0] + ok[19:]
        return lib.mamba_scan_bwd_init(*a)
    assert call_init(None, None) == -1                     # h0 is required
    assert call_init(P[13], vp(0x600000 + 128)) == -7      # dh0 inside dout
    assert call_init(P[13], P[13]) == -7                   # dh0 over h0


def test_sequence_split_validation(lib):
    vp = ctypes.c_void_p
    # argument marshalling as the binding passes it, rejected before any device work
    assert lib.mamba_delta_sum(vp(0x100000), vp(0x200000), 1, vp(0x300000), 0, 4, 8, 1, None) == -2
    assert lib.mamba_delta_sum(None, None, 1, vp(0x300000), 2, 4, 8, 1, None) == -1
    assert lib.mamba_delta_sum(vp(0x100000), None, 1, vp(0x100000 + 8), 2, 4, 8, 1, None) == -7
    assert lib.mamba_state_fold(vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000),
                                2, 4, 16, -1, None) == -2
    assert lib.mamba_state_fold(None, None, vp(0x300000), None, vp(0x500000), 2, 4, 16, 3, None) == -1
    # the output partly over the initial state
    assert lib.mamba_state_fold(vp(0x500000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000 + 4),
                                2, 4, 16, 1, None) == -7
    # the output over the second h_local slice exactly is allowed; mid-slice is not
    ns = 2 * 4 * 16 * 4
    assert lib.mamba_state_fold(None, vp(0x200000), vp(0x300000), vp(0x400000), vp(0x400000 + 12),
                                2, 4, 16, 2, None) == -7
    assert lib.mamba_state_fold(None, vp(0x200000), vp(0x300000), vp(0x400000), vp(0x400000 + ns + 16),
                                2, 4, 16, 2, None) == -7


def test_fused_conv_scan_validation(lib):
    vp = ctypes.c_void_p
    P = [vp(0x100000 * (i + 1)) for i in range(16)]

    def call(x=P[0], width=4, xbs=0, ws=P[12], wsb=1 << 20, dstate=16, L=64, out=P[8], z=None, zbs=0):
        return lib.mamba_scan_fwd_conv(x, P[1], None, width, xbs, P[2], P[3], P[4], P[5], None, z, zbs, None,
                                       None, out, None, None, 2, 8, L, dstate, 1, ws, wsb, None)
    assert call(x=None) == -1
    assert call(width=5) == -3 and call(width=0) == -3
    assert call(dstate=32) == -3              # the lane-split kernel holds 16 states
    assert call(L=60) == -3                   # whole 16-byte chunks of timesteps
    assert call(x=vp(0x100000 + 2)) == -3     # 16-byte alignment
    assert call(xbs=8 * 64 - 8) == -2         # rows would overlap
    assert call(out=vp(0x100000 + 64)) == -7  # out over x
    assert call(ws=None) == -8 and call(wsb=16) == -8


def test_host_memory_scan_validation(lib):
    vp = ctypes.c_void_p
    need = lib.mamba_scan_host_scratch_size(4, 5120, 4096, 16, 1)
    assert need > 0 and lib.mamba_scan_host_scratch_size(0, 8, 8, 16, 1) == 0
    args = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), None, None, None, 1, None,
            vp(0x600000), None, 2, 4, 64, 16, 1]
    assert lib.mamba_scan_fwd_host(*args, None, 0, None) == -8                      # no scratch
    assert lib.mamba_scan_fwd_host(*args, vp(0x1000000), 16, None) == -8            # too small
    bad = list(args)
    bad[0] = None
    assert lib.mamba_scan_fwd_host(*bad, vp(0x1000000), 1 << 30, None) == -1
    bad = list(args)
    bad[15] = 65
    assert lib.mamba_scan_fwd_host(*bad, vp(0x1000000), 1 << 30, None) == -3


def test_checked_build_exports_the_same_abi():
    """The bounds-checked build of the same sources: every declared symbol,
    and it says which build it is (host-only calls)."""
    checked = binding.load_checked_library()
    for name in declared_functions():
        assert hasattr(checked, name), f"{name} not exported by the checked build"
    assert checked.mamba_bounds_checked() == 1
    assert binding.load_library().mamba_bounds_checked() == 0
    assert binding.load_library().mamba_debug_shrink_output_extent(0) == 0


def test_scan_state_validation(lib):
    vp = ctypes.c_void_p
    P = [vp(0x1000000 * (i + 1)) for i in range(8)]
    ws_n = lib.mamba_scan_workspace_size(2, 8, 64, 16, 1)
    # u delta A B bias softplus h0 last_state batch dim L N act ws wsb stream
    ok = [P[0], P[1], P[2], P[3], None, 1, None, P[4], 2, 8, 64, 16, 1, None, 0, None]
    names = ["u", "delta", "A", "B", "bias", "sp", "h0", "last", "batch", "dim", "L", "N", "act", "ws", "wsb"]

    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.mamba_scan_state(*a)
    assert call(u=None) == -1 and call(B=None) == -1 and call(last=None) == -1
    assert call(batch=0) == -2 and call(act=2) == -3
    assert call(last=vp(0x2000000 + 64)) == -7            # last_state inside delta
    assert call(h0=vp(0x5000000 + 4)) == -7               # h0 overlaps last_state, not exactly
    assert call(ws=vp(0x7000008), wsb=ws_n) == -8         # misaligned workspace
    assert call(ws=vp(0x7000000), wsb=ws_n - 16) == -8    # small workspace
    assert call(ws=vp(0x1000000 + 256), wsb=ws_n) == -7   # workspace over u
