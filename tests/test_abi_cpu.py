"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/bimamba.h declares, and rejects bad arguments on
the host (before any CUDA call) with the documented status codes."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssm_b200 import build
    build.build()
    from bidirectional_mamba_ssm_b200 import _lib
    return _lib


def _declared():
    src = open(os.path.join(ROOT, "include", "bimamba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bimamba_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert set(names) == set(lib.EXPORTED)
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(so, n), n


def test_version_and_strerror(lib):
    assert lib.bimamba_version() >> 16 == 1
    for code in range(6):
        assert lib.strerror(code) and lib.strerror(code) != "unknown status"
    assert lib.strerror(99) == "unknown status"


def _call_scan(lib, dims, **ptrs):
    L = lib.library()
    p = dict(xbc=16, dt=16, A=16, D=16, conv_w=None, conv_b=None, init=None, fin=None, y=16,
             ws=None, wsz=0)
    p.update(ptrs)
    return L.bimamba_ssd_fwd_rev(ctypes.byref(dims), p["xbc"], p["dt"], p["A"], p["D"],
                                 p["conv_w"], p["conv_b"], p["init"], p["fin"], p["y"], p["ws"],
                                 p["wsz"], None)


def test_host_validation_codes(lib):
    ok = dict(batch=1, seqlen=8, heads=2, headdim=8, d_state=16, dtype=0)
    d = lib.make_dims(**ok)
    # shape errors (checked before anything touches the device)
    for bad, code in [(dict(heads=0), lib.BIMAMBA_ERR_INVALID),
                      (dict(headdim=-8), lib.BIMAMBA_ERR_INVALID),
                      (dict(batch=-1), lib.BIMAMBA_ERR_INVALID),
                      (dict(headdim=12), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(headdim=136), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(d_state=24), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(d_state=512), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(ngroups=2), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(d_conv=3), lib.BIMAMBA_ERR_UNSUPPORTED),
                      (dict(dtype=7), lib.BIMAMBA_ERR_INVALID)]:
        args = dict(ok)
        args.update(bad)
        assert _call_scan(lib, lib.make_dims(**args)) == code, bad
        assert lib.bimamba_workspace_bytes(lib.make_dims(**args)) == 0
    # pointer errors
    assert _call_scan(lib, d, xbc=None) == lib.BIMAMBA_ERR_INVALID
    assert _call_scan(lib, d, y=None) == lib.BIMAMBA_ERR_INVALID
    assert _call_scan(lib, d, xbc=18) == lib.BIMAMBA_ERR_INVALID          # misaligned
    assert _call_scan(lib, d, conv_b=16) == lib.BIMAMBA_ERR_INVALID       # bias without weights
    # empty batch is a no-op
    assert _call_scan(lib, lib.make_dims(**dict(ok, batch=0))) == lib.BIMAMBA_OK
    L = lib.library()
    # conv entry point
    assert L.bimamba_conv_silu(16, 16 + 4096, 16, None, None, 1, 8, 12, 4, 0, 1, 0, None) \
        == lib.BIMAMBA_ERR_UNSUPPORTED                                      # ch % 8
    assert L.bimamba_conv_silu(16, 32, 16, None, None, 1, 8, 8, 4, 0, 1, 0, None) \
        == lib.BIMAMBA_ERR_INVALID                                          # overlap
    assert L.bimamba_conv_silu(16, 1 << 20, 16, None, 16, 1, 8, 8, 4, 1, 1, 0, None) \
        == lib.BIMAMBA_ERR_INVALID                                          # tail + reverse
    # decode entry point: conv weights, state and tail are required
    r = L.bimamba_block_decode(ctypes.byref(d), 16, 16, 16, 16, None, None, 16, 16, 16, None,
                               None, None, 0, None)
    assert r == lib.BIMAMBA_ERR_INVALID


def test_workspace_size_is_monotone(lib):
    a = lib.bimamba_workspace_bytes(lib.make_dims(8, 4096, 64, 64, 128, 1))
    b = lib.bimamba_workspace_bytes(lib.make_dims(8, 8192, 64, 64, 128, 1))
    assert 0 <= a <= b


def test_launch_plan_covers_the_walk(lib):
    """Segment plans (host only): segments tile the chunk walk, state-only
    items tile the walk before the last segment and nest in the segments, and
    a segmented launch stays within one wave of the 148 SMs."""
    import torch
    assert lib.bimamba_launch_plan(lib.make_dims(1, 256, 4, 32, 16, torch.float32)) == {
        "tensor_core": False, "segments": 1, "seg_chunks": 2, "items": 0}
    # the benchmarked layer (512 CTAs) is not segmented
    assert lib.bimamba_launch_plan(lib.make_dims(8, 4096, 64, 64, 128, torch.bfloat16)) == {
        "tensor_core": True, "segments": 1, "seg_chunks": 32, "items": 0}
    seen_split_items = False
    for bsz in (1, 2, 3, 8):
        for H in (2, 4, 16, 32, 64):
            for L in (1, 127, 128, 513, 1100, 1300, 4096, 131072):
                p = lib.bimamba_launch_plan(lib.make_dims(bsz, L, H, 64, 128, torch.bfloat16))
                nchunks = (L + 127) // 128
                S, sc, items = p["segments"], p["seg_chunks"], p["items"]
                assert p["tensor_core"]
                assert S >= 1 and sc >= 1
                assert (S - 1) * sc < nchunks <= S * sc, (bsz, H, L, p)
                ctas = bsz * H
                if S == 1:
                    assert items == 0
                    continue
                assert ctas * S <= 148 and ctas * items <= 148, (bsz, H, L, p)
                assert items % (S - 1) == 0
                r = items // (S - 1)
                assert sc % r == 0
                seen_split_items |= r > 1
    assert seen_split_items


def test_launch_plan_rejects_bad_arguments(lib):
    import torch
    L = lib.library()
    d = lib.make_dims(1, 8, 0, 64, 128, torch.bfloat16)
    out = (ctypes.c_int * 4)()
    assert L.bimamba_launch_plan(ctypes.byref(d), out) == lib.BIMAMBA_ERR_INVALID
    d = lib.make_dims(1, 8, 2, 64, 128, torch.bfloat16)
    assert L.bimamba_launch_plan(ctypes.byref(d), None) == lib.BIMAMBA_ERR_INVALID


def test_workspace_grows_with_the_state_only_items(lib):
    import torch
    d1 = lib.make_dims(1, 1300, 2, 64, 128, torch.bfloat16)    # 10 items
    flags = 1024                                                 # 11 chunks x 2 counters, 1 KB
    act = 2 * 1 * 1300 * 256 * 2
    items = 2 * 1 * 1 * 10
    assert lib.bimamba_workspace_bytes(d1) == flags + act + items * 2 * 64 * 128 * 4 + items * 2 * 4


def test_untied_host_validation(lib):
    """bimamba_ssd_fwd_rev_untied rejects bad arguments on the host, before
    anything touches a device."""
    import torch
    L = lib.library()
    d = lib.make_dims(1, 8, 2, 64, 128, torch.bfloat16)

    def call(fusion=0, **over):
        a = dict(xf=16, xr=16, dtf=16, dtr=16, Af=16, Ar=16, Df=16, Dr=16, wf=None, wr=None,
                 bf=None, br=None, init=None, fin=None, y=16)
        a.update(over)
        return L.bimamba_ssd_fwd_rev_untied(
            ctypes.byref(d), a["xf"], a["xr"], a["dtf"], a["dtr"], a["Af"], a["Ar"], a["Df"],
            a["Dr"], a["wf"], a["wr"], a["bf"], a["br"], a["init"], a["fin"], a["y"], fusion,
            None, 0, None)

    assert call(fusion=2) == lib.BIMAMBA_ERR_INVALID
    assert call(fusion=-1) == lib.BIMAMBA_ERR_INVALID
    for k in ("xf", "xr", "dtf", "dtr", "Af", "Ar", "Df", "Dr", "y"):
        assert call(**{k: None}) == lib.BIMAMBA_ERR_INVALID, k
    assert call(br=16) == lib.BIMAMBA_ERR_INVALID          # a bias without its taps
    assert call(bf=16, wf=None) == lib.BIMAMBA_ERR_INVALID
    assert call(xr=24) == lib.BIMAMBA_ERR_INVALID          # misaligned
    assert call(fusion=1, dtr=8) == lib.BIMAMBA_ERR_INVALID
    # unsupported / invalid dims are reported the same way as for the tied call
    bad = lib.make_dims(1, 8, 0, 64, 128, torch.bfloat16)
    assert L.bimamba_ssd_fwd_rev_untied(ctypes.byref(bad), *([16] * 8), *([None] * 6), 16, 0,
                                        None, 0, None) == lib.BIMAMBA_ERR_INVALID
    # an empty batch is a valid no-op
    empty = lib.make_dims(0, 8, 2, 64, 128, torch.bfloat16)
    assert L.bimamba_ssd_fwd_rev_untied(ctypes.byref(empty), *([16] * 8), *([None] * 6), 16, 1,
                                        None, 0, None) == lib.BIMAMBA_OK


def _declared_arity():
    """Parameter count of every entry point, from include/bimamba.h."""
    src = open(os.path.join(ROOT, "include", "bimamba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(bimamba_\w+)\s*\(([^)]*)\)\s*;", src):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(lib):
    """Every ctypes prototype has exactly as many arguments as the C
    declaration (a short prototype passes later arguments with the wrong
    types, which crashes the host process)."""
    so = lib.library()
    arity = _declared_arity()
    assert set(arity) == set(lib.EXPORTED)
    for name, n in arity.items():
        assert len(getattr(so, name).argtypes) == n, (name, len(getattr(so, name).argtypes), n)


def test_plain_c_program_uses_the_abi(lib, tmp_path):
    """The boundary is a C ABI: a C99 program that includes only
    include/bimamba.h and links libbimamba.so builds with gcc and gets the
    documented answers from the entry points that need no device."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_host"
    libdir = os.path.dirname(lib.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", libdir, "-lbimamba",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "abi ok"
