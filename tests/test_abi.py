"""The C-ABI library: loads, exports every symbol include/ra.h declares, and
rejects invalid arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ra.h")


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import blockwise_exact_attention_block_b200 as mod
    return mod


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["ra_block_attn", "ra_merge_partial", "ra_ring_attention", "ra_ring_attention_workspace",
              "ra_zigzag_permute", "ra_get_device_status", "ra_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(ra):
    out = subprocess.run(["nm", "-D", "--defined-only", ra.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ra_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(ra.EXPORTED) <= exported


def test_status_strings(ra):
    assert ra.ra_status_string(0) == "RA_OK"
    assert ra.ra_status_string(3) == "RA_ERR_WORKSPACE"
    assert ra.ra_status_string(99) == "RA_ERR_UNKNOWN"
    assert "sm_100a" in ra.ra_version()


FAKE = 1 << 20  # an aligned, non-null address; never dereferenced on these paths


def ring(ra, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=ra.RA_BF16, B=1, S=4096, Hq=8, D=128, n=4, causal=1,
                part=ra.RA_PART_ZIGZAG, groups=1, out=FAKE, out_dtype=ra.RA_F32, lse=FAKE, ws=FAKE,
                ws_bytes=1 << 40, opts=None, stream=None)
    args.update(kw)
    return ra._lib.ra_ring_attention(args["q"], args["k"], args["v"], args["in_dtype"], args["B"], args["S"],
                                     args["Hq"], args["D"], args["n"], args["causal"], args["part"],
                                     args["groups"], args["out"], args["out_dtype"], args["lse"], args["ws"],
                                     args["ws_bytes"], args["opts"], args["stream"])


def test_ring_attention_rejects_bad_arguments(ra):
    E = ra
    assert ring(ra, S=4100) == E.RA_ERR_INVALID_ARG            # S % (2n) != 0 under zigzag
    assert ring(ra, S=4099, part=ra.RA_PART_CONTIGUOUS) == E.RA_ERR_INVALID_ARG
    assert ring(ra, groups=3) == E.RA_ERR_INVALID_ARG          # Hq % groups != 0
    assert ring(ra, D=96) == E.RA_ERR_UNSUPPORTED
    assert ring(ra, n=17) == E.RA_ERR_UNSUPPORTED
    assert ring(ra, n=0) == E.RA_ERR_INVALID_ARG
    assert ring(ra, q=None) == E.RA_ERR_INVALID_ARG
    assert ring(ra, out=FAKE + 4) == E.RA_ERR_INVALID_ARG      # misaligned
    assert ring(ra, in_dtype=7) == E.RA_ERR_INVALID_ARG
    assert ring(ra, part=5) == E.RA_ERR_INVALID_ARG
    assert ring(ra, ws=None, in_dtype=ra.RA_F32) == E.RA_ERR_WORKSPACE     # fp32 inputs are rounded in scratch
    assert ring(ra, ws_bytes=16, in_dtype=ra.RA_F32) == E.RA_ERR_WORKSPACE
    unf = ra.ra_options(0, ra.RA_SCHED_UNFUSED, None, None, 0)
    assert ring(ra, ws=None, opts=ctypes.byref(unf)) == E.RA_ERR_WORKSPACE  # per-step partials
    bad = ra.ra_options(9, 0, None, None, 0)
    assert ring(ra, opts=ctypes.byref(bad)) == E.RA_ERR_INVALID_ARG
    bad_tiling = ra.ra_options(0, 0, None, None, 9)
    assert ring(ra, opts=ctypes.byref(bad_tiling)) == E.RA_ERR_INVALID_ARG
    bad_fault = ra.ra_options(0, 0, None, None, 0, 2)
    assert ring(ra, opts=ctypes.byref(bad_fault)) == E.RA_ERR_INVALID_ARG


def noalloc(ra, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=ra.RA_BF16, B=1, S=4096, Hq=8, D=128, n=4, causal=1,
                part=ra.RA_PART_ZIGZAG, groups=1, out=FAKE, out_dtype=ra.RA_F32, lse=FAKE, opts=None, stream=None)
    args.update(kw)
    return ra._lib.ra_ring_attention_noalloc(args["q"], args["k"], args["v"], args["in_dtype"], args["B"],
                                             args["S"], args["Hq"], args["D"], args["n"], args["causal"],
                                             args["part"], args["groups"], args["out"], args["out_dtype"],
                                             args["lse"], args["opts"], args["stream"])


@pytest.mark.parametrize("kw", [dict(S=4100), dict(groups=3), dict(groups=0), dict(D=96), dict(n=17), dict(n=0),
                                dict(in_dtype=7), dict(out_dtype=9), dict(part=5), dict(q=None),
                                dict(out=FAKE + 4), dict(B=0)],
                         ids=lambda kw: ",".join(f"{k}={v}" for k, v in kw.items()))
def test_noalloc_returns_the_same_status_as_the_workspace_call(ra, kw):
    # Invalid arguments never reach the scratch lookup or a launch (no GPU
    # needed); both entry points must name the same cause.
    expect = ring(ra, **kw)
    assert expect in (ra.RA_ERR_INVALID_ARG, ra.RA_ERR_UNSUPPORTED)
    assert noalloc(ra, **kw) == expect


@pytest.mark.parametrize("entry", ["ra_block_attn", "ra_block_attn_merge"])
def test_block_attn_rejects_bad_arguments(ra, entry):
    # ra_block_attn_merge takes the same arguments, with the running (out, lse)
    # in place of (block_out, block_lse)
    f = getattr(ra._lib, entry)
    ok = dict(q=FAKE, k=FAKE, v=FAKE, dt=ra.RA_BF16, B=1, S=1024, n=4, qb=0, kb=0, Hq=4, Hkv=2, D=128, causal=1,
              part=ra.RA_PART_ZIGZAG, bo=FAKE, bl=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["dt"], a["B"], a["S"], a["n"], a["qb"], a["kb"], a["Hq"], a["Hkv"],
                 a["D"], a["causal"], a["part"], a["bo"], a["bl"], None)

    assert call(dt=ra.RA_F32) == ra.RA_ERR_UNSUPPORTED
    assert call(qb=4) == ra.RA_ERR_INVALID_ARG
    assert call(kb=-1) == ra.RA_ERR_INVALID_ARG
    assert call(Hkv=3) == ra.RA_ERR_INVALID_ARG
    assert call(bo=None) == ra.RA_ERR_INVALID_ARG
    assert call(S=1028) == ra.RA_ERR_INVALID_ARG
    assert call(bl=FAKE + 4) == ra.RA_ERR_INVALID_ARG
    assert call(D=96) == ra.RA_ERR_UNSUPPORTED


def test_merge_and_permute_reject_bad_arguments(ra):
    m = ra._lib.ra_merge_partial
    assert m(FAKE, FAKE, FAKE, FAKE, -1, 128, None) == ra.RA_ERR_INVALID_ARG
    assert m(FAKE, FAKE, FAKE, FAKE, 0, 128, None) == ra.RA_OK          # empty: no-op
    assert m(FAKE, FAKE, FAKE, FAKE, 10, 6, None) == ra.RA_ERR_UNSUPPORTED
    assert m(FAKE + 8, FAKE, FAKE, FAKE, 10, 128, None) == ra.RA_ERR_INVALID_ARG
    p = ra._lib.ra_zigzag_permute
    assert p(FAKE, FAKE + (1 << 30), 1, 100, 2, 8, 2, 3, 0, None) == ra.RA_ERR_INVALID_ARG  # 100 % 6
    assert p(FAKE, FAKE, 1, 96, 2, 8, 2, 3, 0, None) == ra.RA_ERR_INVALID_ARG               # in place
    assert p(FAKE, FAKE + 64, 1, 96, 2, 8, 2, 3, 0, None) == ra.RA_ERR_INVALID_ARG          # overlap
    assert p(FAKE, FAKE + (1 << 30), 1, 96, 2, 8, 3, 3, 0, None) == ra.RA_ERR_INVALID_ARG   # elem bytes


def test_workspace_query(ra):
    # the partition is an index map: bf16 inputs need no scratch on the default path
    assert ra.ra_ring_attention_workspace(1, 24000, 32, 128, 4, 4, "zigzag") == 0
    assert ra.ra_ring_attention_workspace(1, 4096, 8, 128, 4, 1, "contiguous") == 0
    # fp32 inputs: bf16 copies of Q (32 heads) and K, V (8 heads each)
    n = ra.ra_ring_attention_workspace(1, 24000, 32, 128, 4, 4, "zigzag", in_dtype=torch.float32)
    assert n >= 24000 * (32 + 8 + 8) * 128 * 2
    # unfused: fp32 partial out + lse; bf16 output adds the fp32 running output
    n_unf = ra.ra_ring_attention_workspace(1, 4096, 8, 128, 4, 1, "contiguous", sched="unfused")
    assert n_unf >= 4096 * 8 * (128 + 1) * 4
    n_unf16 = ra.ra_ring_attention_workspace(1, 4096, 8, 128, 4, 1, "contiguous", sched="unfused",
                                             out_dtype=torch.bfloat16)
    assert n_unf16 >= n_unf + 4096 * 8 * 128 * 4
    with pytest.raises(ra.RAError):
        ra.ra_ring_attention_workspace(1, 4095, 8, 128, 4, 1, "zigzag")


def decode(ra, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=ra.RA_BF16, B=1, Tq=1, Skv=4096, Hq=8, Hkv=2, D=128, causal=1,
                n_splits=0, out=FAKE, out_dtype=ra.RA_F32, lse=FAKE, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return ra._lib.ra_decode_attention(args["q"], args["k"], args["v"], args["in_dtype"], args["B"], args["Tq"],
                                       args["Skv"], args["Hq"], args["Hkv"], args["D"], args["causal"],
                                       args["n_splits"], args["out"], args["out_dtype"], args["lse"], args["ws"],
                                       args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hkv=4), 1),                 # Hq not a multiple of Hkv
    (dict(Tq=5000), 1),                     # more query tokens than cached ones
    (dict(Skv=0), 1),
    (dict(n_splits=-1), 1),
    (dict(D=96), 2),
    (dict(Hq=32, Hkv=2, Tq=5), 2),          # 16 heads x 5 tokens > 64 rows per KV head
    (dict(in_dtype=0), 2),                  # fp32 cache
    (dict(out_dtype=7), 1),
    (dict(q=None), 1),
    (dict(lse=FAKE + 2), 1),                # misaligned lse
    (dict(ws_bytes=16), 3),                 # workspace too small
    (dict(ws=FAKE + 64), 1),                # workspace not 256-byte aligned
])
def test_decode_rejects_invalid_arguments(ra, kw, status):
    assert decode(ra, **kw) == status


def test_decode_plan(ra):
    # chunks cover the cache in multiples of 64 keys; workspace holds one
    # fp32 partial (out and lse) per chunk and row
    for (B, Tq, Skv, Hq, Hkv, D, n) in [(1, 1, 1048576, 8, 2, 128, 0), (8, 4, 24000, 32, 8, 128, 0),
                                         (2, 3, 1000, 8, 2, 128, 5), (1, 1, 64, 2, 1, 64, 0), (1, 2, 100, 4, 4, 64, 50)]:
        splits = ra.ra_decode_splits(B, Tq, Skv, Hq, Hkv, D, n)
        chunk = -(-Skv // (n if n else splits))
        chunk = -(-chunk // 64) * 64
        assert splits == -(-Skv // chunk)
        assert 1 <= splits <= max(n, 1) if n else splits >= 1
        rows = B * Tq * Hq
        assert ra.ra_decode_workspace(B, Tq, Skv, Hq, Hkv, D, n) >= splits * rows * (D + 1) * 4
    assert ra._lib.ra_decode_splits(1, 1, 10, 8, 3, 128, 0) == -1
    with pytest.raises(ra.RAError):
        ra.ra_decode_workspace(1, 1, 10, 8, 3, 128, 0)


def backward(ra, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=ra.RA_BF16, out=FAKE, out_dtype=ra.RA_F32, lse=FAKE, dout=FAKE,
                B=1, S=4096, Hq=8, D=128, n=4, causal=1, part=ra.RA_PART_ZIGZAG, groups=2, dq=FAKE, dk=FAKE,
                dv=FAKE, ws=FAKE, ws_bytes=1 << 40, opts=None, stream=None)
    args.update(kw)
    a = args
    return ra._lib.ra_ring_attention_backward(a["q"], a["k"], a["v"], a["in_dtype"], a["out"], a["out_dtype"],
                                              a["lse"], a["dout"], a["B"], a["S"], a["Hq"], a["D"], a["n"],
                                              a["causal"], a["part"], a["groups"], a["dq"], a["dk"], a["dv"],
                                              a["ws"], a["ws_bytes"], a["opts"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(S=4100), 1), (dict(groups=3), 1), (dict(D=96), 2), (dict(n=17), 2), (dict(n=0), 1),
    (dict(dout=None), 1), (dict(dq=None), 1), (dict(dk=FAKE + 4), 1), (dict(lse=FAKE + 8), 1),
    (dict(in_dtype=7), 1), (dict(out_dtype=5), 1), (dict(part=2), 1), (dict(ws=None), 3), (dict(ws_bytes=64), 3),
    (dict(ws=FAKE + 16), 1),
])
def test_backward_rejects_invalid_arguments(ra, kw, status):
    assert backward(ra, **kw) == status


def test_backward_workspace_query(ra):
    # Delta and lse * log2(e): two fp32 values per (row, query head)
    n = ra.ra_ring_attention_backward_workspace(1, 24000, 32, 128, 4, 4, "zigzag")
    assert n >= 2 * 24000 * 32 * 4
    # fp32 inputs add bf16 copies of q, k, v and dout
    n32 = ra.ra_ring_attention_backward_workspace(1, 24000, 32, 128, 4, 4, "zigzag", in_dtype=torch.float32)
    assert n32 >= n + 24000 * (32 + 8 + 8 + 32) * 128 * 2
    with pytest.raises(ra.RAError):
        ra.ra_ring_attention_backward_workspace(1, 4095, 8, 128, 4, 1, "zigzag")


def test_c_caller_links_and_runs(ra, tmp_path):
    # the boundary from plain C: include/ra.h, a C compiler and the .so
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(ra.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    build = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", lib_dir, "-lra_b200",
                            f"-Wl,-rpath,{lib_dir}", "-o", exe], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.startswith("ok ")


def test_release_build_is_not_the_checked_build(ra):
    # the checked build is a separate library (libra_b200_debug.so); the
    # release one reports 0, has no bounds record, and rejects the checked
    # build's injected out-of-range row before any launch
    assert ra.ra_debug_build() is False
    assert ra.ra_get_bounds_record() == (0, 0, 0)
    inj = ra.ra_options(0, ra.RA_SCHED_AUTO, None, None, 0, 2)
    assert ring(ra, opts=ctypes.byref(inj)) == ra.RA_ERR_INVALID_ARG


def test_checked_build_exports_the_same_symbols(ra):
    import __graft_entry__
    mod = __graft_entry__._build_module()
    path = mod.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ra_\w+)", out))
    assert not [n for n in declared_functions() if n not in exported]


def test_cta_timeline_setter_validates_on_the_host(ra):
    # host-only: the setter records the buffer for later launches and
    # launches nothing itself; every case ends with the timeline off
    lib = ra._lib
    fake = 0x10000  # never dereferenced: no launch follows while it is set
    try:
        assert lib.ra_set_cta_timeline(None, 0, 0) == ra.RA_OK
        assert lib.ra_set_cta_timeline(None, 0, 7) == ra.RA_ERR_INVALID_ARG   # unknown kernel
        assert lib.ra_set_cta_timeline(fake, 0, 0) == ra.RA_ERR_INVALID_ARG   # no records
        assert lib.ra_set_cta_timeline(fake, -1, 1) == ra.RA_ERR_INVALID_ARG
        assert lib.ra_set_cta_timeline(fake, (1 << 24) + 1, 2) == ra.RA_ERR_INVALID_ARG
        assert lib.ra_set_cta_timeline(fake + 4, 16, 0) == ra.RA_ERR_INVALID_ARG  # misaligned
        for kernel in (0, 1, 2):
            assert lib.ra_set_cta_timeline(fake, 16, kernel) == ra.RA_OK
    finally:
        assert lib.ra_set_cta_timeline(None, 0, 0) == ra.RA_OK
    with pytest.raises(ValueError):
        ra.ra_set_cta_timeline(None, "no_such_kernel")
    with pytest.raises(ValueError):
        ra.ra_set_cta_timeline(torch.zeros((4, 3), dtype=torch.int64), "attn_fwd")
