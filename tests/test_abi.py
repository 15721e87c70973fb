"""The C-ABI library loads, exports every entry point its header declares, and rejects bad
arguments before touching the GPU (these calls launch nothing, so they run without one)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_soft_b200 import build
    build.build()
    import linear_attention_soft_b200 as ra
    return ra.load_library()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(race_[A-Za-z0-9_]+)\s*\(",
                            src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("race_attn_forward", "race_attn_backward", "race_attn_hash_indices",
              "race_attn_workspace_size", "race_attn_ctx_size", "race_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    import linear_attention_soft_b200 as ra
    assert ra.race_status_string(ra.RACE_OK) == "RACE_OK"
    assert ra.race_status_string(ra.RACE_ERR_WORKSPACE) == "RACE_ERR_WORKSPACE"
    assert ra.race_status_string(99) == "RACE_ERR_UNKNOWN"


def test_workspace_queries(lib):
    import linear_attention_soft_b200 as ra
    fw = ra.race_attn_workspace_size(1, 1, 4096, 64, 16, 4, 1, 0, ra.RACE_BF16)
    bw = ra.race_attn_workspace_size(1, 1, 4096, 64, 16, 4, 1, 1, ra.RACE_BF16)
    cx = ra.race_attn_ctx_size(1, 1, 4096, 64, 16, 4, 1)
    # backward: both segment-state buffers, a 16 KB W image and c_i per token (fp32)
    assert fw > 0 and bw == 2 * fw + 16384 + 4096 * 4 and cx == fw
    # state is [segments][L*R][d+1] fp32 per head: a multiple of that size
    assert fw % (256 * 65 * 4) == 0
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_workspace_size(1, 1, 4096, 60, 16, 4, 1, 0, ra.RACE_BF16)
    assert e.value.status == ra.RACE_ERR_UNSUPPORTED
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_workspace_size(1, 1, 4096, 64, 16, 6, 1, 0, ra.RACE_BF16)
    assert e.value.status == ra.RACE_ERR_UNSUPPORTED
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_workspace_size(1, 1, 4096, 64, 64, 5, 1, 0, ra.RACE_BF16)  # L*R = 2048
    assert e.value.status == ra.RACE_ERR_UNSUPPORTED
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_workspace_size(0, 1, 4096, 64, 16, 4, 1, 0, ra.RACE_BF16)
    assert e.value.status == ra.RACE_ERR_INVALID_ARG



def _segments(ra, B, H, N):
    """Segments per sequence the library plans, read off the forward workspace size
    (B*H*nseg states of [L*R][d+1] fp32 for d = 64, L = 16, P = 4)."""
    fw = ra.race_attn_workspace_size(B, H, N, 64, 16, 4, 1, 0, ra.RACE_BF16)
    per = B * H * 256 * 65 * 4
    assert fw % per == 0
    return fw // per


def test_segment_plan_fills_whole_waves(lib):
    """One CTA walks one segment and holds its SM, so the planner picks the segment count
    that wastes the fewest CTA slots: one wave when the heads alone do not fill the GPU."""
    import torch
    import linear_attention_soft_b200 as ra
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    # one long head: one segment per SM
    assert _segments(ra, 1, 1, 1 << 22) == sms
    # 16 heads of 65,536 tokens: one wave (at most sms CTAs), not a nearly empty second one
    n = _segments(ra, 2, 8, 65536)
    assert 16 * n <= sms and 16 * (n + 1) > sms
    # more heads than SMs: one segment each
    assert _segments(ra, 64, 64, 4096) == 1
    # never a segment shorter than one 128-token chunk (unless N is); a short head is cut
    # into chunk-long segments, one CTA each
    for N in (1, 300, 1000, 5000, 70000):
        assert 1 <= _segments(ra, 1, 1, N) <= max(1, -(-N // 128))
    assert _segments(ra, 1, 1, 1024) == 8

def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, W=16, out=16, den=16, ctx=None, ctx_bytes=0, B=1, H=1, N=256, d=64,
             L=16, P=4, tau=0.5, causal=1, dtype=1, ws=16, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.race_attn_forward(a["q"], a["k"], a["v"], a["W"], a["out"], a["den"], a["ctx"],
                                 a["ctx_bytes"], a["B"], a["H"], a["N"], a["d"], a["L"], a["P"],
                                 ctypes.c_float(a["tau"]), a["causal"], a["dtype"], a["ws"],
                                 a["ws_bytes"], a["stream"])


def _bwd(lib, **kw):
    a = dict(q=16, k=16, v=16, W=16, out=16, den=16, dout=16, ctx=None, ctx_bytes=0, dq=16, dk=16,
             dv=16, B=1, H=1, N=256, d=64, L=16, P=4, tau=0.5, causal=1, dtype=1, ws=16,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.race_attn_backward(a["q"], a["k"], a["v"], a["W"], a["out"], a["den"], a["dout"],
                                  a["ctx"], a["ctx_bytes"], a["dq"], a["dk"], a["dv"], a["B"],
                                  a["H"], a["N"], a["d"], a["L"], a["P"], ctypes.c_float(a["tau"]),
                                  a["causal"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


def test_forward_rejects_bad_arguments_without_launching(lib):
    import linear_attention_soft_b200 as ra
    assert _fwd(lib, q=None) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, out=None) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, ws=None) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, k=24) == ra.RACE_ERR_INVALID_ARG            # not 16-byte aligned
    assert _fwd(lib, tau=-1.0) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, tau=float("nan")) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, tau=float("inf")) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, dtype=7) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, N=-1) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, d=12) == ra.RACE_ERR_UNSUPPORTED
    assert _fwd(lib, d=136) == ra.RACE_ERR_UNSUPPORTED
    assert _fwd(lib, P=0) == ra.RACE_ERR_INVALID_ARG
    assert _fwd(lib, P=6) == ra.RACE_ERR_UNSUPPORTED
    assert _fwd(lib, ws_bytes=1024) == ra.RACE_ERR_WORKSPACE
    assert _fwd(lib, ctx=16, ctx_bytes=1024) == ra.RACE_ERR_WORKSPACE
    assert _fwd(lib, N=0, q=None) == ra.RACE_OK                  # empty input: nothing to do


def test_backward_rejects_bad_arguments_without_launching(lib):
    import linear_attention_soft_b200 as ra
    assert _bwd(lib, tau=0.0) == ra.RACE_ERR_UNSUPPORTED        # hard hash has no gradient
    assert _bwd(lib, den=None) == ra.RACE_ERR_INVALID_ARG
    assert _bwd(lib, dv=None) == ra.RACE_ERR_INVALID_ARG
    assert _bwd(lib, dq=8) == ra.RACE_ERR_INVALID_ARG
    assert _bwd(lib, L=128, P=4) == ra.RACE_ERR_UNSUPPORTED     # L*R = 2048 > 1024
    need = ra.race_attn_workspace_size(1, 1, 256, 64, 16, 4, 1, 1, ra.RACE_BF16)
    assert _bwd(lib, ws_bytes=need - 1) == ra.RACE_ERR_WORKSPACE
    assert _bwd(lib, N=0) == ra.RACE_OK


def test_hash_indices_rejects_bad_arguments(lib):
    import linear_attention_soft_b200 as ra
    f = lib.race_attn_hash_indices
    assert f(None, 16, 16, 1, 1, 8, 64, 4, 3, 1, None) == ra.RACE_ERR_INVALID_ARG
    assert f(16, 16, 16, 1, 1, 8, 66, 4, 3, 1, None) == ra.RACE_ERR_UNSUPPORTED
    assert f(16, 16, 16, 1, 1, 0, 64, 4, 3, 1, None) == ra.RACE_OK


def test_product_path_has_no_cpu_fallback():
    """The binding refuses to run without the CUDA library and never imports the oracle."""
    src = open(os.path.join(ROOT, "linear_attention_soft_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("oracle.", "")
    for f in os.listdir(os.path.join(ROOT, "linear_attention_soft_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "linear_attention_soft_b200", "csrc", f)).read().lower()


def test_decode_entry_points_reject_bad_arguments_without_launching(lib):
    import linear_attention_soft_b200 as ra
    sz = ctypes.c_size_t()
    assert lib.race_attn_decode_workspace_size(1, 1, 64, 16, 4, ctypes.byref(sz)) == ra.RACE_OK
    # one share of d+1 fp32 per CTA of each head; at most one CTA per 32 state rows
    assert sz.value % (65 * 4) == 0 and 0 < sz.value // (65 * 4) <= 256 // 32
    assert lib.race_attn_decode_workspace_size(1, 1, 66, 16, 4, ctypes.byref(sz)) == ra.RACE_ERR_UNSUPPORTED
    assert lib.race_attn_decode_workspace_size(1, 1, 64, 16, 6, ctypes.byref(sz)) == ra.RACE_ERR_UNSUPPORTED
    f = lib.race_attn_decode_step
    args = [16, 16, 16, 16, 16, 16, None, 1, 1, 64, 16, 4, ctypes.c_float(0.5), ra.RACE_BF16, 16, 1 << 20, None]
    bad = list(args)
    bad[0] = None                       # q
    assert f(*bad) == ra.RACE_ERR_INVALID_ARG
    bad = list(args)
    bad[4] = 8                          # state not 16-byte aligned
    assert f(*bad) == ra.RACE_ERR_INVALID_ARG
    bad = list(args)
    bad[12] = ctypes.c_float(-0.5)      # tau
    assert f(*bad) == ra.RACE_ERR_INVALID_ARG
    bad = list(args)
    bad[15] = 16                        # workspace too small
    assert f(*bad) == ra.RACE_ERR_WORKSPACE
    g = lib.race_attn_state
    assert g(16, 16, 16, None, 1, 1, 128, 64, 16, 4, ctypes.c_float(0.5), ra.RACE_BF16, 16, 1 << 30, None) == \
        ra.RACE_ERR_INVALID_ARG         # state
    assert g(16, 16, 16, 16, 1, 1, 128, 64, 16, 4, ctypes.c_float(0.5), 7, 16, 1 << 30, None) == \
        ra.RACE_ERR_INVALID_ARG         # dtype
    assert g(16, 16, 16, 16, 1, 1, 128, 64, 16, 4, ctypes.c_float(0.5), ra.RACE_BF16, 16, 16, None) == \
        ra.RACE_ERR_WORKSPACE


def test_shard_entry_points_reject_bad_arguments_without_launching(lib):
    import linear_attention_soft_b200 as ra
    f = lib.race_attn_shard_combine
    assert f(None, 2, 0, 0, 8, 16, None) == ra.RACE_ERR_INVALID_ARG
    assert f(16, 2, 2, 0, 8, 16, None) == ra.RACE_ERR_INVALID_ARG      # shard out of range
    assert f(16, 2, 0, 3, 8, 16, None) == ra.RACE_ERR_INVALID_ARG      # which
    assert f(16, 2, 0, 0, 0, 16, None) == ra.RACE_OK                   # nothing to sum
    fb = lib.race_attn_forward_begin
    args = [16, 16, 16, None, 0, None, 1, 1, 256, 64, 16, 4, ctypes.c_float(0.5), 1, ra.RACE_BF16, 16, 1 << 30,
            None]
    assert fb(*args) == ra.RACE_ERR_INVALID_ARG                        # h_total is required
    args[5] = 8
    assert fb(*args) == ra.RACE_ERR_INVALID_ARG                        # misaligned
    bb = lib.race_attn_backward_begin
    bargs = [16] * 8 + [0, None, 16, None, 1, 1, 256, 64, 16, 4, ctypes.c_float(0.5), 1, ra.RACE_BF16, 16,
                        1 << 30, None]
    assert bb(*bargs) == ra.RACE_ERR_INVALID_ARG                       # g_total is required


def test_dw_entry_points_reject_bad_arguments_without_launching(lib):
    import linear_attention_soft_b200 as ra
    bw = ra.race_attn_workspace_size(1, 1, 4096, 64, 16, 4, 1, 1, ra.RACE_BF16)
    dw = ra.race_attn_dw_workspace_size(1, 1, 4096, 64, 16, 4, 1, ra.RACE_BF16)
    # the backward's workspace, then dLoss/dp of the q and k rows (fp32 [rows][L*P] each)
    assert dw >= bw + 2 * 4096 * 64 * 4
    f = lib.race_attn_backward_dw
    args = [16] * 7 + [None, 0, 16, 16, 16, None, 1, 1, 4096, 64, 16, 4, ctypes.c_float(0.5), 1, ra.RACE_BF16, 16,
                       dw, None]
    assert f(*args) == ra.RACE_ERR_INVALID_ARG                    # dW missing
    args[12] = 16
    args[19] = ctypes.c_float(0.0)
    assert f(*args) == ra.RACE_ERR_UNSUPPORTED                    # hard hashing has no gradient
    args[19] = ctypes.c_float(0.5)
    args[23] = dw - 1
    assert f(*args) == ra.RACE_ERR_WORKSPACE


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C99 program that includes only the header compiles with gcc -Werror, links against
    the library and gets the documented statuses back (argument checks launch nothing)."""
    import shutil
    import subprocess
    import linear_attention_soft_b200 as ra
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(ra.library_path())
    exe = str(tmp_path / "abi_from_c")
    src = os.path.join(os.path.dirname(__file__), "c", "abi_from_c.c")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, src, "-o", exe, "-L", libdir,
                    "-l:" + os.path.basename(ra.library_path()), "-Wl,-rpath," + libdir], check=True)
    p = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert p.returncode == 0, p.stderr
    assert "abi_from_c ok" in p.stdout



def test_noalloc_buffer_size_matches_the_header():
    """The binding's copy of RACE_NOALLOC_SCRATCH_BYTES equals the header's definition (the
    refusal of larger sizes is tested where a GPU runs the entry point)."""
    import linear_attention_soft_b200 as ra
    src = open(os.path.join(ROOT, "include", "race_attn.h")).read()
    m = re.search(r"#define\s+RACE_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", src)
    assert m, "RACE_NOALLOC_SCRATCH_BYTES not found in the header"
    assert ra.RACE_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
