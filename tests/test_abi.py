"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, exports
every function include/fp2.h declares, its structs have the header's layout,
and host-side argument validation returns the documented status codes before
any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from block_sparse_long_blockmean_b200 import build as B
from block_sparse_long_blockmean_b200 import fp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp2.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return fp2.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp2_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["fp2_prefill", "fp2_blockmean", "fp2_score", "fp2_mask", "fp2_attn",
              "fp2_workspace_size", "fp2_get_status"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fp2.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fp2_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)
    assert set(fp2.SIGNATURES) == set(declared_functions())


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++11")])
def test_header_is_strict_c99_and_cxx11(tmp_path, compiler, std):
    """The boundary is plain C: the header compiles alone, warning-free, as
    pedantic C99 and as C++11 (extern "C")."""
    src = tmp_path / "hdr.c"
    src.write_text('#include "fp2.h"\nint main(void) { return (int)sizeof(fp2_params) == 0; }\n')
    cmd = [compiler, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
           os.path.join(ROOT, "include")]
    if compiler == "g++":
        cmd += ["-x", "c++"]
    subprocess.run(cmd + [str(src), "-o", str(tmp_path / "hdr")], check=True)


def test_struct_layout_matches_header(tmp_path):
    fields = [f for f, _ in fp2.Params._fields_]
    lfields = [f for f, _ in fp2.WorkspaceLayout._fields_]
    hfields = [f for f, _ in fp2.HostIO._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "fp2.h"', "int main(void){",
            'printf("%zu\\n", sizeof(fp2_params));']
    prog += [f'printf("%zu\\n", offsetof(fp2_params, {f}));' for f in fields]
    prog += ['printf("%zu\\n", sizeof(fp2_workspace_layout));']
    prog += [f'printf("%zu\\n", offsetof(fp2_workspace_layout, {f}));' for f in lfields]
    prog += ['printf("%zu\\n", sizeof(fp2_host_io));']
    prog += [f'printf("%zu\\n", offsetof(fp2_host_io, {f}));' for f in hfields]
    prog += ["return 0;}"]
    c = tmp_path / "probe.c"
    c.write_text("\n".join(prog))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)],
                   check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    want = [ctypes.sizeof(fp2.Params)] + [getattr(fp2.Params, f).offset for f in fields]
    want += [ctypes.sizeof(fp2.WorkspaceLayout)]
    want += [getattr(fp2.WorkspaceLayout, f).offset for f in lfields]
    want += [ctypes.sizeof(fp2.HostIO)]
    want += [getattr(fp2.HostIO, f).offset for f in hfields]
    assert vals == want


def base_params(**kw):
    P = fp2.Params()
    P.num_seqs = 1
    P.num_q_heads, P.num_kv_heads, P.head_dim = 32, 8, 128
    P.total_q = P.total_k = 131072
    P.max_seqlen_q = P.max_seqlen_k = 131072
    for k, v in kw.items():
        setattr(P, k, v)
    return P


def test_workspace_layout_for_the_128k_layer(lib):
    P = base_params()
    L = fp2.get_workspace_layout(P, 128)
    assert (L.nqb_max, L.nkb_max, L.nw) == (1024, 1024, 32)
    offs = [L.error_word, L.kbar, L.vbar, L.kbar_op, L.vbar_op, L.scores, L.kept_idx,
            L.kept_cnt, L.kept_bits]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert L.scores - L.vbar_op >= 8 * 1024 * 128 * 2
    assert L.kept_idx - L.scores >= 32 * 1024 * 1024 * 4
    assert L.total - L.kept_bits >= 32 * 1024 * 32 * 4
    assert fp2.workspace_size(P, 128) == L.total


@pytest.mark.parametrize("S,Hq,Hkv,d,max_q,max_k,B", [
    (1, 4, 1, 64, 1024, 1024, 64),           # tiny causal layer
    (3, 32, 8, 128, 1000, 5000, 128),        # chunks on prefixes: one extra query block
    (2, 8, 8, 128, 1, 300, 128),             # decode rows only (MHA: G = 1 needs block 128)
    (5, 16, 2, 64, 37, 37, 64),              # ragged, one partial block
    (1, 64, 8, 128, 32768, 262144, 128),     # 32K chunk on a 256K context
    (4, 8, 1, 128, 300, 300, 128),           # more query blocks would exceed the key blocks
])
def test_workspace_regions_follow_the_header(lib, S, Hq, Hkv, d, max_q, max_k, B):
    """Every region of the workspace layout has at least the size the header
    states for it, starts 256-byte aligned, and follows the previous one; the
    padded block counts follow the header's formulas."""
    P = base_params(num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d,
                    total_q=S * max_q, total_k=S * max_k, max_seqlen_q=max_q,
                    max_seqlen_k=max_k)
    L = fp2.get_workspace_layout(P, B)
    nkb = -(-max_k // B)
    nqb = min((max_q + 2 * B - 2) // B, nkb)
    nw = -(-nkb // 32)
    assert (L.nqb_max, L.nkb_max, L.nw) == (nqb, nkb, nw)
    regions = [(L.error_word, 16),
               (L.kbar, 4 * S * Hkv * nkb * d), (L.vbar, 4 * S * Hkv * nkb * d),
               (L.kbar_op, 2 * S * Hkv * nkb * d), (L.vbar_op, 2 * S * Hkv * nkb * d),
               (L.scores, 4 * S * Hq * nqb * nkb), (L.kept_idx, 4 * S * Hq * nqb * nkb),
               (L.kept_cnt, 4 * S * Hq * nqb), (L.kept_bits, 4 * S * Hq * nqb * nw)]
    for (o, size), (o_next, _) in zip(regions, regions[1:] + [(L.total, 0)]):
        assert o % 256 == 0
        assert o_next - o >= size
    assert fp2.workspace_size(P, B) == L.total


@pytest.mark.parametrize("field,value,block,code", [
    ("num_kv_heads", 3, 128, fp2.FP2_ERR_INVALID_ARG),    # 32 % 3 != 0
    ("num_kv_heads", 2, 128, fp2.FP2_ERR_UNSUPPORTED),    # G = 16
    ("head_dim", 96, 128, fp2.FP2_ERR_UNSUPPORTED),
    ("max_seqlen_k", 10, 128, fp2.FP2_ERR_INVALID_ARG),   # < max_seqlen_q
    ("num_seqs", 0, 128, fp2.FP2_ERR_INVALID_ARG),
    (None, None, 96, fp2.FP2_ERR_UNSUPPORTED),            # block 96
])
def test_host_validation_codes(lib, field, value, block, code):
    P = base_params()
    if field:
        setattr(P, field, value)
    L = fp2.WorkspaceLayout()
    assert lib.fp2_get_workspace_layout(ctypes.byref(P), block, ctypes.byref(L)) == code
    assert lib.fp2_workspace_size(ctypes.byref(P), block) == 0


def test_calls_reject_bad_arguments_before_any_cuda_work(lib):
    P = base_params()
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    # no workspace
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_WORKSPACE
    P.workspace = 4096 * 256
    P.workspace_bytes = 16
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_WORKSPACE
    P.workspace_bytes = fp2.workspace_size(P, 128)
    P.workspace = 4096 * 256 + 8  # misaligned
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_WORKSPACE
    P.workspace = 4096 * 256
    # null cu_seqlens, null q, misaligned q, NaN tau, fp8 without scales, fp8 d=64
    assert lib.fp2_prefill(fake, fake, fake, None, None, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_prefill(None, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_prefill(fake + 2, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_prefill(fake, fake, fake, None, fake, float("nan"), 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 1, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 7, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    # paged: page size not a power of two / not dividing the block
    P.page_size, P.max_pages_per_seq, P.num_pages = 48, 4, 4
    assert lib.fp2_prefill(fake, fake, fake, fake, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_UNSUPPORTED
    P.page_size = 512
    assert lib.fp2_prefill(fake, fake, fake, fake, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_UNSUPPORTED
    P.page_size, P.max_pages_per_seq = 64, 0
    assert lib.fp2_prefill(fake, fake, fake, fake, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    assert lib.fp2_mask(fake, float("nan"), 128, ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    # e4m3 output from bf16 inputs needs an explicit out_scale; unknown out dtype
    P.page_size, P.max_pages_per_seq = 64, 4
    P.out_dtype = fp2.FP2_FP8_E4M3
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    P.out_dtype = 5
    assert lib.fp2_prefill(fake, fake, fake, None, fake, 1.0, 128, 0, fake,
                           ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG


def test_status_strings_and_version(lib):
    for code in range(7):
        assert fp2.status_string(code) not in ("", "unknown status")
    assert fp2.status_string(99) == "unknown status"
    assert re.fullmatch(r"\d+\.\d+\.\d+", fp2.version())


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(fp2, "_LIB", None)
    monkeypatch.setattr(fp2, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        fp2.lib()


def test_host_pipeline_rejects_bad_arguments_before_any_cuda_work(lib):
    P = base_params()
    fake = 1 << 20  # never dereferenced
    assert lib.fp2_prefill_host(None, None, fake, 1.0, 128, 0, ctypes.byref(P)) == \
        fp2.FP2_ERR_INVALID_ARG
    io = fp2.HostIO()
    for f, _ in fp2.HostIO._fields_:
        if f not in ("seqlens_k_host", "upload_stream", "download_stream", "num_chunks"):
            setattr(io, f, fake)
    for chunks in (0, 65, -1):
        io.num_chunks = chunks
        assert lib.fp2_prefill_host(ctypes.byref(io), None, fake, 1.0, 128, 0,
                                    ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    io.num_chunks = 4
    io.out_host = None
    assert lib.fp2_prefill_host(ctypes.byref(io), None, fake, 1.0, 128, 0,
                                ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    io.out_host = fake
    P.seqlens_k = fake  # device lengths given but no host copy of them
    assert lib.fp2_prefill_host(ctypes.byref(io), None, fake, 1.0, 128, 0,
                                ctypes.byref(P)) == fp2.FP2_ERR_INVALID_ARG
    P.seqlens_k = None
    # no workspace: the same validation as fp2_prefill
    assert lib.fp2_prefill_host(ctypes.byref(io), None, fake, 1.0, 128, 0,
                                ctypes.byref(P)) == fp2.FP2_ERR_WORKSPACE
