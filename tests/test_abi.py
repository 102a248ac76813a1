"""The C ABI library loads and exports every symbol include/e4b.h declares.

CPU only: no call here launches GPU work.  Argument checks that fail before
any device query are exercised directly.
"""
import ctypes
import os
import re
import subprocess

import pytest

from quantized_moe_expert_nf4_b200 import e4b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "e4b.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(e4b_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(e4b.LIB_PATH):
        from quantized_moe_expert_nf4_b200 import build
        build.build()
    return e4b.load_library()


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("e4b_nf4_quantize_stack", "e4b_moe_route_permute", "e4b_grouped_nf4_gemm",
              "e4b_moe_expert_forward"):
        assert n in names
    assert sorted(e4b.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", e4b.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (e4b_[a-z0-9_]+)", out))
    assert exported == set(_declared_functions())


def test_status_strings_and_version(lib):
    assert lib.e4b_version() == e4b.ABI_VERSION == 3
    assert lib.e4b_status_string(0) == b"E4B_OK"
    assert lib.e4b_status_string(3) == b"E4B_ERR_WORKSPACE"


def test_host_side_rejections_without_gpu(lib):
    # blocksize is checked before any device query
    st = lib.e4b_nf4_quantize_stack(None, 0, 2, 64, 64, 32, None, None, None)
    assert st == 2 and b"blocksize" in lib.e4b_last_error()
    st = lib.e4b_nf4_quantize_stack(None, 0, 2, 3, 5, 64, None, None, None)
    assert st == 2 and b"multiple of 64" in lib.e4b_last_error()
    st = lib.e4b_moe_route_permute(None, 4, 8, 9, 1, None, None, None, None, None, None, 0, None)
    assert st == 1 and b"k must be" in lib.e4b_last_error()
    st = lib.e4b_grouped_nf4_gemm(None, 1, 64, None, None, 2, 1, None, None, 64, 96, None, None, 0, 0.0, 0,
                                  None, 0, None, 0, None)
    assert st == 2 and b"K must be" in lib.e4b_last_error()


def test_workspace_queries_are_host_only(lib):
    assert e4b.e4b_moe_route_permute_workspace_size(1, 64, 8) == 0
    assert e4b.e4b_moe_route_permute_workspace_size(4096, 128, 8) > 4096 * 8 * 4
    # error word, LoRA products (256-byte aligned), gathered rows
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(100, 128, 64, 0) == 256 + 100 * 64 * 2
    xa = (100 * 128 + 255) // 256 * 256   # LoRA products: 128 bytes per row
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(100, 128, 64, 8) == 256 + xa + 100 * 64 * 2
    st = e4b.ExpertStackC(1, 1, 1, 1, None, None, 0, 0.0, 64, 2048, 1024)
    n = lib.e4b_moe_expert_forward_workspace_size(2048, ctypes.byref(st), 8)
    assert n >= 2048 * 8 * (1024 * 2 + 2048 * 4)


def test_gemm_workspace_too_small_is_rejected_on_the_host(lib):
    """The workspace check runs before any device query: a call with one byte
    too few returns E4B_ERR_WORKSPACE and names the size it needs."""
    rows, N, K = 300, 128, 256
    need = e4b.e4b_grouped_nf4_gemm_workspace_size(rows, N, K, 0)
    assert need == 256 + rows * K * 2          # error word + the gathered routed rows
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: rejected before launch
    offs = ctypes.c_void_p(1 << 21)
    st = lib.e4b_grouped_nf4_gemm(fake, rows, K, None, offs, 2, rows, fake, fake, N, K, None, None, 0, 0.0, 0,
                                  fake, 0, fake, need - 1, None)
    assert st == 3 and str(need).encode() in lib.e4b_last_error()


def test_forward_workspace_covers_both_paths(lib):
    """The forward workspace is the larger of the grouped and decode layouts,
    and grows with M."""
    st = e4b.ExpertStackC(1, 1, 1, 1, None, None, 0, 0.0, 64, 2048, 1024)
    sizes = [lib.e4b_moe_expert_forward_workspace_size(M, ctypes.byref(st), 8) for M in (1, 8, 9, 64, 2048)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    # grouped layout at M=9: per slot at least h (2I) + gathered x (2H) + Z (2H) bytes
    assert sizes[2] >= 9 * 8 * (1024 * 2 + 2048 * 2 + 2048 * 2)
    assert lib.e4b_moe_expert_forward_workspace_size(0, ctypes.byref(st), 8) == 0


def test_misaligned_lora_adapter_is_rejected_on_the_host(lib):
    """Kernels read lora_A with 16-byte loads: a misaligned adapter is an
    argument error, never a launch."""
    rows, N, K, r = 64, 128, 128, 8
    need = e4b.e4b_grouped_nf4_gemm_workspace_size(rows, N, K, r)
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    st = lib.e4b_grouped_nf4_gemm(p, rows, K, None, p, 2, rows, p, p, N, K, bad, p, r, 2.0, 0,
                                  p, 0, p, need, None)
    assert st == 1 and b"lora_A and lora_B" in lib.e4b_last_error()
    stk = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, (1 << 20) + 2, 1 << 20, 8, 16.0, 8, 256, 128)
    st = lib.e4b_moe_expert_forward(p, 4, p, 2, 1, ctypes.byref(stk), p, p, 1 << 30, None)
    assert st == 1 and b"lora_A and lora_B" in lib.e4b_last_error()


def test_misaligned_workspace_is_rejected_on_the_host(lib):
    """Workspaces feed bulk and tensor-map copies (16-byte rule): an unaligned
    one is an argument error for every call that takes one, never a launch."""
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    rows, N, K = 64, 128, 128
    need = e4b.e4b_grouped_nf4_gemm_workspace_size(rows, N, K, 0)
    st = lib.e4b_grouped_nf4_gemm(p, rows, K, None, p, 2, rows, p, p, N, K, None, None, 0, 0.0, 0,
                                  p, 0, bad, need, None)
    assert st == 1 and b"gemm workspace must be 16-byte aligned" in lib.e4b_last_error()
    stk = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None, 0, 0.0, 8, 256, 128)
    need = lib.e4b_moe_expert_forward_workspace_size(4, ctypes.byref(stk), 2)
    st = lib.e4b_moe_expert_forward(p, 4, p, 2, 1, ctypes.byref(stk), p, bad, need, None)
    assert st == 1 and b"forward workspace must be 16-byte aligned" in lib.e4b_last_error()
    need = e4b.e4b_moe_route_permute_workspace_size(4096, 64, 8)
    st = lib.e4b_moe_route_permute(p, 4096, 64, 8, 1, p, p, p, p, p, bad, need, None)
    assert st == 1 and b"route workspace must be 16-byte aligned" in lib.e4b_last_error()


def test_error_word_calls_check_their_arguments_on_the_host(lib):
    code = ctypes.c_int32(7)
    assert lib.e4b_workspace_error(None, ctypes.byref(code)) == 1
    assert lib.e4b_workspace_error(ctypes.c_void_p((1 << 20) + 4), ctypes.byref(code)) == 1
    assert b"16-byte aligned" in lib.e4b_last_error()
    assert lib.e4b_workspace_clear_error(None, None) == 1
    assert code.value == 7   # untouched on a rejected call



def test_zero_row_gemm_needs_no_workspace(lib):
    """With no routed rows nothing launches or waits: the size query is 0 and a
    NULL workspace passes the host checks (on a host without a GPU the call then
    stops at the device check, not at the workspace)."""
    p = ctypes.c_void_p(1 << 20)
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(0, 128, 128, 8) == 0
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(1, 128, 128, 0) >= 256 + 128 * 2
    st = lib.e4b_grouped_nf4_gemm(p, 1, 128, None, p, 2, 0, p, p, 128, 128, None, None, 0, 0.0, 0, p, 0, None, 0,
                                  None)
    assert st != 3 and b"workspace" not in lib.e4b_last_error()


def test_noalloc_forward_rejections_on_the_host(lib):
    """The allocation-free forward checks its arguments with the regular
    forward's stack check, then its own token range, scratch limit, null and
    alignment rules, all before any device query."""
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    stk = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None, 0, 0.0, 8, 256, 128)
    fn = lib.e4b_moe_expert_forward_decode_noalloc
    assert fn(p, 1, p, 2, 1, None, p, None) == 1 and b"null expert stack" in lib.e4b_last_error()
    assert fn(p, 0, p, 2, 1, ctypes.byref(stk), p, None) == 2 and b"1 to 8 tokens" in lib.e4b_last_error()
    assert fn(p, 9, p, 2, 1, ctypes.byref(stk), p, None) == 2 and b"1 to 8 tokens" in lib.e4b_last_error()
    assert fn(p, 1, p, 9, 1, ctypes.byref(stk), p, None) == 1 and b"k must be" in lib.e4b_last_error()
    assert fn(None, 1, p, 2, 1, ctypes.byref(stk), p, None) == 1 and b"null x" in lib.e4b_last_error()
    assert fn(p, 1, p, 2, 1, ctypes.byref(stk), bad, None) == 1 and b"16-byte aligned" in lib.e4b_last_error()
    big = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None, 0, 0.0, 32, 128, 8192)
    assert fn(p, 2, p, 32, 1, ctypes.byref(big), p, None) == 2 and b"static scratch" in lib.e4b_last_error()
    lora = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, (1 << 20) + 2, 1 << 20, 8, 16.0, 8, 256, 128)
    assert fn(p, 1, p, 2, 1, ctypes.byref(lora), p, None) == 1 and b"lora_A and lora_B" in lib.e4b_last_error()
    rank = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 17, 16.0, 8, 256, 128)
    assert fn(p, 1, p, 2, 1, ctypes.byref(rank), p, None) == 2 and b"LoRA rank" in lib.e4b_last_error()


def test_dgrad_host_side_rejections(lib):
    """The grouped dgrad checks its arguments before any device query."""
    p = ctypes.c_void_p(1 << 20)
    rows, N, K = 64, 128, 192
    need = e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(rows, N, K, 0)
    # error word, then (with an adapter) dY . lora_B, then room for the dY rows gathered in group order
    assert need == 256 + rows * N * 2
    assert e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(rows, N, K, 8) == \
        256 + (rows * 8 * 4 + 255) // 256 * 256 + rows * N * 2

    def call(**kw):
        a = dict(dY=p, dy_rows=rows, lddy=N, ridx=None, offs=p, E=2, rows=rows, packed=p, absmax=p, N=N, K=K,
                 la=None, lb=None, r=0, scale=0.0, out=p, od=0, ws=p, wsb=need)
        a.update(kw)
        return lib.e4b_grouped_nf4_gemm_dgrad(a["dY"], a["dy_rows"], a["lddy"], a["ridx"], a["offs"], a["E"],
                                              a["rows"], a["packed"], a["absmax"], a["N"], a["K"], a["la"],
                                              a["lb"], a["r"], a["scale"], a["out"], a["od"], a["ws"], a["wsb"],
                                              None)
    assert call(K=96) == 2 and b"K must be" in lib.e4b_last_error()
    assert call(N=100) == 2 and b"N must be" in lib.e4b_last_error()
    assert call(lddy=N - 8) == 1 and b"lddy" in lib.e4b_last_error()
    assert call(lddy=N + 4) == 1 and b"lddy" in lib.e4b_last_error()
    assert call(la=p) == 1 and b"both set" in lib.e4b_last_error()
    assert call(la=p, lb=p, r=17) == 2 and b"rank" in lib.e4b_last_error()
    assert call(absmax=ctypes.c_void_p((1 << 20) + 4)) == 1 and b"16-byte aligned" in lib.e4b_last_error()
    assert call(wsb=need - 1) == 3 and str(need).encode() in lib.e4b_last_error()
    assert call(ws=ctypes.c_void_p((1 << 20) + 8)) == 1 and b"dgrad workspace must be" in lib.e4b_last_error()


def test_lora_grads_host_side_rejections(lib):
    p = ctypes.c_void_p(1 << 20)
    rows, N, K, r = 64, 128, 192, 8
    need = e4b.e4b_grouped_lora_grads_workspace_size(rows, r)
    assert need == 256 + 2 * ((rows * r * 4 + 255) // 256 * 256)
    assert e4b.e4b_grouped_lora_grads_workspace_size(rows, 0) == 0

    def call(**kw):
        a = dict(x=p, x_rows=rows, ldx=K, ridx=None, offs=p, E=2, rows=rows, da=p, ldda=N, N=N, K=K, la=p, lb=p,
                 r=r, scale=1.0, dA=p, dB=p, ws=p, wsb=need)
        a.update(kw)
        return lib.e4b_grouped_lora_grads(a["x"], a["x_rows"], a["ldx"], a["ridx"], a["offs"], a["E"], a["rows"],
                                          a["da"], a["ldda"], a["N"], a["K"], a["la"], a["lb"], a["r"], a["scale"],
                                          a["dA"], a["dB"], a["ws"], a["wsb"], None)
    assert call(r=0) == 2 and b"rank" in lib.e4b_last_error()
    assert call(K=100) == 2 and b"K must be" in lib.e4b_last_error()
    assert call(ldx=K + 4) == 1 and b"ldx" in lib.e4b_last_error()
    assert call(ldda=N - 1) == 1 and b"ldda" in lib.e4b_last_error()
    assert call(dB=None) == 1 and b"null" in lib.e4b_last_error()
    assert call(wsb=need - 1) == 3 and str(need).encode() in lib.e4b_last_error()


def test_backward_host_side_checks(lib):
    p = 1 << 20
    st = e4b.ExpertStackC(p, p, p, p, None, None, 0, 0.0, 8, 256, 128)
    sizes = [lib.e4b_moe_expert_backward_workspace_size(M, ctypes.byref(st), 2) for M in (1, 64, 300)]
    assert sizes[0] < sizes[1] < sizes[2]
    # per routed row at least a (fp32 2I), z and dxg (fp32 H each), dz (bf16 H), dh (fp32 I), da (bf16 2I)
    assert sizes[2] >= 600 * (8 * 128 + 4 * 256 * 2 + 2 * 256 + 4 * 128 + 4 * 128)
    assert lib.e4b_moe_expert_backward_workspace_size(0, ctypes.byref(st), 2) == 0
    vp = ctypes.c_void_p(p)
    need = sizes[1]
    status = lib.e4b_moe_expert_backward(vp, 64, vp, 2, 1, ctypes.byref(st), vp, vp, vp, None, None, vp, need - 1,
                                         None)
    assert status == 3 and str(need).encode() in lib.e4b_last_error()
    stl = e4b.ExpertStackC(p, p, p, p, p, p, 8, 16.0, 8, 256, 128)
    status = lib.e4b_moe_expert_backward(vp, 64, vp, 2, 1, ctypes.byref(stl), vp, vp, vp, None, None, vp, 1 << 40,
                                         None)
    assert status == 1 and b"needs dA and dB" in lib.e4b_last_error()


def test_mxfp4_host_side_rejections(lib):
    p = ctypes.c_void_p(1 << 20)

    def call(**kw):
        a = dict(A=p, a_rows=4, lda=128, ridx=None, offs=p, E=2, rows=4, blocks=p, scales=p, N=128, K=128, epi=0,
                 out=p, od=0, ws=p, wsb=1 << 30)
        a.update(kw)
        return lib.e4b_grouped_mxfp4_gemm(a["A"], a["a_rows"], a["lda"], a["ridx"], a["offs"], a["E"], a["rows"],
                                          a["blocks"], a["scales"], a["N"], a["K"], a["epi"], a["out"], a["od"],
                                          a["ws"], a["wsb"], None)
    need = lib.e4b_grouped_mxfp4_gemm_workspace_size(4, 128, 128)
    assert need == e4b.e4b_grouped_nf4_gemm_workspace_size(4, 128, 128, 0) >= 256 + 4 * 128 * 2
    assert call(wsb=need - 1) == 3 and str(need).encode() in lib.e4b_last_error()
    assert call(ws=ctypes.c_void_p((1 << 20) + 8), wsb=need) == 1 and b"16-byte aligned" in lib.e4b_last_error()
    assert call(K=96) == 2 and b"K must be" in lib.e4b_last_error()
    assert call(N=32) == 2 and b"N must be" in lib.e4b_last_error()
    assert call(lda=100) == 1 and b"lda" in lib.e4b_last_error()
    assert call(epi=7) == 1 and b"epilogue" in lib.e4b_last_error()
    assert call(scales=None) == 1 and b"null" in lib.e4b_last_error()
    assert call(blocks=ctypes.c_void_p((1 << 20) + 4)) == 1 and b"16-byte aligned" in lib.e4b_last_error()


def test_storage_type_is_checked_on_the_host(lib):
    """An e4b_quant_type other than NF4 and FP4 is an argument error from every
    call that takes one, before any device work; FP4 itself passes the host
    checks."""
    p = ctypes.c_void_p(1 << 20)
    assert lib.e4b_quantize_stack(p, 0, 1, 1, 64, 64, 2, p, p, None) == 1
    assert b"quant_type" in lib.e4b_last_error()
    assert lib.e4b_quantize_stack(p, 0, 1, 1, 64, 64, e4b.E4B_QUANT_FP4, p, p, None) != 1
    assert b"quant_type" not in lib.e4b_last_error()
    rows, N, K = 64, 128, 128
    need = e4b.e4b_grouped_nf4_gemm_workspace_size(rows, N, K, 0)
    st = lib.e4b_grouped_4bit_gemm(p, rows, K, None, p, 2, rows, p, p, 5, N, K, None, None, 0, 0.0, 0, p, 0, p, need,
                                   None)
    assert st == 1 and b"quant_type" in lib.e4b_last_error()
    st = lib.e4b_grouped_4bit_gemm_dgrad(p, rows, N, None, p, 2, rows, p, p, -1, N, K, None, None, 0, 0.0, p, 0, p,
                                         1 << 30, None)
    assert st == 1 and b"quant_type" in lib.e4b_last_error()
    stk = e4b.ExpertStackC(1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None, 0, 0.0, 8, 256, 128, 3)
    st = lib.e4b_moe_expert_forward(p, 4, p, 2, 1, ctypes.byref(stk), p, p, 1 << 30, None)
    assert st == 1 and b"quant_type" in lib.e4b_last_error()
    st = lib.e4b_moe_expert_forward_decode_noalloc(p, 4, p, 2, 1, ctypes.byref(stk), p, None)
    assert st == 1 and b"quant_type" in lib.e4b_last_error()


def test_expert_stack_layout_matches_the_header():
    """ctypes mirror of e4b_expert_stack: the storage type follows I."""
    names = [f[0] for f in e4b.ExpertStackC._fields_]
    assert names[-4:] == ["E", "H", "I", "quant_type"]
    assert e4b.ExpertStackC.quant_type.offset == e4b.ExpertStackC.I.offset + 8
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "e4b.h")).read()
    body = hdr[hdr.index("typedef struct {\n  const uint8_t* gu_packed"):hdr.index("} e4b_expert_stack;")]
    assert body.index("int64_t E, H, I;") < body.index("int32_t quant_type;")


def test_zero_row_gemm_needs_no_workspace(lib):
    """With no routed rows nothing launches or waits: the size query is 0 and a
    NULL workspace passes the host checks (on a host without a GPU the call then
    stops at the device check, not at the workspace)."""
    p = ctypes.c_void_p(1 << 20)
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(0, 128, 128, 8) == 0
    assert e4b.e4b_grouped_nf4_gemm_workspace_size(1, 128, 128, 0) >= 256 + 128 * 2
    st = lib.e4b_grouped_nf4_gemm(p, 1, 128, None, p, 2, 0, p, p, 128, 128, None, None, 0, 0.0, 0, p, 0, None, 0,
                                  None)
    assert st != 3 and b"workspace" not in lib.e4b_last_error()


def test_zero_row_dgrad_needs_no_workspace(lib):
    p = ctypes.c_void_p(1 << 20)
    assert e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(0, 128, 128, 8) == 0
    st = lib.e4b_grouped_nf4_gemm_dgrad(p, 1, 128, None, p, 2, 0, p, p, 128, 128, None, None, 0, 0.0, p, 0, None, 0,
                                        None)
    assert st != 3 and b"workspace" not in lib.e4b_last_error()


def test_zero_row_mxfp4_gemm_needs_no_workspace(lib):
    p = ctypes.c_void_p(1 << 20)
    assert lib.e4b_grouped_mxfp4_gemm_workspace_size(0, 128, 128) == 0
    st = lib.e4b_grouped_mxfp4_gemm(p, 1, 128, None, p, 2, 0, p, p, 128, 128, 0, p, 0, None, 0, None)
    assert st != 3 and b"workspace" not in lib.e4b_last_error()


def test_graft_entry_build_checks_the_abi_version():
    """build() compiles (or reuses) the library, loads it and checks its ABI
    version against the binding's."""
    import __graft_entry__ as ge
    ge.build()
