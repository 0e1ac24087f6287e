"""Host-side checks of the C ABI (no GPU needed).

The library builds with nvcc here, loads without a GPU, exports every entry
point the header declares, and rejects bad arguments before touching CUDA.
"""
import ctypes
import os
import re

import pytest
import torch

from tiled_attention_blackwell_b200 import attn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return attn.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]*?\b(attn_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert "attn_fwd" in names and "attn_get_device_status" in names
    assert set(attn.EXPORTED) <= set(names)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {attn.library_path()}").read()
    exported = set(re.findall(r"\b(attn_\w+)\b", out))
    assert set(declared_functions()) == exported


def test_status_strings_and_version(L):
    assert L.attn_abi_version() == 2
    for code in range(8):
        s = L.attn_status_string(code).decode()
        assert s and s != "unknown status"
    assert L.attn_status_string(99).decode() == "unknown status"


def test_default_options(L):
    o = attn.default_options()
    assert o.rescale_threshold == 8.0 and o.exp2_mode == 1 and list(o.reserved) == [0] * 4
    assert o.wait_timeout_us == 0 and o.debug_withhold_kv == 0


# Fake, 16-byte-aligned device addresses: validation must reject the call
# before any CUDA call, so nothing ever dereferences them.
P = 0x10000


def call(L, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=2, Sq=16, Sk=16, D=128, scale=0.1,
             causal=0, wl=-1, wr=-1, docs=None, nd=0, opts=None)
    a.update(kw)
    args = [ctypes.c_void_p(a["q"]), ctypes.c_void_p(a["k"]), ctypes.c_void_p(a["v"]),
            ctypes.c_void_p(a["o"]), ctypes.c_void_p(a["lse"]), a["B"], a["Hq"], a["Hkv"],
            a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"], a["wl"], a["wr"],
            ctypes.c_void_p(a["docs"]) if a["docs"] else None, a["nd"]]
    if a["opts"] is None:
        return L.attn_fwd(*args, None)
    return L.attn_fwd_ex(*args, ctypes.byref(a["opts"]), None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(lse=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(B=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Sq=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Sk=-3), attn.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), attn.ATTN_ERR_INVALID_ARG),
    (dict(D=96), attn.ATTN_ERR_UNSUPPORTED),
    (dict(D=256), attn.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=-1.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), attn.ATTN_ERR_INVALID_ARG),
    (dict(wl=-2), attn.ATTN_ERR_INVALID_ARG),
    (dict(wr=-5), attn.ATTN_ERR_INVALID_ARG),
    (dict(docs=P, nd=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(docs=None, nd=3), attn.ATTN_ERR_INVALID_ARG),
    (dict(docs=P, nd=2, Sk=32), attn.ATTN_ERR_INVALID_ARG),
    (dict(q=P + 8), attn.ATTN_ERR_MISALIGNED),
    (dict(v=P + 2), attn.ATTN_ERR_MISALIGNED),
    (dict(o=P + 4), attn.ATTN_ERR_MISALIGNED),
    (dict(lse=P + 2), attn.ATTN_ERR_MISALIGNED),
])
def test_invalid_arguments_rejected_before_launch(L, kw, status):
    assert call(L, **kw) == status
    assert L.attn_last_error_detail().decode() != ""


@pytest.mark.parametrize("field,value", [("rescale_threshold", -1.0),
                                         ("rescale_threshold", 17.0),
                                         ("rescale_threshold", float("nan")),
                                         ("exp2_mode", 3), ("exp2_mode", -1),
                                         ("wait_timeout_us", -1),
                                         ("wait_timeout_us", 60000001),
                                         ("debug_withhold_kv", 2)])
def test_invalid_options_rejected(L, field, value):
    opts = attn.default_options()
    setattr(opts, field, value)
    assert call(L, opts=opts) == attn.ATTN_ERR_INVALID_ARG


def test_reserved_options_must_be_zero(L):
    opts = attn.default_options()
    opts.reserved[2] = 1
    assert call(L, opts=opts) == attn.ATTN_ERR_INVALID_ARG
    opts = attn.default_options()
    opts.reserved0 = 1
    assert call(L, opts=opts) == attn.ATTN_ERR_INVALID_ARG


def test_default_options_select_no_modifier(L):
    o = attn.default_options()
    assert o.softcap == 0.0 and o.alibi_slopes is None and o.reserved0 == 0


@pytest.mark.parametrize("field,value,status", [
    ("softcap", -1.0, attn.ATTN_ERR_INVALID_ARG),
    ("softcap", float("nan"), attn.ATTN_ERR_INVALID_ARG),
    ("softcap", float("inf"), attn.ATTN_ERR_INVALID_ARG),
    ("alibi_slopes", P + 2, attn.ATTN_ERR_MISALIGNED),
])
def test_invalid_modifiers_rejected(L, field, value, status):
    opts = attn.default_options()
    setattr(opts, field, value)
    assert call(L, opts=opts) == status
    bopts = attn.BwdOptions()
    setattr(bopts, field, value)
    assert call_bwd(L, opts=bopts) == status


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_call_without_gpu_reports_cuda_error(L):
    assert call(L) == attn.ATTN_ERR_CUDA


def call_bwd(L, **kw):
    a = dict(ptr=P, lse=P, ws=P, B=1, Hq=2, Hkv=2, Sq=16, Sk=16, D=128, scale=0.1, causal=1,
             wl=-1, wr=-1, docs=None, nd=0, wsb=1 << 20, opts=None)
    a.update(kw)
    vp = ctypes.c_void_p
    ptrs = [vp(a.get(n, a["ptr"])) for n in ("q", "k", "v", "o")]
    ptrs += [vp(a["lse"])]
    ptrs += [vp(a.get(n, a["ptr"])) for n in ("dout", "dq", "dk", "dv")]
    args = ptrs + [a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"],
                   a["wl"], a["wr"], vp(a["docs"]) if a["docs"] else None, a["nd"], vp(a["ws"]),
                   a["wsb"]]
    if a["opts"] is None:
        return L.attn_bwd(*args, None)
    return L.attn_bwd_ex(*args, ctypes.byref(a["opts"]), None)


def test_bwd_workspace_size(L):
    assert L.attn_bwd_workspace_size(2, 16, 16, 4096, 4096, 128) >= 2 * 16 * 4096 * 4
    assert L.attn_bwd_workspace_size(2, 16, 16, 4096, 4096, 128) % 256 == 0
    assert L.attn_bwd_workspace_size(0, 16, 16, 4096, 4096, 128) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(dq=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(ws=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(D=80), attn.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(wsb=64), attn.ATTN_ERR_INVALID_ARG),
    (dict(dk=P + 8), attn.ATTN_ERR_MISALIGNED),
    (dict(ws=P + 4), attn.ATTN_ERR_MISALIGNED),
    (dict(docs=P, nd=1, Sk=20), attn.ATTN_ERR_INVALID_ARG),
])
def test_bwd_invalid_arguments_rejected_before_launch(L, kw, status):
    assert call_bwd(L, **kw) == status
    assert call_bwd(L, opts=attn.BwdOptions(), **kw) == status


def call_noalloc(L, **kw):
    a = dict(ptr=P, lse=P, B=1, Hq=2, Hkv=2, Sq=16, Sk=16, D=128, scale=0.1, causal=1,
             wl=-1, wr=-1, docs=None, nd=0)
    a.update(kw)
    vp = ctypes.c_void_p
    ptrs = [vp(a.get(n, a["ptr"])) for n in ("q", "k", "v", "o")]
    ptrs += [vp(a["lse"])]
    ptrs += [vp(a.get(n, a["ptr"])) for n in ("dout", "dq", "dk", "dv")]
    return L.attn_bwd_noalloc(*ptrs, a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["D"],
                              a["scale"], a["causal"], a["wl"], a["wr"],
                              vp(a["docs"]) if a["docs"] else None, a["nd"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(dq=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(lse=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(B=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(D=80), attn.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(wl=-2), attn.ATTN_ERR_INVALID_ARG),
    (dict(dk=P + 8), attn.ATTN_ERR_MISALIGNED),
    (dict(lse=P + 2), attn.ATTN_ERR_MISALIGNED),
    (dict(docs=P, nd=1, Sk=20), attn.ATTN_ERR_INVALID_ARG),
    (dict(B=1, Hq=32, Hkv=32, Sq=32769, Sk=32769), attn.ATTN_ERR_UNSUPPORTED),
])
def test_noalloc_invalid_arguments_rejected_before_cuda(L, kw, status):
    """attn_bwd_noalloc checks its arguments like attn_bwd, before it looks up
    its scratch or touches CUDA: on a machine without a GPU a bad argument
    still reports the argument error, not a CUDA error."""
    assert call_noalloc(L, **kw) == status
    assert L.attn_last_error_detail().decode() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_noalloc_call_without_gpu_reports_cuda_error(L):
    assert call_noalloc(L) == attn.ATTN_ERR_CUDA


class _CudaStandIn(torch.Tensor):
    """A CPU tensor that reports itself as a CUDA tensor, so the binding's
    own checks can be exercised on a machine without a GPU (they must raise
    before anything is passed to the library)."""

    @property
    def is_cuda(self):
        return True


def _bwd_stand_ins(B=1, S=16, H=2, D=64):
    def mk(shape, dt):
        return torch.zeros(shape, dtype=dt).as_subclass(_CudaStandIn)
    q, k, v, o, dout = (mk((B, S, H, D), torch.bfloat16) for _ in range(5))
    lse = mk((B, H, S), torch.float32)
    dq = mk((B, S, H, D), torch.float32)
    dk, dv = mk((B, S, H, D), torch.bfloat16), mk((B, S, H, D), torch.bfloat16)
    return dict(q=q, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("fn", ["attn_bwd_noalloc", "attn_bwd"])
def test_backward_bindings_check_tensors_and_doc_offsets(L, fn):
    """Both backward bindings refuse a bf16 dq (the kernel would write fp32
    rows past its end), a non-contiguous tensor, and doc_offsets that are
    not a CUDA int32 tensor (a host pointer or a list), before any call into
    the library."""
    call = getattr(attn, fn)
    extra = ([torch.zeros(1024, dtype=torch.uint8).as_subclass(_CudaStandIn)]
             if fn == "attn_bwd" else [])

    def run(t, **kw):
        names = ("q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv")
        call(*[t[n] for n in names], *extra, scale=0.1, causal=True, stream=0, **kw)

    t = _bwd_stand_ins()
    t["dq"] = torch.zeros(t["dq"].shape, dtype=torch.bfloat16).as_subclass(_CudaStandIn)
    with pytest.raises(TypeError, match="dq"):
        run(t)
    t = _bwd_stand_ins()
    t["dk"] = torch.zeros((1, 2, 16, 64), dtype=torch.bfloat16).transpose(1, 2) \
        .as_subclass(_CudaStandIn)
    with pytest.raises(TypeError, match="dk"):
        run(t)
    t = _bwd_stand_ins()
    t["dv"] = torch.zeros((1, 16, 2, 32), dtype=torch.bfloat16).as_subclass(_CudaStandIn)
    with pytest.raises(TypeError, match="dv"):
        run(t)
    t = _bwd_stand_ins()
    with pytest.raises(TypeError, match="doc_offsets"):
        run(t, doc_offsets=torch.tensor([0, 16], dtype=torch.int32))
    with pytest.raises(TypeError, match="doc_offsets"):
        run(t, doc_offsets=[0, 16])
    with pytest.raises(TypeError, match="doc_offsets"):
        run(t, doc_offsets=torch.tensor([0, 16]).as_subclass(_CudaStandIn))


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_bwd_calls_without_gpu_report_cuda_error(L):
    assert call_bwd(L) == attn.ATTN_ERR_CUDA
    assert call_bwd(L, opts=attn.BwdOptions(softcap=30.0, alibi_slopes=P)) == attn.ATTN_ERR_CUDA


def test_binding_refuses_cpu_tensors(L):
    q = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 4)
    with pytest.raises(TypeError):
        attn.attn_fwd(q, q, q, q, lse, scale=0.1)


def call_fp8(L, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, qd=0.01, kd=0.02, vd=0.03, B=1, Hq=2, Hkv=2, Sq=16,
             Sk=16, D=128, scale=0.1, causal=0, wl=-1, wr=-1, docs=None, nd=0, opts=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return L.attn_fwd_fp8(vp(a["q"]), vp(a["k"]), vp(a["v"]), a["qd"], a["kd"], a["vd"],
                          vp(a["o"]), vp(a["lse"]), a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Sk"],
                          a["D"], a["scale"], a["causal"], a["wl"], a["wr"],
                          vp(a["docs"]) if a["docs"] else None, a["nd"],
                          None if a["opts"] is None else ctypes.byref(a["opts"]), None)


@pytest.mark.parametrize("kw,status", [
    (dict(D=64), attn.ATTN_ERR_UNSUPPORTED),
    (dict(qd=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(kd=-1.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(vd=float("inf")), attn.ATTN_ERR_INVALID_ARG),
    (dict(vd=float("nan")), attn.ATTN_ERR_INVALID_ARG),
    (dict(q=P + 4), attn.ATTN_ERR_MISALIGNED),
    (dict(q=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.default_options(softcap=5.0)), attn.ATTN_ERR_UNSUPPORTED),
    (dict(opts=attn.default_options(alibi_slopes=P)), attn.ATTN_ERR_UNSUPPORTED),
    (dict(opts=attn.default_options(rescale_threshold=9.0)), attn.ATTN_ERR_INVALID_ARG),
])
def test_fp8_invalid_arguments_rejected_before_launch(L, kw, status):
    assert call_fp8(L, **kw) == status


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_fp8_call_without_gpu_reports_cuda_error(L):
    assert call_fp8(L) == attn.ATTN_ERR_CUDA


def test_option_structs_match_the_c_layout(tmp_path):
    """The ctypes mirrors of attn_fwd_options_t / attn_bwd_options_t have the
    C header's size and field offsets (compiled here with gcc)."""
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "attn.h"\n'
        "#define F(T, m) printf(#T \" \" #m \" %zu\\n\", offsetof(T, m))\n"
        "int main(void) {\n"
        '  printf("attn_fwd_options_t size %zu\\n", sizeof(attn_fwd_options_t));\n'
        '  printf("attn_bwd_options_t size %zu\\n", sizeof(attn_bwd_options_t));\n'
        '  printf("attn_fp4_options_t size %zu\\n", sizeof(attn_fp4_options_t));\n'
        "  F(attn_fwd_options_t, rescale_threshold); F(attn_fwd_options_t, exp2_mode);\n"
        "  F(attn_fwd_options_t, wait_timeout_us); F(attn_fwd_options_t, debug_withhold_kv);\n"
        "  F(attn_fwd_options_t, softcap); F(attn_fwd_options_t, reserved0);\n"
        "  F(attn_fwd_options_t, alibi_slopes); F(attn_fwd_options_t, reserved);\n"
        "  F(attn_bwd_options_t, softcap); F(attn_bwd_options_t, reserved0);\n"
        "  F(attn_bwd_options_t, alibi_slopes); F(attn_bwd_options_t, reserved);\n"
        "  F(attn_fp4_options_t, rescale_threshold); F(attn_fp4_options_t, classifier);\n"
        "  F(attn_fp4_options_t, wait_timeout_us); F(attn_fp4_options_t, mma);\n"
        "  F(attn_fp4_options_t, reserved);\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    c = {}
    for line in out.splitlines():
        t, m, v = line.split()
        c[(t, m)] = int(v)
    for name, cls in (("attn_fwd_options_t", attn.FwdOptions), ("attn_bwd_options_t", attn.BwdOptions),
                      ("attn_fp4_options_t", attn.Fp4Options)):
        assert c[(name, "size")] == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert c[(name, field)] == getattr(cls, field).offset, (name, field)


# ------------------------------------------------------------ FP4 Direct-P

def test_fp4_defaults_and_workspace(L):
    o = attn.fp4_options()
    assert o.rescale_threshold == 8.0 and o.classifier == attn.ATTN_DIRECT_P_AFFINE
    assert o.wait_timeout_us == 0 and list(o.reserved) == [0] * 4
    assert o.mma == attn.ATTN_FP4_MMA_AUTO
    # Room for either path: Q, K, V widened to f16 (each rounded up to 256
    # bytes), or the block-scaled path's scale atoms (two 512-byte atoms per
    # 128-row tile of Q -- both tiles of every 256-row query block -- K and V)
    # and V's transposed codes (128 rows of 64 bytes per key tile).
    assert attn.fp4_workspace_size(2, 16, 16, 8192, 8192, 128) == 3 * 2 * 2 * 8192 * 16 * 128
    assert attn.fp4_workspace_size(1, 2, 1, 3, 5, 64) == 768 + 2 * 768  # 768 B, 640 B -> 768
    assert attn.fp4_workspace_size(1, 1, 1, 1, 1, 128) == 2 * 1024 + 1024 + 1024 + 128 * 64
    assert attn.fp4_workspace_size(0, 2, 1, 3, 5, 64) == 0


def call_fp4(L, **kw):
    a = dict(qc=P, qs=P, qg=1.0, kc=P, ks=P, kg=0.5, vc=P, vs=P, vg=1.0, o=P, lse=P, B=1, Hq=2,
             Hkv=2, Sq=16, Sk=16, D=128, scale=0.1, causal=0, wl=-1, wr=-1, docs=None, nd=0,
             ws=P, wsb=1 << 20, opts=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return L.attn_fwd_fp4(vp(a["qc"]), vp(a["qs"]), a["qg"], vp(a["kc"]), vp(a["ks"]), a["kg"],
                          vp(a["vc"]), vp(a["vs"]), a["vg"], vp(a["o"]), vp(a["lse"]), a["B"],
                          a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"],
                          a["wl"], a["wr"], vp(a["docs"]) if a["docs"] else None, a["nd"],
                          vp(a["ws"]), a["wsb"],
                          None if a["opts"] is None else ctypes.byref(a["opts"]), None)


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), attn.ATTN_ERR_UNSUPPORTED),
    (dict(qg=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(kg=float("nan")), attn.ATTN_ERR_INVALID_ARG),
    (dict(vg=-1.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(vs=P + 8), attn.ATTN_ERR_MISALIGNED),
    (dict(ws=P + 4), attn.ATTN_ERR_MISALIGNED),
    (dict(lse=P + 2), attn.ATTN_ERR_MISALIGNED),
    (dict(kc=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(ws=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(wsb=1000), attn.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(Sq=8, docs=P, nd=1), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(classifier=2)), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(rescale_threshold=8.5)), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(rescale_threshold=-1.0)), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(wait_timeout_us=-5)), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(mma=3)), attn.ATTN_ERR_INVALID_ARG),
    (dict(opts=attn.fp4_options(mma=-1)), attn.ATTN_ERR_INVALID_ARG),
    (dict(D=64, opts=attn.fp4_options(mma=attn.ATTN_FP4_MMA_BLOCK_SCALED)),
     attn.ATTN_ERR_UNSUPPORTED),
])
def test_fp4_invalid_arguments_rejected_before_launch(L, kw, status):
    assert call_fp4(L, **kw) == status


def test_fp4_reserved_options_must_be_zero(L):
    o = attn.fp4_options()
    o.reserved[3] = 1
    assert call_fp4(L, opts=o) == attn.ATTN_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_fp4_call_without_gpu_reports_cuda_error(L):
    for classifier in (0, 1):
        for mma in (attn.ATTN_FP4_MMA_AUTO, attn.ATTN_FP4_MMA_F16, attn.ATTN_FP4_MMA_BLOCK_SCALED):
            assert call_fp4(L, opts=attn.fp4_options(classifier=classifier, mma=mma)) == \
                attn.ATTN_ERR_CUDA


def test_fp4_binding_checks_shapes(L):
    q = torch.zeros(1, 4, 1, 32, dtype=torch.uint8)
    with pytest.raises(TypeError):
        attn.attn_fwd_fp4(q, q, 1.0, q, q, 1.0, q, q, 1.0, None, None, None, scale=0.1)
