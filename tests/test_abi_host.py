"""The C-ABI library loads and exports every entry point its header declares, and rejects bad
arguments before touching the device.  CPU only: every call below fails validation, so no
kernel is launched and no pointer is dereferenced (the fake addresses are never used)."""
import ctypes
import os
import re

import pytest

import causal_sliding_window_swa_b200 as swa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
A = 0x7f0000000000          # a 16-byte aligned fake address, never dereferenced


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared_symbols()
    assert len(names) >= 9
    lib = ctypes.CDLL(swa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_version_and_strerror():
    assert swa.swa_attn_version() >= 100
    for code in range(-7, 1):
        assert swa.swa_attn_strerror(code)
    assert swa.swa_attn_strerror(-99) == "unknown status"


def test_workspace_bytes():
    n = 16 * 2048 * 12 * 128
    b0 = swa.swa_attn_workspace_bytes(16, 2048, 12, 128, 0)
    b1 = swa.swa_attn_workspace_bytes(16, 2048, 12, 128, 1)
    gate = 16 * 2048 * 12 * 8                       # (g_hi, g_lo) per (b, t, h)
    assert b0 >= 2 * 2 * n and b1 >= 3 * 2 * n
    assert 2 * n + gate <= b1 - b0 <= 2 * n + gate + 2048
    assert swa.swa_attn_workspace_bytes(0, 2048, 12, 128, 0) == 0
    assert swa.swa_attn_workspace_bytes(1, 16, 1, 96, 0) == 0


def _fwd(**kw):
    args = dict(q=A, k=A, v=A, ve=None, gate_x=None, Wg=None, out=A, lse=A, B=1, T=16, H=1, D=64,
                window=0, rope_base=1e4, eps=1e-6, stream=None)
    args.update(kw)
    return swa.swa_attn_fwd(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), swa.SWA_ERR_INVALID_ARG),
    (dict(T=0), swa.SWA_ERR_INVALID_ARG),
    (dict(H=-1), swa.SWA_ERR_INVALID_ARG),
    (dict(D=96), swa.SWA_ERR_UNSUPPORTED),
    (dict(D=256), swa.SWA_ERR_UNSUPPORTED),
    (dict(B=1 << 14, T=1 << 14, H=1, D=128), swa.SWA_ERR_UNSUPPORTED),   # 2^35 elements
    (dict(q=None), swa.SWA_ERR_INVALID_ARG),
    (dict(v=None), swa.SWA_ERR_INVALID_ARG),
    (dict(out=None), swa.SWA_ERR_INVALID_ARG),
    (dict(ve=A), swa.SWA_ERR_INVALID_ARG),                  # ve without gate_x / Wg
    (dict(ve=A, gate_x=A), swa.SWA_ERR_INVALID_ARG),
    (dict(eps=-1.0), swa.SWA_ERR_INVALID_ARG),
    (dict(eps=float("nan")), swa.SWA_ERR_INVALID_ARG),
    (dict(rope_base=0.0), swa.SWA_ERR_INVALID_ARG),
    (dict(rope_base=float("inf")), swa.SWA_ERR_INVALID_ARG),
    (dict(q=A + 2), swa.SWA_ERR_MISALIGNED),
    (dict(k=A + 8), swa.SWA_ERR_MISALIGNED),
    (dict(out=A + 4), swa.SWA_ERR_MISALIGNED),
    (dict(lse=A + 2), swa.SWA_ERR_MISALIGNED),
    (dict(ve=A + 2, gate_x=A, Wg=A), swa.SWA_ERR_MISALIGNED),
])
def test_fwd_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def test_fwd_ws_rejects_small_or_misaligned_workspace():
    need = swa.swa_attn_workspace_bytes(1, 16, 1, 64, 0)
    base = (A, A, A, None, None, None, A, A, 1, 16, 1, 64, 0, 1e4, 1e-6)
    assert swa.swa_attn_fwd_ws(*base, A, need - 1, None) == swa.SWA_ERR_NO_MEMORY
    assert swa.swa_attn_fwd_ws(*base, A + 8, need, None) == swa.SWA_ERR_MISALIGNED
    assert swa.swa_attn_fwd_ws(*base, None, need, None) == swa.SWA_ERR_INVALID_ARG


def test_stage_entry_points_reject_bad_arguments():
    need = swa.swa_attn_workspace_bytes(1, 16, 1, 64, 0)
    assert swa.swa_attn_prologue(A, A, A, None, None, None, 1, 16, 1, 64, 1e4, 1e-6, A, need - 1, None) \
        == swa.SWA_ERR_NO_MEMORY
    assert swa.swa_attn_rope_table(1, 16, 1, 64, 0, 1e4, A, need - 1, None) == swa.SWA_ERR_NO_MEMORY
    assert swa.swa_attn_rope_table(1, 16, 1, 64, 0, -1.0, A, need, None) == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_attn_attention(None, 0, A, A, 1, 16, 1, 64, 0, A, need, None) == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_attn_attention(A, 0, A, A, 1, 16, 1, 64, 0, A, need - 1, None) == swa.SWA_ERR_NO_MEMORY
    assert swa.swa_attn_attention(A, 0, A, A, 1, 16, 1, 80, 0, A, need, None) == swa.SWA_ERR_UNSUPPORTED


def test_document_forward_rejects_bad_arguments():
    base = dict(q=A, k=A, v=A, ve=None, gate_x=None, Wg=None, doc=A, out=A, lse=A, B=1, T=16, H=2, Hkv=1, D=64,
                window=0, rope_base=1e4, eps=1e-6, stream=None)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return swa.swa_attn_fwd_doc(*a.values())
    assert call(doc=None) == swa.SWA_ERR_INVALID_ARG
    assert call(doc=A + 2) == swa.SWA_ERR_MISALIGNED
    assert call(Hkv=3) == swa.SWA_ERR_INVALID_ARG
    assert call(D=80) == swa.SWA_ERR_UNSUPPORTED
    assert call(q=None) == swa.SWA_ERR_INVALID_ARG


def test_wait_limit_setter():
    prev = swa.swa_attn_set_wait_limit_ms(1500)
    assert prev >= 1
    assert swa.swa_attn_set_wait_limit_ms(0) == 1500      # ignored, returns current
    swa.swa_attn_set_wait_limit_ms(prev)


def test_selftest_wait_rejects_limits_out_of_range():
    # validated before any device query, so this runs without a GPU
    assert swa.swa_attn_selftest_wait(0, None) == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_attn_selftest_wait(10001, None) == swa.SWA_ERR_INVALID_ARG


def test_decode_workspace_and_validation():
    # qhat (B*H*D bf16), 1024-byte aligned; the chunks of a row are combined inside their cluster
    n = swa.swa_attn_decode_workspace_bytes(2, 1000, 3, 64, 0, 0)
    assert n == 1024
    assert swa.swa_attn_decode_workspace_bytes(16, 1000, 12, 128, 1, 200) == 16 * 12 * 128 * 2
    assert swa.swa_attn_decode_workspace_bytes(2, 1000, 3, 96, 0, 0) == 0
    need = swa.swa_attn_decode_workspace_bytes(1, 16, 1, 64, 0, 0)
    base = dict(q=A, k=A, v=A, ve=None, gate_x=None, Wg=None, k_cache=A, v_cache=A, out=A, lse=A,
                B=1, Tmax=16, H=1, D=64, window=0, rope_base=1e4, eps=1e-6, workspace=A, ws_bytes=need, stream=None)

    def call(**kw):
        a = dict(base, **kw)
        return swa.swa_attn_decode(a["q"], a["k"], a["v"], a["ve"], a["gate_x"], a["Wg"], a["k_cache"],
                                   a["v_cache"], a.get("pos", 3), a["out"], a["lse"], a["B"], a["Tmax"],
                                   a["H"], a["D"], a["window"], a["rope_base"], a["eps"], a["workspace"],
                                   a["ws_bytes"], a["stream"])
    assert call(pos=16) == swa.SWA_ERR_INVALID_ARG
    assert call(pos=-1) == swa.SWA_ERR_INVALID_ARG
    assert call(k_cache=None) == swa.SWA_ERR_INVALID_ARG
    assert call(ve=A) == swa.SWA_ERR_INVALID_ARG
    assert call(v_cache=A + 8) == swa.SWA_ERR_MISALIGNED
    assert call(ws_bytes=need - 1) == swa.SWA_ERR_NO_MEMORY
    assert call(D=80) == swa.SWA_ERR_UNSUPPORTED


def test_backward_workspace_and_validation():
    # forward sections + row statistics (B*H*Tp float2)
    # [+ dz and the dWg partial sums on value-embedding layers] + document starts and ends (B*T int32
    # each), each section 1024-byte aligned.
    B, T, H, Hkv, D = 2, 200, 4, 2, 64
    up = lambda x: (x + 1023) // 1024 * 1024
    fwd = swa.swa_attn_workspace_bytes(B, T, H, D, 0)
    n0 = swa.swa_attn_bwd_workspace_bytes(B, T, H, Hkv, D, 0)
    Tp = 256
    kv_fwd = up(B * T * Hkv * D * 2)
    assert n0 == (fwd - 2 * up(B * T * H * D * 2) + 2 * kv_fwd + up(B * T * H * D * 2) - kv_fwd
                  + up(B * H * Tp * 8) + 2 * up(B * T * 4))
    n1 = swa.swa_attn_bwd_workspace_bytes(B, T, H, Hkv, D, 1)
    assert n1 > n0 + up(B * T * Hkv * 4)
    assert swa.swa_attn_bwd_workspace_bytes(B, T, H, 3, D, 0) == 0     # 3 does not divide 4
    assert swa.swa_attn_bwd_workspace_bytes(B, T, H, Hkv, 96, 0) == 0
    base = dict(q=A, k=A, v=A, ve=None, gate_x=None, Wg=None, out=A, lse=A, dout=A, dlse=None, dq=A, dk=A,
                dv=A, dve=None, dgate_x=None, dWg=None, B=B, T=T, H=H, Hkv=Hkv, D=D, window=0,
                rope_base=1e4, eps=1e-6, workspace=A, ws_bytes=n0, stream=None)

    def call(**kw):
        return swa.swa_attn_bwd_gqa(*dict(base, **kw).values())
    assert call(dout=None) == swa.SWA_ERR_INVALID_ARG
    assert call(lse=None) == swa.SWA_ERR_INVALID_ARG
    assert call(dq=None) == swa.SWA_ERR_INVALID_ARG
    assert call(Hkv=3) == swa.SWA_ERR_INVALID_ARG
    assert call(dve=A) == swa.SWA_ERR_INVALID_ARG                      # VE gradients without VE
    assert call(ve=A, gate_x=A, Wg=A, ws_bytes=n1) == swa.SWA_ERR_INVALID_ARG   # VE without its gradients
    assert call(dk=A + 8) == swa.SWA_ERR_MISALIGNED
    assert call(workspace=A + 8) == swa.SWA_ERR_MISALIGNED
    assert call(ws_bytes=n0 - 1) == swa.SWA_ERR_NO_MEMORY
    assert call(D=80) == swa.SWA_ERR_UNSUPPORTED
    assert call(eps=-1.0) == swa.SWA_ERR_INVALID_ARG


def test_saved_backward_and_document_backward_validation():
    # swa_attn_bwd_saved takes the multi-head backward's arguments and checks them the same way;
    # swa_attn_bwd_doc also wants a 4-byte aligned document-id array.
    B, T, H, D = 2, 200, 4, 64
    n0 = swa.swa_attn_bwd_workspace_bytes(B, T, H, H, D, 0)
    base = dict(q=A, k=A, v=A, ve=None, gate_x=None, Wg=None, out=A, lse=A, dout=A, dlse=None, dq=A, dk=A,
                dv=A, dve=None, dgate_x=None, dWg=None, B=B, T=T, H=H, D=D, window=0,
                rope_base=1e4, eps=1e-6, workspace=A, ws_bytes=n0, stream=None)

    def saved(**kw):
        return swa.swa_attn_bwd_saved(*dict(base, **kw).values())
    assert saved(dout=None) == swa.SWA_ERR_INVALID_ARG
    assert saved(workspace=None) == swa.SWA_ERR_INVALID_ARG
    assert saved(dve=A) == swa.SWA_ERR_INVALID_ARG
    assert saved(dq=A + 8) == swa.SWA_ERR_MISALIGNED
    assert saved(ws_bytes=n0 - 1) == swa.SWA_ERR_NO_MEMORY
    assert saved(D=80) == swa.SWA_ERR_UNSUPPORTED
    assert saved(rope_base=0.0) == swa.SWA_ERR_INVALID_ARG

    def doc(**kw):
        a = dict(base, **kw)
        return swa._lib.swa_attn_bwd_doc(a["q"], a["k"], a["v"], a["ve"], a["gate_x"], a["Wg"], a.get("doc", A),
                                         a["out"], a["lse"], a["dout"], a["dlse"], a["dq"], a["dk"], a["dv"],
                                         a["dve"], a["dgate_x"], a["dWg"], a["B"], a["T"], a["H"], a.get("Hkv", H),
                                         a["D"], a["window"], a["rope_base"], a["eps"], a["workspace"],
                                         a["ws_bytes"], a["stream"])
    assert doc(doc=A + 2) == swa.SWA_ERR_MISALIGNED
    assert doc(Hkv=3) == swa.SWA_ERR_INVALID_ARG
    assert doc(ws_bytes=n0 - 1) == swa.SWA_ERR_NO_MEMORY


def test_document_decode_rejects_a_misaligned_id_array():
    need = swa.swa_attn_decode_workspace_bytes(1, 16, 1, 64, 0, 0)

    def call(doc, Hkv=1):
        return swa._lib.swa_attn_decode_doc(A, A, A, None, None, None, A, A, 3, doc, A, A, 1, 16, 1, Hkv, 64, 0,
                                            1e4, 1e-6, A, need, None)
    assert call(A + 2) == swa.SWA_ERR_MISALIGNED
    assert call(A, Hkv=2) == swa.SWA_ERR_INVALID_ARG


def test_saved_backward_binding_wants_the_forward_workspace():
    # the check runs before any tensor is looked at or any workspace is allocated
    import torch
    t = torch.zeros(1)
    with pytest.raises(ValueError, match="saved=True"):
        swa.backward(t, t, t, t, t, t, saved=True)
    with pytest.raises(ValueError, match="saved=True"):
        swa.backward(t, t, t, t, t, t, saved=True, workspace=t, doc=t)


def test_fused_projection_workspace_and_validation():
    B, T, H, Hkv, D, C = 2, 100, 4, 2, 64, 256
    n = swa.swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D)
    assert n > 0 and swa.swa_attn_fwd_x_workspace_bytes(B, T, H, 3, D) == 0
    base = dict(x=A, W=A, ve=None, Wg=None, out=A, lse=A, B=B, T=T, C=C, H=H, Hkv=Hkv, D=D, window=0,
                rope_base=1e4, eps=1e-6, workspace=A, ws_bytes=n, stream=None)

    def call(**kw):
        a = dict(base, **kw)
        return swa.swa_attn_fwd_x(a["x"], a["W"], a["ve"], a["Wg"], a["out"], a["lse"], a["B"], a["T"], a["C"],
                                  a["H"], a["Hkv"], a["D"], a["window"], a["rope_base"], a["eps"],
                                  a["workspace"], a["ws_bytes"], a["stream"])
    assert call(x=None) == swa.SWA_ERR_INVALID_ARG
    assert call(ve=A) == swa.SWA_ERR_INVALID_ARG                 # ve without Wg
    assert call(C=12) == swa.SWA_ERR_UNSUPPORTED                 # C not a multiple of 8
    assert call(ve=A, Wg=A, C=16) == swa.SWA_ERR_INVALID_ARG     # the gate needs 32 channels
    assert call(W=A + 8) == swa.SWA_ERR_MISALIGNED
    assert call(ws_bytes=n - 1) == swa.SWA_ERR_NO_MEMORY
    assert call(Hkv=3) == swa.SWA_ERR_INVALID_ARG
    assert call(D=96) == swa.SWA_ERR_UNSUPPORTED
    assert swa.swa_attn_qkv_prologue(A, A, None, None, None, A, A, B, T, C, H, Hkv, D, 1e4, 1e-6, A, n,
                                     None) == swa.SWA_ERR_INVALID_ARG
    # x with B T C = 2^31 elements (small B T H D): refused before the device is looked at
    big = dict(B=2, T=1 << 14, C=1 << 16, H=1, Hkv=1, D=64)
    nb = swa.swa_attn_fwd_x_workspace_bytes(2, 1 << 14, 1, 1, 64)
    assert nb > 0
    assert call(**big, ws_bytes=nb) == swa.SWA_ERR_UNSUPPORTED
    assert swa.swa_attn_qkv_prologue(A, A, None, None, A, A, A, 2, 1 << 14, 1 << 16, 1, 1, 64, 1e4, 1e-6, A, nb,
                                     None) == swa.SWA_ERR_UNSUPPORTED


def test_header_is_plain_c():
    """include/swa_attn.h compiles as C99 (no C++ or torch types at the boundary), and every entry
    point it declares can be taken by address from C (the source goes to gcc on stdin)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    names = sorted(_declared_symbols())
    src = ('#include "swa_attn.h"\n'
           "typedef void (*swa_fn)(void);\n"
           "swa_fn swa_entry_points[] = {\n" + "".join(f"    (swa_fn)&{n},\n" for n in names) + "};\n")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), "-x", "c", "-"], input=src, capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr


def test_binding_tensor_checks():
    # the helper the tensor-level calls use before handing bare pointers to the C calls
    import torch
    t = torch.zeros((2, 3), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="out is required"):
        swa._want("out", None, (2, 3), torch.bfloat16)
    with pytest.raises(ValueError, match=r"shape \(2, 4\), not \(2, 3\)"):
        swa._want("out", t, (2, 4), torch.bfloat16)
    with pytest.raises(ValueError, match="must be torch.float32"):
        swa._want("lse", t, (2, 3), torch.float32)
    with pytest.raises(ValueError, match="contiguous CUDA"):
        swa._want("out", t, (2, 3), torch.bfloat16)
    with pytest.raises(ValueError, match="workspace"):
        swa._want_workspace(torch.zeros(16, dtype=torch.uint8), torch.device("cpu"))


def test_c_program_links_and_calls_the_library(tmp_path):
    """A plain C99 program includes the header, links libswa_attn.so and calls it: the version,
    strerror, the workspace size, arguments refused before any device work, and (on a machine
    without a GPU) a valid call that reports SWA_ERR_NO_DEVICE instead of computing anything."""
    import shutil
    import subprocess
    import torch
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    lib_dir = os.path.dirname(swa.LIB_PATH)
    no_gpu = int(not torch.cuda.is_available())
    src = tmp_path / "use_swa.c"
    src.write_text(r'''
#include <stdio.h>
#include <stdint.h>
#include "swa_attn.h"

int main(void) {
    void* a = (void*)(uintptr_t)0x7f0000000000ull;   /* aligned, never dereferenced */
    float* l = (float*)a;
    if (swa_attn_version() < 100) return 1;
    if (swa_attn_workspace_bytes(1, 16, 1, 96, 0) != 0) return 2;
    if (swa_attn_workspace_bytes(1, 16, 1, 64, 0) == 0) return 3;
    if (swa_attn_fwd(a, a, a, NULL, NULL, NULL, a, l, 0, 16, 1, 64, 0, 1e4f, 1e-6f, NULL) != SWA_ERR_INVALID_ARG)
        return 4;
    if (swa_attn_fwd(a, a, a, NULL, NULL, NULL, a, l, 1, 16, 1, 96, 0, 1e4f, 1e-6f, NULL) != SWA_ERR_UNSUPPORTED)
        return 5;
    if (swa_attn_fwd((char*)a + 2, a, a, NULL, NULL, NULL, a, l, 1, 16, 1, 64, 0, 1e4f, 1e-6f, NULL) !=
        SWA_ERR_MISALIGNED)
        return 6;
    if (NO_GPU && swa_attn_fwd(a, a, a, NULL, NULL, NULL, a, l, 1, 16, 1, 64, 0, 1e4f, 1e-6f, NULL) !=
        SWA_ERR_NO_DEVICE)
        return 7;
    printf("%s\n", swa_attn_strerror(SWA_ERR_MISALIGNED));
    return 0;
}
''')
    exe = tmp_path / "use_swa"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", f"-DNO_GPU={no_gpu}", "-I",
                        os.path.join(ROOT, "include"), str(src), "-L", lib_dir, "-lswa_attn",
                        f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.strip() == swa.swa_attn_strerror(swa.SWA_ERR_MISALIGNED)


def test_readme_usage_matches_the_binding():
    # every call in the README's usage block binds to the binding's signature (names, order and
    # keywords), so the documented API cannot drift from the code
    import ast
    import inspect
    txt = open(os.path.join(ROOT, "README.md")).read()
    block = txt.split("```python", 1)[1].split("```", 1)[0]
    calls = [n for n in ast.walk(ast.parse(block)) if isinstance(n, ast.Call)
             and isinstance(n.func, ast.Attribute) and isinstance(n.func.value, ast.Name) and n.func.value.id == "swa"]
    assert len(calls) >= 8
    for c in calls:
        fn = getattr(swa, c.func.attr)
        sig = inspect.signature(fn)
        args = [object()] * len(c.args)
        kwargs = {k.arg: object() for k in c.keywords}
        sig.bind(*args, **kwargs)      # raises TypeError on a mismatch


def _prototypes():
    """name -> list of parameter type strings, from the SWA_API declarations of include/*.h."""
    protos = {}
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if not f.endswith(".h"):
            continue
        txt = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
        for m in re.finditer(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(([^)]*)\)\s*;", txt):
            params = [p.strip() for p in m.group(2).split(",")]
            protos[m.group(1)] = [] if params == ["void"] else params
    return protos


def _ctype_of(param: str):
    p = re.sub(r"\b(const|restrict)\b", " ", param)
    if "*" in p or re.search(r"\bswa_stream_t\b", p):
        return "pointer"
    for key, name in (("size_t", "size_t"), ("unsigned", "uint"), ("double", "double"), ("float", "float"),
                      ("int", "int")):
        if re.search(rf"\b{key}\b", p):
            return name
    raise AssertionError(f"unmapped C parameter type: {param!r}")


def test_binding_argtypes_match_the_header():
    # the ctypes signature of every entry point the binding declares has the header's arity and
    # parameter kinds, so no call can pass an argument in the wrong slot or width
    lib = swa.load()
    kinds = {ctypes.c_int: "int", ctypes.c_uint: "uint", ctypes.c_float: "float", ctypes.c_double: "double",
             ctypes.c_size_t: "size_t", ctypes.c_void_p: "pointer", ctypes.c_char_p: "pointer"}
    checked = 0
    for name, params in _prototypes().items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == len(params), (name, len(fn.argtypes), len(params))
        for t, p in zip(fn.argtypes, params):
            got = kinds.get(t, "pointer" if issubclass(t, (ctypes._Pointer, ctypes.c_void_p)) else repr(t))
            assert got == _ctype_of(p), (name, p, t)
        checked += 1
    assert checked == len(_prototypes()) >= 28      # every declared entry point has argtypes


def test_binding_restypes_match_the_header():
    lib = swa.load()
    inc = os.path.join(ROOT, "include")
    want = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p}
    n = 0
    for f in os.listdir(inc):
        if not f.endswith(".h"):
            continue
        txt = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
        for m in re.finditer(r"SWA_API\s+([\w\s\*]+?)\s*\b(swa_\w+)\s*\(", txt):
            ret = re.sub(r"\s+", " ", m.group(1)).replace(" *", "*").strip()
            assert ret in want, (m.group(2), ret)
            assert getattr(lib, m.group(2)).restype is want[ret], (m.group(2), ret)
            n += 1
    assert n >= 28


def test_fuzzed_forward_arguments_get_a_documented_status():
    # Random sizes, pointer alignments and null patterns: every call returns one of the header's
    # statuses without touching memory; on a machine without a GPU, arguments that pass validation
    # end in SWA_ERR_NO_DEVICE (no compute anywhere else).
    import torch
    from hypothesis import given, settings, strategies as st
    codes = {swa.SWA_OK, swa.SWA_ERR_INVALID_ARG, swa.SWA_ERR_UNSUPPORTED, swa.SWA_ERR_MISALIGNED,
             swa.SWA_ERR_CUDA, swa.SWA_ERR_TIMEOUT, swa.SWA_ERR_NO_MEMORY, swa.SWA_ERR_NO_DEVICE}
    no_gpu = not torch.cuda.is_available()
    sizes = st.integers(min_value=-3, max_value=1 << 20)
    ptr = st.one_of(st.none(), st.sampled_from([A, A + 2, A + 8, A + 16]))

    @settings(max_examples=300, deadline=None)
    @given(q=ptr, k=ptr, v=ptr, ve=ptr, gx=ptr, wg=ptr, out=ptr, lse=ptr, B=sizes, T=sizes, H=sizes,
           D=st.sampled_from([0, 32, 64, 96, 128, 256]), window=sizes,
           base=st.sampled_from([1e4, 0.0, -1.0, float("inf"), float("nan")]),
           eps=st.sampled_from([1e-6, 0.0, -1e-6, float("nan")]))
    def check(q, k, v, ve, gx, wg, out, lse, B, T, H, D, window, base, eps):
        rc = swa.swa_attn_fwd(q, k, v, ve, gx, wg, out, lse, B, T, H, D, window, base, eps, None)
        assert rc in codes
        valid = (None not in (q, k, v, out) and len({ve is None, gx is None, wg is None}) == 1
                 and B >= 1 and T >= 1 and H >= 1 and D in (64, 128) and B * T * H * D < (1 << 31)
                 and B <= 65535 and H <= 65535 and base > 0 and base != float("inf") and eps >= 0
                 and all(p % 16 == 0 for p in (q, k, v, out)) and (lse is None or lse % 4 == 0)
                 and (ve is None or (ve % 16 == 0 and gx % 2 == 0 and wg % 2 == 0)))
        assert (rc == swa.SWA_ERR_NO_DEVICE) == (valid and no_gpu) or not no_gpu, (rc, valid)

    check()


def test_fuzzed_decode_arguments_get_a_documented_status():
    import torch
    from hypothesis import given, settings, strategies as st
    no_gpu = not torch.cuda.is_available()
    ptr = st.one_of(st.none(), st.sampled_from([A, A + 4, A + 16]))

    @settings(max_examples=300, deadline=None)
    @given(q=ptr, kc=ptr, vc=ptr, ws=ptr, out=ptr, ve=st.sampled_from([None, A]), B=st.integers(-1, 40),
           Tmax=st.integers(-1, 5000), H=st.integers(-1, 16), Hkv=st.integers(-1, 16), D=st.sampled_from([64, 96, 128]),
           pos=st.integers(-2, 5001), ws_extra=st.integers(-2048, 2048))
    def check(q, kc, vc, ws, out, ve, B, Tmax, H, Hkv, D, pos, ws_extra):
        need = swa.swa_attn_decode_workspace_bytes(max(B, 1), max(Tmax, 1), max(H, 1), D, ve is not None, 0)
        ws_bytes = max(0, need + ws_extra)
        rc = swa._lib.swa_attn_decode_gqa(q, A, A, ve, ve, ve, kc, vc, pos, out, A, B, Tmax, H, Hkv, D, 0,
                                          1e4, 1e-6, ws, ws_bytes, None)
        valid = (None not in (q, kc, vc, ws, out) and B >= 1 and Tmax >= 1 and H >= 1 and D in (64, 128)
                 and 1 <= Hkv <= H and H % Hkv == 0 and 0 <= pos < Tmax
                 and all(p % 16 == 0 for p in (q, kc, vc, ws, out)) and ws_bytes >= need)
        assert rc in range(-7, 1)
        if no_gpu:
            assert (rc == swa.SWA_ERR_NO_DEVICE) == valid, (rc, valid)

    check()


def test_fuzzed_backward_arguments_get_a_documented_status():
    import torch
    from hypothesis import given, settings, strategies as st
    no_gpu = not torch.cuda.is_available()
    ptr = st.one_of(st.none(), st.sampled_from([A, A + 4, A + 16]))

    @settings(max_examples=300, deadline=None)
    @given(out=ptr, lse=ptr, dout=ptr, dq=ptr, dk=ptr, ws=ptr, has_ve=st.booleans(),
           vegrads=st.sampled_from([0, 1, 3]), B=st.integers(-1, 8), T=st.integers(-1, 3000),
           H=st.integers(-1, 12), Hkv=st.integers(-1, 12), D=st.sampled_from([64, 96, 128]),
           ws_extra=st.integers(-2048, 2048))
    def check(out, lse, dout, dq, dk, ws, has_ve, vegrads, B, T, H, Hkv, D, ws_extra):
        ve = A if has_ve else None
        dve, dgx, dwg = [(A, A, A), (A, None, None), (None, None, None)][{3: 0, 1: 1, 0: 2}[vegrads]]
        need = swa.swa_attn_bwd_workspace_bytes(max(B, 1), max(T, 1), max(H, 1), max(Hkv, 1), D, int(has_ve))
        ws_bytes = max(0, need + ws_extra)
        rc = swa.swa_attn_bwd_gqa(A, A, A, ve, ve, ve, out, lse, dout, None, dq, dk, A, dve, dgx, dwg, B, T, H,
                                  Hkv, D, 0, 1e4, 1e-6, ws, ws_bytes, None)
        valid = (None not in (out, lse, dout, dq, dk, ws) and B >= 1 and T >= 1 and H >= 1 and D in (64, 128)
                 and 1 <= Hkv <= H and H % Hkv == 0 and vegrads == (3 if has_ve else 0)
                 and all(p % 16 == 0 for p in (out, dout, dq, dk, ws)) and lse % 4 == 0 and need > 0
                 and ws_bytes >= need)
        assert rc in range(-7, 1)
        if no_gpu:
            assert (rc == swa.SWA_ERR_NO_DEVICE) == valid, (rc, valid)

    check()


def test_fuzzed_fused_layer_arguments_get_a_documented_status():
    # including inputs x too large for int32 indexing (B T C >= 2^31), refused before any work
    import torch
    from hypothesis import given, settings, strategies as st
    no_gpu = not torch.cuda.is_available()
    ptr = st.one_of(st.none(), st.sampled_from([A, A + 4, A + 16]))

    @settings(max_examples=300, deadline=None)
    @given(x=ptr, w=ptr, ws=ptr, out=ptr, ve=st.sampled_from([None, A]), wg=st.sampled_from([None, A]),
           B=st.integers(-1, 1 << 12), T=st.integers(-1, 1 << 14), C=st.sampled_from([0, 12, 16, 32, 768, 1536, 1 << 16]),
           H=st.integers(1, 12), Hkv=st.integers(1, 12), D=st.sampled_from([64, 96, 128]),
           ws_extra=st.integers(-2048, 2048))
    def check(x, w, ws, out, ve, wg, B, T, C, H, Hkv, D, ws_extra):
        need = swa.swa_attn_fwd_x_workspace_bytes(max(B, 1), max(T, 1), H, Hkv, D)
        ws_bytes = max(0, need + ws_extra)
        rc = swa.swa_attn_fwd_x(x, w, ve, wg, out, A, B, T, C, H, Hkv, D, 0, 1e4, 1e-6, ws, ws_bytes, None)
        valid = (None not in (x, w, ws, out) and B >= 1 and T >= 1 and D in (64, 128) and H % Hkv == 0
                 and Hkv <= H and B * T * H * D < (1 << 31) and (ve is None) == (wg is None)
                 and C >= 8 and C % 8 == 0 and (ve is None or C >= 32) and B * T * C < (1 << 31)
                 and all(p % 16 == 0 for p in (x, w, ws, out)) and need > 0 and ws_bytes >= need)
        assert rc in range(-7, 1)
        if no_gpu:
            assert (rc == swa.SWA_ERR_NO_DEVICE) == valid, (rc, valid)

    check()


def test_stream_handle_checks_the_device():
    # a torch stream must be on the inputs' GPU; a raw handle has no device to check
    import types
    import torch
    dev0, dev1 = torch.device("cuda", 0), torch.device("cuda", 1)
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        swa._stream_handle(types.SimpleNamespace(device=dev1, cuda_stream=1234), dev0)
    assert swa._stream_handle(types.SimpleNamespace(device=dev0, cuda_stream=99), dev0) == 99
    assert swa._stream_handle(5678, dev0) == 5678


def test_fuzzed_stage_arguments_get_a_documented_status():
    # the stage entry points (RoPE table, prologue, attention) on random arguments
    import torch
    from hypothesis import given, settings, strategies as st
    no_gpu = not torch.cuda.is_available()
    ptr = st.one_of(st.none(), st.sampled_from([A, A + 4, A + 16]))

    @settings(max_examples=300, deadline=None)
    @given(v=ptr, out=ptr, lse=ptr, ws=ptr, has_ve=st.booleans(), B=st.integers(-1, 16), T=st.integers(-1, 4096),
           H=st.integers(-1, 16), D=st.sampled_from([64, 96, 128]), base=st.sampled_from([1e4, 0.0, float("nan")]),
           ws_extra=st.integers(-2048, 2048))
    def check(v, out, lse, ws, has_ve, B, T, H, D, base, ws_extra):
        need = swa.swa_attn_workspace_bytes(max(B, 1), max(T, 1), max(H, 1), D, int(has_ve))
        wsb = max(0, need + ws_extra)
        sizes_ok = B >= 1 and T >= 1 and H >= 1 and D in (64, 128)
        ws_ok = ws is not None and ws % 16 == 0 and need > 0 and wsb >= need
        ve = A if has_ve else None
        rcs = {
            "rope": (swa.swa_attn_rope_table(B, T, H, D, int(has_ve), base, ws, wsb, None),
                     sizes_ok and base > 0 and ws_ok),
            "prologue": (swa.swa_attn_prologue(A, A, A, ve, ve, ve, B, T, H, D, base, 1e-6, ws, wsb, None),
                         sizes_ok and base > 0 and ws_ok),
            "attention": (swa.swa_attn_attention(v, int(has_ve), out, lse, B, T, H, D, 0, ws, wsb, None),
                          sizes_ok and ws_ok and out is not None and out % 16 == 0
                          and (lse is None or lse % 4 == 0) and (has_ve or (v is not None and v % 16 == 0))),
        }
        for name, (rc, valid) in rcs.items():
            assert rc in range(-7, 1), name
            if no_gpu:
                assert (rc == swa.SWA_ERR_NO_DEVICE) == valid, (name, rc, valid)

    check()


def test_every_entry_point_has_a_binding_of_the_same_name():
    # one Python function per C entry point, taking the C inputs in order; an `unsigned int*`
    # out-parameter is returned by the Python function instead of passed in
    import inspect
    lib = swa.load()
    for name, params in _prototypes().items():
        fn = getattr(swa, name, None)
        assert callable(fn) and name in swa.__all__, name
        inputs = [p for p in params if not re.match(r"unsigned\s+int\s*\*", p)]
        assert len(inspect.signature(fn).parameters) == len(inputs), name
        assert len(params) == len(getattr(lib, name).argtypes), name
