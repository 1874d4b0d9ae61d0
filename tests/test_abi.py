"""The C-ABI library on the CPU: it builds, loads, exports every declared entry
point, its host-only plan matches the oracle bit for bit, and host-side argument
checks reject bad calls before anything touches a GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import build, hsa
from token_sparse_denoising_b200 import synthetic as S

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hsa.h")


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return hsa.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hsa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("T,budgets,fracs,m,kind,shift,N", [
    (8, [8, 4], (0.5, 0.5), 1, 0, 1.0, 1024),
    (40, [40, 20, 10], (0.25, 0.25, 0.5), 4, 1, 5.0, 32760),
    (40, [40, 8, 5, 1], (0.4, 0.2, 0.2, 0.2), 3, 1, 3.0, 1000),
    (12, [12, 6, 4, 3], (0.25, 0.25, 0.25, 0.25), 0, 0, 1.0, 17),
])
def test_plan_matches_oracle_bit_exact(lib, T, budgets, fracs, m, kind, shift, N):
    sizes = S.group_sizes(N, fracs)
    sig, tab, nact = hsa.plan_groups(T, budgets, sizes, N, m, kind, shift)
    assert sig.tobytes() == O.sigma_schedule(T, kind, shift).tobytes()
    want_tab = O.active_table(T, budgets, m)
    assert np.array_equal(tab.astype(bool), want_tab)
    assert np.array_equal(nact, O.active_counts(want_tab, sizes))


@pytest.mark.parametrize("bad", [dict(budgets=[8, 3]), dict(budgets=[4, 4]), dict(sizes=[4, 5]), dict(m=5),
                                 dict(budgets=[4, 8]), dict(kind=2)])
def test_plan_rejects(lib, bad):
    a = dict(T=8, budgets=[8, 4], sizes=[4, 4], N=8, m=1, kind=0)
    a.update(bad)
    with pytest.raises(hsa.HsaError) as e:
        hsa.plan_groups(a["T"], a["budgets"], a["sizes"], a["N"], a["m"], a["kind"], 1.0)
    assert e.value.code == hsa.HSA_EINVAL


def test_device_calls_reject_bad_arguments_on_host(lib):
    null = None
    sizes = (C.c_int * 2)(4, 4)
    assert lib.hsa_select_tokens(null, 8, 0, sizes, null, null, null, 0, null) == hsa.HSA_EINVAL
    assert lib.hsa_select_tokens(null, 8, 2, (C.c_int * 2)(4, 5), null, null, null, 0, null) == hsa.HSA_EINVAL
    assert lib.hsa_select_tokens_pinned(null, null, 8, 0, sizes, null, null, null, 0, null) == hsa.HSA_EINVAL
    assert lib.hsa_select_tokens_pinned(null, null, 8, 2, (C.c_int * 2)(4, 5), null, null, null, 0,
                                        null) == hsa.HSA_EINVAL
    assert lib.hsa_euler_update(null, null, null, null, 0, 8, 6, 0.1, null, null) == hsa.HSA_EINVAL
    act = (C.c_uint8 * 2)(1, 1)
    assert lib.hsa_active_rows(null, 8, 2, (C.c_int * 2)(4, 5), act, null, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_active_rows(null, 8, 0, sizes, act, null, null, null) == hsa.HSA_EINVAL
    m = C.c_int(-1)
    assert lib.hsa_active_rows(null, 8, 2, sizes, (C.c_uint8 * 2)(0, 0), null, C.byref(m), null) == hsa.HSA_OK
    assert m.value == 0                                    # nothing active: no device work
    assert lib.hsa_euler_update(null, null, null, null, 9, 8, 4, 0.1, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_l1_score(null, null, 4, 3, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_layer_step(null, null, null, 8, null, null, null, 1, null, null, null, 0, null, 0,
                              null) == hsa.HSA_EINVAL
    w = hsa.LayerWeightsC(300, 2, 64, hsa.HSA_BF16)           # D != 128 H
    assert lib.hsa_layer_step(C.byref(w), null, null, 8, null, null, null, 1, null, null, null, 0, null, 0,
                              null) == hsa.HSA_EINVAL
    assert lib.hsa_linear(null, 4, 100, null, 64, null, hsa.HSA_BF16, 0, null, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_linear(null, 4, 64, null, 64, null, hsa.HSA_BF16, 9, null, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_linear(null, 0, 64, null, 64, null, hsa.HSA_BF16, 0, null, null, null) == hsa.HSA_OK
    assert lib.hsa_attention(null, 0, null, null, 10, 1, hsa.HSA_BF16, null, null) == hsa.HSA_OK
    assert lib.hsa_attention(null, 4, null, null, 10, 1, 7, null, null) == hsa.HSA_EINVAL
    assert lib.hsa_context_kv(null, 0, 256, hsa.HSA_BF16, null, null, null, null, null, null, 0,
                              null) == hsa.HSA_EINVAL
    assert lib.hsa_patch_embed(null, null, 0, 8, 64, 256, hsa.HSA_BF16, null, null, null, null, 0,
                               null) == hsa.HSA_EINVAL
    assert b"need" in lib.hsa_last_error_string() or len(lib.hsa_last_error_string()) > 0


def test_iteration_host_rejects_bad_arguments_on_host(lib):
    """hsa_iteration_host checks every argument of its steps before it enqueues the upload."""
    null = None
    buf = (C.c_float * 4)()
    slot = hsa.HostSlotC(None, None, None, None)
    assert lib.hsa_iteration_host(null, buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    w = hsa.LayerWeightsC(256, 2, 1024, hsa.HSA_BF16)
    a = hsa.IterationArgsC(C.pointer(w))
    a.N, a.M = 8, 8
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    assert b"events" in lib.hsa_last_error_string()
    fake = 1 << 20                                         # 16-byte aligned stand-ins, never dereferenced
    slot = hsa.HostSlotC(fake, fake, fake, fake)
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    assert b"misaligned" in lib.hsa_last_error_string()    # the weights are NULL
    a.M = 9                                                # M > N
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    w.D = 300                                              # D != 128 H
    a.M = 8
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    # every buffer present (aligned stand-ins): the regrouping arguments are checked too
    w.D = 256
    for name, _ in hsa.LayerWeightsC._fields_[4:15]:
        setattr(w, name, fake)
    for name in ("d_kcache", "d_vcache", "d_idx", "d_pos", "d_xA", "d_vhat", "d_ws", "d_score", "d_group",
                 "d_order", "d_sel_ws"):
        setattr(a, name, fake)
    a.ws_bytes = lib.hsa_layer_step_workspace_size(8, 256, 1024, hsa.HSA_BF16) - 1
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EWORKSPACE
    a.ws_bytes += 1
    a.sel_ws_bytes = 1 << 20
    sizes = (C.c_int * 2)(4, 5)                            # sums to 9, not N = 8
    a.K, a.h_group_sizes = 2, C.cast(sizes, C.c_void_p)
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL
    assert b"sum to N" in lib.hsa_last_error_string()
    a.K = 17                                               # more groups than the selection supports
    assert lib.hsa_iteration_host(C.byref(a), buf, buf, C.byref(slot), null, null, null) == hsa.HSA_EINVAL


def test_workspace_sizes(lib):
    assert hsa.layer_step_workspace_size(32760, 1536, 8960, hsa.HSA_BF16) >= 32760 * (6 * 1536 + 8960) * 2
    assert hsa.layer_step_workspace_size(1024, 256, 1024, hsa.HSA_F32) >= 1024 * (6 * 256 + 1024) * 4
    assert lib.hsa_select_tokens_workspace_size(32760, 3) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    """No CPU fallback: a missing library is an error, not a silent substitute."""
    saved = hsa._lib
    try:
        hsa._lib = None
        with pytest.raises(RuntimeError):
            hsa.load(str(tmp_path / "libhsa.so"))
    finally:
        hsa._lib = saved


def test_attention_workspace_size_follows_the_last_wave(lib):
    """The split scratch is sized only when the last wave of (query tile, head) units is
    incomplete and worth splitting (148 SMs assumed without a device)."""
    bf, f32 = hsa.HSA_BF16, hsa.HSA_F32
    assert lib.hsa_attention_workspace_size(32760, 32760, 12, bf) == 0      # 3072 units: no split pays
    assert lib.hsa_attention_workspace_size(8190, 32760, 12, bf) > 0        # 768 units: 28 in the tail
    assert lib.hsa_attention_workspace_size(8190, 32760, 12, f32) == 0
    assert lib.hsa_attention_workspace_size(300, 256, 2, bf) == 0           # 2 key tiles: nothing to split
    assert lib.hsa_attention_workspace_size(0, 100, 2, bf) == 0


def _c_decls():
    """(name, return type, [parameter types]) of every function declared in include/hsa.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = []
    for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ \*]*?)\b(hsa_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        ret, name, params = m.group(1).strip(), m.group(2), " ".join(m.group(3).split())
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        out.append((name, ret, plist))
    return out


def _kind(c_type: str) -> str:
    t = c_type.strip()
    if "*" in t:
        return "ptr"
    base = t.replace("const", "").split()[0]
    return {"int": "i32", "size_t": "u64", "float": "f32", "uint64_t": "u64"}[base]   # LP64: size_t is 64-bit


def _ctype_kind(ct) -> str:
    if ct in (C.c_void_p, C.c_char_p) or getattr(ct, "__name__", "").startswith("LP_"):
        return "ptr"
    return {C.c_int: "i32", C.c_size_t: "u64", C.c_float: "f32", C.c_uint64: "u64"}[ct]


def test_binding_signatures_match_the_header():
    """Every declared entry point has a binding signature with the same parameter kinds and
    return kind, so the Python side cannot drift from the C ABI."""
    decls = _c_decls()
    assert len(decls) >= 20
    for name, ret, params in decls:
        assert name in hsa._SIGS, f"{name} missing from the binding"
        rtype, argtypes = hsa._SIGS[name]
        want = [_kind(p.rsplit(" ", 1)[0] if not p.endswith("*") else p) for p in params]
        got = [_ctype_kind(a) for a in argtypes]
        assert got == want, f"{name}: binding {got} vs header {want}"
        want_ret = "ptr" if "*" in ret else _kind(ret)
        assert _ctype_kind(rtype) == want_ret, f"{name}: return {rtype} vs {ret}"


def _struct_fields(struct):
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct %s \{(.*?)\} %s;" % (struct, struct), text, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        names = decl.split(None, 1)[1] if not decl.startswith("const") else decl.split(None, 2)[2]
        fields += [n.strip().lstrip("*").strip() for n in names.split(",")]
    return fields


@pytest.mark.parametrize("struct,cls", [("hsa_layer_weights", "LayerWeightsC"), ("hsa_iteration_args", "IterationArgsC"),
                                        ("hsa_host_slot", "HostSlotC")])
def test_struct_layouts_match_the_c_compiler(tmp_path, struct, cls):
    """The ctypes mirrors of the header's structs have the same field names, order, offsets and size
    as the C compiler gives them (gcc on this host, the same LP64 layout nvcc's host compiler uses)."""
    import shutil
    import subprocess
    fields = _struct_fields(struct)
    ctype = getattr(hsa, cls)
    assert fields == [f[0] for f in ctype._fields_]
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', 'int main(void) {',
             f'  printf("%zu\\n", sizeof({struct}));']
    lines += [f'  printf("%zu\\n", offsetof({struct}, {f}));' for f in fields]
    lines += ['  return 0;', '}']
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-o", str(exe), str(src)], check=True, capture_output=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    assert got[0] == C.sizeof(ctype)
    assert got[1:] == [getattr(ctype, f).offset for f in fields]
