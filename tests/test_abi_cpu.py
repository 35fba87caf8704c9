"""Host-side checks of the C-ABI library (no GPU needed, no compute calls)."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from strided_verify_propose_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "isd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(isd_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = binding.lib()
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(binding.EXPORTS) == set(names)


def test_struct_layouts_match_header():
    """The ctypes mirrors have the sizes the C compiler gives the structs."""
    # isd_model_cfg: 14 x 4-byte fields
    assert ctypes.sizeof(binding.ModelCfg) == 14 * 4
    # isd_weights: 3 pointers + 8 pointer-to-pointer
    assert ctypes.sizeof(binding.Weights) == 11 * 8
    # isd_batch: 3 ints, pad, 3 pointers
    assert ctypes.sizeof(binding.Batch) == 16 + 3 * 8
    # isd_kv: 5 pointers + 3 ints (+ pad)
    assert ctypes.sizeof(binding.KV) == 5 * 8 + 16
    assert ctypes.sizeof(binding.Lora) == 8 + 14 * 8


def test_last_error_is_callable_without_gpu():
    assert binding.lib().isd_last_error() is not None


def test_gate_up_packing_interleaves_blocks_of_16():
    torch = pytest.importorskip("torch")
    shape = synth.ModelShape(n_layers=1, hidden=128, n_q_heads=2, n_kv_heads=1, head_dim=64,
                             intermediate=192, vocab=256, page_size=16)
    w = synth.decoder_weights(shape, seed=1)
    packed = binding.pack_weights(shape, w, device="cpu")
    gu = packed["layers"][0]["w_gate_up"].float().numpy()
    g, u = w["layers"][0]["w_gate"], w["layers"][0]["w_up"]
    for t in range(shape.intermediate // 16):
        assert np.array_equal(gu[32 * t:32 * t + 16], g[16 * t:16 * t + 16])
        assert np.array_equal(gu[32 * t + 16:32 * t + 32], u[16 * t:16 * t + 16])
    qkv = packed["layers"][0]["w_qkv"].float().numpy()
    assert np.array_equal(qkv[:shape.q_dim], w["layers"][0]["wq"])
    assert np.array_equal(qkv[shape.q_dim + shape.kv_dim:], w["layers"][0]["wv"])


# ------------------------------------------------ host argument validation --
# Every call below is refused by the library's host-side checks before it
# touches a device, so they run without a GPU.

def _cfg(**kw):
    base = dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, intermediate=704,
                vocab=1024, rope_theta=1e6, rms_eps=1e-6, mask_token_id=1023, page_size=16,
                max_batch=4, max_rows=64, max_position=512)
    base.update(kw)
    return binding.ModelCfg(*[base[f] for f, _ in binding.ModelCfg._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), binding.ISD_E_UNSUPPORTED),
    (dict(page_size=48), binding.ISD_E_UNSUPPORTED),
    (dict(n_q_heads=6, n_kv_heads=2), binding.ISD_E_UNSUPPORTED),    # group of 3
    (dict(hidden=200), binding.ISD_E_UNSUPPORTED),
    (dict(vocab=1000, mask_token_id=999), binding.ISD_E_UNSUPPORTED),
    (dict(max_rows=8192), binding.ISD_E_UNSUPPORTED),
    (dict(max_batch=2048), binding.ISD_E_UNSUPPORTED),
    (dict(mask_token_id=1024), binding.ISD_E_INVALID),
    (dict(hidden=0), binding.ISD_E_INVALID),
])
def test_init_refuses_bad_configs(kw, code):
    lib = binding.lib()
    h = ctypes.c_void_p()
    assert lib.isd_init(ctypes.byref(_cfg(**kw)), None, ctypes.byref(h)) == code
    assert not h.value
    assert lib.isd_last_error()


def test_entry_points_refuse_null_arguments():
    lib = binding.lib()
    h = ctypes.c_void_p()
    assert lib.isd_init(None, None, ctypes.byref(h)) == binding.ISD_E_INVALID
    b = binding.Batch(4, 3, 0, 1, 1, None)
    kv = binding.KV(1, 1, 1, 1, 1, 8, 4, 8)
    assert lib.isd_step(None, ctypes.byref(b), ctypes.byref(kv), 1, None, 1, 1, None, 1,
                        None) == binding.ISD_E_INVALID
    assert lib.isd_prefill(None, ctypes.byref(kv), 1, 8, None, 1, 3, 1, 1, 1, 1,
                           None) == binding.ISD_E_INVALID
    assert lib.isd_load_gated_lora(None, None) == binding.ISD_E_INVALID
    assert lib.isd_accept_propose(None, ctypes.byref(b), ctypes.byref(kv), 16, 1024, 1, None, 1,
                                  1, None, 1, 1 << 20, 1, None) == binding.ISD_E_INVALID
    assert lib.isd_gemm_bf16(None, 1, 1, 64, 128, 64, 1, None, None) == binding.ISD_E_INVALID
    assert lib.isd_profile_enable(None, 1) == binding.ISD_E_INVALID


def test_accept_refuses_out_of_range_sizes():
    lib = binding.lib()
    kv = binding.KV(1, 1, 1, 1, 1, 8, 4, 8)
    for batch, n, vocab, code in [(0, 3, 1024, binding.ISD_E_INVALID),
                                  (4, 9, 1024, binding.ISD_E_INVALID),
                                  (4, 3, 1022, binding.ISD_E_UNSUPPORTED)]:
        b = binding.Batch(batch, n, 0, 1, 1, None)
        assert lib.isd_accept_propose(1, ctypes.byref(b), ctypes.byref(kv), 16, vocab, 1, None, 1,
                                      1, None, 1, 1 << 20, 1, None) == code, (batch, n, vocab)
    # the fixed-scratch variant refuses a batch its array cannot hold
    b = binding.Batch(1024, 8, 0, 1, 1, None)
    assert lib.isd_accept_propose_noalloc(1, ctypes.byref(b), ctypes.byref(kv), 16, 151936, 1,
                                          None, 1, 1, None, 1, None) == binding.ISD_E_UNSUPPORTED
    assert b"fixed array holds" in lib.isd_last_error()


def test_component_calls_refuse_unsupported_shapes():
    lib = binding.lib()
    # GEMM: n not a multiple of 128, k not of 64, too many splits
    assert lib.isd_gemm_bf16(1, 1, 1, 64, 100, 64, 1, None, None) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_gemm_bf16(1, 1, 1, 64, 128, 96, 1, None, None) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_gemm_bf16(1, 1, 1, 64, 128, 128, 3, None, None) == binding.ISD_E_UNSUPPORTED
    # attention: head_dim 96, a group of 3 query heads, 9 rows x 8 heads > 64
    args = [1, 1, 1, 1, 1]
    assert lib.isd_paged_attention(*args, 4, 7, 8, 8, 96, 64, 10, 4, 1, 0, 1, 1, 1 << 20, None,
                                   None) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_paged_attention(*args, 4, 7, 6, 2, 128, 64, 10, 4, 1, 0, 1, 1, 1 << 20, None,
                                   None) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_paged_attention(*args, 4, 9, 64, 8, 128, 64, 10, 4, 1, 0, 1, 1, 1 << 20, None,
                                   None) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_set_wait_limit(10) == binding.ISD_E_INVALID
    # the plan query: an unaligned shape has no plan, a count below 1 is invalid
    out = (ctypes.c_int32 * len(binding.GEMM_PLAN_FIELDS))()
    assert lib.isd_gemm_plan(448, 100, 4096, 0, 8, 148, out) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_gemm_plan(448, 128, 96, 0, 8, 148, out) == binding.ISD_E_UNSUPPORTED
    assert lib.isd_gemm_plan(0, 128, 64, 0, 8, 148, out) == binding.ISD_E_INVALID
    assert lib.isd_gemm_plan(448, 128, 64, 0, 0, 148, out) == binding.ISD_E_INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """The product path has no fallback: without libisd.so the binding raises."""
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libisd.so"))
    with pytest.raises(RuntimeError, match="missing"):
        binding.lib()


def _sources(top, exts):
    for d, _, files in os.walk(os.path.join(ROOT, top)):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_oracle_and_product_share_no_code():
    """Neither side imports, includes or loads the other, and the input
    generators import neither."""
    imp = re.compile(r"^\s*(from|import)\s+([A-Za-z_][\w.]*)", re.M)
    inc = re.compile(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', re.M)
    for path in _sources("strided_verify_propose_b200", (".py",)):
        mods = [m.group(2) for m in imp.finditer(open(path).read())]
        assert not [m for m in mods if m.split(".")[0] == "oracle"], path
    for path in list(_sources("strided_verify_propose_b200", (".cu", ".cuh", ".h"))) + \
            list(_sources("include", (".h",))):
        assert not [h for h in inc.findall(open(path).read()) if "oracle" in h], path
    for path in _sources("oracle", (".py", ".c", ".h")):
        src = open(path).read()
        mods = [m.group(2).split(".")[0] for m in imp.finditer(src)]
        assert "strided_verify_propose_b200" not in mods and "libisd" not in src, path
    for path in _sources("synth", (".py",)):
        mods = [m.group(2).split(".")[0] for m in imp.finditer(open(path).read())]
        assert "oracle" not in mods and "strided_verify_propose_b200" not in mods, path


def test_a_c99_program_calls_the_library(tmp_path):
    """The header is plain C: a C99 program (tests/c/host_calls.c) compiles
    against it with -Wall -Wextra -pedantic -Werror, links libisd.so and,
    without a GPU, gets the same plan and work split as the Python binding."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    pkg = os.path.dirname(binding.LIB_PATH)
    exe = str(tmp_path / "host_calls")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "host_calls.c"),
                    "-L", pkg, "-lisd", f"-Wl,-rpath,{pkg}", "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    vals = {}
    for line in filter(None, out):
        name, v = line.split()
        vals.setdefault(name, []).append(int(v))
    assert vals["plan_rc"] == [binding.ISD_OK] and vals["split_rc"] == [binding.ISD_OK]
    assert vals["refused_rc"] == [binding.ISD_E_UNSUPPORTED]
    plan = binding.gemm_plan(448, 6144, 4096)
    assert vals["plan"] == [plan[f] for f in binding.GEMM_PLAN_FIELDS]
    segs, max_parts = binding.attention_split(3, 7, 32, 8, 128, 64, 64, [100, 1500, 4096], num_sms=16)
    assert vals["segments"] == [len(segs)] and vals["max_parts"] == [max_parts]
    assert vals["seg"] == np.asarray(segs).reshape(-1).tolist()


def _prototypes():
    """name -> (return type, [parameter types]) from include/isd.h."""
    src = open(os.path.join(ROOT, "include", "isd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"#[^\n]*", "", src)
    out = {}
    for ret, name, params in re.findall(r"([A-Za-z_][\w\s\*]*?)\b(isd_\w+)\s*\(([^)]*)\)\s*;", src):
        ps = [p.strip() for p in params.split(",")] if params.strip() not in ("", "void") else []
        # drop the parameter name, keep its type
        types = [re.sub(r"\b\w+$", "", p).strip() if not p.endswith("*") else p for p in ps]
        out[name] = (ret.strip(), types)
    return out


def _kind_of_c(t):
    t = t.replace("const", "").strip()
    if "*" in t:
        return "ptr"
    return {"int32_t": "i32", "int": "i32", "size_t": "size", "long long": "i64", "void": "void"}[
        " ".join(t.split())]


def _kind_of_ctypes(t):
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(t, ctypes._Pointer):
        return "ptr"
    if t in (ctypes.c_int32, ctypes.c_int):       # both 32-bit on this ABI
        return "i32"
    return {ctypes.c_size_t: "size", ctypes.c_longlong: "i64"}[t]


def test_binding_signatures_match_the_header():
    """Every prototype's parameters and return type, by kind (pointer, 32-bit
    int, size_t, long long, void), equal the binding's ctypes declaration."""
    lib = binding.lib()
    protos = _prototypes()
    assert set(protos) == set(_declared_functions())
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        want = [_kind_of_c(p) for p in params]
        if params:
            assert fn.argtypes is not None, f"{name}: no argtypes"
            got = [_kind_of_ctypes(t) for t in fn.argtypes]
            assert got == want, (name, got, want)
        assert _kind_of_ctypes(fn.restype) == _kind_of_c(ret), (name, fn.restype, ret)


def _header_structs():
    """struct name -> field names in declaration order, from include/isd.h."""
    src = open(os.path.join(ROOT, "include", "isd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for body, name in re.findall(r"typedef struct\s*\{(.*?)\}\s*(\w+)\s*;", src, flags=re.S):
        fields = []
        for decl in filter(None, (d.strip() for d in body.split(";"))):
            # the type ends where the first declarator's name begins
            m = re.match(r"^(.*?[\s\*])(\w+\s*(\[\d+\])?\s*(,\s*\**\s*\w+\s*(\[\d+\])?\s*)*)$", decl, flags=re.S)
            assert m, decl
            fields += [re.sub(r"[\s\*]|\[\d+\]", "", d) for d in m.group(2).split(",")]
        out[name] = fields
    return out


def test_struct_field_offsets_match_the_c_compiler(tmp_path):
    """Each ctypes mirror's fields sit at the offsets, and have the sizes, gcc
    gives the header's struct, field by field; the struct sizes agree."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    structs = _header_structs()
    mirrors = {"isd_model_cfg": binding.ModelCfg, "isd_weights": binding.Weights,
               "isd_batch": binding.Batch, "isd_kv": binding.KV, "isd_lora": binding.Lora}
    assert set(structs) == set(mirrors)
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "isd.h"', "int main(void) {"]
    for s, fields in structs.items():
        lines.append(f'  printf("{s} sizeof %zu\\n", sizeof({s}));')
        for f in fields:
            lines.append(f'  printf("{s} {f} %zu %zu\\n", offsetof({s}, {f}), sizeof((({s} *)0)->{f}));')
    lines += ["  return 0;", "}"]
    c = tmp_path / "offsets.c"
    c.write_text("\n".join(lines) + "\n")
    exe = str(tmp_path / "offsets")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(c),
                    "-o", exe], check=True)
    got = {}
    for line in subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n"):
        if line:
            s, f, *v = line.split()
            got.setdefault(s, []).append((f, tuple(int(x) for x in v)))
    for s, mirror in mirrors.items():
        size = dict(got[s])["sizeof"][0]
        fields = [v for f, v in got[s] if f != "sizeof"]
        assert ctypes.sizeof(mirror) == size, s
        mine = [(getattr(mirror, name).offset, getattr(mirror, name).size) for name, *_ in mirror._fields_]
        assert mine == fields, (s, mine, fields)


def test_accept_workspace_is_the_size_the_header_states():
    """batch * (2N-1) * ceil(vocab / 8192) chunk statistics of 16 bytes, then
    4 bytes per request, plus at most alignment padding; the headline shape
    fits the fixed 4 MiB array of the no-allocation entry point."""
    lib = binding.lib()
    rng = np.random.default_rng(4)
    for _ in range(200):
        B, N, V = int(rng.integers(1, 1025)), int(rng.integers(1, 9)), int(rng.integers(1, 131073)) * 4
        want = B * (2 * N - 1) * (-(-V // 8192)) * 16 + 4 * B
        got = lib.isd_accept_workspace_bytes(B, N, V)
        assert want <= got <= want + 512, (B, N, V, got, want)
    assert lib.isd_accept_workspace_bytes(1024, 4, 151936) <= 4 << 20
