"""The ctypes binding declares every C-ABI entry point with the header's
argument count, argument kinds and return kind (no GPU needed)."""
import ctypes
import re

from quantized_moe_expert_histogram_b200 import moeq


def _kind(decl: str) -> str:
    decl = decl.strip()
    if decl.count("*") >= 2:
        return "ptrptr"
    if "*" in decl or decl.split()[0] in ("moe_stream_t",) or "moe_slot_cache" in decl or "moe_predictor" in decl:
        return "ptr"
    base = decl.replace("const", "").split()[0]
    return {"int": "int", "int32_t": "int", "unsigned": "int", "size_t": "size", "double": "double",
            "float": "float", "int64_t": "i64"}[base]


def _ctype_kind(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p):
        return "ptr"
    if t is ctypes.c_int:
        return "int"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_double:
        return "double"
    if isinstance(t, type) and issubclass(t, ctypes._Pointer):
        return "ptrptr"
    raise AssertionError(t)


def _prototypes():
    with open(moeq.HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(r"MOE_API\s+([\w\s\*]+?)\s*\b(moe_\w+)\s*\(([^)]*)\)\s*;", text):
        params = params.strip()
        args = [] if params in ("", "void") else [p.rsplit(None, 1)[0] if not p.strip().endswith("*") else p
                                                  for p in params.split(",")]
        args = [a.replace("*", " * ") for a in args]
        ret = ret.strip()
        rk = "void" if ret == "void" else ("ptr" if "*" in ret else {"moe_status_t": "int", "size_t": "size"}[ret])
        out[name] = (rk, [_kind(a) for a in args])
    return out


def test_binding_matches_header():
    protos = _prototypes()
    assert set(protos) == set(moeq._SIGS), set(protos) ^ set(moeq._SIGS)
    for name, (rk, kinds) in protos.items():
        res, args = moeq._SIGS[name]
        got = [_ctype_kind(a) for a in args]
        assert _ctype_kind(res) == rk, name
        assert got == kinds, (name, got, kinds)
