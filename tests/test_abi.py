"""Host-only checks of the C ABI: the library loads without a GPU, exports every entry point
include/moe.h declares, sizes workspaces and names statuses (no kernel is launched)."""
import os
import re

import moe_expert_layer_prefix_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"^\s*(?:moe_status|size_t|const char\*|uint64_t)\s+(moe_\w+)\(",
                                    src, re.M))
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared()
    assert {"moe_route", "moe_dispatch", "moe_expert_linear1", "moe_expert_linear2",
            "moe_fused_ffn", "moe_combine", "moe_forward", "moe_workspace_size",
            "moe_get_device_error", "moe_status_string"} <= declared
    for n in declared:
        assert hasattr(M._lib, n), n
    assert set(M.EXPORTS) == declared


def test_status_strings():
    for code, name in M.STATUS.items():
        assert M.moe_status_string(code) == name
    assert M.moe_status_string(12345) == "MOE_ERR_UNKNOWN"


def test_workspace_sizes():
    T, H, E, k, I = 8192, 7168, 256, 8, 2048
    S = T * k
    assert M.moe_workspace_size("linear1", T, H, E, k, I, "e4m3", "e4m3") == 0
    ffn = M.moe_workspace_size("fused_ffn", S, H, E, 1, I, "e4m3", "e4m3")
    assert ffn >= S * I + S * (I // 128) * 4
    fwd = M.moe_workspace_size("forward", T, H, E, k, I, "e4m3", "e4m3")
    assert fwd >= S * H + S * I + 2 * S * H     # x_perm + h + y (BF16)
    assert M.moe_workspace_size("dispatch", T, H, E, k, I, "e4m3", "e4m3") >= (T // 32) * E * 4
    # invalid queries size to zero
    assert M.moe_workspace_size("forward", T, H, E, k, I, "bf16", "e4m3") == 0
    assert M.moe_workspace_size(99, T, H, E, k, I, "e4m3", "e4m3") == 0
    assert M.moe_workspace_size("forward", 0, H, E, k, I, "e4m3", "e4m3") == 0


def test_tile_shape_knob_accepts_the_documented_values_only():
    # host-side setting (no launch): 0 auto, 1 single, 2 pair, 3 small
    try:
        for mode in ("auto", "single", "pair", "small", 0, 1, 2, 3):
            M.moe_set_gemm_tiles(mode)
        for bad in (-1, 4):
            try:
                M.moe_set_gemm_tiles(bad)
            except M.MoeError as e:
                assert "MOE_ERR_INVALID_ARG" in str(e)
            else:
                raise AssertionError(f"mode {bad} accepted")
    finally:
        M.moe_set_gemm_tiles("auto")


def test_argument_errors_need_no_gpu():
    # argument checks run before anything touches a device, so they work on a host alone
    P = None
    st = M._route_ex(P, P, 4, 256, 8, 0, 1, None, P, P, P)
    assert M.moe_status_string(st) == "MOE_ERR_INVALID_ARG"            # NULL logits
    st = M._dispatch_quant(P, 4, 256, 8, 2, P, P, P, P, P, P, P, 0, P)
    assert M.moe_status_string(st) == "MOE_ERR_INVALID_ARG"            # NULL buffers
    # a group configuration the GPU router does not take is refused before any launch (the
    # aligned dummy addresses are never dereferenced)
    import ctypes
    fake = ctypes.c_void_p(1 << 20)
    g = M.MoeRouterGroups(3, 1, 1.0)                                  # 256 experts / 3 groups
    st = M._route_ex(fake, None, 4, 256, 8, 0, 1, ctypes.byref(g), fake, fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"


def test_scale_format_checked_before_launch():
    import ctypes
    fake = ctypes.c_void_p(1 << 20)
    for fmt, act, wt, want in ((7, 2, 2, "MOE_ERR_INVALID_ARG"), (1, 2, 3, "MOE_ERR_UNSUPPORTED"),
                               (1, 1, 1, "MOE_ERR_UNSUPPORTED")):
        W = M.MoeWeights(act, wt, fake, fake, fake, fake, fmt)
        st = M._linear1(fake, fake, fake, 256, 256, 128, 4, ctypes.byref(W), fake, fake, None, 0,
                        None)
        assert M.moe_status_string(st) == want, (fmt, act, wt)


def test_wait_limit_and_selftest_arguments_checked_before_any_device_call():
    assert M.moe_status_string(M._set_wait_limit(-1)) == "MOE_ERR_INVALID_ARG"
    assert M.moe_status_string(M._selftest_wait(7, None)) == "MOE_ERR_INVALID_ARG"


def test_slot_count_beyond_32_bits_is_refused_before_launch():
    # slot indices t*k + j are 32-bit on the device: T*k > 2^31 - 1 is refused, and sizes
    # to zero, on the host (the dummy addresses are never dereferenced)
    import ctypes
    fake = ctypes.c_void_p(1 << 20)
    T = (1 << 31) // 8                                                 # T * 8 = 2^31
    st = M._route_ex(fake, None, T, 256, 8, 0, 1, None, fake, fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"
    st = M._dispatch_quant(fake, T, 256, 256, 8, fake, fake, fake, fake, fake, fake, fake,
                           1 << 40, None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"
    assert M.moe_workspace_size("forward", T, 7168, 256, 8, 2048, "e4m3", "e4m3") == 0
    assert M.moe_workspace_size("forward", T - 1, 7168, 256, 8, 2048, "e4m3", "e4m3") > 0



def test_backward_arguments_are_checked_before_launch():
    import ctypes
    fake = ctypes.c_void_p(1 << 20)
    assert M.moe_status_string(M._backward(None, None, 0, None)) == "MOE_ERR_INVALID_ARG"
    a = M.MoeBackwardArgs(64, 256, 8, 2, 128, 0, 1, 1.0)     # every pointer NULL
    assert M.moe_status_string(M._backward(ctypes.byref(a), fake, 1 << 30, None)) == \
        "MOE_ERR_INVALID_ARG"
    assert M.moe_workspace_size("backward", 64, 256, 8, 2, 128, "bf16", "bf16") >= \
        64 * 2 * (256 * 2 * 2 + 256 * 2 * 2 + 128 * 2)
    assert M.moe_workspace_size("backward", 64, 256, 8, 2, 128, "e4m3", "e4m3") == 0
    # transposes: packed E2M1 is refused, overlapping buffers too
    st = M._transpose(fake, M.DTYPES["e2m1"], 2, 64, 64, ctypes.c_void_p(1 << 30), None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"
    st = M._transpose(fake, M.DTYPES["bf16"], 2, 64, 64, ctypes.c_void_p((1 << 20) + 64), None)
    assert M.moe_status_string(st) == "MOE_ERR_INVALID_ARG"


def _header_struct(name):
    """(field, C type) pairs of `typedef struct name {...}` in include/moe.h, in order."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    body = {m.group(2): m.group(1)
            for m in re.finditer(r"typedef struct(?: \w+)? \{(.*?)\}\s*(\w+);", src, re.S)}[name]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        m = re.match(r"((?:const\s+)?\w+\s*\**)\s*(.*)", decl, re.S)
        base = m.group(1).replace(" ", "")
        for part in m.group(2).split(","):
            part = part.strip()
            stars = len(part) - len(part.lstrip("*"))
            fields.append((part.lstrip("*").strip(), "ptr" if "*" in base or stars else base))
    return fields


def _ctypes_kind(t):
    import ctypes
    if t is ctypes.c_void_p:
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_float: "float"}[t]


def test_binding_structs_match_the_header():
    # the ctypes mirrors of the header's structs: same fields, same order, same kinds
    for cname, py in (("moe_weights", M.MoeWeights), ("moe_router_groups", M.MoeRouterGroups),
                      ("moe_backward_args", M.MoeBackwardArgs)):
        hdr = _header_struct(cname)
        mine = [(n, _ctypes_kind(t)) for n, t in py._fields_]
        assert [n for n, _ in hdr] == [n for n, _ in mine], cname
        for (n, ht), (_, pk) in zip(hdr, mine):
            assert (ht == "ptr") == (pk == "ptr") and (ht != "float" or pk == "float"), (cname, n)


def test_binding_argument_counts_match_the_header():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = {m.group(1): m.group(2) for m in re.finditer(
        r"^\s*(?:moe_status|size_t|const char\*|uint64_t)\s+(moe_\w+)\((.*?)\);", src, re.M | re.S)}
    assert set(decls) == set(M.EXPORTS)
    for name, params in decls.items():
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(M._lib, name).argtypes or []) == n, name
