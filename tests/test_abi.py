"""C-ABI library checks that need no GPU: it loads, exports every symbol the
header declares, and rejects bad arguments on the host before launching."""
import ctypes
import os
import re

import pytest

from block_sparse_full_b200 import ssa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssa_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(ssa.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(ssa.EXPORTS) == names


def _prototypes():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return {name: args.strip()
            for name, args in re.findall(r"\b(ssa_\w+)\s*\(([^;{)]*)\)\s*;", src)}


def _ctype_class(c_decl):
    # the ctypes argument class a C parameter declaration needs
    t = re.sub(r"\b(const|restrict)\b", "", c_decl).strip()
    if "ssa_params_t" in t:
        return "params"
    if "*" in t or t.startswith("cudaStream_t"):
        return "pointer"
    base = t.split()[:-1] if len(t.split()) > 1 else t.split()
    base = " ".join(base)
    # size_t and unsigned long long are both unsigned 64-bit here (and one
    # ctypes type on LP64)
    return {"int": "int", "size_t": "u64", "float": "float", "unsigned long long": "u64"}[base]


def test_binding_signatures_match_the_header():
    # every prototype's parameter list, argument by argument, against the
    # ctypes signature the binding installs: a drift between the two would pass
    # wrong-width arguments silently
    cls = {ctypes.c_void_p: "pointer", ctypes.c_int: "int", ctypes.c_size_t: "u64",
           ctypes.c_float: "float", ctypes.c_ulonglong: "u64"}
    assert ctypes.sizeof(ctypes.c_size_t) == ctypes.sizeof(ctypes.c_ulonglong) == 8
    protos = _prototypes()
    assert sorted(protos) == declared_functions()
    for name, args in protos.items():
        want = [] if args in ("", "void") else [_ctype_class(a) for a in args.split(",")]
        got = [("params" if a is ssa._P else cls[a]) for a in ssa._SIGNATURES[name][1]]
        assert got == want, (name, got, want)


def test_exports_are_c_symbols():
    # plain C names, no C++ mangling
    out = os.popen(f"nm -D --defined-only {ssa.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_version_and_status_strings():
    assert ssa.ssa_version() >> 16 == 1
    assert ssa.ssa_status_string(0) == "ok"
    assert "timed out" in ssa.ssa_status_string(ssa.SSA_ERR_TIMEOUT)
    assert ssa.ssa_status_string(12345) == "unknown status"


GOOD = dict(B=1, H=2, T=1024, D=128, block=64, topk=4, dtype=ssa.SSA_BF16)


def P(**kw):
    a = {**GOOD, **kw}
    return ssa.make_params(a["B"], a["H"], a["T"], a["D"], a["block"], a["topk"], a["dtype"],
                           kw.get("sm_scale"), kw.get("flags", 0))


@pytest.mark.parametrize("kw,code", [
    (dict(T=1000), ssa.SSA_ERR_INVALID_ARG),           # T % block
    (dict(block=32), ssa.SSA_ERR_UNSUPPORTED),
    (dict(D=96), ssa.SSA_ERR_UNSUPPORTED),
    (dict(topk=0), ssa.SSA_ERR_INVALID_ARG),
    (dict(topk=17), ssa.SSA_ERR_INVALID_ARG),          # > T/block
    (dict(topk=1, flags=ssa.SSA_FLAG_FORCE_SINK), ssa.SSA_ERR_INVALID_ARG),
    (dict(flags=8), ssa.SSA_ERR_INVALID_ARG),
    (dict(dtype=7), ssa.SSA_ERR_INVALID_ARG),
    (dict(B=0), ssa.SSA_ERR_INVALID_ARG),
    (dict(sm_scale=-1.0), ssa.SSA_ERR_INVALID_ARG),
    (dict(sm_scale=float("inf")), ssa.SSA_ERR_INVALID_ARG),
])
def test_bad_params_rejected_before_launch(kw, code):
    p = P(**kw)
    fake = 1 << 20  # never dereferenced: validation fails first
    st = ssa.ssa_select_blocks(p, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == code, ssa.ssa_last_error()
    assert ssa.ssa_last_error()
    assert ssa.ssa_workspace_size(p, 0) == ctypes.c_size_t(-1).value
    assert ssa.ssa_kernel_path(p) == -1


def test_null_and_misaligned_pointers_rejected():
    p = P()
    a = 1 << 20
    assert ssa.ssa_select_blocks(p, None, a, a, a, a, a, 1 << 30, None) == ssa.SSA_ERR_INVALID_ARG
    assert "q is NULL" in ssa.ssa_last_error()
    assert ssa.ssa_select_blocks(p, a + 2, a, a, a, a, a, 1 << 30, None) == ssa.SSA_ERR_INVALID_ARG
    assert "aligned" in ssa.ssa_last_error()
    st = ssa.ssa_attn_fwd_dual(p, a, a, a, None, None, None, a, a, a, a, a, a, a, 1 << 30, None)
    assert st == ssa.SSA_ERR_INVALID_ARG and "mask" in ssa.ssa_last_error()
    st = ssa.ssa_attn_bwd(p, a, a, a, None, None, a, a, a, a, a, None, None, 0.0, 0.0,
                          a, a, None, a, 1 << 40, None)
    assert st == ssa.SSA_ERR_INVALID_ARG and "dv" in ssa.ssa_last_error()
    st = ssa.ssa_align_loss(p, a, float("nan"), 1.0, a, a, 1 << 20, None)
    assert st == ssa.SSA_ERR_INVALID_ARG


def test_workspace_too_small_rejected():
    p = P()
    need = ssa.ssa_workspace_size(p, ssa.SSA_WS_SELECT)
    assert need > 0
    a = 1 << 20
    st = ssa.ssa_select_blocks(p, a, a, a, a, a, a, need - 1, None)
    assert st == ssa.SSA_ERR_WORKSPACE
    st = ssa.ssa_select_blocks(p, a, a, a, a, a, None, need, None)
    assert st == ssa.SSA_ERR_WORKSPACE
    st = ssa.ssa_select_blocks(p, a, a, a, a, a, a + 16, need, None)  # not 256-aligned
    assert st == ssa.SSA_ERR_INVALID_ARG


def test_workspace_sizes_scale_with_shape():
    small, big = P(T=1024), P(T=4096, topk=4)
    for w in (ssa.SSA_WS_SELECT, ssa.SSA_WS_LOSS, ssa.SSA_WS_BWD):
        assert ssa.ssa_workspace_size(big, w) >= ssa.ssa_workspace_size(small, w)
    # select: Qbar and Kbar in float64
    assert ssa.ssa_workspace_size(small, 0) == 2 * 1 * 2 * 16 * 128 * 8


def test_kernel_path_choice():
    assert ssa.ssa_kernel_path(P(dtype=ssa.SSA_F32)) == 0
    assert ssa.ssa_kernel_path(P(D=64)) == 1   # bf16 d = 64 runs on the tensor cores too
    assert ssa.ssa_kernel_path(P(flags=ssa.SSA_FLAG_FORCE_SIMT)) == 0


def test_bwd_head_groups_bound_the_ds_workspace():
    # the tensor-core backward stores bf16 dS blocks of the causal triangle:
    # (T - 128 J) / 64 blocks of 16 KB for key tile J, within 4 GiB per group
    def blocks(T):
        ntk = (T + 127) // 128
        return ntk * (T // 64) - ntk * (ntk - 1)
    assert blocks(192) == 4 and blocks(8192) == 4160
    bench = P(B=1, H=16, T=8192, block=64, topk=16)
    assert ssa.ssa_bwd_heads_per_group(bench) == 16
    sink = P(B=1, H=8, T=65536, block=128, topk=16)
    assert ssa.ssa_bwd_heads_per_group(sink) == 1
    train = P(B=4, H=32, T=4096, block=64, topk=8)
    per_head = blocks(4096) * 16 * 1024
    assert ssa.ssa_bwd_heads_per_group(train) == min(128, (4 << 30) // per_head)
    assert ssa.ssa_bwd_heads_per_group(P(dtype=ssa.SSA_F32)) == -1
    # the workspace holds exactly one group's blocks on top of the row data
    g = ssa.ssa_bwd_heads_per_group(train)
    assert ssa.ssa_workspace_size(train, ssa.SSA_WS_BWD) >= g * per_head


def test_ds_budget_hook_sets_the_head_groups():
    train = P(B=4, H=32, T=4096, block=64, topk=8)
    ntk = 4096 // 128
    per_head = (ntk * (4096 // 64) - ntk * (ntk - 1)) * 16 * 1024
    default = ssa.ssa_bwd_heads_per_group(train)
    try:
        ssa.ssa_debug_set_ds_budget_bytes(1)  # below one head: still one head per group
        assert ssa.ssa_bwd_heads_per_group(train) == 1
        ssa.ssa_debug_set_ds_budget_bytes(int(2.5 * per_head))
        assert ssa.ssa_bwd_heads_per_group(train) == 2
        ws2 = ssa.ssa_workspace_size(train, ssa.SSA_WS_BWD)
        ssa.ssa_debug_set_ds_budget_bytes(5 * per_head)
        assert ssa.ssa_workspace_size(train, ssa.SSA_WS_BWD) == ws2 + 3 * per_head
    finally:
        ssa.ssa_debug_set_ds_budget_bytes(0)
    assert ssa.ssa_bwd_heads_per_group(train) == default
