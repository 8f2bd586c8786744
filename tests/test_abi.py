"""C-ABI checks that need no GPU: the library loads, exports every function
include/lora.h declares, and validates arguments on the host exactly as the
entry points do (no CUDA call is made on these paths)."""
import ctypes
import re

import pytest

ALIGNED = 0x7f0000001000      # never dereferenced: validation only


def test_library_loads_and_exports_every_header_function(built_lib):
    L = built_lib
    names = L.header_functions()
    assert len(names) >= 10, names
    so = L.lib()
    for n in names:
        assert hasattr(so, n), f"{n} declared in include/lora.h but not exported"
    assert L.lora_abi_version() == 4


def test_header_declares_the_hot_path_entry_points(built_lib):
    names = set(built_lib.header_functions())
    for n in ("lora_fwd", "lora_fwd_save", "lora_bwd", "lora_bwd_ex", "lora_bwd_workspace_size", "lora_merge", "lora_merge_batched",
              "lora_restore", "lora_get_device_status", "lora_check_args", "lora_status_string"):
        assert n in names


def test_status_strings(built_lib):
    L = built_lib
    for code, name in L.STATUS.items():
        assert L.lora_status_string(code).startswith(name)


def _ptrs(n, base=ALIGNED, step=1 << 32):
    return [base + i * step for i in range(n)]


@pytest.mark.parametrize("M,d_in,d_out,r,expect", [
    (256, 512, 512, 16, "LORA_OK"),
    (0, 512, 512, 16, "LORA_OK"),
    (3, 8, 8, 8, "LORA_OK"),
    (-1, 512, 512, 16, "LORA_ERR_SHAPE"),
    (256, 0, 512, 16, "LORA_ERR_SHAPE"),
    (256, 516, 512, 16, "LORA_ERR_SHAPE"),
    (256, 512, 100, 16, "LORA_ERR_SHAPE"),
    (256, 512, 512, 12, "LORA_ERR_RANK"),
    (256, 512, 512, 0, "LORA_ERR_RANK"),
    (256, 512, 512, 136, "LORA_ERR_RANK"),
    (256, 512, 512, 128, "LORA_OK"),
])
def test_fwd_shape_and_rank_validation(built_lib, M, d_in, d_out, r, expect):
    L = built_lib
    assert L.STATUS[L.lora_check_args(0, _ptrs(5), M, d_in, d_out, r)] == expect


def test_fwd_null_align_alias(built_lib):
    L = built_lib
    p = _ptrs(5)
    assert L.STATUS[L.lora_check_args(0, p[:4] + [0], 8, 8, 8, 8)] == "LORA_ERR_NULL"
    q = list(p)
    q[2] += 8
    assert L.STATUS[L.lora_check_args(0, q, 8, 8, 8, 8)] == "LORA_ERR_ALIGN"
    q = list(p)
    q[4] = q[0] + 16                       # Y inside X
    assert L.STATUS[L.lora_check_args(0, q, 8, 8, 8, 8)] == "LORA_ERR_ALIAS"


def test_bwd_workspace_rules(built_lib):
    L = built_lib
    M, d_in, d_out, r = 1000, 520, 264, 24
    need = L.lora_bwd_workspace_size(M, d_in, d_out, r)
    assert need > 0 and need % 256 == 0
    assert L.lora_bwd_workspace_size(0, d_in, d_out, r) == 0
    assert L.lora_bwd_workspace_size(M, d_in, d_out, 12) == 0          # invalid -> 0
    # T and dT, each bf16 [M, r_pad] at a 256-byte aligned offset
    r_pad = 32
    assert need == 2 * ((M * r_pad * 2 + 255) // 256 * 256)
    assert L.lora_bwd_workspace_size(2 * M, d_in, d_out, r) > need
    p = _ptrs(9)
    assert L.STATUS[L.lora_check_args(1, p, M, d_in, d_out, r, need)] == "LORA_OK"
    assert L.STATUS[L.lora_check_args(1, p, M, d_in, d_out, r, need - 256)] == "LORA_ERR_WORKSPACE"
    q = list(p)
    q[8] = 0
    assert L.STATUS[L.lora_check_args(1, q, M, d_in, d_out, r, need)] == "LORA_ERR_WORKSPACE"
    q = list(p)
    q[8] += 128                             # workspace must be 256-byte aligned
    assert L.STATUS[L.lora_check_args(1, q, M, d_in, d_out, r, need)] == "LORA_ERR_ALIGN"
    q = list(p)
    q[5] = q[4]                             # dX aliases dY
    assert L.STATUS[L.lora_check_args(1, q, M, d_in, d_out, r, need)] == "LORA_ERR_ALIAS"
    q = list(p)
    q[6] = q[8] + 256                       # dA inside the workspace
    assert L.STATUS[L.lora_check_args(1, q, M, d_in, d_out, r, need)] == "LORA_ERR_ALIAS"
    # M = 0 needs no workspace at all
    q = list(p)
    q[8] = 0
    assert L.STATUS[L.lora_check_args(1, q, 0, d_in, d_out, r, 0)] == "LORA_OK"


def test_merge_validation(built_lib):
    L = built_lib
    p = _ptrs(4)
    assert L.STATUS[L.lora_check_args(2, p, 0, 2560, 4096, 32)] == "LORA_OK"
    q = list(p)
    q[3] = q[0]                             # in place is allowed
    assert L.STATUS[L.lora_check_args(2, q, 0, 2560, 4096, 32)] == "LORA_OK"
    q = list(p)
    q[3] = q[0] + 64                        # partial overlap is not
    assert L.STATUS[L.lora_check_args(2, q, 0, 2560, 4096, 32)] == "LORA_ERR_ALIAS"
    q = list(p)
    q[3] = q[1]                             # W_dst over A
    assert L.STATUS[L.lora_check_args(2, q, 0, 2560, 4096, 32)] == "LORA_ERR_ALIAS"
    assert L.STATUS[L.lora_check_args(2, p, 0, 2560, 4090, 32)] == "LORA_ERR_SHAPE"
    assert L.STATUS[L.lora_check_args(2, p, 0, 2560, 4096, 20)] == "LORA_ERR_RANK"
    assert L.STATUS[L.lora_check_args(2, [0] + p[1:], 0, 2560, 4096, 32)] == "LORA_ERR_NULL"


def test_unknown_op_rejected(built_lib):
    assert built_lib.STATUS[built_lib.lora_check_args(7, _ptrs(5), 8, 8, 8, 8)] == "LORA_ERR_SHAPE"


def test_binding_rejects_cpu_tensors_before_any_cuda_call(built_lib):
    import torch
    X = torch.zeros(8, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        built_lib.lora_fwd(X, X, X[:8], X, X.clone(), 16.0)


def test_fwd_batched_validation_before_any_cuda_call(built_lib):
    """lora_fwd_batched checks every entry (lora_fwd's rules) and that no
    entry's Y overlaps another entry's inputs or Y, before touching the GPU."""
    L = built_lib
    so = L.lib()

    def call(entries, r=16, n=None):
        arr = (L._FwdDesc * max(len(entries), 1))(*[L._FwdDesc(*e) for e in entries])
        return L.STATUS[so.lora_fwd_batched(arr, len(entries) if n is None else n, r, 32.0, None)]

    a = _ptrs(5, base=ALIGNED)
    b = _ptrs(5, base=ALIGNED + (1 << 40))
    ok_a = (*a, 256, 512, 512)
    ok_b = (*b, 128, 1024, 256)
    assert L.STATUS[so.lora_fwd_batched(None, 1, 16, 32.0, None)] == "LORA_ERR_NULL"
    assert call([ok_a], n=-1) == "LORA_ERR_SHAPE"
    assert call([ok_a, (*b, 128, 1020, 256)]) == "LORA_ERR_SHAPE"     # d_in % 8 != 0
    assert call([ok_a, ok_b], r=12) == "LORA_ERR_RANK"
    assert call([ok_a, (b[0], b[1], b[2], b[3], 0, 128, 1024, 256)]) == "LORA_ERR_NULL"
    assert call([ok_a, (b[0] + 8, *b[1:], 128, 1024, 256)]) == "LORA_ERR_ALIGN"
    # entry 1 writes its Y into entry 0's X
    assert call([ok_a, (*b[:4], a[0] + 4096, 128, 1024, 256)]) == "LORA_ERR_ALIAS"
    # two entries share one Y
    assert call([ok_a, (*b[:4], a[4], 128, 1024, 256)]) == "LORA_ERR_ALIAS"


def test_bwd_ex_refuses_unknown_flags_before_any_cuda_call(built_lib):
    """The flags word is checked first: an unknown bit is LORA_ERR_FLAGS even
    with pointers that are never dereferenced and no GPU present."""
    L = built_lib
    so = L.lib()
    p = [ctypes.c_void_p(x) for x in _ptrs(9)]
    args = p[:8] + [256, 512, 512, 16, ctypes.c_float(32.0), p[8], 1 << 30]
    for flags in (4, 8, 0x80000000, 0xFFFFFFFC, 0xFFFFFFFF):
        assert L.STATUS[so.lora_bwd_ex(*args, flags, None)] == "LORA_ERR_FLAGS"
    # known flags pass the flags check and stop at the next rule (alignment)
    bad_align = list(p)
    bad_align[6] = ctypes.c_void_p(ALIGNED + 8)        # dA not 16-byte aligned
    for flags in (L.LORA_BWD_FP32_GRADS, L.LORA_BWD_T_SAVED, L.LORA_BWD_FP32_GRADS | L.LORA_BWD_T_SAVED):
        code = so.lora_bwd_ex(*(bad_align[:8] + args[8:]), flags, None)
        assert L.STATUS[code] == "LORA_ERR_ALIGN"


def test_size_limits(built_lib):
    """Sizes up to 2^30 rows / columns pass validation, one step past is
    LORA_ERR_SHAPE (validation only: the pointers are never dereferenced)."""
    L = built_lib
    big = 1 << 30
    p = _ptrs(5, step=1 << 42)       # 4 TiB apart: a 2^30-row tensor is 1 TiB here
    assert L.STATUS[L.lora_check_args(0, p, big, 512, 512, 16)] == "LORA_OK"
    assert L.STATUS[L.lora_check_args(0, p, big + 1, 512, 512, 16)] == "LORA_ERR_SHAPE"
    assert L.STATUS[L.lora_check_args(0, p, 256, big, 512, 16)] == "LORA_OK"
    assert L.STATUS[L.lora_check_args(0, p, 256, big + 8, 512, 16)] == "LORA_ERR_SHAPE"
    assert L.STATUS[L.lora_check_args(0, p, 256, 512, big + 8, 16)] == "LORA_ERR_SHAPE"
    assert L.lora_bwd_workspace_size(big + 1, 512, 512, 16) == 0


def test_two_call_backward_validation(built_lib):
    """lora_bwd_grads / lora_bwd_dx refuse bad arguments on the host before
    any CUDA call (the pointers are never dereferenced)."""
    L = built_lib
    so = L.lib()
    M, d_in, d_out, r = 256, 512, 512, 16
    need = L.lora_bwd_workspace_size(M, d_in, d_out, r)
    X, A, B, dY, dA, dB, W, dX = _ptrs(8)
    ws = ALIGNED + (20 << 32)
    c = lambda *a: L.STATUS[so.lora_bwd_grads(*[ctypes.c_void_p(x) if isinstance(x, int) and x > 1 << 20 else x
                                                  for x in a])]
    f = ctypes.c_float(32.0)
    assert c(X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need, 4, None) == "LORA_ERR_FLAGS"
    assert c(X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need - 256, L.LORA_BWD_T_SAVED,
             None) == "LORA_ERR_WORKSPACE"
    assert c(X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need - 256, 0, None) == "LORA_ERR_WORKSPACE"
    assert c(X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws + 16, need, 0, None) == "LORA_ERR_ALIGN"
    assert c(X, A, B, dY, dA, dB, M, d_in, d_out, 12, f, ws, need, 0, None) == "LORA_ERR_RANK"
    assert c(X, A, B, dY, X + 16, dB, M, d_in, d_out, r, f, ws, need, 0, None) == "LORA_ERR_ALIAS"
    assert c(X, A, B, dY, dA, dA, M, d_in, d_out, r, f, ws, need, 0, None) == "LORA_ERR_ALIAS"
    assert c(0, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need, 0, None) == "LORA_ERR_NULL"
    d = lambda *a: L.STATUS[so.lora_bwd_dx(*[ctypes.c_void_p(x) if isinstance(x, int) and x > 1 << 20 else x
                                               for x in a])]
    assert d(W, A, dY, dX, M, d_in, d_out, r, ws, 0, None) == "LORA_ERR_WORKSPACE"
    assert d(W, A, dY, ws + 256, M, d_in, d_out, r, ws, need, None) == "LORA_ERR_ALIAS"   # dX inside the workspace
    assert d(W, A, dY, W, M, d_in, d_out, r, ws, need, None) == "LORA_ERR_ALIAS"
    assert d(W, A, dY, dX + 8, M, d_in, d_out, r, ws, need, None) == "LORA_ERR_ALIGN"
    assert d(0, A, dY, dX, M, d_in, d_out, r, ws, need, None) == "LORA_ERR_NULL"


def test_fwd_save_validation(built_lib):
    """lora_fwd_save applies lora_fwd's rules plus the workspace rules of the
    backward, and refuses a workspace that overlaps an input or Y, all on the
    host before any CUDA call (the pointers are never dereferenced)."""
    L = built_lib
    so = L.lib()
    M, d_in, d_out, r = 256, 512, 512, 16
    need = L.lora_bwd_workspace_size(M, d_in, d_out, r)
    X, W, A, B, Y = _ptrs(5)
    ws = ALIGNED + (20 << 32)
    c = lambda *a: L.STATUS[so.lora_fwd_save(*[ctypes.c_void_p(x) if isinstance(x, int) and x > 1 << 20 else x
                                                 for x in a])]
    f = ctypes.c_float(32.0)
    assert c(X, W, A, B, Y, M, d_in, d_out, r, f, None, need, None) == "LORA_ERR_WORKSPACE"
    assert c(X, W, A, B, Y, M, d_in, d_out, r, f, ws, need - 1, None) == "LORA_ERR_WORKSPACE"
    assert c(X, W, A, B, Y, M, d_in, d_out, r, f, ws + 16, need, None) == "LORA_ERR_ALIGN"
    for p in (X, W, A, B, Y):                    # the workspace starts inside each operand in turn
        assert c(X, W, A, B, Y, M, d_in, d_out, r, f, p, need, None) == "LORA_ERR_ALIAS"
    # lora_fwd's own rules come first
    assert c(X, W, A, B, 0, M, d_in, d_out, r, f, ws, need, None) == "LORA_ERR_NULL"
    assert c(X, W, A, B, Y, M, d_in, d_out, 12, f, ws, need, None) == "LORA_ERR_RANK"
    assert c(X, W, A, B, X, M, d_in, d_out, r, f, ws, need, None) == "LORA_ERR_ALIAS"


def _header_structs(path):
    """{typedef name: [(field, C type)]} for the plain structs of the header
    (comments removed; several names in one declaration allowed)."""
    text = re.sub(r"/\*.*?\*/", " ", open(path).read(), flags=re.S)
    out = {}
    for body, name in re.findall(r"typedef struct \{(.*?)\}\s*(\w+)\s*;", text, flags=re.S):
        fields = []
        for decl in body.split(";"):
            decl = " ".join(decl.split())
            if not decl:
                continue
            m = re.match(r"((?:const )?[a-z0-9_]+\s*\*?)\s*(.*)", decl)
            ctype = m.group(1).replace(" ", "")
            for n in m.group(2).split(","):
                n = n.strip()
                if n.startswith("*"):
                    ctype, n = ctype + "*", n[1:]
                fields.append((n, ctype))
        out[name] = fields
    return out


def test_ctypes_structs_mirror_the_header(built_lib):
    """The binding's ctypes structures have the header structs' fields, in
    order, with matching types (a mismatch would corrupt every call)."""
    L = built_lib
    c = {"constvoid*": ctypes.c_void_p, "void*": ctypes.c_void_p, "int64_t": ctypes.c_int64,
         "int32_t": ctypes.c_int32, "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64}
    structs = _header_structs(L.HEADER_PATH)
    for cname, cls in (("lora_fwd_desc_t", L._FwdDesc), ("lora_merge_desc_t", L._MergeDesc),
                       ("lora_plan_t", L._Plan)):
        want = [(n, c[t]) for n, t in structs[cname]]
        assert [(n, t) for n, t in cls._fields_] == want, cname
    assert ctypes.sizeof(L._Plan) == 96 and ctypes.sizeof(L._FwdDesc) == 64 and ctypes.sizeof(L._MergeDesc) == 48


def _call(so, name, *args):
    return int(getattr(so, name)(*args))


@pytest.mark.parametrize("M,d_in,d_out,r,ptr_fix", [
    (256, 512, 512, 16, None),            # valid: both reach the device step (no GPU here)
    (-1, 512, 512, 16, None),             # bad size
    (256, 516, 512, 16, None),
    (256, 512, 512, 12, None),            # bad rank
    (256, 512, 512, 16, ("null", 1)),     # NULL W
    (256, 512, 512, 16, ("odd", 2)),      # A not 16-byte aligned
    (256, 512, 512, 16, ("alias", 4)),    # Y on top of X
])
def test_scaled_forms_apply_the_alpha_forms_rules(built_lib, M, d_in, d_out, r, ptr_fix):
    """Each *_scaled entry point takes `scale` where its alpha form takes
    alpha and otherwise validates exactly the same way: the same status for
    valid and invalid arguments (fake pointers, never dereferenced; on a
    machine without a GPU a valid call stops at the device check)."""
    L = built_lib
    so = L.lib()
    p = _ptrs(10)
    if ptr_fix is not None:
        kind, i = ptr_fix
        p[i] = 0 if kind == "null" else (p[i] + 8 if kind == "odd" else p[0])
    X, W, A, B, Y, dY, dX, dA, dB, ws = (ctypes.c_void_p(v) for v in p)
    f = ctypes.c_float(32.0)
    need = L.lora_bwd_workspace_size(max(M, 0), d_in, d_out, r) if M >= 0 and r in (8, 16, 128) else 1 << 20
    pairs = [
        (("lora_fwd", X, W, A, B, Y, M, d_in, d_out, r, f, None),
         ("lora_fwd_scaled", X, W, A, B, Y, M, d_in, d_out, r, f, None)),
        (("lora_fwd_save", X, W, A, B, Y, M, d_in, d_out, r, f, ws, need, None),
         ("lora_fwd_save_scaled", X, W, A, B, Y, M, d_in, d_out, r, f, ws, need, None)),
        (("lora_bwd_ex", X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, f, ws, need, 0, None),
         ("lora_bwd_scaled", X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, f, ws, need, 0, None)),
        (("lora_bwd_grads", X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need, 0, None),
         ("lora_bwd_grads_scaled", X, A, B, dY, dA, dB, M, d_in, d_out, r, f, ws, need, 0, None)),
        (("lora_merge", W, A, B, Y, d_out, d_in, r, f, None),
         ("lora_merge_scaled", W, A, B, Y, d_out, d_in, r, f, None)),
    ]
    for a, b in pairs:
        ca, cb = _call(so, *a), _call(so, *b)
        assert ca == cb, (a[0], L.STATUS.get(ca), b[0], L.STATUS.get(cb))
    # an unknown flag bit is refused by the scaled backward as by lora_bwd_ex
    assert L.STATUS[_call(so, "lora_bwd_scaled", X, W, A, B, dY, dX, dA, dB, 256, 512, 512, 16, f, ws,
                          1 << 26, 1 << 7, None)] == "LORA_ERR_FLAGS"


def test_scaled_batched_forms_apply_the_alpha_forms_rules(built_lib):
    L = built_lib
    so = L.lib()
    p = _ptrs(12)
    f = ctypes.c_float(2.0)
    fwd = (L._FwdDesc * 2)(L._FwdDesc(*p[0:5], 256, 512, 512), L._FwdDesc(*p[5:10], 128, 512, 520))
    mrg = (L._MergeDesc * 2)(L._MergeDesc(*p[0:4], 512, 512), L._MergeDesc(*p[4:8], 100, 512))  # bad d_out
    for n in (0, 1, 2, -1):
        assert _call(so, "lora_fwd_batched", fwd, n, 16, f, None) == _call(so, "lora_fwd_batched_scaled", fwd, n, 16,
                                                                              f, None)
        assert _call(so, "lora_merge_batched", mrg, n, 16, f, None) == _call(so, "lora_merge_batched_scaled", mrg,
                                                                              n, 16, f, None)
    assert L.STATUS[_call(so, "lora_merge_batched_scaled", mrg, 2, 16, f, None)] == "LORA_ERR_SHAPE"
    assert L.STATUS[_call(so, "lora_fwd_batched_scaled", fwd, 2, 12, f, None)] == "LORA_ERR_RANK"
