"""C ABI checks that need no GPU: the library loads, exports every entry point that
include/sas.h declares, builds the gate rotary tables on the host, and rejects bad
arguments with a status code and a reason before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "gated_block_sparse_sas_b200", "libsas_b200.so")


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(sas_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def sas():
    if not os.path.exists(LIB):
        import __graft_entry__
        __graft_entry__.build()
    import gated_block_sparse_sas_b200 as m
    return m


def test_every_declared_symbol_is_exported(sas):
    lib = ctypes.CDLL(LIB)
    names = _declared()
    assert len(names) >= 12, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_rope_tables_host(sas):
    c, s = sas.rope_tables(1000, 32, 1e6)
    i = np.arange(16)
    ang = np.arange(1000)[:, None] * (1e6 ** (-2.0 * i / 32))[None, :]
    np.testing.assert_allclose(c, np.cos(ang).astype(np.float32), rtol=0, atol=1.2e-7)
    np.testing.assert_allclose(s, np.sin(ang).astype(np.float32), rtol=0, atol=1.2e-7)
    with pytest.raises(sas.SasError) as e:
        sas.rope_tables(10, 31)
    assert e.value.status == sas.SAS_ERR_INVALID_ARG


def _prob(sas, **kw):
    base = dict(batch=1, total_tokens=128, max_seqlen=128, num_q_heads=8, num_kv_heads=2,
                head_dim=128, block=64, topk=3, gate_hidden=128, rms_eps=1e-6, dtype=sas.SAS_BF16,
                cu_seqlens=0x1000, gate_rope_cos=0x2000, gate_rope_sin=0x3000)
    base.update(kw)
    return sas.SasProblem(**base)


def _call_pool(sas, prob, k=0x10000, out=0x20000):
    lib = sas.lib_handle()
    return lib.sas_pool_keys(ctypes.byref(prob), k, out, None), lib.sas_last_error().decode()


@pytest.mark.parametrize("field,value,status,frag", [
    ("head_dim", 96, -2, "head_dim"),
    ("block", 48, -2, "block"),
    ("num_q_heads", 5, -1, "multiple"),
    ("num_q_heads", 6 * 2 * 3, -2, "per KV head"),
    ("gate_hidden", 100, -2, "gate_hidden"),
    ("topk", 0, -1, "topk"),
    ("batch", 0, -1, "batch"),
    ("cu_seqlens", None, -1, "cu_seqlens"),
    ("max_seqlen", 64 * 4096, -2, "blocks"),
    ("gate_heads", 3, -1, "gate_heads"),
])
def test_invalid_problem_rejected(sas, field, value, status, frag):
    p = _prob(sas, **{field: value})
    st, msg = _call_pool(sas, p)
    assert st == status and frag in msg, (st, msg)


def test_null_and_misaligned_pointers(sas):
    p = _prob(sas)
    st, msg = _call_pool(sas, p, k=0)
    assert st == sas.SAS_ERR_INVALID_ARG and "NULL" in msg
    st, msg = _call_pool(sas, p, k=0x10008)
    assert st == sas.SAS_ERR_INVALID_ARG and "aligned" in msg
    lib = sas.lib_handle()
    assert lib.sas_pool_keys(None, 0x10000, 0x20000, None) == sas.SAS_ERR_INVALID_ARG


def test_workspace_sizes_and_shortfall(sas):
    lib = sas.lib_handle()
    p = _prob(sas)
    n = ctypes.c_size_t(0)
    assert lib.sas_attn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    assert n.value >= 128 * 8 * 4
    ptrs = [0x10000 + 0x100 * i for i in range(12)]
    st = lib.sas_attn_bwd(ctypes.byref(p), *ptrs, 0x90000, 16, None)
    assert st == sas.SAS_ERR_WORKSPACE and "workspace" in lib.sas_last_error().decode()
    d = sas.SasDecodeProblem(batch=4, capacity=4096, num_q_heads=32, num_kv_heads=8, head_dim=128,
                             block=64, topk=31, gate_hidden=128, rms_eps=1e-6, dtype=sas.SAS_BF16,
                             seqlens=0x1000, gate_rope_cos=0x2000, gate_rope_sin=0x3000)
    assert lib.sas_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    assert n.value >= 4 * 8 * 32 * 8
    d.num_q_heads = 30
    assert lib.sas_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)) == sas.SAS_ERR_INVALID_ARG


def test_empty_problem_is_a_no_op(sas):
    """T = 0: validated, nothing launched (no GPU needed)."""
    lib = sas.lib_handle()
    p = _prob(sas, total_tokens=0)
    ptrs = [0x10000 + 0x100 * i for i in range(8)]
    assert lib.sas_attn_fwd(ctypes.byref(p), *ptrs[:7], 0x90000, 256, None) == 0
    assert lib.sas_topk(ctypes.byref(p), *ptrs[:4], None) == 0


def test_binding_argument_counts_match_the_header(sas):
    """Every ctypes signature of the binding takes as many arguments as include/sas.h
    declares (a mismatch would pass a wrong stream or size without any error)."""
    import re
    src = open(os.path.join(ROOT, "include", "sas.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = dict(re.findall(r"\b(sas_\w+)\s*\(([^)]*)\)\s*;", src))
    assert decls, "no declarations parsed"
    for name, (args, _res) in sas._SIGS.items():
        params = decls[name].strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert n == len(args), f"{name}: header {n} parameters, binding {len(args)}"


def test_gate_bwd_argument_checks(sas):
    """Router backward: NULL outputs and unsupported shapes are rejected before any launch."""
    lib = sas.lib_handle()
    p = _prob(sas)
    ptrs = [0x10000 + 0x100 * i for i in range(13)]
    ptrs[12] = 0   # dknorm_w
    st = lib.sas_gate_bwd(ctypes.byref(p), *ptrs, 0x90000, 1 << 30, None)
    assert st == sas.SAS_ERR_INVALID_ARG and "NULL" in lib.sas_last_error().decode()
    n = ctypes.c_size_t(0)
    p32 = _prob(sas, dtype=sas.SAS_FP32)
    assert lib.sas_gate_bwd_workspace_size(ctypes.byref(p32), ctypes.byref(n)) == sas.SAS_ERR_UNSUPPORTED
    assert "gate_bwd" in lib.sas_last_error().decode()


def test_decode_ungated_flag_is_checked(sas):
    lib = sas.lib_handle()
    n = ctypes.c_size_t(0)
    d = sas.SasDecodeProblem(batch=4, capacity=4096, num_q_heads=32, num_kv_heads=8, head_dim=128,
                             block=64, topk=31, gate_hidden=128, rms_eps=1e-6, dtype=sas.SAS_BF16,
                             seqlens=0x1000, gate_rope_cos=0x2000, gate_rope_sin=0x3000, ungated=1)
    assert lib.sas_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    d.ungated = 2
    assert lib.sas_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)) == sas.SAS_ERR_INVALID_ARG
    assert "ungated" in lib.sas_last_error().decode()
