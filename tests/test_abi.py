"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/lidx.h declares, agrees with the binding's struct layouts, and
rejects bad arguments synchronously (before touching a device)."""
import ctypes as C
import os
import re

import pytest

import lightning_indexer_top_index_b200 as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    hdr = open(os.path.join(ROOT, "include", "lidx.h")).read()
    return sorted(set(re.findall(r"LIDX_API\s+[\w\s\*]+?\b(lidx_\w+)\s*\(", hdr)))


@pytest.fixture(scope="module")
def lib():
    from lightning_indexer_top_index_b200 import build
    build.build()
    return L.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(L.EXPORTS) <= set(names)
    hdr = open(os.path.join(ROOT, "include", "lidx.h")).read()
    assert lib.lidx_abi_version() == int(re.search(r"#define LIDX_ABI_VERSION (\d+)", hdr).group(1))


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-x", "c", "-std=c11", "-pedantic"]),
                                            ("g++", ["-x", "c++", "-std=c++17"])])
def test_plain_c_consumer(lib, tmp_path, compiler, flags):
    """include/lidx.h compiles as strict C11 and as C++ without CUDA or torch
    headers, links against liblidx.so, and agrees with the library's struct
    layouts and host-only calls."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"no {compiler}")
    pkg = os.path.dirname(L.__file__)
    exe = str(tmp_path / "consumer")
    subprocess.run([compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_consumer.c"), "-x", "none", "-L", pkg, "-llidx",
                    f"-Wl,-rpath,{pkg}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "OK", r.stdout + r.stderr


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without liblidx.so every call raises: there is no fallback path."""
    import torch
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "liblidx.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(ImportError):
        L.lib()
    with pytest.raises(ImportError):
        L.topk_select(torch.zeros(1, 1, 8), 2)


def test_struct_sizes_match(lib):
    for i, s in enumerate(L._STRUCTS):
        assert lib.lidx_struct_size(i) == C.sizeof(s)
    assert C.sizeof(L.KVArgs) == 64


def test_status_strings(lib):
    for s in range(5):
        assert L.status_string(s)
    assert L.status_string(99) == "unknown status"


def _kv(dtype=L.BF16, dim=128, ld=128, data=0x1000, batch_rows=0):
    return L.KVArgs(dtype, dim, data, None, None, ld, 0, 0, batch_rows)


def test_score_argument_errors(lib):
    ok = L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(), 0x3000, 100)
    n = C.c_size_t(99)
    assert lib.lidx_workspace_size(L.OP_SCORE, C.byref(ok), C.byref(n)) == L.OK and n.value == 0
    bad = [
        L.ScoreArgs(1, 1, 64, 100, L.BF16, None, 0x2000, _kv(), 0x3000, 100),        # null q
        L.ScoreArgs(1, 1, 64, 0, L.BF16, 0x1000, 0x2000, _kv(), 0x3000, 100),        # N = 0
        L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(), 0x3000, 99),       # ld < N
        L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(ld=100), 0x3000, 100),  # ld*2 % 16
        L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(data=0x1004), 0x3000, 100),  # misaligned
        L.ScoreArgs(2, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(batch_rows=50), 0x3000, 100),  # rows overlap
    ]
    for a in bad:
        assert lib.lidx_index_score(C.byref(a), None) == L.ERR_INVALID_ARG
    f16 = L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(dtype=L.F16), 0x3000, 100)
    assert lib.lidx_index_score(C.byref(f16), None) == L.ERR_UNSUPPORTED
    mixed = L.ScoreArgs(1, 1, 64, 100, L.F32, 0x1000, 0x2000, _kv(), 0x3000, 100)
    assert lib.lidx_index_score(C.byref(mixed), None) == L.ERR_UNSUPPORTED
    dim = L.ScoreArgs(1, 1, 64, 100, L.BF16, 0x1000, 0x2000, _kv(dim=64), 0x3000, 100)
    assert lib.lidx_index_score(C.byref(dim), None) == L.ERR_UNSUPPORTED


def test_topk_argument_errors_and_workspace(lib):
    a = L.TopkArgs(2, 1, 1000, 64, 0x1000, 1000, None, 0, 0x2000, None, None, None)
    n = C.c_size_t(0)
    assert lib.lidx_workspace_size(L.OP_TOPK, C.byref(a), C.byref(n)) == L.OK and n.value >= 256
    assert lib.lidx_topk_select(C.byref(a), None, 0, None) == L.ERR_WORKSPACE
    for bad in [L.TopkArgs(2, 1, 1000, 0, 0x1000, 1000, None, 0, 0x2000, None, None, None),
                L.TopkArgs(2, 1, 1000, 64, None, 1000, None, 0, 0x2000, None, None, None),
                L.TopkArgs(2, 1, 1000, 64, 0x1000, 1000, 0x5000, 10, 0x2000, None, None, None)]:
        assert lib.lidx_topk_select(C.byref(bad), C.c_void_p(0x10000), 1 << 20, None) == L.ERR_INVALID_ARG


def test_attn_argument_errors_and_workspace(lib):
    kv = _kv(dim=512, ld=512)
    sw = _kv(dim=512, ld=512, data=0x8000)
    a = L.AttnArgs(1, 64, L.BF16, 0x1000, kv, 16384, 0x2000, 512, 512, None, sw, 128, 0.044, 0x3000, None)
    n = C.c_size_t(0)
    assert lib.lidx_workspace_size(L.OP_ATTN, C.byref(a), C.byref(n)) == L.OK and n.value > 256
    cnt = C.c_int(0)
    assert lib.lidx_launch_count(L.OP_ATTN, C.byref(a), C.byref(cnt)) == L.OK and cnt.value == 2
    assert lib.lidx_sparse_attn_decode(C.byref(a), None, 0, None) == L.ERR_WORKSPACE
    kv16 = _kv(dtype=L.F16, dim=512, ld=512)
    f16 = L.AttnArgs(1, 64, L.BF16, 0x1000, kv16, 16384, 0x2000, 512, 512, None, sw, 128, 0.044, 0x3000, None)
    assert lib.lidx_sparse_attn_decode(C.byref(f16), C.c_void_p(0x10000), 1 << 30, None) == L.ERR_UNSUPPORTED
    nan = L.AttnArgs(1, 64, L.BF16, 0x1000, kv, 16384, 0x2000, 512, 512, None, sw, 128, float("nan"), 0x3000, None)
    assert lib.lidx_sparse_attn_decode(C.byref(nan), C.c_void_p(0x10000), 1 << 30, None) == L.ERR_INVALID_ARG


def test_launch_count_arguments(lib):
    """lidx_launch_count runs the call's own argument checks; the score call
    is one kernel."""
    kv = _kv()
    a = L.ScoreArgs(1, 1, 64, 1000, L.BF16, 0x1000, 0x2000, kv, 0x3000, 1000, 0, None, None)
    n = C.c_int(-1)
    assert lib.lidx_launch_count(L.OP_SCORE, C.byref(a), C.byref(n)) == L.OK and n.value == 1
    bad = L.ScoreArgs(1, 1, 64, 0, L.BF16, 0x1000, 0x2000, kv, 0x3000, 1000, 0, None, None)
    assert lib.lidx_launch_count(L.OP_SCORE, C.byref(bad), C.byref(n)) == L.ERR_INVALID_ARG
    assert lib.lidx_launch_count(L.OP_SCORE, C.byref(a), None) == L.ERR_INVALID_ARG
    assert lib.lidx_launch_count(L.OP_SCORE, None, C.byref(n)) == L.ERR_INVALID_ARG
    assert lib.lidx_launch_count(99, C.byref(a), C.byref(n)) == L.ERR_INVALID_ARG
    t = L.TopkArgs(2, 1, 1000, 64, 0x1000, 1000, None, 0, 0x2000, None, None, None)
    assert lib.lidx_launch_count(L.OP_TOPK, C.byref(t), C.byref(n)) == L.OK and n.value == 1


def test_eval_argument_errors(lib):
    a = L.EvalArgs()
    a.ops = 0
    assert lib.lidx_selection_eval(C.byref(a), C.c_void_p(0x10000), 1 << 20, None) == L.ERR_INVALID_ARG
    a.ops = L.EVAL_TOPP
    a.N, a.L, a.T = 100, 1, 1
    a.probs, a.topp_bits = 0x1000, 0x2000
    a.top_p_num, a.top_p_den = 3, 0
    assert lib.lidx_selection_eval(C.byref(a), C.c_void_p(0x10000), 1 << 20, None) == L.ERR_INVALID_ARG


def test_schedule_constants():
    """21 CSA layers (even 2..42); gate layers 10/12/20 sit at CSA stack
    positions 4/5/9; 64K tokens at 4:1 give 16384 entries, of which 512 is
    about 3%; at 128:1 an HCA layer has 512 entries."""
    import json
    facts = json.load(open(os.path.join(ROOT, "tests", "golden", "page_facts.json")))
    assert len(L.CSA_LAYERS) == facts["csa_layer_count"]["value"] == 21
    assert L.GATE_LAYERS == (4, 5, 9)
    assert tuple(facts["gate_layers"]["value"]) == L.GATE_MODEL_LAYERS
    assert 65536 // facts["csa_layers"]["ratio"] == facts["csa_entries_at_64k"]["value"]
    assert abs(facts["top_k"]["value"] / 16384 - facts["top_k_share_at_64k"]["value"]) < 0.002
    assert 65536 // facts["hca_layers"]["ratio"] == facts["hca_entries_at_64k"]["value"]
    assert len(L.CSA_LAYERS) + len(L.HCA_LAYERS) + len(facts["swa_layers"]["value"]) == facts["model_layers"]["value"]


def test_logical_kv_size_at_64k():
    """The architecture post's ~871 MiB of KV at 64K: 21 CSA layers of 16384
    entries x (512 + 128) fp32, 20 HCA layers of 512 entries x 512, and a
    128-row window of 512 in each of the 43 layers."""
    import json
    facts = json.load(open(os.path.join(ROOT, "tests", "golden", "page_facts.json")))
    kv = L.logical_kv_bytes(65536)
    mib = 1 << 20
    assert kv["csa"] == 840 * mib
    assert kv["hca"] == 20 * mib
    assert kv["swa"] == 10.75 * mib
    assert abs(kv["total"] / mib - facts["kv_logical_mib_at_64k"]["value"]) < 0.5
    # entries per layer at 64K as the post gives them
    assert kv["csa"] // (len(L.CSA_LAYERS) * 640 * 4) == facts["csa_entries_at_64k"]["value"]
    assert kv["hca"] // (len(L.HCA_LAYERS) * 512 * 4) == facts["hca_entries_at_64k"]["value"]


def test_oracle_and_product_share_nothing():
    """The oracle and the CUDA path import / include nothing of each other."""
    pkg = os.path.join(ROOT, "lightning_indexer_top_index_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", txt, re.M), f
                assert "oracle.c" not in txt and "liboracle" not in txt, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            txt = open(os.path.join(ROOT, "oracle", f)).read()
            assert "lightning_indexer_top_index_b200" not in txt and "lidx.h" not in txt, f
