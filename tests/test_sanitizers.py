"""Host code under AddressSanitizer and UndefinedBehaviorSanitizer (CPU).

The C oracle and the native block manager (plain C++, no CUDA) are rebuilt with
-fsanitize=address,undefined in a temporary directory and driven from a child Python process with the
ASan runtime preloaded: every oracle operation on small ragged cases (decode attention in all cache
formats, prefill over 16-bit and per-block FP8 caches, reshape_and_cache, copy_blocks, swap_blocks, the codecs), and a seeded block-manager
session checked call by call against the manager's oracle. Any out-of-bounds access, use after free or
undefined behaviour aborts the child.
"""
import os
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r'''
    import ctypes, sys
    import numpy as np
    sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
    import oracle
    from helpers import random_paged_case, bits16
    from oracle.block_manager import BlockManagerOracle, OracleBlockError
    import torch

    with oracle.use_library(ORACLE_SO):
        rng = np.random.default_rng(0)
        for kvd in ("bf16", "fp8_e4m3", "fp8_e4m3_block"):
            inputs, q, _, _ = random_paged_case(rng, [1, 9, 40], 8, 2, 32, 8, "bf16")
            NB, Hkv = inputs["key_cache"].shape[0], 2
            if kvd != "bf16":
                ks = np.full((NB, Hkv) if kvd.endswith("block") else (Hkv,), 0.01, np.float32)
                quant = oracle.quantize_e4m3_blocks if kvd.endswith("block") else oracle.quantize_e4m3
                kc = quant(inputs["key_cache"], "bf16", ks)
                vc = quant(inputs["value_cache"], "bf16", ks)
                inputs = dict(inputs, key_cache=kc, value_cache=vc, kv_dtype=kvd, k_scale=ks, v_scale=ks)
            oracle.paged_attention(scale=0.2, **inputs)
        inputs, q, _, _ = random_paged_case(rng, [17, 30], 4, 2, 16, 4, "bf16")
        qp = bits16(torch.randn(20, 4, 16).to(torch.bfloat16))
        oracle.paged_prefill(qp, "bf16", inputs["key_cache"], inputs["value_cache"], "bf16", inputs["block_tables"],
                             inputs["context_lens"], np.array([0, 10, 20], np.int32), 0.3)
        NBp = inputs["key_cache"].shape[0]
        bsc = np.full((NBp, 2), 0.01, np.float32)
        oracle.paged_prefill(qp, "bf16", oracle.quantize_e4m3_blocks(inputs["key_cache"], "bf16", bsc),
                             oracle.quantize_e4m3_blocks(inputs["value_cache"], "bf16", bsc), "fp8_e4m3_block",
                             inputs["block_tables"], inputs["context_lens"], np.array([0, 10, 20], np.int32), 0.3,
                             k_scale=bsc, v_scale=bsc)
        kc = inputs["key_cache"].copy(); vc = inputs["value_cache"].copy()
        NB = kc.shape[0]
        x = bits16(torch.randn(5, 2, 16).to(torch.bfloat16))
        oracle.reshape_and_cache(x, x, "bf16", kc, vc, "bf16", np.array([0, -1, 7, NB * 4 - 1, NB * 4], np.int64))
        oracle.copy_blocks(kc, vc, "bf16", np.array([[0, 1], [2, 3]], np.int64))
        hk = np.zeros((3,) + kc.shape[1:], kc.dtype); hv = np.zeros_like(hk)
        oracle.swap_blocks(hk, hv, kc, vc, "bf16", np.array([[1, 0], [3, 2]], np.int64))
        oracle.e4m3_from_float(np.linspace(-500, 500, 1001).astype(np.float32))

    bm = ctypes.CDLL(BM_SO)
    p, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    h = p()
    assert bm.pa_bm_create(24, 4, 12, ctypes.byref(h)) == 0
    ref = BlockManagerOracle(24, 4, 12)
    rng = np.random.default_rng(1)
    ids = []
    for step in range(300):
        op = rng.integers(5)
        live = sorted(ref.tables)
        try:
            if op == 0:
                n = int(rng.integers(0, 12)); sid = len(ids); ids.append(sid)
                slots = np.empty(max(n, 1), np.int64); k = ctypes.c_int64()
                st = bm.pa_bm_add_sequence(h, i64(sid), i64(n), i64(-1), i64(0), p(slots.ctypes.data), i64(n), ctypes.byref(k))
                try:
                    want = ref.add_sequence(sid, n); assert st == 0 and slots[:k.value].tolist() == want
                except OracleBlockError:
                    assert st != 0
            elif op == 1 and live:
                sel = np.array(live[:int(rng.integers(1, len(live) + 1))], np.int64)
                slots = np.empty(len(sel), np.int64); pairs = np.empty((len(sel), 2), np.int64); k = ctypes.c_int()
                st = bm.pa_bm_append_slots(h, p(sel.ctypes.data), i(len(sel)), p(slots.ctypes.data), p(pairs.ctypes.data), ctypes.byref(k))
                try:
                    s_, pr = ref.append_slots(sel.tolist()); assert st == 0 and slots.tolist() == s_
                except OracleBlockError:
                    assert st != 0
            elif op == 2 and live:
                sid = len(ids); ids.append(sid)
                st = bm.pa_bm_fork(h, i64(live[0]), i64(sid)); ref.fork(live[0], sid); assert st == 0
            elif op == 3 and live:
                v = live[int(rng.integers(len(live)))]
                assert bm.pa_bm_free_sequence(h, i64(v)) == 0; ref.free_sequence(v)
            elif op == 4 and live:
                v = live[int(rng.integers(len(live)))]
                m = np.empty((16, 2), np.int64); k = ctypes.c_int()
                st = bm.pa_bm_swap_out(h, i64(v), p(m.ctypes.data), i(16), ctypes.byref(k))
                try:
                    want = ref.swap_out(v); assert st == 0 and [tuple(r) for r in m[:k.value].tolist()] == want
                except OracleBlockError:
                    assert st != 0
        except AssertionError:
            raise
    tables = np.empty((len(ref.tables), 8), np.int32); lens = np.empty(max(len(ref.tables), 1), np.int32)
    sel = np.array(sorted(ref.tables), np.int64)
    if len(sel):
        bm.pa_bm_block_tables(h, p(sel.ctypes.data), i(len(sel)), p(tables.ctypes.data), i(8), ctypes.c_int32(-1), p(lens.ctypes.data))
    bm.pa_bm_destroy(h)
    print("sanitized run ok")
''')


def test_oracle_and_block_manager_under_asan_and_ubsan(tmp_path):
    asan = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    if not asan or not os.path.exists(asan):
        pytest.skip("no ASan runtime on this host")
    flags = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer", "-g", "-O1",
             "-fPIC", "-shared"]
    oracle_so = tmp_path / "liboracle_asan.so"
    bm_so = tmp_path / "libbm_asan.so"
    subprocess.run(["gcc", "-std=c11", *flags, "-pthread", "-o", str(oracle_so),
                    os.path.join(ROOT, "oracle", "pa_oracle.c"), "-lm"], check=True)
    subprocess.run(["g++", "-std=c++17", *flags, "-I", os.path.join(ROOT, "include"), "-o", str(bm_so),
                    os.path.join(ROOT, "pagedattention_paged_kv_attention_b200", "csrc", "pa_block_manager.cpp")],
                   check=True)
    script = tmp_path / "child.py"
    script.write_text(f"ROOT = {ROOT!r}\nORACLE_SO = {str(oracle_so)!r}\nBM_SO = {str(bm_so)!r}\n" + CHILD)
    env = dict(os.environ, LD_PRELOAD=asan, ASAN_OPTIONS="detect_leaks=0:abort_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([sys.executable, str(script)], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0 and "sanitized run ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
