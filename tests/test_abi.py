"""The C-ABI library loads, exports every entry point include/lbca.h declares,
matches the header's struct layouts, and rejects bad arguments on the host
(before any CUDA call, so these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lbca.h")


@pytest.fixture(scope="module")
def L():
    from block_compressed_long_b200 import build
    build.build()
    from block_compressed_long_b200 import lbca
    return lbca


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lbca_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(L._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.ENTRY_POINTS)


def test_struct_layout_matches_header(L, tmp_path):
    prog = tmp_path / "sz.c"
    prog.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "lbca.h"\n'
                    'int main(void){printf("%zu %zu %zu %zu %zu\\n", sizeof(lbca_config), sizeof(lbca_cache),'
                    ' offsetof(lbca_config, rope_theta), offsetof(lbca_config, dtype),'
                    ' offsetof(lbca_cache, batch));return 0;}\n')
    exe = tmp_path / "sz"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [ctypes.sizeof(L.lbca_config), ctypes.sizeof(L.lbca_cache), L.lbca_config.rope_theta.offset,
            L.lbca_config.dtype.offset, L.lbca_cache.batch.offset]
    assert got == want


def _cfg(L, **kw):
    base = dict(n_q_heads=24, n_kv_heads=8, head_dim=128, shared_kv=False, block_m=64, n_win=128,
                rope_dims=128)
    base.update(kw)
    return L.config(**base)


def test_ring_slots(L):
    assert L.lbca_ring_slots(_cfg(L)) == 192                       # m=64, w=128
    assert L.lbca_ring_slots(_cfg(L, block_m=16)) == 144
    assert L.lbca_ring_slots(_cfg(L, n_q_heads=64, n_kv_heads=1, head_dim=512, shared_kv=True,
                                  block_m=128, rope_dims=64)) == 256
    assert L.lbca_ring_slots(_cfg(L, block_m=1, n_win=0)) == 1
    assert L.lbca_ring_slots(_cfg(L, block_m=0)) == -1


@pytest.mark.parametrize("bad", [dict(n_q_heads=25), dict(head_dim=100), dict(head_dim=1024),
                                 dict(block_m=0), dict(n_win=-1), dict(rope_dims=3),
                                 dict(rope_dims=256), dict(rope_theta=0.0)])
def test_bad_config_rejected(L, bad):
    cfg = _cfg(L, **bad)
    A = 0x10000
    st = L._lib.lbca_pool(ctypes.byref(cfg), 0, A, A, A, None, 1, 64, 0, A, 1, None)
    assert st == L.LBCA_ERR_ARG


def test_pool_argument_checks(L):
    cfg = _cfg(L)
    A = 0x10000
    f = lambda *a: L._lib.lbca_pool(ctypes.byref(cfg), *a)  # noqa: E731
    assert f(0, None, A, A, None, 1, 64, 0, A, 1, None) == L.LBCA_ERR_ARG        # null x
    assert f(0, A, A, A, None, 1, 64, 3, A, 8, None) == L.LBCA_ERR_ARG           # pos0 % m
    assert f(0, A, A, A, None, 1, 640, 0, A, 9, None) == L.LBCA_ERR_ARG          # out_blocks too small
    assert f(0, A + 8, A, A, None, 1, 64, 0, A, 1, None) == L.LBCA_ERR_ALIGN     # misaligned
    assert f(7, A, A, A, None, 1, 64, 0, A, 1, None) == L.LBCA_ERR_ARG           # series
    shared = _cfg(L, n_q_heads=4, n_kv_heads=1, shared_kv=True)
    assert L._lib.lbca_pool(ctypes.byref(shared), 1, A, A, A, None, 1, 64, 0, A, 1, None) == L.LBCA_ERR_ARG
    # a valid call with no GPU present must not succeed: there is no CPU fallback
    assert f(0, A, A, A, None, 1, 64, 0, A, 1, None) in (L.LBCA_ERR_CUDA, L.LBCA_ERR_UNSUPPORTED)
    g = lambda *a: L._lib.lbca_pool_f32(ctypes.byref(cfg), *a)  # noqa: E731
    assert g(0, A, A, A, None, 1, 64, 0, None, 1, None) == L.LBCA_ERR_ARG          # null out
    assert g(0, A, A, A, None, 1, 640, 0, A, 9, None) == L.LBCA_ERR_ARG            # out_blocks too small
    assert g(0, A, A, A, None, 1, 64, 0, A + 4, 1, None) == L.LBCA_ERR_ALIGN       # misaligned out
    assert g(0, A, A, A, None, 1, 64, 0, A, 1, None) in (L.LBCA_ERR_CUDA, L.LBCA_ERR_UNSUPPORTED)
    # both series in one call: k, v, zk, zv, b_pos_k, b_pos_v, gamma, B, T, pos0, pooled_k, pooled_v, out_blocks
    h = lambda *a: L._lib.lbca_pool_kv(ctypes.byref(cfg), *a)  # noqa: E731
    assert h(A, None, A, A, A, A, None, 1, 64, 0, A, A, 1, None) == L.LBCA_ERR_ARG      # null v
    assert h(A, A, A, A, A, A, None, 1, 64, 0, A, None, 1, None) == L.LBCA_ERR_ARG      # null pooled_v
    assert h(A, A, A, A, A, A, None, 1, 64, 3, A, A, 8, None) == L.LBCA_ERR_ARG         # pos0 % m
    assert h(A, A, A, A, A, A, None, 1, 640, 0, A, A, 9, None) == L.LBCA_ERR_ARG        # out_blocks too small
    assert h(A, A, A, A, A + 8, A, None, 1, 64, 0, A, A, 1, None) == L.LBCA_ERR_ALIGN   # misaligned b_pos_k
    assert h(A, A, A, A, A, A, None, 1, 64, 0, A, A + 4, 1, None) == L.LBCA_ERR_ALIGN   # misaligned pooled_v
    assert L._lib.lbca_pool_kv(ctypes.byref(shared), A, A, A, A, A, A, None, 1, 64, 0, A, A, 1,
                               None) == L.LBCA_ERR_ARG                                   # no value series
    assert h(A, A, A, A, A, A, None, 1, 64, 0, A, A, 1, None) in (L.LBCA_ERR_CUDA, L.LBCA_ERR_UNSUPPORTED)


def test_cache_and_decode_checks(L):
    cfg = _cfg(L)
    A = 0x10000
    cache = L.lbca_cache(A, A, A, A, A, A, 1, 600, 192, 0)
    small = L.lbca_cache(A, A, A, A, A, A, 1, 600, 100, 0)
    shared_bad = L.lbca_cache(A, None, A, None, A, A, 1, 600, 192, 0)
    ws = L.lbca_decode_workspace_bytes(cfg, 1, 32769)
    assert ws > 0
    dec = lambda c, wsb: L._lib.lbca_decode(ctypes.byref(cfg), A, ctypes.byref(c), None, None, None, 32769,  # noqa
                                            A, A, wsb, None, None)
    assert dec(small, ws) == L.LBCA_ERR_CAPACITY          # ring too small for the window
    assert dec(shared_bad, ws) == L.LBCA_ERR_ARG          # GQA needs pooled_v / ring_v
    assert dec(cache, ws - 1) == L.LBCA_ERR_CAPACITY      # workspace too small
    assert dec(cache, ws) in (L.LBCA_ERR_CUDA, L.LBCA_ERR_UNSUPPORTED)
    app = L._lib.lbca_append(ctypes.byref(cfg), A, None, A, A, A, A, None, ctypes.byref(cache), None, None)
    assert app == L.LBCA_ERR_ARG                          # GQA needs v
    pre = L._lib.lbca_prefill(ctypes.byref(cfg), A, A, A, A, A, A, A, None, None, None, 1, 64, None, None,
                              None, 0, None, None)
    assert pre == L.LBCA_ERR_ARG                          # neither out nor cache
    pre = L._lib.lbca_prefill(ctypes.byref(cfg), A, A, A, A, A, A, A, None, None, None, 1, 6400, A, None,
                              None, 0, None, None)
    assert pre == L.LBCA_ERR_CAPACITY                     # pooled entries need a workspace


def test_decode_step_launches(L):
    """One fused kernel for the GQA step shapes and for the shared-entry
    D = 512 form with one kv head; append + decode for two kv heads of that
    form and for no window; -1 for a bad config."""
    assert L.lbca_decode_step_launches(_cfg(L), 1, 32769) == 1
    assert L.lbca_decode_step_launches(_cfg(L, n_win=0), 1, 32769) == 2
    hca = _cfg(L, n_q_heads=64, n_kv_heads=1, head_dim=512, shared_kv=True, block_m=128, rope_dims=64)
    assert L.lbca_decode_step_launches(hca, 8, 131073) == 1
    assert L.lbca_decode_step_launches(_cfg(L, n_q_heads=128, n_kv_heads=2, head_dim=512, shared_kv=True,
                                            block_m=128, rope_dims=64), 8, 131073) == 2
    assert L.lbca_decode_step_launches(_cfg(L, block_m=0), 1, 100) == -1


def test_decode_step_form(L):
    """A few (sequence, head group) pairs take the cluster kernel, many (the
    32-sequence ragged batch: 256 pairs) the persistent evenly split one; the
    persistent form's workspace grows with the longest context it may meet."""
    cfg = _cfg(L)
    assert L.lbca_decode_step_form(cfg, 1, 32769) == L.LBCA_STEP_CLUSTER
    assert L.lbca_decode_step_form(cfg, 32, 65600) == L.LBCA_STEP_PERSISTENT
    assert L.lbca_decode_step_form(_cfg(L, n_win=0), 32, 65600) == L.LBCA_STEP_TWO_CALLS
    hca = _cfg(L, n_q_heads=64, n_kv_heads=1, head_dim=512, shared_kv=True, block_m=128, rope_dims=64)
    assert L.lbca_decode_step_form(hca, 8, 131073) == L.LBCA_STEP_SHARED_TC
    assert L.lbca_decode_step_form(_cfg(L, n_q_heads=64, n_kv_heads=1, head_dim=512, shared_kv=True, block_m=128,
                                        rope_dims=64, n_win=0), 8, 131073) == L.LBCA_STEP_TWO_CALLS
    assert L.lbca_decode_step_form(_cfg(L, block_m=0), 32, 100) == -1
    small = L.lbca_decode_step_workspace_bytes(cfg, 32, 4096)
    big = L.lbca_decode_step_workspace_bytes(cfg, 32, 65600)
    assert 0 < small < big


def test_shared_entry_step_forms(L):
    """The fused tensor-core step takes the shared-entry form with 64 query
    heads per kv head, one kv head, D 256 or 512, bf16 and a raw window;
    other shared-entry shapes run the two calls (the CUDA-core fused forms
    serve the GQA form only).  Its workspace query returns a small positive
    size (it uses none)."""
    hca = dict(n_q_heads=64, n_kv_heads=1, head_dim=512, shared_kv=True, block_m=128, rope_dims=64, n_win=128)
    assert L.lbca_decode_step_form(_cfg(L, **hca), 8, 131073) == L.LBCA_STEP_SHARED_TC
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, head_dim=256)), 8, 131073) == L.LBCA_STEP_SHARED_TC
    assert 0 < L.lbca_decode_step_workspace_bytes(_cfg(L, **hca), 8, 131073) <= 4096
    # not the tensor-core shape: 48 heads per kv head, f32, D = 128
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, n_q_heads=48)), 8, 131073) != L.LBCA_STEP_SHARED_TC
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, dtype="f32")), 8, 131073) != L.LBCA_STEP_SHARED_TC
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, head_dim=128)), 8, 131073) == L.LBCA_STEP_TWO_CALLS
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, n_q_heads=4, head_dim=128)), 32, 4096) == L.LBCA_STEP_TWO_CALLS
    # a list longer than 16 CTAs x 128 rows can hold: no tensor-core plan at all
    assert L.lbca_decode_step_form(_cfg(L, **dict(hca, block_m=16)), 1, 131073) != L.LBCA_STEP_SHARED_TC


def test_status_strings(L):
    for s in range(7):
        assert L.lbca_status_string(s)


def test_every_binding_wrapper_reaches_the_library(L, monkeypatch):
    """Each Python wrapper marshals its arguments into the C entry point it
    names: called with host tensors (no GPU here) it must come back with a
    library status, never with a ctypes arity or type error.  Every wrapper
    of the binding is among the calls."""
    import inspect
    import re

    import torch
    reached = set()
    check = L._check

    def record(fn, st):
        reached.add(fn)
        return check(fn, st)

    monkeypatch.setattr(L, "_check", record)
    cfg = L.config(4, 2, 32, False, 4, 8, rope_dims=8)
    hca = L.config(64, 1, 256, True, 4, 8, rope_dims=8, rmsnorm=True)
    q = torch.zeros(1, 8, 4, 32)
    kv = torch.zeros(1, 8, 2, 32)
    tok = torch.zeros(1, 2, 32)
    bp = torch.zeros(4, 64)
    q1 = torch.zeros(1, 4, 32)
    ws = torch.zeros(4096, dtype=torch.uint8)
    st = torch.zeros(1, dtype=torch.int32)
    cache = L.Cache(cfg, 1, 2, L.lbca_ring_slots(cfg), torch.zeros(1, 2, 2, 32), torch.zeros(1, 2, 2, 32),
                    torch.zeros(1, 2, 12, 32), torch.zeros(1, 2, 12, 32), torch.zeros(L.lbca_pool_state_elems(cfg, 1)),
                    torch.zeros(1, dtype=torch.int32))
    hcache = L.Cache(hca, 1, 2, L.lbca_ring_slots(hca), torch.zeros(1, 1, 2, 256), None, torch.zeros(1, 1, 12, 256),
                     None, torch.zeros(L.lbca_pool_state_elems(hca, 1)), torch.zeros(1, dtype=torch.int32))
    grads = {n: torch.zeros(1) for n in ("dq", "dk", "dv", "dzk", "dzv", "dbk", "dbv")}
    bws = torch.zeros(L.lbca_prefill_backward_workspace_bytes(cfg, 1, 8), dtype=torch.uint8)
    calls = [
        lambda: L.lbca_pool(cfg, 0, kv, kv, bp, None, torch.zeros(1, 2, 2, 32)),
        lambda: L.lbca_pool_dual(cfg, 0, kv, kv, kv, kv, bp, bp, None, torch.zeros(1, 2, 2, 32)),
        lambda: L.lbca_pool_kv(cfg, kv, kv, kv, kv, bp, bp, None, torch.zeros(1, 2, 2, 32), torch.zeros(1, 2, 2, 32)),
        lambda: L.lbca_pool_f32(cfg, 0, kv, kv, bp, None, torch.zeros(1, 2, 2, 32)),
        lambda: L.lbca_prefill_rows(cfg, q, 0, kv, kv, 0, torch.zeros(1, 2, 2, 32), torch.zeros(1, 2, 2, 32), None,
                                    None, None, torch.zeros_like(q)),
        lambda: L.lbca_append(cfg, tok, tok, tok, tok, bp, bp, None, cache, st),
        lambda: L.lbca_decode(cfg, q1, cache, None, None, None, torch.zeros_like(q1), ws, 8, st),
        lambda: L.lbca_decode_noalloc(cfg, q1, cache, None, None, None, torch.zeros_like(q1), 8, st),
        lambda: L.lbca_decode_step(cfg, tok, tok, tok, tok, bp, bp, None, q1, cache, None, None,
                                   torch.zeros_like(q1), ws, 8, st),
        lambda: L.lbca_prefill(cfg, q, kv, kv, kv, kv, bp, bp, None, None, None, torch.zeros_like(q), None, ws),
        lambda: L.lbca_prefill_backward(cfg, q, kv, kv, kv, kv, bp, bp, None, None, None, q, grads, bws),
        lambda: L.lbca_decode_sparse(hca, torch.zeros(1, 64, 256), hcache, torch.zeros(1, 4, dtype=torch.int32),
                                     None, None, None, torch.zeros(1, 64, 256), st),
        lambda: L.lbca_indexer_topk(torch.zeros(1, 64, 128), torch.zeros(1, 64), torch.zeros(1, 16, 128),
                                    torch.zeros(1, dtype=torch.int32), 4, torch.zeros(1, 4, dtype=torch.int32), None,
                                    torch.zeros(256, dtype=torch.uint8), st),
        lambda: L.lbca_selftest_bounded_wait(False, 1000, st),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(L.LbcaError):
            call()
    wrappers = set(re.findall(r'_check\("(\w+)"', inspect.getsource(L)))
    assert wrappers == reached, sorted(wrappers ^ reached)


def test_cache_struct_follows_field_changes(L):
    """The C struct of a Cache is built once and rebuilt after any field
    change (a decode loop marshals its cache once; a flag or tensor swap is
    still seen by the next call)."""
    import torch
    cfg = _cfg(L)
    t = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)  # noqa: E731
    c = L.Cache(cfg, 1, 4, 192, t(1, 2, 4, 32), t(1, 2, 4, 32), t(1, 2, 192, 32), t(1, 2, 192, 32),
                torch.zeros(16), torch.zeros(1, dtype=torch.int32))
    first = c.c()
    assert c.c() is first
    c.flags = L.LBCA_CACHE_OVERLAP_PREV
    assert c.c().flags == L.LBCA_CACHE_OVERLAP_PREV
    other = t(1, 2, 4, 32)
    c.pooled_k = other
    assert c.c().pooled_k == other.data_ptr()


def test_f32_pool_exchange_wrappers_check_dtypes(L):
    """The context-parallel exchange format is f32: the wrappers refuse other
    dtypes before any call reaches the library."""
    import torch
    cfg = _cfg(L)
    kv = torch.zeros(1, 64, 8, 128, dtype=torch.bfloat16)
    bp = torch.zeros(64, 8 * 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        L.lbca_pool_f32(cfg, 0, kv, kv, bp, None, torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16))
    q = torch.zeros(1, 16, 24, 128, dtype=torch.bfloat16)
    pk = torch.zeros(1, 8, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        L.lbca_prefill_rows(cfg, q, 240, kv, kv, 192, pk, pk, None, None, None, torch.empty_like(q))


def test_checked_variant_exports_the_same_symbols(L):
    """The bounds-checked build (loaded with LBCA_CHECKED=1) is the same
    library compiled with -DLBCA_CHECKED: every declared entry point is there."""
    path = os.path.join(os.path.dirname(L._LIB_PATH), "liblbca_checked.so")
    if not os.path.exists(path):
        pytest.skip("the checked variant is built by build(); not present here")
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n
