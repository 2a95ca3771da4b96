"""Host-side checks of the C ABI that need no GPU.

The library must load, export every function include/parallax.h declares, and
reject bad arguments on the host before any CUDA call.  The split plan is
pure host logic and is checked against its documented rule.
"""

import ctypes
import os
import re

import pytest
import torch

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "parallax.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(parallax_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def binding():
    from parallax_local_linear_b200 import binding as b
    return b


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("parallax_decode", "parallax_decode_projected", "parallax_prefill", "parallax_prefill_paged",
                 "parallax_decode_workspace_size",
                 "parallax_last_device_error", "parallax_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(binding):
    lib = ctypes.CDLL(binding.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_abi_version_and_status_strings(binding):
    assert binding.lib.parallax_abi_version() == 10
    for code, name in binding.STATUS.items():
        assert binding.lib.parallax_status_string(code).decode() == name


def _params(binding, **kw):
    base = dict(batch=8, num_q_heads=16, num_kv_heads=8, head_dim=128, kv_len=4096, page_size=0,
                num_pages=0, max_pages_per_seq=0, in_dtype=1, out_dtype=1, scale=0.088, num_ctas=0)
    base.update(kw)
    return binding.DecodeParams(**base)


@pytest.mark.parametrize("bad", [
    dict(batch=0), dict(num_q_heads=12, num_kv_heads=8), dict(kv_len=-1), dict(in_dtype=7),
    dict(out_dtype=9), dict(scale=float("inf")), dict(num_ctas=-2),
    dict(page_size=64, num_pages=0, max_pages_per_seq=64),
    dict(page_size=64, num_pages=10, max_pages_per_seq=3),
])
def test_invalid_decode_params_are_rejected(binding, bad):
    p = _params(binding, **bad)
    assert binding.lib.parallax_decode_num_ctas(ctypes.byref(p), 148) == -1
    assert binding.lib.parallax_decode_workspace_size(ctypes.byref(p), 148) == binding.SIZE_MAX
    st = binding.lib.parallax_decode(None, None, None, None, None, None, None, None, 0, ctypes.byref(p), None)
    assert st == 1


@pytest.mark.parametrize("unsup", [dict(head_dim=96), dict(page_size=32, num_pages=4, max_pages_per_seq=200),
                                   dict(num_q_heads=32, num_kv_heads=2), dict(batch=9000)])
def test_unsupported_decode_params(binding, unsup):
    p = _params(binding, **unsup)
    st = binding.lib.parallax_decode(None, None, None, None, None, None, None, None, 0, ctypes.byref(p), None)
    assert st == 2


def test_null_and_misaligned_pointers_rejected_before_launch(binding):
    p = _params(binding)
    st = binding.lib.parallax_decode(None, None, None, None, None, None, None, None, 0, ctypes.byref(p), None)
    assert st == 1
    buf = ctypes.create_string_buffer(64)
    addr = ctypes.addressof(buf)
    odd = ctypes.c_void_p(addr + 2)
    al = ctypes.c_void_p((addr + 15) & ~15)
    st = binding.lib.parallax_decode(odd, al, al, al, None, None, al, None, 0, ctypes.byref(p), None)
    assert st == 1
    # contiguous cache given a page table
    st = binding.lib.parallax_decode(al, al, al, al, al, None, al, None, 0, ctypes.byref(p), None)
    assert st == 1
    pp = _params(binding, page_size=64, num_pages=4, max_pages_per_seq=64)
    st = binding.lib.parallax_decode(al, al, al, al, None, None, al, None, 0, ctypes.byref(pp), None)
    assert st == 1   # paged without a page table / seq_lens


def test_projected_decode_rejects_bad_arguments_before_launch(binding):
    buf = ctypes.create_string_buffer(256)
    addr = ctypes.addressof(buf)
    al = ctypes.c_void_p((addr + 15) & ~15)
    odd = ctypes.c_void_p(((addr + 15) & ~15) + 2)
    p = _params(binding)

    def call(x=al, wq=al, wr=al, hidden=2048, params=p):
        return binding.lib.parallax_decode_projected(x, wq, wr, hidden, al, al, None, None, al, al, al, None, 0,
                                                     ctypes.byref(params), None)

    assert call(params=_params(binding, batch=0)) == 1          # decode parameters checked first
    assert call(x=None) == 1
    assert call(wr=None) == 1
    assert call(wq=odd) == 1
    assert call(hidden=0) == 1
    assert call(hidden=-32) == 1
    assert call(hidden=48) == 2                                 # not a multiple of 32
    assert call(params=_params(binding, in_dtype=0, out_dtype=0)) == 2   # fp32 cache


def test_projected_decode_rejects_overlapping_outputs_before_launch(binding):
    # Fake, 16-byte aligned device addresses: the overlap checks run on the
    # host before any CUDA call.  B=8, Hq*d=2048, hidden=2048: q and rho are
    # 32 KiB each, x 32 KiB, each weight 8 MiB.
    p = _params(binding)
    X, WQ, WR = 1 << 32, 2 << 32, 3 << 32
    Q, R, OUT = 4 << 32, 5 << 32, 6 << 32
    V = ctypes.c_void_p

    def call(q=Q, r=R, x=X, wq=WQ, wr=WR):
        return binding.lib.parallax_decode_projected(V(x), V(wq), V(wr), 2048, V(7 << 32), V(8 << 32), None, None,
                                                     V(q), V(r), V(OUT), None, 0, ctypes.byref(p), None)

    # disjoint buffers pass these checks and fail later: no device (CPU) or no workspace (GPU)
    assert call() in (3, 4)
    assert call(q=X + 16) == 1                 # q inside x
    assert call(r=WQ + (8 << 20) - 16) == 1    # rho straddles the end of w_q
    assert call(q=WR) == 1                     # q on w_rho
    assert call(r=Q + 32768 - 16) == 1         # rho overlaps q
    assert call(q=None) == 1


@pytest.mark.parametrize("bad", [dict(seq_len=0), dict(head_dim=64), dict(in_dtype=0), dict(causal=2), dict(cta_pair=2),
                                 dict(num_heads=6, num_kv_heads=4), dict(scale=-0.1), dict(scale=0.0)])
def test_invalid_prefill_params_are_rejected(binding, bad):
    base = dict(batch=1, num_heads=4, num_kv_heads=0, seq_len=16, head_dim=128, in_dtype=1, out_dtype=1,
                scale=0.088, causal=1)
    base.update(bad)
    p = binding.PrefillParams(**base)
    st = binding.lib.parallax_prefill(None, None, None, None, None, ctypes.byref(p), None)
    assert st in (1, 2)


def _paged_prefill_params(binding, **kw):
    base = dict(batch=2, num_heads=4, num_kv_heads=2, head_dim=128, total_q=300, max_q_len=200, page_size=64,
                num_pages=20, max_pages_per_seq=10, in_dtype=1, out_dtype=0, scale=0.088, causal=1)
    base.update(kw)
    return binding.PrefillPagedParams(**base)


@pytest.mark.parametrize("bad,status", [
    (dict(batch=0), 1), (dict(num_heads=6, num_kv_heads=4), 1), (dict(total_q=-1), 1),
    (dict(max_q_len=-5), 1), (dict(num_pages=0), 1), (dict(max_pages_per_seq=0), 1),
    (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(in_dtype=3), 1), (dict(out_dtype=5), 1),
    (dict(causal=-1), 1), (dict(head_dim=64), 2), (dict(page_size=16), 2), (dict(in_dtype=0), 2),
    (dict(num_pages=1 << 24, num_kv_heads=4), 2), (dict(max_pages_per_seq=1 << 26), 2),
])
def test_invalid_paged_prefill_params_are_rejected(binding, bad, status):
    p = _paged_prefill_params(binding, **bad)
    st = binding.lib.parallax_prefill_paged(None, None, None, None, None, None, None, None, ctypes.byref(p), None)
    assert st == status


def test_paged_prefill_pointer_checks_and_empty_calls(binding):
    p = _paged_prefill_params(binding)
    nul = [None] * 8
    assert binding.lib.parallax_prefill_paged(*nul, ctypes.byref(p), None) == 1
    buf = ctypes.create_string_buffer(64)
    addr = ctypes.addressof(buf)
    al = ctypes.c_void_p((addr + 15) & ~15)
    odd = ctypes.c_void_p(((addr + 15) & ~15) + 8)
    args = [al, al, al, al, al, al, al, odd]          # out only 8-byte aligned
    assert binding.lib.parallax_prefill_paged(*args, ctypes.byref(p), None) == 1
    # no query rows: valid, and nothing is launched or dereferenced
    for empty in (dict(total_q=0), dict(max_q_len=0)):
        pe = _paged_prefill_params(binding, **empty)
        assert binding.lib.parallax_prefill_paged(*nul, ctypes.byref(pe), None) == 0


def _expected_plan(B, units, heads_per_unit, L, d=128, num_sms=148, forced=0, f32=False, paged=False):
    tiles = B * units * (-(-L // 64))
    ctas = forced if forced else num_sms
    n_units = B * units
    if not forced and not f32 and not paged and n_units <= num_sms:
        k = num_sms // n_units
        if 4 * n_units * k >= 3 * num_sms:
            ctas = n_units * k
    # by default an fp32 CTA (eight warps of 32 tokens) takes at least four 64-token tiles
    per_cta = 4 if (not forced and f32) else 1
    ctas = max(1, min(ctas, -(-tiles // per_cta)))
    counters = -(-(B * units * 4) // 256) * 256
    return ctas, counters + 2 * ctas * heads_per_unit * (2 * d + 4) * 4


@pytest.mark.parametrize("B,Hq,Hkv,L,forced,dtype", [
    (8, 16, 8, 4096, 0, 1), (64, 32, 8, 32768, 0, 1), (128, 16, 4, 65536, 0, 1), (1, 1, 1, 256, 0, 0),
    (1, 4, 4, 65, 0, 1), (8, 16, 8, 4096, 3, 1), (2, 2, 1, 100, 16, 1), (4, 8, 2, 1, 0, 1), (2, 6, 2, 4096, 0, 0),
])
def test_work_plan_and_workspace_size(binding, B, Hq, Hkv, L, forced, dtype):
    p = _params(binding, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, kv_len=L, num_ctas=forced, in_dtype=dtype,
                out_dtype=dtype)
    ctas = binding.lib.parallax_decode_num_ctas(ctypes.byref(p), 148)
    units, hpu = (Hkv, Hq // Hkv) if dtype == 1 else (Hq, 1)
    exp_ctas, exp_ws = _expected_plan(B, units, hpu, L, forced=forced, f32=dtype == 0)
    assert ctas == exp_ctas
    assert binding.lib.parallax_decode_workspace_size(ctypes.byref(p), 148) == exp_ws


def test_workspace_does_not_grow_with_length(binding):
    sizes = [binding.lib.parallax_decode_workspace_size(ctypes.byref(_params(binding, kv_len=L)), 148)
             for L in (4096, 65536, 1 << 20)]
    assert sizes[0] == sizes[1] == sizes[2]


def test_no_cpu_fallback(binding):
    q = torch.zeros(1, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        binding.decode(q, q, torch.zeros(1, 1, 4, 64), torch.zeros(1, 1, 4, 64))


def _train_params(binding, **kw):
    base = dict(batch=2, num_heads=4, num_kv_heads=2, seq_len=300, head_dim=128, in_dtype=1, out_dtype=0,
                scale=0.088, causal=1)
    base.update(kw)
    return binding.PrefillParams(**base)


def test_backward_workspace_size_and_validation(binding):
    p = _train_params(binding)
    assert binding.lib.parallax_prefill_backward_workspace_size(ctypes.byref(p)) == (2 * 4 * 300 * 16 + 255) // 256 * 256 + 2 * 4 * 300 * 128
    bad = _train_params(binding, head_dim=64)
    assert binding.lib.parallax_prefill_backward_workspace_size(ctypes.byref(bad)) == binding.SIZE_MAX
    nul = [None] * 13
    assert binding.lib.parallax_prefill_backward(*nul, 0, ctypes.byref(bad), None) == 2
    assert binding.lib.parallax_prefill_backward(*nul, 0, ctypes.byref(p), None) == 1
    assert binding.lib.parallax_prefill_train(*([None] * 7), ctypes.byref(p), None) == 1
    buf = ctypes.create_string_buffer(64)
    al = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)
    # every pointer present and aligned, workspace too small
    assert binding.lib.parallax_prefill_backward(*([al] * 13), 16, ctypes.byref(p), None) == 3


def test_decode_binding_checks_cache_shapes_before_any_launch(binding):
    # Host tensors: each call must fail on the shape check, which runs before
    # the device checks, so no launch is ever reached.
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16)
    k = torch.zeros((2, 2, 256, 64), dtype=torch.bfloat16)        # head_dim 64 against q's 128
    out = torch.zeros_like(q)
    for fn in (lambda: binding.decode(q, q, k, k),
               lambda: binding.decode_noalloc(q, q, k, k, out=out)):
        with pytest.raises(ValueError, match="head_dim"):
            fn()
    k = torch.zeros((2, 2, 256, 128), dtype=torch.bfloat16)
    for kv_len in (100, 300):   # a contiguous cache is addressed with its own length
        for fn in (lambda: binding.decode(q, q, k, k, kv_len=kv_len),
                   lambda: binding.decode_noalloc(q, q, k, k, out=out, kv_len=kv_len)):
            with pytest.raises(ValueError, match="kv_len"):
                fn()
    with pytest.raises(ValueError, match="one sequence per row"):
        binding.decode(q, q, torch.zeros((3, 2, 256, 128), dtype=torch.bfloat16),
                       torch.zeros((3, 2, 256, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="KV heads"):
        binding.decode(q, q, torch.zeros((2, 3, 256, 128), dtype=torch.bfloat16),
                       torch.zeros((2, 3, 256, 128), dtype=torch.bfloat16))
    x = torch.zeros((2, 256), dtype=torch.bfloat16)
    w = torch.zeros((4 * 128, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="kv_len"):
        binding.decode_projected(x, w, w, k, k, kv_len=100)
    # a paged pool must hold 64-token pages, and kv_len fits the page table
    pool = torch.zeros((8, 2, 64, 128), dtype=torch.bfloat16)
    table = torch.zeros((2, 4), dtype=torch.int32)
    lens = torch.zeros((2,), dtype=torch.int32)
    with pytest.raises(ValueError, match="kv_len"):
        binding.decode(q, q, pool, pool, seq_lens=lens, page_table=table, kv_len=4 * 64 + 1)


def test_decode_plan_rejects_bad_arguments_before_any_launch(binding):
    p = _params(binding)
    handle = ctypes.c_void_p(1234)
    st = binding.lib.parallax_decode_plan_create(None, None, None, None, None, None, None, None, 0,
                                                 ctypes.byref(p), ctypes.byref(handle))
    assert st == 1 and not handle.value   # the plan pointer is cleared on error
    bad = _params(binding, batch=0)
    assert binding.lib.parallax_decode_plan_create(None, None, None, None, None, None, None, None, 0,
                                                   ctypes.byref(bad), ctypes.byref(handle)) == 1
    assert binding.lib.parallax_decode_plan_run(None, None) == 1
    binding.lib.parallax_decode_plan_destroy(None)   # a no-op
