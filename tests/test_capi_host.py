"""libpa.so loads on a CPU-only machine, exports every symbol the headers in
include/ declare, and rejects bad arguments on the host without touching a
device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_455_b200 import build
    build.build()
    from paged_kv_cache_455_b200 import pa as mod
    return mod


def _declared_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(pa):
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(pa.lib, n), f"{n} declared in include/ but not exported"
        assert n in pa.SIGNATURES, f"{n} has no binding"


def test_status_strings(pa):
    assert pa.lib.pa_status_string(0) == b"ok"
    for s in range(1, 5):
        assert pa.lib.pa_status_string(s) not in (b"ok", b"unknown status")
    assert pa.lib.pa_status_string(99) == b"unknown status"


def test_size_helpers(pa):
    assert pa.pa_num_partitions(8192, 256) == 32
    assert pa.pa_num_partitions(8193, 256) == 33
    assert pa.pa_num_partitions(0, 256) == 1
    assert pa.pa_splitk_workspace_bytes(8, 16, 256, 32) == 8 * 16 * 32 * (256 + 2) * 4
    # two partial slots (G*d + 2G + 1 floats, rounded up to 4) per CTA and KV
    # head of the group, rounded up to 128 bytes; a 128-byte line per arrival
    # counter (CTA, head); for up to 256 CTAs
    def ws(heads, slot):
        return -(-(2 * heads * slot * 4) // 128) * 128 + heads * 128
    slot = -(-(4 * 256 + 2 * 4 + 1) // 4) * 4
    assert pa.pa_decode_workspace_bytes(8, 16, 4, 256, 8192) == ws(256 * 4, slot)
    # two KV heads form one group of two
    slot8 = -(-(8 * 128 + 2 * 8 + 1) // 4) * 4
    assert pa.pa_decode_workspace_bytes(3, 16, 2, 128, 64) == ws(256 * 2, slot8)
    assert pa.pa_decode_workspace_bytes(8, 16, 4, 256, 1) == \
        pa.pa_decode_workspace_bytes(8, 16, 4, 256, 8192)
    assert pa.pa_decode_workspace_bytes(8, 16, 5, 256, 64) == 0        # Hq % Hkv != 0


# Fake device addresses: every call below fails validation before any CUDA
# call, so none of them is dereferenced.
A = 0x10000          # 16-byte aligned
M = 0x10008          # misaligned


def _attn(pa, **kw):
    args = dict(out=A, query=A, k_pool=A, v_pool=A, block_tables=A, max_blocks=4,
                context_lens=A, num_seqs=3, max_ctx=16, hq=8, hkv=2, d=64, bs=4, nb=16,
                scale=0.125, dtype=0, ws=None, ws_bytes=0, status=None, stream=None)
    args.update(kw)
    a = args
    return pa.lib.pa_decode_attention(a["out"], a["query"], a["k_pool"], a["v_pool"],
                                      a["block_tables"], a["max_blocks"], a["context_lens"],
                                      a["num_seqs"], a["max_ctx"], a["hq"], a["hkv"], a["d"],
                                      a["bs"], a["nb"], a["scale"], a["dtype"], a["ws"],
                                      a["ws_bytes"], a["status"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(out=None), 1), (dict(query=None), 1), (dict(block_tables=None), 1),
    (dict(context_lens=None), 1), (dict(num_seqs=-1), 1), (dict(hq=6, hkv=4), 1),
    (dict(hq=12, hkv=4), 2), (dict(hq=32, hkv=2), 2), (dict(d=96), 2), (dict(d=512), 2),
    (dict(bs=24), 2), (dict(bs=64), 2), (dict(bs=2), 2), (dict(dtype=7), 2),
    (dict(max_ctx=17), 1), (dict(nb=0), 1), (dict(max_blocks=0), 1),
    (dict(out=M), 1), (dict(k_pool=M), 1), (dict(nb=1 << 40), 1),
])
def test_decode_attention_host_validation(pa, kw, want):
    assert _attn(pa, **kw) == want


def test_zero_sequences_is_a_no_op(pa):
    assert _attn(pa, num_seqs=0, out=None, query=None) == 0


def test_splitk_host_validation(pa):
    L = pa.lib

    def call(P=16, maxp=1, tmp=A, ml=A, es=A, max_ctx=16):
        return L.pa_decode_splitk(A, A, A, A, A, 4, A, 3, max_ctx, 8, 2, 64, 4, 16, 0.125, 0,
                                  P, maxp, tmp, ml, es, None, None)
    assert call(P=24) == 1                      # not a multiple of 16
    assert call(P=0) == 1
    assert call(P=16, maxp=0) == 1
    assert call(P=16, maxp=1, max_ctx=16) != 4  # enough partitions (fails later only on CUDA)
    assert call(P=8 * 2, maxp=1, max_ctx=16) != 4
    assert L.pa_decode_splitk(A, A, A, A, A, 8, A, 3, 32, 8, 2, 64, 4, 16, 0.125, 0,
                              16, 1, A, A, A, None, None) == 4      # 32 tokens need 2 parts
    assert call(tmp=None) == 1
    assert L.pa_splitk_reduce(A, A, A, A, A, 3, 8, 64, 24, 2, 0, None) == 1
    assert L.pa_splitk_reduce(A, A, A, A, A, 3, 8, 96, 16, 2, 0, None) == 2
    assert L.pa_splitk_reduce(None, A, A, A, A, 3, 8, 64, 16, 2, 0, None) == 1


def test_reshape_and_cache_host_validation(pa):
    L = pa.lib

    def call(**kw):
        a = dict(key=A, value=A, kp=A, vp=A, slots=A, T=3, hkv=2, d=64, bs=4, nb=16, dt=0)
        a.update(kw)
        return L.pa_reshape_and_cache(a["key"], a["value"], a["kp"], a["vp"], a["slots"],
                                      a["T"], a["hkv"], a["d"], a["bs"], a["nb"], a["dt"],
                                      None, None)
    assert call(key=None) == 1
    assert call(slots=None) == 1
    assert call(T=-1) == 1
    assert call(bs=12) == 2
    assert call(d=100) == 2
    assert call(dt=5) == 2
    assert call(value=M) == 1
    assert call(T=0, key=None) == 0


def test_copy_blocks_host_validation(pa):
    L = pa.lib

    def call(**kw):
        a = dict(kp=A, vp=A, mapping=A, n=2, nb=16, bs=16, hkv=4, d=256, dt=1)
        a.update(kw)
        return L.pa_copy_blocks(a["kp"], a["vp"], a["mapping"], a["n"], a["nb"], a["bs"],
                                a["hkv"], a["d"], a["dt"], None, None)
    assert call(n=-1) == 1
    assert call(nb=0) == 1
    assert call(hkv=0) == 1
    assert call(d=100) == 2
    assert call(bs=12) == 2
    assert call(dt=5) == 2
    assert call(mapping=None) == 1
    assert call(kp=None) == 1
    assert call(n=0, kp=None, vp=None, mapping=None) == 0   # nothing to copy: no launch


def test_swap_blocks_host_validation(pa):
    L = pa.lib

    def call(**kw):
        a = dict(dk=A, dv=A, dnb=8, sk=A, sv=A, snb=16, mapping=A, n=2, bs=16, hkv=4, d=256,
                 dt=1)
        a.update(kw)
        return L.pa_swap_blocks(a["dk"], a["dv"], a["dnb"], a["sk"], a["sv"], a["snb"],
                                a["mapping"], a["n"], a["bs"], a["hkv"], a["d"], a["dt"],
                                None, None)
    assert call(n=-1) == 1
    assert call(dnb=0) == 1
    assert call(snb=0) == 1
    assert call(d=100) == 2
    assert call(dt=7) == 2
    assert call(sk=None) == 1
    assert call(dv=M) == 1
    assert call(n=0, dk=None, dv=None, sk=None, sv=None, mapping=None) == 0


def test_prefill_host_validation(pa):
    L = pa.lib

    def call(**kw):
        a = dict(out=A, q=A, cu=A, total=10, maxq=8, kp=A, vp=A, tab=A, maxb=4, lens=A, B=2,
                 maxctx=64, hq=16, hkv=4, d=256, bs=16, nb=32, dt=1)
        a.update(kw)
        return L.pa_prefill_attention(a["out"], a["q"], a["cu"], a["total"], a["maxq"], a["kp"],
                                      a["vp"], a["tab"], a["maxb"], a["lens"], a["B"],
                                      a["maxctx"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"],
                                      0.0625, a["dt"], None, None)
    assert call(dt=0) == 2                  # fp32: not built
    assert call(hq=12) == 2                 # group 3
    assert call(d=96) == 2
    assert call(bs=12) == 2
    assert call(hq=15) == 1                 # Hq % Hkv != 0
    assert call(maxctx=65) == 1             # beyond the table
    assert call(maxq=65, maxctx=64) == 1    # chunk longer than any context
    assert call(maxb=4096, maxctx=40000) == 2   # more than 2048 blocks
    assert call(cu=None) == 1
    assert call(out=M) == 1
    assert call(B=0, out=None) == 0         # nothing to do: no launch
    assert call(maxq=0, out=None) == 0


def test_binding_rejects_cpu_tensors(pa):
    import torch
    x = torch.zeros(3, 8, 64)
    with pytest.raises(ValueError):
        pa.pa_decode_attention(x, x, torch.zeros(16, 4, 2, 64), torch.zeros(16, 4, 2, 64),
                               torch.zeros(3, 2, dtype=torch.int32),
                               torch.zeros(3, dtype=torch.int32), 8, 0.125)


def test_fp8_host_validation(pa):
    L = pa.lib

    def cache(**kw):
        a = dict(key=A, value=A, kp=A, vp=A, slots=A, T=3, hkv=2, d=128, bs=16, nb=16, ks=0.02,
                 vs=0.02)
        a.update(kw)
        return L.pa_reshape_and_cache_fp8(a["key"], a["value"], a["kp"], a["vp"], a["slots"],
                                          a["T"], a["hkv"], a["d"], a["bs"], a["nb"], a["ks"],
                                          a["vs"], None, None)

    def attn(**kw):
        a = dict(out=A, query=A, kp=A, vp=A, tab=A, maxb=4, lens=A, B=3, max_ctx=64, hq=8, hkv=2,
                 d=128, bs=16, nb=16, scale=0.1, ks=0.02, vs=0.02)
        a.update(kw)
        return L.pa_decode_attention_fp8(a["out"], a["query"], a["kp"], a["vp"], a["tab"],
                                         a["maxb"], a["lens"], a["B"], a["max_ctx"], a["hq"],
                                         a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["ks"],
                                         a["vs"], None, 0, None, None)
    assert cache(key=None) == 1
    assert cache(ks=0.0) == 1 and cache(vs=-1.0) == 1 and cache(ks=float("inf")) == 1
    assert cache(d=64) == 2 and cache(bs=8) == 2
    assert cache(kp=M) == 1
    assert cache(T=0, key=None) == 0
    assert attn(out=None) == 1
    assert attn(ks=float("nan")) == 1 and attn(vs=0.0) == 1
    assert attn(d=64) == 2 and attn(bs=4) == 2
    assert attn(hq=6, hkv=4) == 1
    assert attn(max_ctx=65) == 1
    assert attn(B=0, out=None, query=None) == 0
    # copies of E4M3 pools are accepted; an unknown element type is not
    assert L.pa_copy_blocks(A, A, A, 1, 16, 16, 2, 128, 2, None, None) != 2
    assert L.pa_copy_blocks(A, A, A, 1, 16, 16, 2, 128, 3, None, None) == 2
