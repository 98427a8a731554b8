"""Chunked-prefill paged attention on the GPU, through the C ABI, against the
fp64 oracle ("vLLM Architecture, Memory and Benchmarks Deep Dive", section
4, chunked prefill).  Tolerance: max |gpu - oracle| <= 2e-2 (bf16 data, fp32
accumulation, outputs of order 1)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_cache_455_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = 2e-2


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_455_b200 import pa as mod
    return mod


def _case(seed, ctxs, chunks, hq, hkv, d, bs, spare=5):
    """Random pools and tables; sequence b has ctxs[b] cached tokens, the last
    chunks[b] of them being its chunk."""
    rng = np.random.default_rng(seed)
    need = [-(-c // bs) for c in ctxs]
    nb = sum(need) + spare
    perm = rng.permutation(nb)
    tables = np.full((len(ctxs), max(need + [1])), -1, np.int32)
    pos = 0
    for b, k in enumerate(need):
        tables[b, :k] = perm[pos:pos + k]
        pos += k
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    k_pool = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    # NaN in every slot past each context and in every block no sequence owns,
    # so that a masking slip shows as a non-finite output
    valid = np.zeros((nb, bs), bool)
    for b, c in enumerate(ctxs):
        t = np.arange(c)
        valid[tables[b, t // bs], t % bs] = True
    invalid = torch.from_numpy(~valid).to(DEV)
    k_pool[invalid] = float("nan")
    v_pool[invalid] = float("nan")
    cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), hq, d, generator=g, device=DEV).to(torch.bfloat16)
    return q, k_pool, v_pool, tables, np.array(ctxs, np.int32), cu


def _run(pa, q, kp, vp, tables, lens, cu, scale, status=None):
    out = torch.full_like(q, float("nan"))
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
    chunks = np.diff(cu)
    pa.pa_prefill_attention(out, q, torch.from_numpy(cu).to(DEV), int(chunks.max()), kp, vp,
                            torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV),
                            int(lens.max()), scale, status)
    torch.cuda.synchronize()
    return out, int(status.item())


def _oracle(q, kp, vp, tables, lens, cu, scale):
    return O.prefill_attention_np(W.to_numpy_elems(q), W.to_numpy_elems(kp),
                                  W.to_numpy_elems(vp), tables, lens, cu, scale, "bf16")


@pytest.mark.parametrize("d,hq,hkv,bs", [(256, 16, 4, 16), (128, 8, 8, 32), (64, 16, 2, 4),
                                         (128, 16, 8, 8), (256, 8, 4, 32), (64, 16, 2, 16),
                                         (128, 32, 4, 32), (256, 8, 1, 16)])
def test_random_chunks_match_oracle(pa, d, hq, hkv, bs):
    ctxs = [1, 40, 300, 97, 513, 64]
    chunks = [1, 40, 37, 1, 129, 33]           # whole prompts, prefix + chunk, single tokens
    q, kp, vp, tab, lens, cu = _case(d + hq + bs, ctxs, chunks, hq, hkv, d, bs)
    scale = d ** -0.5
    out, status = _run(pa, q, kp, vp, tab, lens, cu, scale)
    assert status == 0
    ref = _oracle(q, kp, vp, tab, lens, cu, scale)
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL


@pytest.mark.parametrize("bs", [16, 32])
def test_every_tail_length_up_to_80(pa, bs):
    """Contexts of 1 .. 80 tokens (every position of the last block, and
    chunks that are whole prompts or end part-way into a 64-token tile) on
    the tensor-core path (blocks of 16 and 32)."""
    ctxs = list(range(1, 81))
    chunks = [c if c % 3 else max(1, c // 2) for c in ctxs]
    q, kp, vp, tab, lens, cu = _case(100 + bs, ctxs, chunks, 8, 2, 128, bs)
    scale = 128 ** -0.5
    out, status = _run(pa, q, kp, vp, tab, lens, cu, scale)
    assert status == 0
    ref = _oracle(q, kp, vp, tab, lens, cu, scale)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL


def test_512_token_chunk_after_a_long_prefix(pa):
    """A 512-token chunk at the end of a 4096-token context, qwen-shaped heads."""
    q, kp, vp, tab, lens, cu = _case(7, [4096, 2000], [512, 300], 16, 4, 256, 16)
    scale = 1.0 / 16.0
    out, status = _run(pa, q, kp, vp, tab, lens, cu, scale)
    assert status == 0
    ref = _oracle(q, kp, vp, tab, lens, cu, scale)
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL


def test_one_token_chunks_agree_with_decode(pa):
    q, kp, vp, tab, lens, cu = _case(8, [17, 250, 1], [1, 1, 1], 16, 4, 256, 16)
    scale = 1.0 / 16.0
    out, status = _run(pa, q, kp, vp, tab, lens, cu, scale)
    dec = torch.empty_like(q)
    pa.pa_decode_attention(dec, q, kp, vp, torch.from_numpy(tab).to(DEV),
                           torch.from_numpy(lens).to(DEV), int(lens.max()), scale)
    torch.cuda.synchronize()
    assert status == 0
    assert (out.float() - dec.float()).abs().max().item() <= TOL


def test_empty_chunks_are_skipped(pa):
    q, kp, vp, tab, lens, cu = _case(9, [30, 50, 20], [5, 0, 7], 8, 2, 128, 16)
    out, status = _run(pa, q, kp, vp, tab, lens, cu, 0.1)
    assert status == 0
    ref = _oracle(q, kp, vp, tab, lens, cu, 0.1)
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL


def test_bad_block_and_bad_chunk_set_status_and_zero(pa):
    q, kp, vp, tab, lens, cu = _case(10, [40, 40], [10, 10], 8, 2, 128, 16)
    bad = tab.copy()
    bad[0, 1] = kp.shape[0] + 3
    out, status = _run(pa, q, kp, vp, bad, lens, cu, 0.1)
    assert status & pa.PA_DEV_BAD_BLOCK
    assert (out[:10].float() == 0).all()
    ref = _oracle(q, kp, vp, tab, lens, cu, 0.1)
    assert np.abs(out[10:].double().cpu().numpy() - ref[10:]).max() <= TOL
    short = lens.copy()
    short[1] = 5                                   # chunk of 10 longer than its context
    out, status = _run(pa, q, kp, vp, tab, short, cu, 0.1)
    assert status & pa.PA_DEV_BAD_CONTEXT
    assert (out[10:].float() == 0).all()
