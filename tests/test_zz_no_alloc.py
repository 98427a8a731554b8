"""pa_decode_attention_static: the entry point for callers that cannot
allocate device memory (plug-in interfaces that pass only inputs and outputs,
memory owned by another framework, code paths where an allocation is not
allowed).  It must give the same result as pa_decode_attention with a
workspace, through the C ABI, on consecutive calls that share its fixed
scratch array.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = 2e-2   # bf16 attention tolerance used by every GPU test


def _case(seed, B, lens, hq=16, hkv=4, d=256, bs=16):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    need = -(-lens // bs)
    nb = int(need.sum()) + 16
    perm = rng.permutation(nb)
    tables = np.full((B, int(need.max())), -1, np.int32)
    pos = 0
    for b in range(B):
        tables[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = torch.randn(B, hq, d, generator=g, device=DEV).to(torch.bfloat16)
    kp = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    vp = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    return (q, kp, vp, torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV),
            int(lens.max()), d ** -0.5)


def _with_workspace(pa, q, kp, vp, tab, lens, mc, scale):
    out = torch.empty_like(q)
    B, hq, d = q.shape
    ws = torch.empty(pa.pa_decode_workspace_bytes(B, hq, kp.shape[2], d, mc), dtype=torch.uint8,
                     device=DEV)
    pa.pa_decode_attention(out, q, kp, vp, tab, lens, mc, scale, ws)
    return out


def _oracle(args):
    from oracle import oracle as O
    from paged_kv_cache_455_b200 import workloads as W
    q, kp, vp, tab, lens, mc, scale = args
    return O.paged_attention(W.to_numpy_elems(q), W.to_numpy_elems(kp), W.to_numpy_elems(vp),
                             tab.cpu().numpy(), lens.cpu().numpy(), scale, "bf16")


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    from paged_kv_cache_455_b200 import pa
    # long contexts so that sequences are spread over several CTAs and the
    # scratch really holds partial results.  The second batch differs, and
    # the third has a smaller head dimension, so its partial slots are
    # smaller and its counter words sit where the earlier calls left partial
    # results: every call runs on the previous call's leftover contents.
    cases = [_case(11, 6, [3000, 1, 777, 4096, 1500, 2049]),
             _case(12, 9, [5000, 64, 65, 1, 2500, 4100, 300, 3333, 17]),
             _case(13, 5, [4000, 2222, 9, 1200, 3100], d=128)]
    for args in cases + cases[:1]:
        ref = _with_workspace(pa, *args)
        out = torch.full_like(ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        q, kp, vp, tab, lens, mc, scale = args
        pa.pa_decode_attention_static(out, q, kp, vp, tab, lens, mc, scale, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # same kernel, same grid, pieces merged in a fixed order: bit-identical
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        err = np.abs(out.double().cpu().numpy() - _oracle(args)).max()
        assert err <= TOL


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    from paged_kv_cache_455_b200 import pa
    # group 8 at d = 256: two partial slots per SM and KV head of 8*256 + 17
    # floats (rounded to 2068) plus a flag each; on a GPU with enough SMs that
    # is more than the fixed scratch, and the call must refuse (launching
    # nothing) rather than fall back silently
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    need = 2 * sms * 4 * 2068 * 4 + 2 * sms * 4 * 4
    if need <= pa.PA_STATIC_SCRATCH_BYTES:
        pytest.skip("this GPU's grid fits the scratch")
    B = 64
    q = torch.zeros(B, 32, 256, dtype=torch.bfloat16, device=DEV)
    kp = torch.zeros(8, 16, 4, 256, dtype=torch.bfloat16, device=DEV)
    tab = torch.zeros(B, 8, dtype=torch.int32, device=DEV)
    lens = torch.full((B,), 128, dtype=torch.int32, device=DEV)
    out = torch.zeros_like(q)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_attention_static(out, q, kp, kp, tab, lens, 128, 0.0625)
    assert e.value.status == pa.PA_ERR_WORKSPACE
