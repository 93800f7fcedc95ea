"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded fp16 inputs.  Needs a B200."""
import numpy as np
import pytest
import torch

from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.inputs import make_qkv, WORKLOADS, sweep_points
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from dnn_compiler_pipelining_b200.build import build
    build()
    attn.load()
    torch.cuda.set_device(0)
    attn.device_status()  # clear


# small shapes that still span several tiles: the oracle checks every row
SMALL = [
    (1, 1, 1, 128), (1, 2, 1, 256), (1, 4, 2, 384), (2, 8, 2, 512), (1, 8, 8, 256),
    (3, 6, 3, 640),
    (2, 32, 1, 300),  # multi-query: one kv head for 32 query heads, ragged S
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", SMALL)
def test_small_full(B, Hq, Hkv, S, causal):
    parity.full_check(B, Hq, Hkv, S, 128, causal, seed=7)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", [(1, 4, 2, 512), (2, 8, 2, 256)])
def test_small_stress_full(B, Hq, Hkv, S, causal):
    """Q, K ~ N(0, 4^2): logits with standard deviation 16 stress the running max."""
    parity.full_check(B, Hq, Hkv, S, 128, causal, seed=11, qk_std=4.0)


# S not a multiple of 128: the last row / key block is ragged
RAGGED = [(1, 4, 2, 1), (1, 4, 2, 77), (2, 4, 2, 200), (1, 8, 2, 383), (2, 6, 3, 1000)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", RAGGED)
def test_ragged_full(B, Hq, Hkv, S, causal):
    """Keys past S are masked and rows past S are computed but not stored."""
    parity.full_check(B, Hq, Hkv, S, 128, causal, seed=13)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_stress_full(causal):
    parity.full_check(1, 8, 2, 329, 128, causal, seed=17, qk_std=4.0)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_writes_stay_in_bounds(causal):
    """O and LSE end inside larger buffers whose tails hold a sentinel: the
    last head's rows past S (inside the ragged block) must not be stored."""
    B, Hq, Hkv, S, D = 1, 2, 1, 150, 128
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=19, device="cuda")
    n_o, n_l, pad = B * Hq * S * D, B * Hq * S, 128 * D
    o_buf = torch.full((n_o + pad,), 7.0, dtype=torch.float16, device="cuda")
    l_buf = torch.full((n_l + 4 * 128,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[:n_o].view(B, Hq, S, D)
    lse = l_buf[:n_l].view(B, Hq, S)
    attn.attn_fwd(q, k, v, causal, o=o, lse=lse)
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    assert bool((o_buf[n_o:] == 7.0).all().item()), "O written past its end"
    assert bool((l_buf[n_l:] == 7.0).all().item()), "LSE written past its end"
    o_ref, lse_ref = parity.oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                             v.cpu().double().numpy(), causal)
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        "ragged in-bounds causal=%d" % causal)


# head dimension 64: one 64-column panel per tile, 4 K-steps in Q K^T, N = 64 in P V
D64 = [(1, 4, 2, 128), (2, 8, 2, 384), (1, 6, 3, 200), (1, 4, 1, 1000)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", D64)
def test_d64_full(B, Hq, Hkv, S, causal):
    parity.full_check(B, Hq, Hkv, S, 64, causal, seed=23)


@pytest.mark.parametrize("causal", [True, False])
def test_d64_stress_full(causal):
    parity.full_check(1, 8, 2, 512, 64, causal, seed=29, qk_std=4.0)


@pytest.mark.parametrize("causal", [True, False])
def test_d64_sampled(causal):
    q, k, v = make_qkv(4, 32, 8, 4096, 64, seed=31, device="cuda")
    o, lse = parity.run_gpu(q, k, v, causal)
    parity.sampled_check(q, k, v, o, lse, causal, n_random=512, seed=31)


# head dimension 256: one 128-row tile per work item, 64-key blocks, S
# double-buffered in TMEM
D256 = [(1, 2, 1, 64), (1, 4, 2, 384), (2, 4, 2, 200), (1, 6, 3, 1000), (1, 2, 2, 1)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", D256)
def test_d256_full(B, Hq, Hkv, S, causal):
    parity.full_check(B, Hq, Hkv, S, 256, causal, seed=61)


@pytest.mark.parametrize("causal", [True, False])
def test_d256_stress_full(causal):
    parity.full_check(1, 8, 2, 700, 256, causal, seed=63, qk_std=4.0)


@pytest.mark.parametrize("causal", [True, False])
def test_d256_large_outputs(causal):
    """Every row with |O| >= 4: every item goes through the exact pass."""
    B, Hq, Hkv, S, D = 1, 4, 2, 640, 256
    q, k, _ = make_qkv(B, Hq, Hkv, S, D, seed=65, qk_std=4.0, device="cuda")
    v = _large_v(B, Hkv, S, D, 66)
    attn.device_status_ex()
    o, lse = parity.run_gpu(q, k, v, causal)
    import oracle
    o_ref, lse_ref = oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                      v.cpu().double().numpy(), causal)
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        "D256 large V causal=%d" % causal)


@pytest.mark.parametrize("causal", [True, False])
def test_d256_qk(causal):
    q, k, v = _qk_inputs(1, 4, 2, 200, 450, 256, seed=67)
    _qk_check(q, k, v, causal, "D256 Sq200 Sk450")


@pytest.mark.parametrize("causal", [True, False])
def test_d256_sampled(causal):
    q, k, v = make_qkv(4, 16, 4, 4096, 256, seed=69, device="cuda")
    o, lse = parity.run_gpu(q, k, v, causal)
    parity.sampled_check(q, k, v, o, lse, causal, n_random=256, seed=69)


@pytest.mark.parametrize("variant", [1, 2, 4, 15])
def test_d256_variants(variant):
    q, k, v = make_qkv(1, 8, 2, 520, 256, seed=71, qk_std=4.0, device="cuda")
    _variant_check(q, k, v, True, variant, "D256 %s" % attn.variant_name(variant))


# Sq query rows over Sk keys (attn_fwd_qk); causal windows aligned bottom-right
QK = [(1, 4, 2, 1, 513), (2, 4, 2, 77, 300), (1, 8, 2, 128, 1000), (1, 6, 3, 257, 1024),
      (2, 4, 1, 300, 300)]


def _qk_inputs(B, Hq, Hkv, Sq, Sk, D, seed, qk_std=1.0):
    q, _, _ = make_qkv(B, Hq, Hkv, Sq, D, seed=seed, qk_std=qk_std, device="cuda")
    _, k, v = make_qkv(B, Hq, Hkv, Sk, D, seed=seed + 100, qk_std=qk_std, device="cuda")
    return q, k, v


def _qk_check(q, k, v, causal, what):
    o, lse = parity.run_gpu(q, k, v, causal)
    o_ref, lse_ref = parity.oracle.attention_qk(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                                v.cpu().double().numpy(), causal)
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref, what)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk", QK)
def test_qk_full(B, Hq, Hkv, Sq, Sk, causal):
    q, k, v = _qk_inputs(B, Hq, Hkv, Sq, Sk, 128, seed=37)
    _qk_check(q, k, v, causal, "Sq%d Sk%d causal=%d" % (Sq, Sk, causal))


def test_qk_noncausal_more_queries_than_keys():
    q, k, v = _qk_inputs(1, 4, 2, 500, 130, 128, seed=43)
    _qk_check(q, k, v, False, "Sq500 Sk130")


@pytest.mark.parametrize("causal", [True, False])
def test_qk_stress_and_d64(causal):
    q, k, v = _qk_inputs(1, 8, 2, 100, 700, 128, seed=47, qk_std=4.0)
    _qk_check(q, k, v, causal, "stress Sq100 Sk700")
    q, k, v = _qk_inputs(1, 4, 2, 200, 450, 64, seed=53)
    _qk_check(q, k, v, causal, "D64 Sq200 Sk450")


def test_qk_prefill_over_long_prefix():
    """64 new queries over 8192 cached keys (causal, bottom-right)."""
    q, k, v = _qk_inputs(2, 32, 8, 64, 8192, 128, seed=59)
    _qk_check(q, k, v, True, "Sq64 Sk8192")


def test_qk_causal_more_queries_than_keys_rejected():
    q, k, v = _qk_inputs(1, 4, 2, 300, 200, 128, seed=61)
    with pytest.raises(attn.AttnError):
        attn.attn_fwd(q, k, v, True)


def test_llama3_8b_s512_b1_full():
    w = WORKLOADS["llama3-8b-s512-b1"]
    parity.full_check(w["B"], w["Hq"], w["Hkv"], w["S"], w["D"], w["causal"], seed=0)


@pytest.mark.parametrize("name", ["llama3-8b-s8192-b1", "llama3-8b-s2048-b64",
                                  "llama3-8b-s8192-b64", "llama3-70b-s8192-b64",
                                  "gqa32x8-d256-s8192-b16"])
def test_workload_sampled(name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w["B"], w["Hq"], w["Hkv"], w["S"], w["D"], seed=0, device="cuda")
    o, lse = parity.run_gpu(q, k, v, w["causal"])
    assert not torch.isnan(o).any().item() and not torch.isnan(lse).any().item()
    parity.sampled_check(q, k, v, o, lse, w["causal"], n_random=1024)
    del q, k, v, o, lse
    torch.cuda.empty_cache()


SWEEP = sweep_points()


@pytest.mark.parametrize("pt", SWEEP, ids=lambda p: "Hq%d-S%d-B%d-%s" % (
    p["Hq"], p["S"], p["B"], "causal" if p["causal"] else "full"))
def test_stress_sweep(pt):
    """The 40-point sweep, Q, K ~ N(0,4^2), V ~ N(0,1): full check when the
    oracle is cheap (B=1, S<=1024), else sampled rows."""
    B, Hq, Hkv, S, D, causal = pt["B"], pt["Hq"], pt["Hkv"], pt["S"], pt["D"], pt["causal"]
    seed = 100 + SWEEP.index(pt)
    if B == 1 and S <= 1024:
        parity.full_check(B, Hq, Hkv, S, D, causal, seed=seed, qk_std=4.0)
        return
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=seed, qk_std=4.0, device="cuda")
    o, lse = parity.run_gpu(q, k, v, causal)
    assert not torch.isnan(o).any().item() and not torch.isnan(lse).any().item()
    parity.sampled_check(q, k, v, o, lse, causal, n_random=256, seed=seed,
                         full_heads=(S <= 2048))
    del q, k, v, o, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S", [(8, 24, 8, 1000), (4, 32, 8, 1100), (2, 24, 8, 6000)])
def test_default_head_pairs(B, Hq, Hkv, S, causal):
    """Calls the table sends to the head-pair ping-pong (enough heads for
    two-tile items): an even group pairs the same rows of two heads, an odd
    one (24 / 8 = 3) falls back to row pairs; ragged S in both."""
    from tests.test_variants import table_rules, expected_variant
    var = attn.variant_select(B, Hq, Hkv, S, S, 128, 1 if causal else 0)
    assert var == expected_variant(table_rules(), 128, 1 if causal else 0, S)
    q, k, v = make_qkv(B, Hq, Hkv, S, 128, seed=41, device="cuda")
    o, lse = parity.run_gpu(q, k, v, causal)
    parity.sampled_check(q, k, v, o, lse, causal, n_random=384, seed=42)


def test_deterministic():
    q, k, v = make_qkv(2, 8, 2, 1024, 128, seed=3, device="cuda")
    o1, l1 = parity.run_gpu(q, k, v, True)
    o2, l2 = parity.run_gpu(q, k, v, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_output_only_16_byte_aligned(D):
    """O at an address that is 16- but not 32-byte aligned goes out as 16-byte
    stores instead of full-sector ones; it must hold exactly what the call
    with an aligned O stores, and nothing past it may change."""
    B, Hq, Hkv, S = 2, 8, 2, 300
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=5, device="cuda")
    o1, l1 = attn.attn_fwd(q, k, v, True)
    buf = torch.full((q.numel() + 16,), 7.0, dtype=torch.float16, device="cuda")
    o2 = buf[8:8 + q.numel()].view_as(q)  # +16 bytes from a 256-byte aligned base
    assert o2.data_ptr() % 32 == 16
    _, l2 = attn.attn_fwd(q, k, v, True, o=o2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.all(buf[:8] == 7.0) and torch.all(buf[8 + q.numel():] == 7.0)


def test_concurrent_streams():
    """Calls on two streams run at the same time, each with its own status
    block: large-V inputs (every item recomputed by the exact pass) on one
    stream and N(0,1) inputs on the other give the same bytes as the same
    calls made one after another on the default stream."""
    B, Hq, Hkv, S, D = 2, 8, 2, 640, 128
    qa, ka, _ = make_qkv(B, Hq, Hkv, S, D, seed=71, device="cuda")
    va = _large_v(B, Hkv, S, D, seed=73)
    qb, kb, vb = make_qkv(B, Hq, Hkv, S, D, seed=79, device="cuda")
    ref_a = parity.run_gpu(qa, ka, va, True)
    ref_b = parity.run_gpu(qb, kb, vb, False)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            oa, la = attn.attn_fwd(qa, ka, va, True, stream=s1)
        with torch.cuda.stream(s2):
            ob, lb = attn.attn_fwd(qb, kb, vb, False, stream=s2)
        outs.append((oa, la, ob, lb))
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    for oa, la, ob, lb in outs:
        assert torch.equal(oa, ref_a[0]) and torch.equal(la, ref_a[1])
        assert torch.equal(ob, ref_b[0]) and torch.equal(lb, ref_b[1])


def test_zero_query_prefix_mean():
    """Q = 0: O_i = mean of V_0..V_i (causal), LSE_i = ln(i+1)."""
    B, Hq, Hkv, S, D = 1, 4, 2, 512, 128
    _, k, v = make_qkv(B, Hq, Hkv, S, D, seed=5, device="cuda")
    q = torch.zeros(B, Hq, S, D, dtype=torch.float16, device="cuda")
    o, lse = parity.run_gpu(q, k, v, True)
    vv = v.double()
    prefix = vv.cumsum(dim=2) / torch.arange(1, S + 1, device="cuda", dtype=torch.float64)[:, None]
    ref = prefix.repeat_interleave(Hq // Hkv, dim=1)
    assert (o.double() - ref).abs().max().item() <= parity.O_TOL
    ln = torch.log(torch.arange(1, S + 1, device="cuda", dtype=torch.float64))
    assert (lse.double() - ln).abs().max().item() <= parity.LSE_TOL


def test_constant_v():
    B, Hq, Hkv, S, D = 1, 4, 1, 384, 128
    q, k, _ = make_qkv(B, Hq, Hkv, S, D, seed=6, qk_std=4.0, device="cuda")
    c = torch.randn(D, device="cuda").half()
    v = c.expand(B, Hkv, S, D).contiguous()
    for causal in (True, False):
        o, _ = parity.run_gpu(q, k, v, causal)
        assert (o.double() - c.double()).abs().max().item() <= parity.O_TOL


@pytest.mark.parametrize("B,Hq,Hkv,S,D,pinned", [(1, 8, 2, 512, 128, True),
                                                 (11, 4, 2, 384, 128, True),
                                                 (3, 1, 1, 77, 64, True),
                                                 (5, 2, 1, 200, 128, False),
                                                 (3, 4, 2, 300, 256, True)])
def test_host_entry_matches_device_entry(B, Hq, Hkv, S, D, pinned):
    """The host-buffer entry (a pipeline over up to 16 batch chunks on the
    library's own streams) gives the device entry's bytes, including chunks
    whose LSE slices start off a 16-byte boundary, and from pageable memory."""
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=9, device="cuda")
    o, lse = parity.run_gpu(q, k, v, True)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    oh = torch.full_like(qh, float("nan"))
    lh = torch.full((B, Hq, S), float("nan"), dtype=torch.float32)
    if pinned:
        qh, kh, vh, oh, lh = (t.pin_memory() for t in (qh, kh, vh, oh, lh))
    ws = torch.empty(attn.host_workspace_bytes(B, Hq, Hkv, S, D), dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(qh, kh, vh, oh, lh, True, ws)
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu())


def test_host_entry_concurrent_threads():
    """Two host threads call the host-buffer entry at the same time on one device
    (ctypes drops the GIL, and the library runs the calls one after another on
    its pipeline streams): every call gives the device entry's bytes."""
    import threading
    cases = []
    for i, (B, Hq, Hkv, S) in enumerate([(6, 4, 2, 384), (5, 8, 2, 256)]):
        q, k, v = make_qkv(B, Hq, Hkv, S, 128, seed=70 + i, device="cuda")
        o, lse = parity.run_gpu(q, k, v, True)
        host = [t.cpu().pin_memory() for t in (q, k, v)]
        oh = torch.empty_like(host[0]).pin_memory()
        lh = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
        ws = torch.empty(attn.host_workspace_bytes(B, Hq, Hkv, S, 128), dtype=torch.uint8,
                         device="cuda")
        cases.append((host, oh, lh, ws, o.cpu(), lse.cpu()))
    torch.cuda.synchronize()
    errors = []

    def run(c):
        try:
            torch.cuda.set_device(0)
            for _ in range(3):
                c[1].fill_(float("nan"))
                c[2].fill_(float("nan"))
                attn.attn_fwd_host(*c[0], c[1], c[2], True, c[3])
                assert torch.equal(c[1], c[4]) and torch.equal(c[2], c[5])
        except Exception as e:  # reported by the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(c,)) for c in cases]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors


def test_bounded_wait_reports_timeout():
    """A wait on an mbarrier nobody completes ends after its bound with
    ATTN_ERR_DEVICE_TIMEOUT, and the context stays usable."""
    assert attn.selftest_wait_timeout(20_000_000) == attn.ATTN_ERR_DEVICE_TIMEOUT
    assert attn.device_status() == (attn.ATTN_OK, 0)
    parity.full_check(1, 2, 1, 256, 128, True, seed=1)


def test_unsupported_shape_raises():
    q = torch.zeros(1, 2, 128, 96, dtype=torch.float16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_fwd(q, q, q)


def _large_v(B, Hkv, S, D, seed):
    """V in [4, 6] with random signs: every output row has |O| >= 4, where the
    fp16 output rounding leaves only ~5e-5 for everything else."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    mag = 4.0 + 2.0 * torch.rand(B, Hkv, S, D, generator=g, device="cuda")
    sign = torch.where(torch.rand(B, Hkv, S, D, generator=g, device="cuda") < 0.5, -1.0, 1.0)
    return (mag * sign).half()


@pytest.mark.parametrize("causal", [True, False])
def test_large_outputs_exact_rows(causal):
    """All rows exceed the fixup threshold (list mode): peaky logits mix a
    few large values, and every row must still be within 2e-3."""
    B, Hq, Hkv, S, D = 1, 4, 2, 1024, 128
    q, k, _ = make_qkv(B, Hq, Hkv, S, D, seed=21, qk_std=4.0, device="cuda")
    v = _large_v(B, Hkv, S, D, 22)
    o, lse = parity.run_gpu(q, k, v, causal)
    import oracle
    o_ref, lse_ref = oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                      v.cpu().double().numpy(), causal)
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        "large V causal=%d" % causal)


def test_large_outputs_every_item_exact():
    """Every 256-row item of every CTA is marked (many per CTA): the exact
    pass recomputes all of them in the same launch.  Sampled rows against the
    oracle, and the call's status block counts every item."""
    B, Hq, Hkv, S, D = 4, 16, 4, 2048, 128   # 512 items of 256 rows, all marked
    q, k, _ = make_qkv(B, Hq, Hkv, S, D, seed=23, qk_std=4.0, device="cuda")
    v = _large_v(B, Hkv, S, D, 24)
    attn.device_status_ex()  # clear
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device="cuda")
    attn.attn_fwd(q, k, v, True, o=o, lse=lse)
    st, site, n_exact = attn.device_status_ex()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    assert n_exact == B * Hq * (S // 256), n_exact
    parity.sampled_check(q, k, v, o, lse, True, n_random=512, seed=25, full_heads=True)
    # nothing carries over: a plain call right after still passes
    parity.full_check(1, 2, 1, 256, 128, True, seed=26)


@pytest.mark.parametrize("large_keys", ["first", "second"])
def test_exact_pass_one_tile_of_an_item(large_keys):
    """Items of 256 rows (the ping-pong kernel, variant 0, with enough heads
    for two-tile items) where only one 128-row tile has |O| >= 4.  V is large
    (|v| in [4, 6]) only on keys 0-127 ("first": the first rows of tile A
    follow those values, tile B averages them with small ones under diffuse
    logits) or only on keys 128-255 ("second": peaked logits, so rows of tile
    B follow single large values, while tile A never sees those keys).  The
    exact pass runs the marked tile alone; every row must match the oracle,
    and the call counts each item with a marked tile once."""
    B, Hq, Hkv, S, D = 8, 32, 8, 256, 128   # one 256-row item per head, 256 items
    qk_std = 0.5 if large_keys == "first" else 4.0
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=31, qk_std=qk_std, device="cuda")
    big = _large_v(B, Hkv, S, D, 32)
    small = (v.float() * 0.01).half()
    keys = torch.arange(S, device="cuda").view(1, 1, S, 1)
    in_large = keys < 128 if large_keys == "first" else keys >= 128
    v = torch.where(in_large, big, small).contiguous()
    attn.device_status_ex()  # clear
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device="cuda")
    attn.attn_fwd_variant(q, k, v, True, 0, o=o, lse=lse)
    st, site, n_exact = attn.device_status_ex()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    import oracle
    o_ref, lse_ref = oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                      v.cpu().double().numpy(), True)
    row_max = np.abs(o_ref).max(axis=-1)                      # [B, Hq, S]

    def marked(thr):
        return (row_max >= thr).reshape(B, Hq, 2, 128).any(axis=-1)   # [B, Hq, tile]
    # the kernel applies the threshold to its own O; rows within 0.01 of it
    # may go either way
    surely, maybe = marked(3.98 + 0.01), marked(3.98 - 0.01)
    if large_keys == "first":
        assert surely[..., 0].all() and not maybe[..., 1].any()
    else:
        assert surely[..., 1].any() and not maybe[..., 0].any()
    assert int(surely.any(axis=-1).sum()) <= n_exact <= int(maybe.any(axis=-1).sum()), n_exact
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        "one tile marked (%s)" % large_keys)


def test_exact_pass_only_where_needed():
    """N(0,1) inputs at a long sequence: outputs average many V rows, so only
    the first rows of a head can reach |O| >= 3.98 -- few items, all of them
    in the last row block of the walk order (row block 0 of each head)."""
    B, Hq, Hkv, S, D = 2, 16, 4, 4096, 128
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=27, device="cuda")
    attn.device_status_ex()
    o, lse = attn.attn_fwd(q, k, v, True)
    st, site, n_exact = attn.device_status_ex()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    assert n_exact <= B * Hq, n_exact
    parity.sampled_check(q, k, v, o, lse, True, n_random=256, seed=27, full_heads=False)


def test_status_blocks_are_per_stream():
    """A wait that runs out on one stream is reported by that stream's status
    and not by another stream's, even while that other stream runs attention."""
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    q, k, v = make_qkv(1, 8, 2, 1024, 128, seed=31, device="cuda")
    assert attn.selftest_wait_timeout(20_000_000, stream=s1) == attn.ATTN_ERR_DEVICE_TIMEOUT
    with torch.cuda.stream(s2):
        attn.attn_fwd(q, k, v, True, stream=s2)
    assert attn.device_status(s2) == (attn.ATTN_OK, 0)
    # the self-test read (and cleared) s1's block itself; nothing is left there
    assert attn.device_status(s1) == (attn.ATTN_OK, 0)


# Items of two 128-row tiles (the launch has at least as many 256-row items as
# SMs): full oracle checks, including an odd number of row blocks (the last
# item has tile A only) and a ragged last tile.
TWO_TILE = [(2, 40, 8, 512, 128, 1.0), (1, 64, 8, 600, 128, 1.0), (1, 64, 8, 700, 128, 4.0),
            (1, 80, 8, 520, 64, 1.0)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S,D,qk_std", TWO_TILE)
def test_two_tile_items_full(B, Hq, Hkv, S, D, qk_std, causal):
    parity.full_check(B, Hq, Hkv, S, D, causal, seed=33, qk_std=qk_std)


def test_call_split_into_launches():
    """More items than one launch's per-CTA marks hold (2048 per CTA): the
    call runs as several launches over batch ranges.  Sampled rows from the
    first and the last batch elements."""
    B, Hq, Hkv, S, D = 2500, 64, 8, 300, 64   # 320000 items of 256 rows
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=35, device="cuda")
    o, lse = parity.run_gpu(q, k, v, True)
    import oracle
    for b in (0, 1, B // 2, B - 2, B - 1):
        for hq in (0, Hq - 1):
            o_ref, lse_ref = oracle.attention(q[b:b + 1, hq:hq + 1].cpu().double().numpy(),
                                              k[b:b + 1, hq // 8:hq // 8 + 1].cpu().double().numpy(),
                                              v[b:b + 1, hq // 8:hq // 8 + 1].cpu().double().numpy(),
                                              True)
            parity.assert_close(o[b:b + 1, hq:hq + 1].cpu().double().numpy(), o_ref,
                                lse[b:b + 1, hq:hq + 1].cpu().double().numpy(), lse_ref,
                                "split call b=%d hq=%d" % (b, hq))
    del q, k, v, o, lse
    torch.cuda.empty_cache()


def test_fastdiv_device_matches_floor_division():
    """The kernels' item decode divides with a multiply-high and a shift; on
    the device it is exact floor division for numerators below 2^31."""
    rng = np.random.default_rng(11)
    ds = list(range(1, 130)) + [255, 256, 257, 4095, 4096, 4097, 2 ** 30 + 1, 2 ** 31 - 1]
    ds += [int(x) for x in rng.integers(1, 2 ** 31 - 1, 16)]
    for d in ds:
        ns = np.concatenate([np.arange(0, 4096), rng.integers(0, 2 ** 31, 8192),
                             np.array([2 ** 31 - 1, 2 ** 31 - 2]),
                             (np.arange(1, 64) * d - 1) % 2 ** 31, (np.arange(1, 64) * d) % 2 ** 31])
        n = torch.from_numpy(ns.astype(np.int32)).cuda()
        q = attn.selftest_fastdiv(d, n).cpu().numpy().astype(np.int64)
        assert np.array_equal(q, ns.astype(np.int64) // d), d


def test_fma_pipe_exp2_error_bound():
    """The polynomial 2^x available to the fused pass for part of its
    exponentials: relative error <= 8e-5 against fp64 exp2 for x in
    [-125, 8] (results of normal fp32 range), and non-negative results below
    2^-124 (they round to 0 in fp16) further down, including -inf."""
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 20, generator=g, device="cuda") * 133.0 - 125.0,
                   torch.arange(-125, 9, device="cuda", dtype=torch.float32)])
    y = attn.selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs().max().item()
    assert rel <= 8e-5, rel
    lo = attn.selftest_exp2(torch.tensor([-125.3, -125.9, -126.0, -127.0, -200.0, -1e30,
                                          float("-inf")], device="cuda"))
    assert torch.all(lo >= 0) and torch.all(lo < 2.0 ** -124), lo


# Every fused-kernel variant (two-tile ping-pong over row pairs or head
# pairs, one tile with S double-buffered and one or two softmax warps per lane
# quadrant, x 0..4 of every 8 exponential pairs from the FMA-pipe polynomial)
# through attn_fwd_variant, against the oracle: both head dims, a ragged
# tail, logits of standard deviation 1 and 16, one-tile and two-tile items.
VARIANT_CASES = [(2, 4, 2, 383, 128, 1.0), (1, 8, 2, 512, 128, 4.0), (2, 4, 2, 329, 64, 1.0),
                 (1, 4, 2, 640, 64, 4.0), (1, 64, 8, 700, 128, 1.0), (2, 48, 8, 520, 128, 4.0),
                 (1, 96, 8, 384, 64, 1.0), (2, 32, 1, 300, 128, 1.0)]


def _variant_check(q, k, v, causal, variant, what):
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    attn.attn_fwd_variant(q, k, v, causal, variant, o=o, lse=lse)
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    o_ref, lse_ref = parity.oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                             v.cpu().double().numpy(), causal)
    parity.assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        what)


@pytest.mark.parametrize("variant", range(20))
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,Hq,Hkv,S,D,qk_std", VARIANT_CASES)
def test_variant_full(B, Hq, Hkv, S, D, qk_std, causal, variant):
    assert attn.variant_count() == 20
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=41, qk_std=qk_std, device="cuda")
    _variant_check(q, k, v, causal, variant, "%s B%d Hq%d S%d D%d std%g causal=%d" % (
        attn.variant_name(variant), B, Hq, S, D, qk_std, causal))


@pytest.mark.parametrize("variant", [2, 4, 5, 7, 10, 12, 15, 17])
def test_variant_large_outputs(variant):
    """Large V: every item goes through the exact pass after an emulating fast pass."""
    q, k, _ = make_qkv(1, 8, 2, 384, 128, seed=43, device="cuda")
    v = _large_v(1, 2, 384, 128, seed=47)
    _variant_check(q, k, v, True, variant, "large V, %s" % attn.variant_name(variant))


def test_variant_default_is_table_choice():
    """attn_fwd runs the variant attn_variant_select names: same bytes."""
    for D in (64, 128):
        q, k, v = make_qkv(1, 8, 2, 1024, D, seed=53, device="cuda")
        var = attn.variant_select(1, 8, 2, 1024, 1024, D, True)
        assert 0 <= var < attn.variant_count()
        o1, l1 = parity.run_gpu(q, k, v, True)
        o2, l2 = attn.attn_fwd_variant(q, k, v, True, var)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
