"""attn_fwd_noalloc: the entry point for callers that cannot let the library
allocate device memory (everything planned up front, their own caching
allocator, or no room for the device synchronization a cudaMalloc may cause).
Its scratch is a fixed array inside the library.  Called through the C ABI and
compared with attn_fwd, the entry point that allocates its scratch, on two
calls in a row, with inputs that do and do not use the scratch list.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import pytest
import torch

from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.inputs import make_qkv
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
    attn.device_status()


def _noalloc(q, k, v, causal):
    B, Hq, S, D = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=q.device)
    st = attn.attn_fwd_noalloc_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), B, Hq, k.shape[1], S, D, causal,
                                   int(torch.cuda.current_stream().cuda_stream))
    assert st == attn.ATTN_OK, attn.status_string(st)
    assert attn.device_status() == (attn.ATTN_OK, 0)
    return o, lse


def _large_v_like(v, seed):
    # values in [4, 6] with random signs: rows cross |O| >= 4, so the fast
    # pass lists items in the scratch array and the second pass redoes them
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    mag = 4.0 + 2.0 * torch.rand(v.shape, generator=g, device="cuda")
    sign = torch.where(torch.rand(v.shape, generator=g, device="cuda") < 0.5, -1.0, 1.0)
    return (mag * sign).half()


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_attn_fwd_two_calls(causal):
    cases = []
    q, k, v = make_qkv(2, 8, 2, 1280, 128, seed=41, device="cuda")
    cases.append((q, k, v))                                    # scratch list stays empty
    q2, k2, _ = make_qkv(2, 8, 2, 1280, 128, seed=42, qk_std=4.0, device="cuda")
    cases.append((q2, k2, _large_v_like(v, 43)))               # many items listed
    for call in range(2):  # two calls in a row: the shared array must not carry state over
        for q_, k_, v_ in cases:
            o_ref, lse_ref = parity.run_gpu(q_, k_, v_, causal)
            o, lse = _noalloc(q_, k_, v_, causal)
            eo = (o.double() - o_ref.double()).abs().max().item()
            el = (lse.double() - lse_ref.double()).abs().max().item()
            assert eo <= parity.O_TOL and el <= parity.LSE_TOL, (call, eo, el)


def test_noalloc_rejects_more_work_than_its_scratch():
    # B * Hq * ceil(S/256) = 2 * 64 * 1025 > 131072 items: rejected before any launch
    st = attn.attn_fwd_noalloc_raw(16, 16, 16, 16, 16, 2, 64, 8, 262400, 128, True, 0)
    assert st == attn.ATTN_ERR_TOO_LARGE, attn.status_string(st)
