"""paged_decode_attention_noalloc: the decode entry point for callers that
cannot allocate device memory (a plug-in whose host owns all device
allocations, or a path that must not allocate), checked against the
workspace-taking paged_decode_attention on two calls in a row.

Kept in its own file, named so pytest collects it last.
"""
import numpy as np
import pytest
import torch

from gpu_cases import build_cache, to_device
from helpers import TOL
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cfg = W.LONG32K  # one layer of the 32K-token sequence: split-KV is chosen, so the scratch is used
    P = cfg.page_size
    st = build_cache(cfg, W.cached_lengths(cfg))
    S = K.paged_decode_num_splits(cfg.B, cfg.H_kv, st.max_blocks, P, 0)
    need = K.paged_decode_workspace_bytes(cfg.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, P, 0)
    assert S > 1 and 0 < need <= K.KV_NOALLOC_SCRATCH_BYTES
    tab = torch.from_numpy(st.tab).cuda()
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    atol, rtol = TOL[cfg.dtype]
    for step in range(2):
        lens32 = st.lens.astype(np.int32).copy()
        slots = st.pool.append_slots(st.tab, lens32)
        tab.copy_(torch.from_numpy(st.tab))
        k_new, v_new = W.new_token_kv(cfg, 0, step)
        K.kv_append(st.k_pages, st.v_pages, to_device(k_new, cfg.dtype), to_device(v_new, cfg.dtype),
                    torch.from_numpy(slots).cuda(), P)
        st.lens = st.lens + 1
        q = to_device(W.queries(cfg, 0, step), cfg.dtype)
        lens = torch.from_numpy(lens32).cuda()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = torch.empty((cfg.B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
        got = torch.full_like(ref, float("nan"))
        K.paged_decode_attention(ref, q, st.k_pages, st.v_pages, tab, lens, cfg.scale, workspace=ws, err_flag=err)
        K.paged_decode_attention_noalloc(got, q, st.k_pages, st.v_pages, tab, lens, cfg.scale, err_flag=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        r, g = ref.cpu().numpy().astype(np.float64), got.cpu().numpy()
        assert np.isfinite(g).all()
        assert (np.abs(g - r) <= atol + rtol * np.abs(r)).all(), f"call {step}: max diff {np.abs(g - r).max():.3e}"


def test_noalloc_refuses_partials_beyond_the_scratch():
    B, H_q, H_kv, Dh, P, max_blocks = 64, 32, 8, 128, 16, 300
    splits = 128
    assert K.paged_decode_workspace_bytes(B, H_q, H_kv, Dh, max_blocks, P, splits) > K.KV_NOALLOC_SCRATCH_BYTES
    k_pages = torch.zeros((4, H_kv, P, Dh), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((B, H_q, Dh), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((B, H_q, Dh), dtype=torch.float32, device="cuda")
    tab = torch.zeros((B, max_blocks), dtype=torch.int32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    with pytest.raises(K.KvError) as e:
        K.paged_decode_attention_noalloc(out, q, k_pages, k_pages, tab, lens, 0.1, num_splits=splits)
    assert e.value.name == "WORKSPACE"
    # without splits the scratch is not needed at all
    K.paged_decode_attention_noalloc(out, q, k_pages, k_pages, tab, lens, 0.1, num_splits=1)
    torch.cuda.synchronize()
