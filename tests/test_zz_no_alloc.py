"""paged_decode_attention_noalloc: the decode entry point for callers that
cannot allocate device memory (a plug-in whose host owns all device
allocations, or a path that must not allocate), checked on two calls in a row
against the workspace-taking paged_decode_attention and against the fp64
oracle, on the three launch forms that can reach the shared scratch array:
a grid split of one long row, a device-planned launch (plan header, item list
and partials all in the array), and an automatic split count that is lowered
because its partials would not fit.

Kept in its own file, named so pytest collects it last.
"""
import numpy as np
import pytest
import torch

from gpu_cases import build_cache, check_close, to_device
from helpers import TOL
from oracle import reference as R
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _two_calls(st, splits_ws):
    """Two decode steps: append the new token (kv_append), then decode through both entry points.
    The workspace entry point runs with `splits_ws`, the no-allocation one with num_splits = 0."""
    cfg = st.cfg
    P = cfg.page_size
    B = len(st.lens)
    tab = torch.from_numpy(st.tab).cuda()
    need = K.paged_decode_workspace_bytes(B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, P, splits_ws)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    atol, rtol = TOL[cfg.dtype]
    for step in range(2):
        lens32 = st.lens.astype(np.int32).copy()
        mlens = [int(x) for x in st.lens]
        slots = st.pool.append_slots(st.tab, lens32)
        assert list(slots) == st.mpool.append_slots(st.mtab, st.max_blocks, mlens)
        tab.copy_(torch.from_numpy(st.tab))
        k_new, v_new = W.new_token_kv(cfg, 0, step)
        k_new, v_new = k_new[:B], v_new[:B]
        for b in range(B):
            page, off = divmod(int(slots[b]), P)
            st.kp[page, :, off, :] = k_new[b]
            st.vp[page, :, off, :] = v_new[b]
        K.kv_append(st.k_pages, st.v_pages, to_device(k_new, cfg.dtype), to_device(v_new, cfg.dtype),
                    torch.from_numpy(slots).cuda(), P)
        st.lens = st.lens + 1
        qh = W.queries(cfg, 0, step)[:B]
        q = to_device(qh, cfg.dtype)
        lens = torch.from_numpy(lens32).cuda()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
        got = torch.full_like(ref, float("nan"))
        K.paged_decode_attention(ref, q, st.k_pages, st.v_pages, tab, lens, cfg.scale, num_splits=splits_ws,
                                 workspace=ws, err_flag=err)
        K.paged_decode_attention_noalloc(got, q, st.k_pages, st.v_pages, tab, lens, cfg.scale, err_flag=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        r, g = ref.cpu().numpy().astype(np.float64), got.cpu().numpy()
        assert np.isfinite(g).all()
        assert (np.abs(g - r) <= atol + rtol * np.abs(r)).all(), f"call {step}: max diff {np.abs(g - r).max():.3e}"
        oracle = R.paged_decode(qh, st.kp, st.vp, st.tab, lens32, cfg.scale, cfg.dtype)
        check_close(g, oracle, cfg.dtype, f"no-allocation entry point vs oracle, call {step}")


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cfg = W.LONG32K  # one layer of the 32K-token sequence: split-KV is chosen, so the scratch is used
    P = cfg.page_size
    st = build_cache(cfg, W.cached_lengths(cfg))
    S = K.paged_decode_num_splits(cfg.B, cfg.H_kv, st.max_blocks, P, 0)
    need = K.paged_decode_workspace_bytes(cfg.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, P, 0)
    assert S > 1 and 0 < need <= K.KV_NOALLOC_SCRATCH_BYTES
    _two_calls(st, 0)


def test_noalloc_planned_launch_on_two_calls():
    """A device-planned launch (many rows, skewed lengths): plan, items and partials share the array."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H_kv = 8
    B = max(256, (4 * sms) // H_kv + 8)
    cfg = W.DecodeConfig(f"noalloc-planned-B{B}", "bf16", B=B, H_q=32, H_kv=H_kv, Dh=128, page_size=16, seed=31)
    st = build_cache(cfg, W.ragged_lengths(B, 16, cfg.seed), slack_pages=B)
    assert K.paged_decode_num_splits(B, H_kv, st.max_blocks, 16, 0) == 0  # planned
    need = K.paged_decode_workspace_bytes(B, cfg.H_q, H_kv, cfg.Dh, st.max_blocks, 16, 0)
    assert 0 < need <= K.KV_NOALLOC_SCRATCH_BYTES
    _two_calls(st, 0)


def test_noalloc_lowers_an_automatic_split_that_does_not_fit():
    """MQA batch with a wide block table: the automatic split count's partials exceed the array, so the
    no-allocation entry point lowers it; its output still matches the workspace entry point and the oracle."""
    B, P = 256, 16
    cfg = W.DecodeConfig("noalloc-mqa-B256", "bf16", B=B, H_q=32, H_kv=1, Dh=128, page_size=P, seed=32)
    max_blocks = -(-(16384 + 26) // P) + 1  # the mixed sweep's table width
    st = build_cache(cfg, W.ragged_lengths(B, P, cfg.seed), max_blocks=max_blocks, slack_pages=B)
    S = K.paged_decode_num_splits(B, 1, max_blocks, P, 0)
    assert S > 1
    assert K.paged_decode_workspace_bytes(B, cfg.H_q, 1, cfg.Dh, max_blocks, P, 0) > K.KV_NOALLOC_SCRATCH_BYTES
    _two_calls(st, 0)


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
