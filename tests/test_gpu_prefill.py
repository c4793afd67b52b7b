"""GPU parity of paged_prefill_attention (chunk of new tokens per sequence,
causal within the chunk) against the oracle's fp64 restatement."""
import numpy as np
import pytest
import torch

from gpu_cases import build_cache, check_close, to_device
from oracle import reference as R
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run(cfg, totals, chunks, max_q_len=None, expect_err=0):
    """Cache holds `totals[b]` tokens of sequence b (its chunk included); the chunk is its last chunks[b]."""
    st = build_cache(cfg, totals, slack_pages=2)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    rows = [W.all_queries(cfg, 0, b, int(L))[int(L) - int(n):] if n <= L else
            W.all_queries(cfg, 0, b, int(n)) for b, (L, n) in enumerate(zip(totals, chunks))]
    q = np.concatenate(rows) if rows else np.zeros((0, cfg.H_q, cfg.Dh), np.uint16)
    lens = np.asarray(totals, np.int32)
    out = torch.full((int(q_start[-1]), cfg.H_q, cfg.Dh), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.paged_prefill_attention(out, to_device(q, cfg.dtype), torch.from_numpy(q_start).cuda(),
                              max(chunks) if max_q_len is None else max_q_len, st.k_pages, st.v_pages,
                              torch.from_numpy(st.tab).cuda(), torch.from_numpy(lens).cuda(), cfg.scale, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == expect_err
    got = out.cpu().numpy()
    return got, q, q_start, st, lens


PREFILL_SHAPES = [
    # dtype, Dh, P, H_q, H_kv
    ("bf16", 128, 16, 32, 8), ("fp16", 128, 16, 32, 8), ("bf16", 64, 32, 16, 4), ("bf16", 128, 16, 8, 8),
    ("fp16", 128, 32, 64, 8), ("bf16", 128, 16, 32, 1), ("fp16", 64, 16, 12, 4), ("bf16", 128, 16, 64, 1),
]


@pytest.mark.parametrize("dtype,Dh,P,H_q,H_kv", PREFILL_SHAPES)
def test_prefill_against_oracle(dtype, Dh, P, H_q, H_kv):
    cfg = W.DecodeConfig(f"prefill-{dtype}-{Dh}-{P}-{H_q}-{H_kv}", dtype, B=5, H_q=H_q, H_kv=H_kv, Dh=Dh, page_size=P,
                         seed=80)
    totals = [700, 233, 95, 40, 1]     # cached tokens after the chunk's append
    chunks = [100, 64, 95, 17, 1]      # a prompt extension, a tile-sized chunk, a whole prompt, ...
    got, q, q_start, st, lens = _run(cfg, totals, chunks)
    ref = R.paged_prefill(q, q_start, st.kp, st.vp, st.tab, lens, cfg.scale, dtype)
    check_close(got, ref, dtype, cfg.name)


def test_prefill_edge_chunks():
    cfg = W.DecodeConfig("prefill-edge", "bf16", B=4, H_q=32, H_kv=8, Dh=128, page_size=16, seed=81)
    totals = [50, 16, 33, 17]
    chunks = [0, 16, 33, 2]            # an empty chunk, a whole page, a whole prompt, a chunk across a page edge
    got, q, q_start, st, lens = _run(cfg, totals, chunks, max_q_len=48)
    ref = R.paged_prefill(q, q_start, st.kp, st.vp, st.tab, lens, cfg.scale, "bf16")
    check_close(got, ref, "bf16", "prefill edge chunks")


def test_prefill_long_context_chunk_sampled():
    cfg = W.DecodeConfig("prefill-long", "bf16", B=2, H_q=32, H_kv=8, Dh=128, page_size=16, seed=82)
    totals = [8192 + 512, 3000]
    chunks = [512, 1]
    got, q, q_start, st, lens = _run(cfg, totals, chunks)
    ref = R.paged_prefill(q, q_start, st.kp, st.vp, st.tab, lens, cfg.scale, "bf16")
    check_close(got, ref, "bf16", "prefill long")


def test_prefill_one_token_chunks_equal_decode():
    cfg = W.DecodeConfig("prefill-as-decode", "bf16", B=3, H_q=32, H_kv=8, Dh=128, page_size=16, seed=83)
    totals = [300, 47, 1000]
    got, q, q_start, st, lens = _run(cfg, totals, [1, 1, 1])
    out = torch.empty_like(torch.from_numpy(got)).cuda()
    K.paged_decode_attention(out, to_device(q, "bf16"), st.k_pages, st.v_pages, torch.from_numpy(st.tab).cuda(),
                             torch.from_numpy(lens).cuda(), cfg.scale, num_splits=1)
    torch.cuda.synchronize()
    check_close(got, out.cpu().numpy().astype(np.float64), "bf16", "one-token chunks vs decode")


def test_prefill_chunk_longer_than_sequence_sets_error():
    cfg = W.DecodeConfig("prefill-bad", "bf16", B=2, H_q=8, H_kv=2, Dh=128, page_size=16, seed=84)
    got, q, q_start, st, lens = _run(cfg, [20, 10], [5, 12], expect_err=K.KV_DEV_ERR_SEQ_LEN)
    assert np.count_nonzero(got[q_start[1]:q_start[2]]) == 0  # the invalid chunk is zeroed
    ref = R.paged_prefill(q[:5], q_start[:2], st.kp, st.vp, st.tab[:1], lens[:1], cfg.scale, "bf16")
    check_close(got[:5], ref, "bf16", "valid chunk next to an invalid one")


@pytest.mark.parametrize("H_q,H_kv", [(8, 8), (32, 8)])
def test_prefill_repeated_launches_identical(H_q, H_kv):
    """The same launch repeated 40 times over a pool whose unused rows hold NaN: every run gives the same bits,
    and the first matches the oracle. The softmax warps may run stages ahead of the V stream; the stale V rows
    past the chunk must still be zeroed in the right fill of their ring entry, or a NaN row reaches P.V."""
    cfg = W.DecodeConfig(f"prefill-repeat-{H_q}-{H_kv}", "bf16", B=5, H_q=H_q, H_kv=H_kv, Dh=128, page_size=16,
                         seed=86)
    totals = [700, 233, 95, 40, 1]
    chunks = [100, 64, 95, 17, 1]
    got, q, q_start, st, lens = _run(cfg, totals, chunks)
    ref = R.paged_prefill(q, q_start, st.kp, st.vp, st.tab, lens, cfg.scale, "bf16")
    check_close(got, ref, "bf16", cfg.name)
    d_q = to_device(q, "bf16")
    d_qs, d_tab, d_lens = torch.from_numpy(q_start).cuda(), torch.from_numpy(st.tab).cuda(), torch.from_numpy(lens).cuda()
    out = torch.empty((int(q_start[-1]), H_q, 128), dtype=torch.float32, device="cuda")
    first = torch.from_numpy(got).cuda()
    for _ in range(40):
        out.fill_(float("nan"))
        K.paged_prefill_attention(out, d_q, d_qs, max(chunks), st.k_pages, st.v_pages, d_tab, d_lens, cfg.scale)
        torch.cuda.synchronize()
        assert torch.equal(out, first)


def test_prefill_refuses_fp32():
    k = torch.zeros((2, 2, 16, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(K.KvError):
        K.paged_prefill_attention(torch.zeros((1, 4, 64), device="cuda"), torch.zeros((1, 4, 64), device="cuda"),
                                  torch.tensor([0, 1], dtype=torch.int32, device="cuda"), 1, k, k,
                                  torch.zeros((1, 2), dtype=torch.int32, device="cuda"),
                                  torch.ones(1, dtype=torch.int32, device="cuda"), 0.1)


def test_prefill_bench_shape_sampled():
    """The chunked-prefill workload the benchmark times (8 sequences x 512-token chunk over 4096 cached
    tokens); sequences 0 and 7 are checked against the oracle."""
    cfg = W.DecodeConfig("prefill-bench", "bf16", B=8, H_q=32, H_kv=8, Dh=128, page_size=16, seed=85)
    totals, chunks = [4096 + 512] * 8, [512] * 8
    got, q, q_start, st, lens = _run(cfg, totals, chunks)
    for b in (0, 7):
        rows = slice(int(q_start[b]), int(q_start[b + 1]))
        ref = R.paged_prefill(q[rows], np.array([0, 512], np.int32), st.kp, st.vp, st.tab[b:b + 1], lens[b:b + 1],
                              cfg.scale, "bf16")
        check_close(got[rows], ref, "bf16", f"prefill bench shape, sequence {b}")


@pytest.mark.parametrize("dtype,P,H_q,H_kv", [("bf16", 16, 32, 8), ("fp16", 32, 32, 1)])
def test_prefill_warp_mma_kernel(dtype, P, H_q, H_kv):
    """Dh = 128 chunks through the warp-MMA kernel (the automatic choice there is the tcgen05 kernel)."""
    cfg = W.DecodeConfig(f"prefill-mma-{dtype}-{P}-{H_q}-{H_kv}", dtype, B=3, H_q=H_q, H_kv=H_kv, Dh=128,
                         page_size=P, seed=86)
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_MMA)
    try:
        got, q, q_start, st, lens = _run(cfg, [300, 95, 40], [100, 95, 17])
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
    ref = R.paged_prefill(q, q_start, st.kp, st.vp, st.tab, lens, cfg.scale, dtype)
    check_close(got, ref, dtype, cfg.name)
