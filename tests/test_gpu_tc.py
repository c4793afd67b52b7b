"""GPU parity of the fifth-generation tensor-core (tcgen05) decode kernel
against the fp64 oracle: selected explicitly (KV_DECODE_KERNEL_TCGEN05) for
GQA groups of 4, 8, 16 and 32 heads, the automatic choice for groups of 32
(MQA-shaped), bf16/fp16 K/V, Dh = 128.

Covers: ragged and edge lengths (1, P-1, P, P+1, a full table, a row longer
than one 128-token stage), grid splits and device-planned launches, the fused
append, empty rows, continuous batching with churn, rows whose later scores
grow far past the first stage's maximum (the reference maximum and the
accumulated output are rescaled), and the device error bits.
"""
import numpy as np
import pytest
import torch

from gpu_cases import append_and_decode, build_cache, check_close, replace_sequence, to_device
from oracle import reference as R
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)
    yield
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)


def _assert_tc(cfg, max_blocks, splits):
    S, kind = K.paged_decode_launch_info(cfg.B, cfg.H_q, cfg.H_kv, cfg.Dh, max_blocks, cfg.page_size, cfg.dtype, splits)
    assert kind == K.KV_DECODE_KERNEL_TCGEN05
    return S


TC_SHAPES = [("bf16", 16, 32, 1), ("fp16", 32, 32, 1), ("bf16", 32, 64, 2), ("fp16", 16, 96, 3),
             ("bf16", 16, 32, 8), ("fp16", 32, 16, 2), ("bf16", 16, 32, 2), ("fp16", 16, 8, 1)]


@pytest.mark.parametrize("dtype,P,H_q,H_kv", TC_SHAPES)
@pytest.mark.parametrize("splits", [1, 2, 0])
@pytest.mark.parametrize("fused", [False, True])
def test_tc_edge_lengths(dtype, P, H_q, H_kv, splits, fused):
    cfg = W.DecodeConfig(f"tc-edge-{dtype}-{P}-{H_q}-{H_kv}", dtype, B=7, H_q=H_q, H_kv=H_kv, Dh=128, page_size=P,
                         seed=41)
    # after the append: 1, P-1, P, P+1, one 128-token stage + 5, three stages + 1, and (one step) a full table
    lens = [0, P - 2, P - 1, P, 133 - 1, 3 * 128, 30 * P - 1]
    st = build_cache(cfg, lens, extra_blocks=1 if fused else 0, slack_pages=8)
    if not fused:
        assert st.max_blocks * P == lens[-1] + 1
    S = _assert_tc(cfg, st.max_blocks, splits)
    assert (S == 0) == (splits == 0)
    for step in range(2 if fused else 1):
        out, ref, err = append_and_decode(st, step=step, num_splits=splits, fused=fused, check_pools=True)
        assert err == 0
        check_close(out, ref, dtype, f"{cfg.name} splits={splits} step {step}")
        if step == 0:
            v_new = W.new_token_kv(cfg, 0, 0)[1]
            v0 = R.decode_storage(v_new[0], dtype)
            g = H_q // H_kv
            for h in range(H_q):  # one token: that token's V exactly
                assert np.array_equal(out[0, h], v0[h // g].astype(np.float32))


@pytest.mark.parametrize("P", [16, 32])
def test_tc_mixed_batch_with_churn(P):
    base = W.mixed_config(1, P)
    B = 40
    lens = W.cached_lengths(base)[:B]
    steps = 3
    max_blocks = -(-(16384 + steps + 1) // P) + 1
    st = build_cache(W.DecodeConfig(base.name + "-B40", "bf16", B=B, H_q=32, H_kv=1, Dh=128, page_size=P,
                                    seed=base.seed), lens, slack_pages=2 * max_blocks, max_blocks=max_blocks)
    assert _assert_tc(st.cfg, max_blocks, 0) == 0  # device-planned
    events = W.churn_events(base, steps, exit_prob=0.25)
    for step in range(steps):
        ev = events[step]
        for b, L in zip(ev.exits, ev.new_lengths):
            if b < B:
                replace_sequence(st, int(b), int(L), tag=200 + step)
        out, ref, err = append_and_decode(st, step=step, num_splits=0, fused=True, check_pools=(step == steps - 1))
        assert err == 0
        check_close(out, ref, "bf16", f"tc mixed P={P} step {step}")


# Balanced plan (num_splits = 0): CTA c streams pages [c T / G, (c + 1) T / G) of the rows laid end to end;
# rows cut by a boundary are merged by the combine kernel from two partial slots per CTA.
BALANCED_CASES = [
    # one row spanning every CTA's range (many pieces of one row), beside a one-token row
    ("span", "bf16", 16, 32, 1, [0, 148 * 3 * 128 + 37]),
    # 16384 one-page rows: about 110 pieces per CTA, past the shared-memory work list
    ("many", "bf16", 16, 32, 8, [0] * 2048),
    # 296 rows of 16 pages: every CTA takes exactly two whole rows (boundaries coincide, no partials)
    ("aligned", "fp16", 16, 32, 1, [16 * 16 - 1] * 296),
    # fewer pages than two stages per CTA: a handful of CTAs carry the work
    ("small", "bf16", 32, 32, 2, [3, 40, 0, 17, 100]),
]


@pytest.mark.parametrize("name,dtype,P,H_q,H_kv,lens", BALANCED_CASES, ids=[c[0] for c in BALANCED_CASES])
def test_tc_balanced_plan(name, dtype, P, H_q, H_kv, lens):
    cfg = W.DecodeConfig(f"tc-balanced-{name}", dtype, B=len(lens), H_q=H_q, H_kv=H_kv, Dh=128, page_size=P,
                         seed=46)
    st = build_cache(cfg, lens, extra_blocks=1, slack_pages=len(lens) + 8)  # a page per row for the second step
    assert _assert_tc(cfg, st.max_blocks, 0) == 0
    for step in range(2):
        out, ref, err = append_and_decode(st, step=step, num_splits=0, fused=True, check_pools=(step == 1))
        assert err == 0
        check_close(out, ref, dtype, f"{cfg.name} step {step}")


@pytest.mark.parametrize("splits", [0, 3])
def test_tc_growing_scores_rescale(splits):
    """Keys whose scores rise far above the first stage's maximum: the reference maximum moves
    (with O^T and the row sums rescaled) several times within one row."""
    cfg = W.DecodeConfig("tc-growing", "bf16", B=3, H_q=32, H_kv=1, Dh=128, page_size=16, seed=43)
    P = cfg.page_size
    lens = [700, 1000, 300]
    st = build_cache(cfg, lens, slack_pages=4)
    q = W.queries(cfg, 0, 0)
    qf = R.decode_storage(q, "bf16")
    # overwrite the cached keys: key t leans towards the mean query direction with a weight growing in t,
    # so later scores exceed earlier ones by many multiples of 2^8 (in log2 units)
    for b, L in enumerate(lens):
        qdir = qf[b].mean(axis=0)
        qdir = qdir / np.linalg.norm(qdir)
        t = np.arange(L, dtype=np.float64)[:, None]
        base_k = R.decode_storage(W.kv_rows(cfg, 0, b, L)[0], "bf16")[:, 0, :]
        keys = base_k + (t / 5.0) * qdir[None, :]
        kraw = W.round_to_storage(keys.astype(np.float32)[:, None, :], "bf16")
        R.scatter_to_pages(st.kp, st.mtab[b], kraw)
        sl = torch.from_numpy(K.kv_slots_for_range(st.tab[b], P, 0, L)).cuda()
        K.kv_append(st.k_pages, st.v_pages, to_device(kraw, "bf16"), to_device(v_rows(st, b, L), "bf16"), sl, P)
    out, ref, err = append_and_decode(st, num_splits=splits, check_pools=True)
    assert err == 0
    check_close(out, ref, "bf16", f"tc growing scores splits={splits}")


def v_rows(st, b, L):
    """Logical V rows of sequence b read back from the oracle pool (storage bits), for re-appending."""
    P = st.cfg.page_size
    t = np.arange(L)
    pages = np.asarray(st.mtab[b], dtype=np.int64)[t // P]
    return st.vp[pages, :, t % P, :]


def test_tc_empty_rows_and_error_bits():
    cfg = W.DecodeConfig("tc-zero", "bf16", B=3, H_q=32, H_kv=1, Dh=128, page_size=16, seed=44)
    k_pages = torch.full((4, 1, 16, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_pages = k_pages.clone()
    q = to_device(W.queries(cfg, 0, 0), "bf16")
    for splits in (1, 2, 0):
        out = torch.full((3, 32, 128), 7.0, device="cuda")
        ws = torch.zeros(max(1 << 20, K.paged_decode_workspace_bytes(3, 32, 1, 128, 2, 16, splits)),
                         dtype=torch.uint8, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        K.paged_decode_attention(out, q, k_pages, v_pages, torch.full((3, 2), -1, dtype=torch.int32, device="cuda"),
                                 torch.zeros(3, dtype=torch.int32, device="cuda"), cfg.scale, num_splits=splits,
                                 workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        assert torch.count_nonzero(out).item() == 0 and int(err.item()) == 0
    # a block-table entry outside the pool is never loaded; a length beyond the table zeroes the row
    out = torch.empty((1, 32, 128), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    k_pages.zero_()
    v_pages.zero_()
    K.paged_decode_attention(out, q[:1], k_pages, v_pages, torch.tensor([[1, 99]], dtype=torch.int32, device="cuda"),
                             torch.tensor([20], dtype=torch.int32, device="cuda"), 0.1, num_splits=1, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_PAGE_RANGE and torch.isfinite(out).all()
    err.zero_()
    K.paged_decode_attention(out, q[:1], k_pages, v_pages, torch.tensor([[1, 2]], dtype=torch.int32, device="cuda"),
                             torch.tensor([33], dtype=torch.int32, device="cuda"), 0.1, num_splits=1, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_SEQ_LEN and torch.count_nonzero(out).item() == 0


def test_auto_selection_takes_tc_for_32_head_groups_and_many_rows():
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
    try:
        assert K.paged_decode_launch_info(256, 32, 1, 128, 1030, 16, "bf16", 0) == (0, K.KV_DECODE_KERNEL_TCGEN05)
        assert K.paged_decode_launch_info(64, 32, 8, 128, 270, 16, "bf16", 0)[1] == K.KV_DECODE_KERNEL_MMA
        # many (sequence, KV head) rows: the balanced plan of the tcgen05 kernel
        assert K.paged_decode_launch_info(256, 32, 8, 128, 1030, 16, "bf16", 0) == (0, K.KV_DECODE_KERNEL_TCGEN05)
        assert K.paged_decode_launch_info(256, 32, 8, 128, 1030, 16, "bf16", 2)[1] == K.KV_DECODE_KERNEL_MMA
        assert K.paged_decode_launch_info(4, 32, 1, 64, 100, 16, "bf16", 0)[1] == K.KV_DECODE_KERNEL_MMA
        assert K.paged_decode_launch_info(4, 32, 1, 128, 100, 16, "fp32", 0)[1] == K.KV_DECODE_KERNEL_SIMT
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)


def test_tc_matches_warp_mma_kernel():
    """Same inputs through the tcgen05 kernel and the warp-MMA kernel: both within the oracle's tolerance."""
    cfg = W.DecodeConfig("tc-vs-mma", "bf16", B=9, H_q=32, H_kv=1, Dh=128, page_size=16, seed=45)
    lens = W.cached_lengths(W.mixed_config(1, 16))[:9]
    st = build_cache(cfg, lens, slack_pages=4)
    out_tc, ref, err = append_and_decode(st, num_splits=0, check_pools=True)
    assert err == 0
    check_close(out_tc, ref, "bf16", "tc")
    lens32 = st.lens.astype(np.int32)
    q = to_device(W.queries(cfg, 0, 0), "bf16")
    out = torch.empty((cfg.B, 32, 128), device="cuda")
    ws = torch.zeros(K.paged_decode_workspace_bytes(cfg.B, 32, 1, 128, st.max_blocks, 16, 0) + 16, dtype=torch.uint8,
                     device="cuda")
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_MMA)
    try:
        K.paged_decode_attention(out, q, st.k_pages, st.v_pages, torch.from_numpy(st.tab).cuda(),
                                 torch.from_numpy(lens32).cuda(), cfg.scale, num_splits=0, workspace=ws)
        torch.cuda.synchronize()
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)
    check_close(out.cpu().numpy(), ref, "bf16", "warp mma")


@pytest.mark.parametrize("H_q,H_kv,splits", [(32, 1, 0), (32, 8, 0), (32, 1, 3)])
def test_tc_repeated_launches_identical(H_q, H_kv, splits):
    """The same decode repeated 30 times over a pool whose unused slots hold NaN: every launch gives the bits
    of the first, which matches the oracle. A barrier wait passing on an older phase, or a stale V row reaching
    P.V, would show as a changed or non-finite element in some launch."""
    cfg = W.DecodeConfig(f"tc-repeat-{H_q}-{H_kv}-{splits}", "bf16", B=24, H_q=H_q, H_kv=H_kv, Dh=128, page_size=16,
                         seed=48)
    lens = W.generator(48, W.S_LENGTHS, 24).integers(1, 700, 24)
    lens[::5] = [1, 15, 16, 17, 128][: len(lens[::5])]
    st = build_cache(cfg, lens, extra_blocks=1, slack_pages=32)
    S = _assert_tc(cfg, st.max_blocks, splits)
    assert (S == 0) == (splits == 0)
    got, ref, err = append_and_decode(st, step=0, num_splits=splits, fused=False, check_pools=False)
    assert err == 0
    check_close(got, ref, "bf16", cfg.name)
    B = len(st.lens)
    q = to_device(W.queries(cfg, 0, 0)[:B], "bf16")
    tab, lens32 = torch.from_numpy(st.tab).cuda(), torch.from_numpy(st.lens.astype(np.int32)).cuda()
    ws = torch.zeros(max(16, K.paged_decode_workspace_bytes(B, H_q, H_kv, 128, st.max_blocks, 16, splits)),
                     dtype=torch.uint8, device="cuda")
    first = torch.from_numpy(got).cuda()
    out = torch.empty_like(first)
    for _ in range(30):
        out.fill_(float("nan"))
        K.paged_decode_attention(out, q, st.k_pages, st.v_pages, tab, lens32, cfg.scale, num_splits=splits, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out, first)
