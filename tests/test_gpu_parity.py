"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Integer work (block tables, slots, the physical pools written by kv_append) is
compared bit-exactly; attention outputs within the dtype tolerance of
tests/helpers.py. All inputs come from the seeded generators.
"""
import math

import numpy as np
import pytest
import torch

from gpu_cases import (TORCH_DT, append_and_decode, build_cache, check_close, oracle_pool, replace_sequence,
                       to_device)
from oracle import reference as R
from oracle.pool_model import PoolModel, PrefixModel
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.fixture(params=["mma", "simt"])
def kernel(request):
    """Run the test with the tensor-core kernel (default for 16-bit K/V) and with the CUDA-core kernel."""
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_MMA if request.param == "mma" else K.KV_DECODE_KERNEL_SIMT)
    yield request.param
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)


# ---------------------------------------------------------------- tiny (fp32)
@pytest.mark.parametrize("splits", [1, 2, 0])
def test_tiny_fp32_against_oracle_and_full_causal(splits):
    cfg = W.TINY
    lens = W.cached_lengths(cfg)
    st = build_cache(cfg, lens, slack_pages=W.TINY_POOL_PAGES - 4, keep_logical=True)
    assert st.num_pages == W.TINY_POOL_PAGES
    out, ref, err = append_and_decode(st, num_splits=splits)
    assert err == 0
    check_close(out, ref, "fp32", "tiny vs oracle")
    # full causal recompute over the logical rows (cached + new token): row T == decode
    k_new, v_new = W.new_token_kv(cfg, 0, 0)
    q = W.queries(cfg, 0, 0)
    for b in range(cfg.B):
        T = int(lens[b])
        Kall = np.concatenate([st.logical_k[b], k_new[b:b + 1]])
        Vall = np.concatenate([st.logical_v[b], v_new[b:b + 1]])
        Qall = np.concatenate([W.all_queries(cfg, 0, b, T), q[b:b + 1]])
        full = R.causal_attention(Qall, Kall, Vall, cfg.scale)
        check_close(out[b], full[T], "fp32", f"tiny seq {b} vs causal")


# ---------------------------------------------------------------- Llama-3.1-8B-shaped layer (bf16)
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_llama8b_reduced_batch(splits, kernel):
    cfg = W.LLAMA8B
    lens = W.cached_lengths(cfg)[:8]
    st = build_cache(cfg, lens)
    for step in range(2):
        out, ref, err = append_and_decode(st, step=step, num_splits=splits)
        assert err == 0
        check_close(out, ref, cfg.dtype, f"8B reduced step {step}")


@pytest.mark.parametrize("splits", [0, 1])
def test_llama8b_full_size(splits, kernel):
    """The full workload (B=64, lengths U[512, 4096]) in the launch configuration the benchmark times."""
    cfg = W.LLAMA8B
    st = build_cache(cfg, W.cached_lengths(cfg))
    out, ref, err = append_and_decode(st, num_splits=splits, check_pools=(splits == 0))
    assert err == 0
    check_close(out, ref, cfg.dtype, "8B full")


# ---------------------------------------------------------------- 32K context (fp16, split-KV)
@pytest.mark.parametrize("layer,splits", [(0, 0), (31, 0), (0, 1), (0, 7)])
def test_long_context_layer(layer, splits, kernel):
    cfg = W.LONG32K
    st = build_cache(cfg, W.cached_lengths(cfg), layer=layer)
    if splits == 0:
        assert K.paged_decode_num_splits(cfg.B, cfg.H_kv, st.max_blocks, cfg.page_size, 0) > 1
    out, ref, err = append_and_decode(st, layer=layer, num_splits=splits, check_pools=(splits == 0))
    assert err == 0
    check_close(out, ref, cfg.dtype, f"32K layer {layer} splits {splits}")


# ---------------------------------------------------------------- shared prefix (bf16)
def test_shared_prefix_batch(kernel):
    cfg = W.SHARED_PREFIX
    P = cfg.page_size
    wl = W.prefix_workload(cfg)
    lens = W.cached_lengths(cfg)
    B = cfg.B
    num_pages = W.PREFIX_LEN // P + int(sum(-(-(int(L) + 1 - W.PREFIX_LEN) // P) for L in lens)) + 4
    max_blocks = max(-(-(int(L) + 1) // P) for L in lens) + 1
    order = W.page_order(num_pages, cfg.seed)
    pool, mpool = K.KvPool(num_pages, P, order), PoolModel(num_pages, P, order)
    ix, mix = K.KvPrefixIndex(P, salt=42), PrefixModel(P, salt=42)
    tab = np.full((B, max_blocks), -1, np.int32)
    mtab = [[-1] * max_blocks for _ in range(B)]
    kp, vp = oracle_pool(num_pages, cfg)
    dt = TORCH_DT[cfg.dtype]
    shape = (num_pages, cfg.H_kv, P, cfg.Dh)
    k_pages = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    v_pages = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    # K/V depend only on the token prefix: the shared prefix rows are drawn once
    pk, pv = W.kv_rows(cfg, 0, 10_000, W.PREFIX_LEN)
    for b in range(B):
        toks = wl.tokens(b)
        hit, mhit = ix.match(toks), mix.match(toks)
        assert list(hit) == mhit
        pool.incref(hit)
        mpool.incref(mhit)
        k = -(-len(toks) // P) - len(hit)
        own = pool.alloc(k)
        assert list(own) == mpool.alloc(k)
        row = np.concatenate([hit, own]).astype(np.int32)
        tab[b, :row.size] = row
        mtab[b][:row.size] = row.tolist()
        ix.register(pool, toks, row)
        mix.register(mpool, toks, row.tolist())
        start = len(hit) * P
        sk, sv = W.kv_rows(cfg, 0, b, len(toks) - W.PREFIX_LEN)
        rk = np.concatenate([pk, sk])[start:]
        rv = np.concatenate([pv, sv])[start:]
        for t0 in range(rk.shape[0]):
            pg, off = divmod(start + t0, P)
            kp[mtab[b][pg], :, off, :] = rk[t0]
            vp[mtab[b][pg], :, off, :] = rv[t0]
        sl = torch.from_numpy(K.kv_slots_for_range(tab[b], P, start, rk.shape[0])).cuda()
        K.kv_append(k_pages, v_pages, to_device(rk, cfg.dtype), to_device(rv, cfg.dtype), sl, P)
    assert all(pool.refcount(int(p)) == B for p in tab[0, : W.PREFIX_LEN // P])
    # divergence probes: floor(d / P) reusable pages
    for b in range(B):
        assert len(ix.match(wl.probe(b))) == int(wl.divergence[b]) // P
    # one decode step
    lens32 = lens.astype(np.int32).copy()
    mlens = [int(x) for x in lens]
    slots = pool.append_slots(tab, lens32)
    assert list(slots) == mpool.append_slots(mtab, max_blocks, mlens)
    k_new, v_new = W.new_token_kv(cfg, 0, 0)
    q = W.queries(cfg, 0, 0)
    for b in range(B):
        pg, off = divmod(int(slots[b]), P)
        kp[pg, :, off, :] = k_new[b]
        vp[pg, :, off, :] = v_new[b]
    ref = R.paged_decode(q, kp, vp, np.asarray(mtab, np.int32), np.asarray(mlens, np.int32), cfg.scale, cfg.dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kv_append(k_pages, v_pages, to_device(k_new, cfg.dtype), to_device(v_new, cfg.dtype), torch.from_numpy(slots).cuda(), P,
                err_flag=err)
    out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, K.paged_decode_workspace_bytes(B, cfg.H_q, cfg.H_kv, cfg.Dh, max_blocks, P)), dtype=torch.uint8,
                     device="cuda")
    K.paged_decode_attention(out, to_device(q, cfg.dtype), k_pages, v_pages, torch.from_numpy(tab).cuda(),
                             torch.from_numpy(lens32).cuda(), cfg.scale, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_close(out.cpu().numpy(), ref, cfg.dtype, "shared prefix")


# ---------------------------------------------------------------- mixed continuous batching
@pytest.mark.parametrize("H_kv,P", W.MIXED_POINTS)
def test_mixed_sweep_with_churn(H_kv, P, kernel):
    base = W.mixed_config(H_kv, P)
    B = 24
    lens = W.cached_lengths(base)[:B]
    steps = 3
    max_blocks = -(-(16384 + steps + 1) // P) + 1
    st = build_cache(base, lens, slack_pages=2 * max_blocks, max_blocks=max_blocks)
    events = W.churn_events(base, steps, exit_prob=0.25)
    for step in range(steps):
        ev = events[step]
        for b, L in zip(ev.exits, ev.new_lengths):
            if b < B:
                replace_sequence(st, int(b), int(L), tag=100 + step)
        out, ref, err = append_and_decode(st, step=step, num_splits=0, check_pools=(step == steps - 1))
        assert err == 0
        check_close(out, ref, base.dtype, f"mixed Hkv={H_kv} P={P} step {step}")


# ---------------------------------------------------------------- fused append + decode
FUSED_CASES = [("tiny", 1), ("tiny", 2), ("8b", 0), ("8b", 1), ("32k", 0), ("edge", 1), ("edge", 3)]


@pytest.mark.parametrize("case,splits", FUSED_CASES)
def test_fused_append_decode(case, splits, kernel):
    """paged_decode_attention_append == kv_append + paged_decode_attention: same pool bytes, same oracle match."""
    if case == "tiny":
        cfg, lens = W.TINY, W.cached_lengths(W.TINY)
    elif case == "8b":
        cfg, lens = W.LLAMA8B, W.cached_lengths(W.LLAMA8B)[:12]
    elif case == "32k":
        cfg, lens = W.LONG32K, W.cached_lengths(W.LONG32K)
    else:
        cfg = W.DecodeConfig("edge-fused", "fp16", B=6, H_q=12, H_kv=4, Dh=64, page_size=32, seed=13)
        lens = [0, 30, 31, 32, 100, 127]
    st = build_cache(cfg, lens)
    for step in range(2):
        out, ref, err = append_and_decode(st, step=step, num_splits=splits, fused=True, check_pools=True)
        assert err == 0
        check_close(out, ref, cfg.dtype, f"fused {case} step {step}")


# ---------------------------------------------------------------- edge cases
EDGE_SHAPES = [
    # dtype, Dh, P, H_q, H_kv
    ("bf16", 128, 16, 32, 8), ("fp16", 128, 32, 32, 8), ("bf16", 64, 16, 8, 8), ("fp16", 64, 32, 12, 4),
    ("fp32", 128, 16, 4, 2), ("fp32", 64, 32, 6, 6), ("bf16", 128, 16, 32, 1), ("bf16", 128, 32, 16, 2),
    ("fp16", 128, 16, 7, 1), ("bf16", 64, 16, 20, 4),
    # head slices of 9..16 rows (residual in a second MMA) and a 16 + 4 split
    ("bf16", 128, 16, 24, 2), ("fp16", 64, 16, 40, 2),
]


@pytest.mark.parametrize("dtype,Dh,P,H_q,H_kv", EDGE_SHAPES)
@pytest.mark.parametrize("splits", [1, 2, 0])
def test_edge_lengths_and_shapes(dtype, Dh, P, H_q, H_kv, splits, kernel):
    cfg = W.DecodeConfig(f"edge-{dtype}-{Dh}-{P}-{H_q}-{H_kv}", dtype, B=6, H_q=H_q, H_kv=H_kv, Dh=Dh, page_size=P, seed=9)
    # after the append: 1, P-1, P, P+1, 3P+5 tokens, and one sequence filling its table exactly
    lens = [0, P - 2, P - 1, P, 3 * P + 4, 4 * P - 1]
    st = build_cache(cfg, lens, extra_blocks=0)
    assert st.max_blocks * P == lens[-1] + 1
    out, ref, err = append_and_decode(st, num_splits=splits)
    assert err == 0
    check_close(out, ref, dtype, cfg.name)
    # one token: the output is that token's V exactly (rounded to fp32)
    v_new = W.new_token_kv(cfg, 0, 0)[1]
    g = H_q // H_kv
    v0 = R.decode_storage(v_new[0], dtype)
    for h in range(H_q):
        assert np.array_equal(out[0, h], v0[h // g].astype(np.float32))


def test_zero_length_rows_are_zero(kernel):
    cfg = W.DecodeConfig("zero", "bf16", B=3, H_q=8, H_kv=2, Dh=128, page_size=16, seed=12)
    P = cfg.page_size
    k_pages = torch.full((4, 2, P, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_pages = k_pages.clone()
    tab = torch.full((3, 2), -1, dtype=torch.int32, device="cuda")
    lens = torch.zeros(3, dtype=torch.int32, device="cuda")
    q = to_device(W.queries(cfg, 0, 0), "bf16")
    for splits in (1, 2, 0):
        out = torch.full((3, 8, 128), 7.0, device="cuda")
        ws = torch.zeros(max(1 << 16, K.paged_decode_workspace_bytes(3, 8, 2, 128, 2, 16, 0)), dtype=torch.uint8,
                         device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        K.paged_decode_attention(out, q, k_pages, v_pages, tab, lens, cfg.scale, num_splits=splits, workspace=ws,
                                 err_flag=err)
        torch.cuda.synchronize()
        assert torch.count_nonzero(out).item() == 0 and int(err.item()) == 0


# ---------------------------------------------------------------- planned launches
def _planned_B(H_kv: int, extra: int) -> int:
    """Rows past the automatic planned-launch threshold (4 x SM count) on this GPU."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return (4 * sms) // H_kv + extra


PLANNED_SHAPES = [
    # dtype, Dh, P, H_q, H_kv, extra rows
    ("bf16", 128, 16, 32, 8, 20), ("fp16", 64, 32, 16, 4, 9), ("bf16", 128, 16, 64, 1, 5), ("fp16", 128, 32, 8, 8, 3),
]


@pytest.mark.parametrize("dtype,Dh,P,H_q,H_kv,extra", PLANNED_SHAPES)
@pytest.mark.parametrize("uniform", [False, True])
@pytest.mark.parametrize("fused", [False, True])
def test_planned_launch(dtype, Dh, P, H_q, H_kv, extra, uniform, fused):
    """num_splits = 0 with many rows: the device plan chunks rows by their actual lengths."""
    B = _planned_B(H_kv, extra)
    cfg = W.DecodeConfig(f"planned-{dtype}-{Dh}-{P}-{H_q}-{H_kv}-B{B}", dtype, B=B, H_q=H_q, H_kv=H_kv, Dh=Dh,
                         page_size=P, seed=21)
    st = build_cache(cfg, W.ragged_lengths(B, P, cfg.seed, uniform), slack_pages=B)  # room for a second step
    assert K.paged_decode_num_splits(B, H_kv, st.max_blocks, P, 0) == 0
    for step in range(2):
        out, ref, err = append_and_decode(st, step=step, num_splits=0, fused=fused, check_pools=(step == 1))
        assert err == 0
        check_close(out, ref, dtype, f"{cfg.name} step {step}")


def test_planned_launch_zero_length_rows():
    """Planned launch with empty rows (seq_len 0): those rows are zeros, the rest match the oracle."""
    cfg = W.DecodeConfig("planned-zero", "bf16", B=_planned_B(2, 4), H_q=8, H_kv=2, Dh=128, page_size=16, seed=22)
    st = build_cache(cfg, W.ragged_lengths(cfg.B, cfg.page_size, cfg.seed))
    out, ref, err = append_and_decode(st, num_splits=0)
    assert err == 0
    check_close(out, ref, cfg.dtype, "planned before zeroing")
    lens = st.lens.astype(np.int32).copy()
    lens[1::3] = 0
    q = to_device(W.queries(cfg, 0, 0), cfg.dtype)
    ws = torch.zeros(K.paged_decode_workspace_bytes(cfg.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, 16, 0),
                     dtype=torch.uint8, device="cuda")
    for lens_case in (lens, np.zeros_like(lens)):
        got = torch.full((cfg.B, cfg.H_q, cfg.Dh), 7.0, device="cuda")
        errt = torch.zeros(1, dtype=torch.int32, device="cuda")
        K.paged_decode_attention(got, q, st.k_pages, st.v_pages, torch.from_numpy(st.tab).cuda(),
                                 torch.from_numpy(lens_case).cuda(), cfg.scale, num_splits=0, workspace=ws,
                                 err_flag=errt)
        torch.cuda.synchronize()
        g = got.cpu().numpy()
        assert int(errt.item()) == 0
        zero = lens_case == 0
        assert np.count_nonzero(g[zero]) == 0
        if (~zero).any():
            check_close(g[~zero], ref[~zero], cfg.dtype, "planned with empty rows")


def test_page_permutation_invariance_bitwise(kernel):
    """Same logical content behind two different physical page orders -> bit-identical output."""
    cfg = W.LLAMA8B
    lens = W.cached_lengths(cfg)[:6]
    outs = []
    for layer in (0, 1):  # page_order differs per layer; K/V are drawn per (layer, b) -> keep layer 0 values
        st = build_cache(W.DecodeConfig(cfg.name, cfg.dtype, 6, cfg.H_q, cfg.H_kv, cfg.Dh, cfg.page_size, seed=cfg.seed),
                         lens, layer=0, slack_pages=11 + 7 * layer)
        out, ref, err = append_and_decode(st, num_splits=1, check_pools=False)
        assert err == 0
        outs.append(out)
    assert np.array_equal(outs[0], outs[1])


# ---------------------------------------------------------------- device error flags (host-checked, no faults)
def test_device_error_flags(kernel):
    P, Dh = 16, 128
    k_pages = torch.zeros((4, 2, P, Dh), dtype=torch.bfloat16, device="cuda")
    v_pages = torch.zeros_like(k_pages)
    q = torch.zeros((1, 4, Dh), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, 4, Dh), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a block-table entry outside the pool is skipped, never read
    K.paged_decode_attention(out, q, k_pages, v_pages, torch.tensor([[1, 99]], dtype=torch.int32, device="cuda"),
                             torch.tensor([20], dtype=torch.int32, device="cuda"), 0.1, num_splits=1, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_PAGE_RANGE
    # a length beyond the table is refused (row zeroed)
    err.zero_()
    K.paged_decode_attention(out, q, k_pages, v_pages, torch.tensor([[1, 2]], dtype=torch.int32, device="cuda"),
                             torch.tensor([33], dtype=torch.int32, device="cuda"), 0.1, num_splits=1, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_SEQ_LEN and torch.count_nonzero(out).item() == 0
    # a slot beyond the pool is skipped by kv_append
    err.zero_()
    before = k_pages.clone()
    K.kv_append(k_pages, v_pages, torch.ones((1, 2, Dh), dtype=torch.bfloat16, device="cuda"),
                torch.ones((1, 2, Dh), dtype=torch.bfloat16, device="cuda"),
                torch.tensor([4 * P], dtype=torch.int64, device="cuda"), P, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_SLOT and torch.equal(before, k_pages)
    # slot -1 is a no-op without error
    err.zero_()
    K.kv_append(k_pages, v_pages, torch.ones((1, 2, Dh), dtype=torch.bfloat16, device="cuda"),
                torch.ones((1, 2, Dh), dtype=torch.bfloat16, device="cuda"),
                torch.tensor([-1], dtype=torch.int64, device="cuda"), P, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and torch.equal(before, k_pages)


def test_workspace_too_small_is_refused():
    cfg = W.LONG32K
    P = cfg.page_size
    k_pages = torch.zeros((8, cfg.H_kv, P, cfg.Dh), dtype=torch.float16, device="cuda")
    q = torch.zeros((1, cfg.H_q, cfg.Dh), dtype=torch.float16, device="cuda")
    out = torch.empty((1, cfg.H_q, cfg.Dh), device="cuda")
    tab = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    lens = torch.tensor([100], dtype=torch.int32, device="cuda")
    with pytest.raises(K.KvError) as e:
        K.paged_decode_attention(out, q, k_pages, k_pages, tab, lens, 0.1, num_splits=4,
                                 workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.name == "WORKSPACE"


# ---------------------------------------------------------------- copy-on-write (beam fork)
@pytest.mark.parametrize("dtype,P", [("bf16", 16), ("fp16", 32), ("fp32", 16)])
def test_beam_fork_copy_on_write(dtype, P, kernel):
    """Fork sequences that share every page (beam search), give each one a
    private copy of the shared partial tail (kv_pool_cow_tails + kv_copy_pages),
    then append different tokens and decode: pools bit-exact, outputs within
    tolerance of the oracle, and the forks diverge only at the new token."""
    cfg = W.DecodeConfig(f"fork-{dtype}-{P}", dtype, B=4, H_q=8, H_kv=2, Dh=128 if dtype != "fp32" else 64,
                         page_size=P, seed=21)
    lens = [37, 70]  # parents; rows 2 and 3 fork them
    st = build_cache(cfg, lens + [0, 0], slack_pages=8)
    for child, parent in ((2, 0), (3, 1)):
        ids = [int(x) for x in st.tab[parent] if x >= 0]
        st.pool.incref(ids)
        st.mpool.incref(ids)
        st.tab[child] = st.tab[parent]
        st.mtab[child] = list(st.mtab[parent])
    st.lens = np.array(lens + lens, dtype=np.int64)
    src, dst = st.pool.cow_tails(st.tab, st.lens.astype(np.int32))
    pairs = st.mpool.cow_tails(st.mtab, st.max_blocks, [int(x) for x in st.lens])
    assert list(zip(src.tolist(), dst.tolist())) == pairs and len(pairs) == 2 and st.tab.tolist() == st.mtab
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kv_copy_pages(st.k_pages, st.v_pages, torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda(), err_flag=err)
    for s_, d_ in pairs:
        st.kp[d_] = st.kp[s_]
        st.vp[d_] = st.vp[s_]
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    out, ref, err2 = append_and_decode(st, num_splits=0, check_pools=True)
    assert err2 == 0
    check_close(out, ref, dtype, "beam fork")
    assert not np.allclose(out[0], out[2])  # same history, different new token


def test_copy_pages_refuses_bad_ids():
    k_pages = torch.zeros((4, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    v_pages = torch.zeros_like(k_pages)
    k_pages[1] = 1.0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kv_copy_pages(k_pages, v_pages, torch.tensor([1, 9], dtype=torch.int32, device="cuda"),
                    torch.tensor([2, 3], dtype=torch.int32, device="cuda"), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KV_DEV_ERR_PAGE_RANGE
    assert torch.equal(k_pages[2], k_pages[1]) and torch.count_nonzero(k_pages[3]).item() == 0
