"""GPU parity of the FP8 (E4M3) K/V cache: kv_append_fp8 codes bit-exact
against the oracle's quantiser, paged_decode_attention_fp8 within the
attention tolerance of the oracle's fp64 decode over the same codes."""
import numpy as np
import pytest
import torch

from gpu_cases import check_close, to_device
from oracle import fp8 as F
from oracle.pool_model import PoolModel
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _scales(H_kv):
    k = (0.010 + 0.002 * np.arange(H_kv)).astype(np.float32)  # distinct per head: a head mix-up shows
    v = (0.012 + 0.001 * np.arange(H_kv)).astype(np.float32)
    return k, v


class Fp8Cache:
    """An E4M3 cache filled on both sides from the same seeded rows."""

    def __init__(self, cfg, lens, extra_blocks=1, slack_pages=None):
        self.cfg = cfg
        P = cfg.page_size
        self.lens = np.asarray(lens, dtype=np.int64)
        B = len(self.lens)
        need = [-(-(int(L) + 1) // P) for L in self.lens]
        self.max_blocks = max(need) + extra_blocks
        self.num_pages = int(sum(need)) + (B if slack_pages is None else slack_pages)
        order = W.page_order(self.num_pages, cfg.seed)
        self.pool = K.KvPool(self.num_pages, P, order)
        self.mpool = PoolModel(self.num_pages, P, order)
        self.tab = np.full((B, self.max_blocks), -1, np.int32)
        self.mtab = [[-1] * self.max_blocks for _ in range(B)]
        for b in range(B):
            k = -(-int(self.lens[b]) // P)
            self.tab[b, :k] = self.pool.alloc(k)
            self.mtab[b][:k] = self.mpool.alloc(k)
        assert self.tab.tolist() == self.mtab
        self.ks, self.vs = _scales(cfg.H_kv)
        self.dks, self.dvs = torch.from_numpy(self.ks).cuda(), torch.from_numpy(self.vs).cuda()
        shape = (self.num_pages, cfg.H_kv, P, cfg.Dh)
        self.kc = np.full(shape, 0x7F, np.uint8)  # NaN codes in unused slots
        self.vc = np.full(shape, 0x7F, np.uint8)
        self.k_pages = torch.from_numpy(self.kc).cuda()
        self.v_pages = torch.from_numpy(self.vc).cuda()
        for b in range(B):
            L = int(self.lens[b])
            if L == 0:
                continue
            slots = K.kv_slots_for_range(self.tab[b], P, 0, L)
            kr, vr = W.kv_rows(cfg, 0, b, L)
            F.append_fp8(self.kc, self.vc, kr, vr, cfg.dtype, self.ks, self.vs, slots)
            K.kv_append_fp8(self.k_pages, self.v_pages, to_device(kr, cfg.dtype), to_device(vr, cfg.dtype), self.dks,
                            self.dvs, torch.from_numpy(slots).cuda(), P)
        torch.cuda.synchronize()

    def check_codes(self):
        assert np.array_equal(self.k_pages.cpu().numpy(), self.kc), "K codes"
        assert np.array_equal(self.v_pages.cpu().numpy(), self.vc), "V codes"

    def step(self, step=0, num_splits=0, q_dtype=None):
        """Append one token per sequence (quantising), then decode. Returns (gpu, ref, err)."""
        cfg = self.cfg
        P = cfg.page_size
        lens32 = self.lens.astype(np.int32).copy()
        mlens = [int(x) for x in self.lens]
        slots = self.pool.append_slots(self.tab, lens32)
        mslots = self.mpool.append_slots(self.mtab, self.max_blocks, mlens)
        assert list(slots) == mslots
        B = len(self.lens)
        kn, vn = W.new_token_kv(cfg, 0, step)
        kn, vn = kn[:B], vn[:B]
        q = W.queries(cfg, 0, step)[:B]
        F.append_fp8(self.kc, self.vc, kn, vn, cfg.dtype, self.ks, self.vs, mslots)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        K.kv_append_fp8(self.k_pages, self.v_pages, to_device(kn, cfg.dtype), to_device(vn, cfg.dtype), self.dks,
                        self.dvs, torch.from_numpy(slots).cuda(), P, err_flag=err)
        ref = F.paged_decode_fp8(q, cfg.dtype, self.kc, self.vc, self.ks, self.vs, np.asarray(self.mtab, np.int32),
                                 np.asarray(mlens, np.int32), cfg.scale)
        out = torch.full((B, cfg.H_q, cfg.Dh), float("nan"), dtype=torch.float32, device="cuda")
        nb = K.paged_decode_workspace_bytes(B, cfg.H_q, cfg.H_kv, cfg.Dh, self.max_blocks, P, num_splits)
        ws = torch.zeros(max(nb, 16), dtype=torch.uint8, device="cuda")
        K.paged_decode_attention_fp8(out, to_device(q, cfg.dtype), self.k_pages, self.v_pages, self.dks, self.dvs,
                                     torch.from_numpy(self.tab).cuda(), torch.from_numpy(lens32).cuda(), cfg.scale,
                                     num_splits=num_splits, workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        self.lens = self.lens + 1
        return out.cpu().numpy(), ref, int(err.item())


# ---------------------------------------------------------------- quantising append
@pytest.mark.parametrize("src", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("Dh", [64, 128])
def test_append_fp8_codes_bit_exact(src, Dh):
    cfg = W.DecodeConfig(f"fp8-append-{src}-{Dh}", src, B=37, H_q=8, H_kv=4, Dh=Dh, page_size=16, seed=60)
    P, B = 16, 37
    num_pages = 4
    g = W.generator(60, W.S_SUFFIX, Dh)
    slots = g.permutation(num_pages * P)[:B].astype(np.int64)
    slots[::7] = -1
    kn, vn = W.new_token_kv(cfg, 0, 0)
    kn = kn * 1 if src != "fp32" else kn * np.float32(40.0)  # fp32 rows: push some values past 448 * scale
    ks, vs = _scales(4)
    kc = np.zeros((num_pages, 4, P, Dh), np.uint8)
    vc = np.zeros_like(kc)
    F.append_fp8(kc, vc, kn, vn, src, ks, vs, slots)
    kd = torch.zeros((num_pages, 4, P, Dh), dtype=torch.uint8, device="cuda")
    vd = torch.zeros_like(kd)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kv_append_fp8(kd, vd, to_device(kn, src), to_device(vn, src), torch.from_numpy(ks).cuda(),
                    torch.from_numpy(vs).cuda(), torch.from_numpy(slots).cuda(), P, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(kd.cpu().numpy(), kc) and np.array_equal(vd.cpu().numpy(), vc)
    if src == "fp32":
        assert (kc == 0x7E).any() or (kc == 0xFE).any()  # saturation was exercised


# ---------------------------------------------------------------- decode
FP8_SHAPES = [
    # q dtype, Dh, P, H_q, H_kv, B, lengths
    ("bf16", 128, 16, 32, 8, 8, "llama"), ("fp16", 128, 16, 32, 8, 8, "llama"), ("bf16", 64, 32, 16, 4, 6, "llama"),
    ("fp16", 64, 16, 12, 4, 6, "edge"), ("bf16", 128, 32, 32, 1, 4, "llama"), ("bf16", 128, 16, 64, 1, 3, "edge"),
    ("fp16", 128, 16, 24, 2, 5, "edge"), ("bf16", 128, 16, 8, 8, 6, "edge"),
]


def _lengths(kind, B, P, seed):
    if kind == "llama":
        return W.generator(seed, W.S_LENGTHS, B).integers(100, 1500, B)
    return np.array([0, P - 2, P - 1, P, 3 * P + 4, 4 * P - 1, 7 * P + 3][:B])


@pytest.mark.parametrize("q_dtype,Dh,P,H_q,H_kv,B,kind", FP8_SHAPES)
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_fp8_decode_against_oracle(q_dtype, Dh, P, H_q, H_kv, B, kind, splits):
    cfg = W.DecodeConfig(f"fp8-{q_dtype}-{Dh}-{P}-{H_q}-{H_kv}", q_dtype, B=B, H_q=H_q, H_kv=H_kv, Dh=Dh, page_size=P,
                         seed=61)
    c = Fp8Cache(cfg, _lengths(kind, B, P, 61))
    c.check_codes()
    for step in range(2):
        out, ref, err = c.step(step, num_splits=splits)
        assert err == 0
        check_close(out, ref, "bf16", f"{cfg.name} splits={splits} step {step}")
    c.check_codes()


TC_FP8_SHAPES = [
    # q dtype, P, H_q, H_kv, B, lengths (g = 4, 8 and 16; the edge lengths include an empty row)
    ("bf16", 16, 32, 8, 8, "llama"), ("fp16", 32, 32, 8, 6, "edge"), ("bf16", 32, 16, 2, 5, "llama"),
    ("fp16", 16, 16, 2, 7, "edge"), ("bf16", 16, 64, 4, 4, "edge"), ("fp16", 32, 48, 3, 3, "llama"),
]


@pytest.mark.parametrize("q_dtype,P,H_q,H_kv,B,kind", TC_FP8_SHAPES)
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_fp8_tcgen05_against_oracle(q_dtype, P, H_q, H_kv, B, kind, splits):
    """The tcgen05 kernel over E4M3 pages (widened to fp16 on the SM), forced for every split mode."""
    cfg = W.DecodeConfig(f"fp8-tc-{q_dtype}-{P}-{H_q}-{H_kv}", q_dtype, B=B, H_q=H_q, H_kv=H_kv, Dh=128, page_size=P,
                         seed=65)
    c = Fp8Cache(cfg, _lengths(kind, B, P, 65))
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)
    try:
        _, kern = K.paged_decode_launch_info(B, H_q, H_kv, 128, c.max_blocks, P, "e4m3", splits)
        assert kern == K.KV_DECODE_KERNEL_TCGEN05
        for step in range(2):
            out, ref, err = c.step(step, num_splits=splits)
            assert err == 0
            check_close(out, ref, "bf16", f"{cfg.name} splits={splits} step {step}")
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
    c.check_codes()


def test_fp8_kernel_choice():
    # under AUTO, E4M3 pools stay on the warp-MMA kernel; TCGEN05 selects the tcgen05 kernel for groups of
    # 4 / 8 / 16 at Dh = 128 and leaves the other shapes on the warp-MMA kernel
    assert K.paged_decode_launch_info(64, 32, 8, 128, 300, 16, "e4m3", 0)[1] == K.KV_DECODE_KERNEL_MMA
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)
    try:
        assert K.paged_decode_launch_info(64, 32, 8, 128, 300, 16, "e4m3", 0) == (0, K.KV_DECODE_KERNEL_TCGEN05)
        assert K.paged_decode_launch_info(64, 32, 8, 128, 300, 16, "e4m3", 2)[1] == K.KV_DECODE_KERNEL_TCGEN05
        assert K.paged_decode_launch_info(64, 32, 1, 128, 300, 16, "e4m3", 0)[1] == K.KV_DECODE_KERNEL_MMA
        assert K.paged_decode_launch_info(64, 16, 4, 64, 300, 16, "e4m3", 0)[1] == K.KV_DECODE_KERNEL_MMA
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)


def test_fp8_long_context_split_and_planned_many_rows():
    # one 32K-token sequence (auto splits), then a batch past the planned-launch row threshold
    cfg = W.DecodeConfig("fp8-long", "fp16", B=1, H_q=32, H_kv=8, Dh=128, page_size=16, seed=62)
    c = Fp8Cache(cfg, [32768])
    assert K.paged_decode_num_splits(1, 8, c.max_blocks, 16, 0) > 1
    out, ref, err = c.step(0)
    assert err == 0
    check_close(out, ref, "fp16", "fp8 32K")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B = (4 * sms) // 8 + 7
    cfg = W.DecodeConfig("fp8-planned", "bf16", B=B, H_q=32, H_kv=8, Dh=128, page_size=16, seed=63)
    c = Fp8Cache(cfg, W.ragged_lengths(B, 16, 63))
    assert K.paged_decode_num_splits(B, 8, c.max_blocks, 16, 0) == 0
    out, ref, err = c.step(0)
    assert err == 0
    check_close(out, ref, "bf16", "fp8 planned")


def test_fp8_refusals():
    cfg = W.DecodeConfig("fp8-refuse", "bf16", B=2, H_q=8, H_kv=2, Dh=128, page_size=16, seed=64)
    c = Fp8Cache(cfg, [20, 5])
    out = torch.zeros((2, 8, 128), dtype=torch.float32, device="cuda")
    q = to_device(W.queries(cfg, 0, 0)[:2], "bf16")
    tab, lens = torch.from_numpy(c.tab).cuda(), torch.from_numpy(c.lens.astype(np.int32)).cuda()
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_SIMT)  # E4M3 runs on the tensor cores regardless
    try:
        K.paged_decode_attention_fp8(out, q, c.k_pages, c.v_pages, c.dks, c.dvs, tab, lens, cfg.scale, num_splits=1)
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
    with pytest.raises(K.KvError):  # q must be bf16 / fp16
        K.paged_decode_attention_fp8(out, q.float(), c.k_pages, c.v_pages, c.dks, c.dvs, tab, lens, cfg.scale)
    with pytest.raises(K.KvError):  # the 16-bit entry point does not take E4M3 pools (q of the pools' type)
        K.paged_decode_attention(out, q.view(torch.uint8).reshape(2, 8, 256)[..., :128].contiguous(), c.k_pages,
                                 c.v_pages, tab, lens, cfg.scale)
    torch.cuda.synchronize()


def test_fp8_llama8b_full_size():
    """The 8B-shaped layer at full size (B=64, lengths U[512, 4096]) with an E4M3 cache, automatic splits."""
    cfg = W.LLAMA8B
    c = Fp8Cache(cfg, W.cached_lengths(cfg))
    out, ref, err = c.step(0)
    assert err == 0
    check_close(out, ref, "bf16", "fp8 8B full")


def test_fp8_tcgen05_repeated_launches_identical():
    """The tcgen05 E4M3 kernel repeated 30 times over a pool whose unused slots hold NaN codes: every launch
    gives the bits of the first (converters, issuers and softmax warps meet on the right barrier phases)."""
    cfg = W.DecodeConfig("fp8-tc-repeat", "bf16", B=12, H_q=32, H_kv=8, Dh=128, page_size=16, seed=66)
    c = Fp8Cache(cfg, _lengths("llama", 12, 16, 66))
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_TCGEN05)
    try:
        out, ref, err = c.step(0, num_splits=0)
        assert err == 0
        check_close(out, ref, "bf16", cfg.name)
        q = to_device(W.queries(cfg, 0, 0)[:12], "bf16")
        tab, lens = torch.from_numpy(c.tab).cuda(), torch.from_numpy(c.lens.astype(np.int32)).cuda()
        ws = torch.zeros(max(16, K.paged_decode_workspace_bytes(12, 32, 8, 128, c.max_blocks, 16, 0)),
                         dtype=torch.uint8, device="cuda")
        first = torch.from_numpy(out).cuda()
        got = torch.empty_like(first)
        for _ in range(30):
            got.fill_(float("nan"))
            K.paged_decode_attention_fp8(got, q, c.k_pages, c.v_pages, c.dks, c.dvs, tab, lens, cfg.scale,
                                         num_splits=0, workspace=ws)
            torch.cuda.synchronize()
            assert torch.equal(got, first)
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
