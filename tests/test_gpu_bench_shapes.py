"""GPU parity in the exact launch configurations that bench.py times.

* the Llama-3.1-8B-shaped layer (B=64) through the fused
  paged_decode_attention_append with the automatic split count, two steps,
  every output against the fp64 oracle and both pools bit for bit;
* the mixed continuous-batching sweep at its real batch (B=256) for all six
  (H_kv, page size) points, after churn (exits and admits at the benchmark's
  rate), with the benchmark's block-table width and pool size, so the
  automatic split / planned-launch choice is the timed one; the oracle checks
  a seeded sample of rows element by element;
* the 32K-context layer through a captured CUDA graph replayed for two steps,
  as the 32-layer benchmark step runs it.

Oracle inputs come from the seeded host generators only. Rows outside the
sample of the mixed sweep are filled on the device (their outputs are not
compared) so the launch sees the full batch.
"""
import numpy as np
import pytest
import torch

from gpu_cases import (TORCH_DT, append_and_decode, build_cache, check_close, device_bits, to_device)
from oracle import reference as R
from oracle.pool_model import PoolModel
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu

# bench.py defaults (driver run: --steps 20 --warmup 5; the layer bench keeps room for an e2e pass too)
BENCH_STEPS, BENCH_WARM = 20, 5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


# ---------------------------------------------------------------- 8B-shaped layer, fused, automatic splits
def test_llama8b_fused_as_benchmarked():
    cfg = W.LLAMA8B
    lens = W.cached_lengths(cfg)
    P = cfg.page_size
    n_steps = 2 * (BENCH_WARM + BENCH_STEPS)  # timed pass + e2e pass, as the layer bench sizes its table
    max_blocks = max(-(-(int(L) + n_steps) // P) for L in lens) + 1
    st = build_cache(cfg, lens, max_blocks=max_blocks, slack_pages=8)
    S = K.paged_decode_num_splits(cfg.B, cfg.H_kv, max_blocks, P, 0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert S > 1 and cfg.B * cfg.H_kv <= 4 * sms  # grid split, not the planned launch
    for step in range(2):
        out, ref, err = append_and_decode(st, step=step, num_splits=0, fused=True, check_pools=True)
        assert err == 0
        check_close(out, ref, cfg.dtype, f"8B fused B=64 S={S} step {step}")


# ---------------------------------------------------------------- mixed sweep at B=256
class SampledBatch:
    """A full batch on the device; the oracle holds only the sampled rows, each in its own compact
    pool (pages in logical order), filled from the host generators."""

    def __init__(self, cfg, lens, max_blocks, num_pages, sample):
        self.cfg, self.P = cfg, cfg.page_size
        self.B = len(lens)
        self.max_blocks = max_blocks
        self.sample = list(sample)
        order = W.page_order(num_pages, cfg.seed)
        self.pool = K.KvPool(num_pages, self.P, order)
        self.mpool = PoolModel(num_pages, self.P, order)
        self.tab = np.full((self.B, max_blocks), -1, np.int32)
        self.mtab = [[-1] * max_blocks for _ in range(self.B)]
        self.lens = np.zeros(self.B, np.int64)
        shape = (num_pages, cfg.H_kv, self.P, cfg.Dh)
        self.k_pages = torch.full(shape, float("nan"), dtype=TORCH_DT[cfg.dtype], device="cuda")
        self.v_pages = torch.full(shape, float("nan"), dtype=TORCH_DT[cfg.dtype], device="cuda")
        self.gen = torch.Generator(device="cuda")
        self.gen.manual_seed(cfg.seed * 31 + cfg.H_kv + cfg.page_size)
        self.rows = {}  # b -> (k rows, v rows) on the host, storage dtype, logical order
        for b in range(self.B):
            self.admit(b, int(lens[b]), tag=0)

    def admit(self, b, n, tag):
        P, cfg = self.P, self.cfg
        k = -(-n // P)
        self.tab[b, :] = -1
        self.tab[b, :k] = self.pool.alloc(k)
        self.mtab[b] = [-1] * self.max_blocks
        self.mtab[b][:k] = self.mpool.alloc(k)
        assert self.tab[b].tolist() == self.mtab[b]
        self.lens[b] = n
        if n == 0:
            return
        slots = torch.from_numpy(K.kv_slots_for_range(self.tab[b], P, 0, n)).cuda()
        if b in self.sample:
            kr, vr = W.kv_rows(cfg, tag, b, n)
            self.rows[b] = (kr, vr)
            kd, vd = to_device(kr, cfg.dtype), to_device(vr, cfg.dtype)
        else:
            kd = torch.randn((n, cfg.H_kv, cfg.Dh), generator=self.gen, device="cuda").to(TORCH_DT[cfg.dtype])
            vd = torch.randn((n, cfg.H_kv, cfg.Dh), generator=self.gen, device="cuda").to(TORCH_DT[cfg.dtype])
        K.kv_append(self.k_pages, self.v_pages, kd, vd, slots, P)

    def release(self, b):
        held = [int(p) for p in self.tab[b] if p >= 0]
        self.pool.free(held)
        self.mpool.free_pages(held)
        self.tab[b, :] = -1
        self.mtab[b] = [-1] * self.max_blocks
        self.lens[b] = 0
        self.rows.pop(b, None)

    def step(self, step, splits=0):
        """Fused append + decode of one new token per row; returns (gpu out [sample], oracle [sample])."""
        cfg, P = self.cfg, self.P
        lens32 = self.lens.astype(np.int32).copy()
        mlens = [int(x) for x in self.lens]
        slots = self.pool.append_slots(self.tab, lens32)
        assert list(slots) == self.mpool.append_slots(self.mtab, self.max_blocks, mlens)
        assert self.tab.tolist() == self.mtab and lens32.tolist() == mlens
        k_new, v_new = W.new_token_kv(cfg, 0, step)
        q = W.queries(cfg, 0, step)
        for b in self.sample:
            kr, vr = self.rows[b]
            self.rows[b] = (np.concatenate([kr, k_new[b:b + 1]]), np.concatenate([vr, v_new[b:b + 1]]))
        out = torch.empty((self.B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = torch.zeros(max(16, K.paged_decode_workspace_bytes(self.B, cfg.H_q, cfg.H_kv, cfg.Dh, self.max_blocks, P,
                                                                splits)), dtype=torch.uint8, device="cuda")
        K.paged_decode_attention_append(out, to_device(q, cfg.dtype), to_device(k_new, cfg.dtype),
                                        to_device(v_new, cfg.dtype), self.k_pages, self.v_pages,
                                        torch.from_numpy(self.tab).cuda(), torch.from_numpy(lens32).cuda(), cfg.scale,
                                        num_splits=splits, workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        self.lens = self.lens + 1
        # every row's new token sits at its slot, bit for bit
        sl = torch.from_numpy(slots).cuda()
        pg, off = sl // P, sl % P
        got_k = self.k_pages[pg, :, off, :]
        got_v = self.v_pages[pg, :, off, :]
        assert np.array_equal(device_bits(got_k), k_new) and np.array_equal(device_bits(got_v), v_new)
        # oracle on the sample: compact pool per row, pages in logical order
        gpu, ref = [], []
        for b in self.sample:
            kr, vr = self.rows[b]
            n = kr.shape[0]
            npg = -(-n // P)
            kp = np.zeros((npg, cfg.H_kv, P, cfg.Dh), kr.dtype)
            vp = np.zeros_like(kp)
            ident = np.arange(npg, dtype=np.int32)
            R.scatter_to_pages(kp, ident, kr)
            R.scatter_to_pages(vp, ident, vr)
            ref.append(R.paged_decode(q[b:b + 1], kp, vp, ident[None, :], np.array([n], np.int32), cfg.scale,
                                      cfg.dtype)[0])
            # the row's device pages, read back through its block table, hold the same bits
            pages = torch.from_numpy(self.tab[b, :npg].astype(np.int64)).cuda()
            dk = device_bits(self.k_pages[pages]).reshape(npg, cfg.H_kv, P, cfg.Dh)
            dv = device_bits(self.v_pages[pages]).reshape(npg, cfg.H_kv, P, cfg.Dh)
            t = np.arange(n)
            assert np.array_equal(dk[t // P, :, t % P, :], kr) and np.array_equal(dv[t // P, :, t % P, :], vr)
            gpu.append(out[b].cpu().numpy())
        return np.stack(gpu), np.stack(ref)


def _sample_rows(lens, n, seed):
    """Seeded sample of rows that always holds the longest and the shortest row."""
    g = np.random.default_rng(seed)
    pick = {int(np.argmax(lens)), int(np.argmin(lens))}
    for b in g.permutation(len(lens)):
        if len(pick) >= n:
            break
        pick.add(int(b))
    return sorted(pick)


@pytest.mark.parametrize("H_kv,P", W.MIXED_POINTS)
def test_mixed_sweep_full_batch(H_kv, P):
    cfg = W.mixed_config(H_kv, P)
    lens = W.cached_lengths(cfg)
    n = BENCH_WARM + BENCH_STEPS
    # bench.py's table width and pool size for this point
    max_blocks = -(-(16384 + n + 1) // P) + 1
    num_pages = int(sum(-(-(int(L) + n) // P) for L in lens)) * 3 // 2 + 4 * max_blocks
    events = W.churn_events(cfg, n)
    # the sample: seeded rows plus every row that churns in the two checked steps
    churned = sorted(set(int(b) for ev in events[:2] for b in ev.exits))
    sample = sorted(set(_sample_rows(lens, 14, cfg.seed + H_kv + P)) | set(churned))
    sb = SampledBatch(cfg, lens, max_blocks, num_pages, sample)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    planned = cfg.B * H_kv > 4 * sms
    S, kind = K.paged_decode_launch_info(cfg.B, cfg.H_q, H_kv, cfg.Dh, max_blocks, P, cfg.dtype, 0)
    planned = planned or kind == K.KV_DECODE_KERNEL_TCGEN05  # the tcgen05 kernel plans every multi-row batch
    assert (S == 0) == planned
    for step in range(2):
        ev = events[step]
        for b, L in zip(ev.exits, ev.new_lengths):
            sb.release(int(b))
            sb.admit(int(b), int(L), tag=100 + step)
        gpu, ref = sb.step(step)
        check_close(gpu, ref, cfg.dtype, f"mixed B=256 Hkv={H_kv} P={P} ({'planned' if planned else f'S={S}'}) "
                                         f"step {step}")


# ---------------------------------------------------------------- 32K context through a CUDA graph
def test_long_context_cuda_graph_replay():
    """Two layers of the 32K-context step captured in one CUDA graph (fused append + decode + combine,
    automatic split), replayed for two steps with inputs staged into the captured buffers."""
    cfg = W.LONG32K
    P = cfg.page_size
    layers = (0, 31)
    lens = W.cached_lengths(cfg)
    sts = [build_cache(cfg, lens, layer=layer, slack_pages=4) for layer in layers]
    B = cfg.B
    max_blocks = sts[0].max_blocks
    S = K.paged_decode_num_splits(B, cfg.H_kv, max_blocks, P, 0)
    assert S > 1
    dt = TORCH_DT[cfg.dtype]
    cur = {"q": torch.empty((len(layers), B, cfg.H_q, cfg.Dh), dtype=dt, device="cuda"),
           "kn": torch.empty((len(layers), B, cfg.H_kv, cfg.Dh), dtype=dt, device="cuda"),
           "vn": torch.empty((len(layers), B, cfg.H_kv, cfg.Dh), dtype=dt, device="cuda"),
           "lens": torch.empty(B, dtype=torch.int32, device="cuda")}
    tabs = [torch.from_numpy(st.tab).cuda() for st in sts]
    out = torch.empty((len(layers), B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
    ws = torch.zeros(K.paged_decode_workspace_bytes(B, cfg.H_q, cfg.H_kv, cfg.Dh, max_blocks, P, 0),
                     dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def layers_pass(stream):
        for i, st in enumerate(sts):
            K.paged_decode_attention_append(out[i], cur["q"][i], cur["kn"][i], cur["vn"][i], st.k_pages, st.v_pages,
                                            tabs[i], cur["lens"], cfg.scale, num_splits=0, workspace=ws, err_flag=err,
                                            stream=stream)

    # the first call configures the library outside any capture; it runs on zero-length rows
    cur["lens"].zero_()
    layers_pass(torch.cuda.current_stream())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=side):
        layers_pass(side)
    torch.cuda.synchronize()
    for step in range(2):
        # host bookkeeping per layer (each layer's pools have their own page order), oracle append
        refs = []
        for i, (st, layer) in enumerate(zip(sts, layers)):
            mlens = [int(x) for x in st.lens]
            lens32 = st.lens.astype(np.int32).copy()
            slots = st.pool.append_slots(st.tab, lens32)  # lens32 now counts the new token
            assert list(slots) == st.mpool.append_slots(st.mtab, st.max_blocks, mlens)
            assert st.tab.tolist() == st.mtab
            tabs[i].copy_(torch.from_numpy(st.tab))  # a page added at a block boundary reaches the captured table
            k_new, v_new = W.new_token_kv(cfg, layer, step)
            q = W.queries(cfg, layer, step)
            for b in range(B):
                page, off = divmod(int(slots[b]), P)
                st.kp[page, :, off, :] = k_new[b]
                st.vp[page, :, off, :] = v_new[b]
            cur["q"][i].copy_(to_device(q, cfg.dtype))
            cur["kn"][i].copy_(to_device(k_new, cfg.dtype))
            cur["vn"][i].copy_(to_device(v_new, cfg.dtype))
            refs.append(R.paged_decode(q, st.kp, st.vp, st.tab, lens32, cfg.scale, cfg.dtype))
        cur["lens"].copy_(torch.from_numpy(lens32))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for i, st in enumerate(sts):
            check_close(out[i].cpu().numpy(), refs[i], cfg.dtype, f"32K graph layer {layers[i]} step {step}")
            assert np.array_equal(device_bits(st.k_pages), st.kp) and np.array_equal(device_bits(st.v_pages), st.vp)
            st.lens = st.lens + 1
    del graph
