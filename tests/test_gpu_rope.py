"""GPU parity of kv_rope_append (rotary embedding fused with the KV append)
against the oracle's stored-precision rotation: bit-exact pools and q."""
import numpy as np
import pytest
import torch

from gpu_cases import TORCH_DT, device_bits, to_device
from oracle import rope as RP
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_433_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


NAN_BITS = {"bf16": 0x7FC0, "fp16": 0x7E00}


def _pool(num_pages, H_kv, P, Dh, dtype):
    """NaN-poisoned pool on both sides."""
    if dtype == "fp32":
        host = np.full((num_pages, H_kv, P, Dh), np.nan, np.float32)
    else:
        host = np.full((num_pages, H_kv, P, Dh), NAN_BITS[dtype], np.uint16)
    return host, to_device(host, dtype)


def _case(dtype, Dh, style, B, H_q, H_kv, P, seed, with_q=True, in_place=False, max_pos=8192):
    num_pages = (B + P - 1) // P + 3
    g = W.generator(seed, W.S_SUFFIX, B)
    slots = g.permutation(num_pages * P)[:B].astype(np.int64)
    slots[3::11] = -1
    positions = g.integers(0, max_pos, B).astype(np.int32)
    table = RP.rope_table(max_pos, Dh, 500000.0)
    k_new = W.normal_storage(seed, W.S_KNEW, (B,), (B, H_kv, Dh), dtype)
    v_new = W.normal_storage(seed, W.S_VNEW, (B,), (B, H_kv, Dh), dtype)
    q = W.normal_storage(seed, W.S_Q, (B,), (B, H_q, Dh), dtype)
    kp_h, kp = _pool(num_pages, H_kv, P, Dh, dtype)
    vp_h, vp = _pool(num_pages, H_kv, P, Dh, dtype)
    RP.rope_append(kp_h, vp_h, k_new, v_new, slots, positions, table, style, dtype)
    q_ref = RP.apply_rope(q, positions, table, style, dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qd = to_device(q, dtype) if with_q else None
    q_out = (qd if in_place else torch.empty_like(qd)) if with_q else None
    K.kv_rope_append(kp, vp, to_device(k_new, dtype), to_device(v_new, dtype), torch.from_numpy(slots).cuda(),
                     torch.from_numpy(positions).cuda(), torch.from_numpy(table).cuda(), P, style=style, q=qd,
                     q_out=q_out, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    view = (lambda a: a.view(np.uint32)) if dtype == "fp32" else (lambda a: a)
    assert np.array_equal(device_bits(kp), view(kp_h)), "K pool bits"
    assert np.array_equal(device_bits(vp), view(vp_h)), "V pool bits"
    if with_q:
        assert np.array_equal(device_bits(q_out), view(q_ref)), "rotated q bits"


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("Dh", [64, 128])
@pytest.mark.parametrize("style", RP.STYLES)
def test_rope_append_bit_exact(dtype, Dh, style):
    _case(dtype, Dh, style, B=67, H_q=32, H_kv=8, P=16, seed=40)


@pytest.mark.parametrize("style", RP.STYLES)
def test_rope_append_in_place_q_and_k_only(style):
    _case("bf16", 128, style, B=33, H_q=12, H_kv=4, P=32, seed=41, in_place=True)
    _case("fp16", 128, style, B=33, H_q=12, H_kv=4, P=32, seed=42, with_q=False)


def test_rope_append_prefill_sized_grid_stride():
    # 8192 tokens x (32 + 2 x 8) rows x 8 units: more units than one pass of the capped grid
    _case("bf16", 128, "half", B=8192, H_q=32, H_kv=8, P=16, seed=43, max_pos=16384)


def test_rope_append_error_bits():
    dtype, Dh, P, H_kv, B = "bf16", 128, 16, 2, 4
    table = torch.from_numpy(RP.rope_table(64, Dh)).cuda()
    kp = torch.zeros((2, H_kv, P, Dh), dtype=TORCH_DT[dtype], device="cuda")
    vp = torch.zeros_like(kp)
    kn = torch.ones((B, H_kv, Dh), dtype=TORCH_DT[dtype], device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.tensor([0, 1, 2, 99], dtype=torch.int64, device="cuda")  # 99 >= 2 * 16
    pos = torch.tensor([0, 64, -1, 5], dtype=torch.int32, device="cuda")   # 64 and -1 outside [0, 64)
    K.kv_rope_append(kp, vp, kn, kn, slots, pos, table, P, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == (K.KV_DEV_ERR_POSITION | K.KV_DEV_ERR_SLOT)
    assert torch.count_nonzero(kp[0, :, 0]).item() == H_kv * Dh  # token 0 written (position 0: identity)
    assert torch.count_nonzero(kp[0, :, 1:3]).item() == 0  # tokens 1 and 2 skipped
    with pytest.raises(K.KvError):  # Dh * 2 bytes not a multiple of 32
        K.kv_rope_append(kp[..., :8].contiguous(), vp[..., :8].contiguous(), kn[..., :8].contiguous(),
                         kn[..., :8].contiguous(), slots, pos, table[:, :8].contiguous(), P)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("style", RP.STYLES)
@pytest.mark.parametrize("splits", [1, 0])
def test_fused_rope_append_decode(dtype, style, splits):
    """paged_decode_attention_rope_append: pools bit-exact vs the oracle's rotate-then-append, output within the
    attention tolerance of the oracle, and bit-identical to kv_rope_append followed by paged_decode_attention."""
    from gpu_cases import build_cache, check_close
    from oracle import reference as R

    cfg = W.DecodeConfig(f"fused-rope-{dtype}-{style}", dtype, B=12, H_q=32, H_kv=8, Dh=128, page_size=16, seed=44)
    lens = [15, 16, 1, 300, 47, 1000, 31, 32, 2047, 5, 64, 129]
    st = build_cache(cfg, lens)
    P = cfg.page_size
    lens32 = st.lens.astype(np.int32).copy()
    mlens = [int(x) for x in st.lens]
    slots = st.pool.append_slots(st.tab, lens32)
    mslots = st.mpool.append_slots(st.mtab, st.max_blocks, mlens)
    assert list(slots) == mslots
    positions = np.asarray(lens, np.int32)  # the new token's position = its cached length before the append
    table = RP.rope_table(4096, cfg.Dh, 500000.0)
    k_new, v_new = W.new_token_kv(cfg, 0, 0)
    q = W.queries(cfg, 0, 0)
    # oracle: rotate, append, fp64 decode
    RP.rope_append(st.kp, st.vp, k_new, v_new, mslots, positions, table, style, dtype)
    q_rot = RP.apply_rope(q, positions, table, style, dtype)
    ref = R.paged_decode(q_rot, st.kp, st.vp, np.asarray(st.mtab, np.int32), np.asarray(mlens, np.int32), cfg.scale,
                         dtype)
    # product, fused, on a copy of the pools; then the two-step path on the original pools
    kp2, vp2 = st.k_pages.clone(), st.v_pages.clone()
    tab = torch.from_numpy(st.tab).cuda()
    d_lens = torch.from_numpy(lens32).cuda()
    d_table = torch.from_numpy(table).cuda()
    nb = K.paged_decode_workspace_bytes(cfg.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, P, splits)
    ws = torch.zeros(max(nb, 16), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((cfg.B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
    K.paged_decode_attention_rope_append(out, to_device(q, dtype), to_device(k_new, dtype), to_device(v_new, dtype), kp2,
                                         vp2, tab, d_lens, d_table, cfg.scale, style=style, num_splits=splits,
                                         workspace=ws, err_flag=err)
    q_out = torch.empty_like(to_device(q, dtype))
    K.kv_rope_append(st.k_pages, st.v_pages, to_device(k_new, dtype), to_device(v_new, dtype),
                     torch.from_numpy(slots).cuda(), torch.from_numpy(positions).cuda(), d_table, P, style=style,
                     q=to_device(q, dtype), q_out=q_out, err_flag=err)
    out2 = torch.empty_like(out)
    K.paged_decode_attention(out2, q_out, st.k_pages, st.v_pages, tab, d_lens, cfg.scale, num_splits=splits,
                             workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(device_bits(kp2), st.kp) and np.array_equal(device_bits(vp2), st.vp), "fused pools"
    assert np.array_equal(device_bits(q_out), q_rot), "rotated q"
    check_close(out.cpu().numpy(), ref, dtype, "fused rope + append + decode")
    assert torch.equal(out, out2), "fused launch differs from rotate-append then decode"
