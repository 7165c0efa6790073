"""GPU parity: every kernel, called through the C-ABI binding, against the CPU
oracle on the same seeded inputs.  Bit-exact for the tensor scale, packed
codes, scale bytes and FP8 bytes; attention within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle over the same FP8 values.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from cases import Case, assert_attention_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import bit_decode_attention_b200 as nv
    return nv


# ---------------------------------------------------------------------------
# calibration
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [1, 7, 1000, (1 << 20) + 3])
def test_calib_bit_exact(nv, dtype, n):
    w = synthetic.shrink(synthetic.get("long64k"), dtype=dtype)
    x = synthetic.kv_tokens(w, (n + 1023) // 1024, "k").reshape(-1)[:n]
    for offset in (0, 1):       # aligned and misaligned base pointer
        xs = x[offset:] if n > 1 else x
        st, want = oracle.tensor_scale(xs.numpy())
        dev = to_dev(x, dtype)[offset:] if n > 1 else to_dev(x, dtype)
        got = nv.nvfp4_calib_tensor_scale(dev).item()
        assert st == 0
        assert np.float32(got).view(np.uint32) == np.float32(want).view(np.uint32)


def test_calib_zero_and_nonfinite(nv):
    z = torch.zeros(100, device="cuda", dtype=torch.bfloat16)
    assert nv.nvfp4_calib_tensor_scale(z).item() == 1.0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.ones(100, device="cuda")
    x[37] = float("nan")
    s = nv.nvfp4_calib_tensor_scale(x, status=status)
    assert np.isnan(s.item()) and status.item() == nv.NVFP4_ERR_NONFINITE
    st_o, _ = oracle.tensor_scale(x.cpu().numpy())
    assert st_o == 4


# ---------------------------------------------------------------------------
# quantize + append, dequant
# ---------------------------------------------------------------------------
def _check_planes(case, batch_indices=None):
    bs = list(range(case.w.B)) if batch_indices is None else list(batch_indices)
    for b in bs:
        kc, ks, vc, vs = case.oracle_planes(b)
        L = case.lens[b]
        np.testing.assert_array_equal(case.k.codes[b, :, :L].cpu().numpy(), kc[0, :, :L])
        np.testing.assert_array_equal(case.k.scales[b, :, :L].cpu().numpy(), ks[0, :, :L])
        np.testing.assert_array_equal(case.v.codes[b, :, :L].cpu().numpy(), vc[0, :, :L])
        np.testing.assert_array_equal(case.v.scales[b, :, :L].cpu().numpy(), vs[0, :, :L])


SMALL_CASES = {
    "tiny": lambda: Case(synthetic.get("tiny")),
    "gqa_ragged": lambda: Case(synthetic.shrink(synthetic.get("gqa"), B=4), lens=[4097, 1, 33, 640]),
    "long_outliers": lambda: Case(synthetic.shrink(synthetic.get("long64k"), L=20000)),
    "ragged16": lambda: Case(synthetic.shrink(synthetic.get("ragged"), B=16)),
    "moe_g12_chunked": lambda: Case(synthetic.shrink(synthetic.get("moe128k"), L=5000),
                                    prefill_chunk=2048),
}


@pytest.fixture(scope="module", params=list(SMALL_CASES))
def case(request):
    c = SMALL_CASES[request.param]()
    assert c.status.item() == 0
    return c


def test_tensor_scale_matches(case):
    for dev, want in ((case.sk, case.sk_o), (case.sv, case.sv_o)):
        assert np.float32(dev.item()).view(np.uint32) == np.float32(want).view(np.uint32)


def test_quantize_append_bit_exact(case):
    _check_planes(case)


def test_dequant_fp8_bit_exact(nv, case):
    out = nv.nvfp4_kv_dequant_fp8(case.k, case.sk, case.seq_lens).cpu().numpy()
    kc, ks, vc, vs = case.oracle_planes()
    want = oracle.dequant_planes(kc, ks, case.sk_o, np.array(case.lens, np.int32))
    for b, L in enumerate(case.lens):
        np.testing.assert_array_equal(out[b, :, :L], want[b, :, :L])


def test_attention_parity(case):
    got = case.gpu_attention().cpu().numpy()
    want = case.oracle_attention()
    assert_attention_close(got, want)
    assert case.status.item() == 0


def test_special_blocks_bit_exact(nv):
    rows = synthetic.special_blocks(128)
    for dtype in ("f32", "bf16"):
        x = rows.to(torch.bfloat16).float() if dtype == "bf16" else rows
        x = x.view(1, rows.shape[0], 1, 128).contiguous()      # B=1, n tokens, H=1
        for st in (np.float32(1.0), np.float32(0.01), np.float32(1e-30), np.float32(3e4)):
            plane = nv.KVPlane.allocate(1, 1, 16, 128)
            s = torch.tensor([st], device="cuda")
            start = torch.zeros(1, dtype=torch.int32, device="cuda")
            nv.nvfp4_kv_quantize_append(to_dev(x, dtype), start, s, plane)
            kc, ks = oracle.new_planes(1, 1, 16, 128)
            assert oracle.quantize_append(x.numpy(), np.zeros(1, np.int32), st, kc, ks) == 0
            n = rows.shape[0]
            np.testing.assert_array_equal(plane.codes[0, 0, :n].cpu().numpy(), kc[0, 0, :n])
            np.testing.assert_array_equal(plane.scales[0, 0, :n].cpu().numpy(), ks[0, 0, :n])


def test_nonfinite_blocks_bit_exact(nv):
    # NaN and infinite elements: no status (the append does not check its
    # input), codes and scales as the oracle's -- a NaN element gives code 0x7
    rows = synthetic.nonfinite_blocks(128)
    x = rows.view(1, rows.shape[0], 1, 128).contiguous()
    for st in (np.float32(1.0), np.float32(0.01)):
        plane = nv.KVPlane.allocate(1, 1, 16, 128)
        s = torch.tensor([st], device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_kv_quantize_append(x.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), s, plane,
                                    status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        kc, ks = oracle.new_planes(1, 1, 16, 128)
        assert oracle.quantize_append(x.numpy(), np.zeros(1, np.int32), st, kc, ks) == 0
        n = rows.shape[0]
        np.testing.assert_array_equal(plane.codes[0, 0, :n].cpu().numpy(), kc[0, 0, :n])
        np.testing.assert_array_equal(plane.scales[0, 0, :n].cpu().numpy(), ks[0, 0, :n])


def test_quantize_wide_range_f32_bit_exact(nv):
    # fp32 inputs over 60 binades and tensor scales over 40: the division by
    # correction and the hardware E2M1 conversion give the oracle's codes
    g = torch.Generator().manual_seed(2024)
    n_tok, H, D = 512, 4, 128
    mag = torch.exp2(torch.empty(n_tok, H, D).uniform_(-30.0, 30.0, generator=g))
    sign = torch.where(torch.rand(n_tok, H, D, generator=g) < 0.5, -1.0, 1.0)
    x = (mag * sign).view(1, n_tok, H, D).contiguous()
    for st in (np.float32(3.7e-9), np.float32(0.0123), np.float32(1.0), np.float32(2.9e3), np.float32(6.1e5)):
        plane = nv.KVPlane.allocate(1, H, n_tok, D)
        s = torch.tensor([st], device="cuda")
        nv.nvfp4_kv_quantize_append(x.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), s, plane)
        kc, ks = oracle.new_planes(1, H, n_tok, D)
        assert oracle.quantize_append(x.numpy(), np.zeros(1, np.int32), st, kc, ks) == 0
        np.testing.assert_array_equal(plane.codes.cpu().numpy(), kc)
        np.testing.assert_array_equal(plane.scales.cpu().numpy(), ks)


def _e2m1_tie_blocks(st, n_tok, H, D, seed):
    """fp32 rows [1][n_tok][H][D] whose 16-element blocks take an E4M3 scale
    value V under the tensor scale st (one element is RN(RN(6 st) V), so the
    block maximum over 6 st rounds to V), every other element being RN(t den)
    or one of its four nearest neighbours, den = RN(V st) the block divisor
    and t a rounding tie of the E2M1 grid: quotients within a few ulps of a
    tie, where a misrounded division changes the code."""
    rng = np.random.default_rng(seed)
    st = np.float32(st)
    n_blk = n_tok * H * D // 16
    V = ((1.0 + rng.integers(0, 8, n_blk) / 8.0) * np.exp2(rng.integers(-6, 9, n_blk))).astype(np.float32)
    V = np.minimum(V, np.float32(448.0))
    den = V * st
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    t = ties[rng.integers(0, ties.size, (n_blk, 16))]
    a = (t * den[:, None]).astype(np.float32)
    a = (a.view(np.int32) + rng.integers(-2, 3, (n_blk, 16)).astype(np.int32)).view(np.float32)
    a[np.arange(n_blk), rng.integers(0, 16, n_blk)] = (np.float32(6.0) * st) * V
    a = np.where(rng.random((n_blk, 16)) < 0.5, -a, a).astype(np.float32)
    return torch.from_numpy(a.reshape(1, n_tok, H, D).copy())


@pytest.mark.parametrize("st", [3.1e-33, 7.3e-31, 1.7e-28, 0.37])
def test_quantize_near_ties_tiny_tensor_scales_bit_exact(nv, st):
    """Blocks whose divisor den lies far below 1 (down to about 2^-114, where
    the residual of a division by correction would underflow) or near 1, with
    elements next to E2M1 rounding ties: codes and scales equal the oracle's,
    through the quantize-append kernel and the append of the fused
    append + attention kernel."""
    n_tok, H, D = 64, 2, 128
    x = _e2m1_tie_blocks(st, n_tok, H, D, seed=int(st * 1e3) % 1000 + 7)
    st32 = np.float32(st)
    s = torch.tensor([st32], device="cuda")
    plane = nv.KVPlane.allocate(1, H, n_tok, D)
    nv.nvfp4_kv_quantize_append(x.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), s, plane)
    kc, ks = oracle.new_planes(1, H, n_tok, D)
    assert oracle.quantize_append(x.numpy(), np.zeros(1, np.int32), st32, kc, ks) == 0
    np.testing.assert_array_equal(plane.codes.cpu().numpy(), kc)
    np.testing.assert_array_equal(plane.scales.cpu().numpy(), ks)
    # the same rows as n_tok sequences of one new token each
    xb = x.view(n_tok, 1, H, D).contiguous()
    q = torch.randn(n_tok, 4 * H, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    kp = nv.KVPlane.allocate(n_tok, H, 16, D)
    vp = nv.KVPlane.allocate(n_tok, H, 16, D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start = torch.zeros(n_tok, dtype=torch.int32, device="cuda")
    out = nv.nvfp4_decode_attention_append(q.cuda(), xb.cuda(), xb.cuda(), start, kp, vp, s, s, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0 and bool(torch.isfinite(out).all())
    kc, ks = oracle.new_planes(n_tok, H, 16, D)
    assert oracle.quantize_append(xb.numpy(), np.zeros(n_tok, np.int32), st32, kc, ks) == 0
    for p in (kp, vp):
        np.testing.assert_array_equal(p.codes[:, :, :1].cpu().numpy(), kc[:, :, :1])
        np.testing.assert_array_equal(p.scales[:, :, :1].cpu().numpy(), ks[:, :, :1])


@pytest.mark.parametrize("D", [64, 128])
def test_dequant_random_planes_bit_exact(nv, D):
    B, H, S = 2, 3, 64
    codes, scales = synthetic.random_planes(7 + D, B, H, S, D)
    plane = nv.KVPlane(codes.cuda(), scales.cuda())
    lens = np.array([64, 37], np.int32)
    for st in (1.0, 0.0371, 2.0 ** -20, 1e-8, 7.5):
        s = torch.tensor([st], dtype=torch.float32, device="cuda")
        got = nv.nvfp4_kv_dequant_fp8(plane, s, torch.from_numpy(lens).cuda()).cpu().numpy()
        want = oracle.dequant_planes(codes.numpy(), scales.numpy(), np.float32(st), lens)
        for b in range(B):
            np.testing.assert_array_equal(got[b, :, :lens[b]], want[b, :, :lens[b]])


def test_append_capacity_and_new_lens(nv):
    w = synthetic.shrink(synthetic.get("gqa"), B=3, Hkv=2, Hq=4)
    x = synthetic.kv_tokens(w, 5, "k")
    plane = nv.KVPlane.allocate(3, 2, 16, 128)
    s = torch.tensor([0.01], device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start = torch.tensor([0, 12, 11], dtype=torch.int32, device="cuda")
    new_lens = torch.full((3,), -7, dtype=torch.int32, device="cuda")
    nv.nvfp4_kv_quantize_append(to_dev(x, "bf16"), start, s, plane, new_lens=new_lens, status=status)
    assert status.item() == nv.NVFP4_ERR_CAPACITY
    assert new_lens.tolist() == [5, -7, 16]
    assert not plane.codes[1].any().item()
    kc, ks = oracle.new_planes(3, 2, 16, 128)
    assert oracle.quantize_append(x.numpy(), start.cpu().numpy(), np.float32(0.01), kc, ks) == 3
    np.testing.assert_array_equal(plane.codes.cpu().numpy(), kc)
    np.testing.assert_array_equal(plane.scales.cpu().numpy(), ks)


def test_bad_tensor_scale_reports(nv):
    plane = nv.KVPlane.allocate(1, 1, 16, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.ones(1, 1, 1, 64, device="cuda")
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        status.zero_()
        nv.nvfp4_kv_quantize_append(x, torch.zeros(1, dtype=torch.int32, device="cuda"),
                                    torch.tensor([bad], device="cuda"), plane, status=status)
        assert status.item() == nv.NVFP4_ERR_NONFINITE
    assert not plane.codes.any().item()


# ---------------------------------------------------------------------------
# attention edge cases
# ---------------------------------------------------------------------------
def test_attention_empty_and_short_sequences(nv):
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=5, Hq=8, Hkv=2), lens=[0, 5, 0, 1, 31])
    got = c.gpu_attention().cpu().numpy()
    assert not got[0].any() and not got[2].any()
    assert_attention_close(got, c.oracle_attention())


def test_attention_q_dtypes_and_scale(nv):
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=2, Hq=16, Hkv=2, D=64), lens=[300, 77],
             q_dtype="f32")
    assert_attention_close(c.gpu_attention().cpu().numpy(), c.oracle_attention())
    assert_attention_close(c.gpu_attention(softmax_scale=0.05).cpu().numpy(),
                           c.oracle_attention(softmax_scale=0.05))
    c2 = Case(synthetic.shrink(synthetic.get("tiny"), B=2, Hq=4, Hkv=1, dtype="bf16"), lens=[256, 40])
    assert_attention_close(c2.gpu_attention().cpu().numpy(), c2.oracle_attention())


def test_attention_fewer_tiles_than_ctas(nv):
    # one unit spread over CTAs with empty ranges in between (94 tiles < grid)
    c = Case(synthetic.shrink(synthetic.get("long64k"), Hq=2, Hkv=1, L=3000))
    assert_attention_close(c.gpu_attention().cpu().numpy(), c.oracle_attention())


def test_attention_group_sizes(nv):
    for g in (1, 2, 3, 8, 12, 16):
        c = Case(synthetic.shrink(synthetic.get("gqa"), B=2, Hq=2 * g, Hkv=2), lens=[700, 129])
        assert_attention_close(c.gpu_attention().cpu().numpy(), c.oracle_attention())


def test_attention_large_batch_is_chunked(nv):
    w = synthetic.shrink(synthetic.get("ragged"), B=600, Hq=2, Hkv=1, L_range=(1, 40))
    c = Case(w)
    assert_attention_close(c.gpu_attention().cpu().numpy(), c.oracle_attention())


def test_attention_workspace_reuse_and_repeatability(nv):
    c = Case(synthetic.shrink(synthetic.get("long64k"), L=9000))
    ws = nv.new_workspace(1, 64, 8, 128)
    a = c.gpu_attention(workspace=ws).cpu()
    b = c.gpu_attention(workspace=ws).cpu()
    assert torch.equal(a, b)
    counters = ws[: 8 * 4].view(torch.int32)
    assert not counters.any().item()      # arrival counters are left at zero


def test_attention_length_past_capacity_reports(nv):
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=2, Hq=8, Hkv=2), lens=[40, 16])
    bad = torch.tensor([40, c.S_max + 5], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = nv.nvfp4_decode_attention(c.q_dev, c.k, c.v, c.sk, c.sv, bad, status=status)
    torch.cuda.synchronize()
    assert status.item() == nv.NVFP4_ERR_CAPACITY
    assert torch.isfinite(out).all().item()


@pytest.mark.parametrize("D,q_dtype", [(128, "bf16"), (128, "f32"), (64, "bf16")])
def test_attention_ignores_bytes_past_the_sequence(nv, D, q_dtype):
    # cache slots past each sequence's length hold 0xFF bytes (E4M3 NaN scales,
    # code -6): the output must not see them, P = 0 there must not meet a NaN V
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=3, Hq=16, Hkv=2, D=D), lens=[130, 1, 259],
             q_dtype=q_dtype)
    for b, L in enumerate(c.lens):
        for plane in (c.k, c.v):
            plane.codes[b, :, L:] = 0xFF
            plane.scales[b, :, L:] = 0xFF
    got = c.gpu_attention().cpu().numpy()
    assert c.status.item() == 0
    assert_attention_close(got, c.oracle_attention())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_append_kv_matches_two_calls(nv, dtype):
    # one launch for K and V gives the same planes (and new lengths) as two calls,
    # and both match the oracle
    w = synthetic.shrink(synthetic.get("gqa"), B=3, Hq=8, Hkv=2, dtype=dtype)
    n_new = 37
    xk = synthetic.kv_tokens(w, n_new, "k")
    xv = synthetic.kv_tokens(w, n_new, "v")
    start = torch.tensor([0, 5, 100], dtype=torch.int32, device="cuda")
    S_max = synthetic.capacity(100 + n_new)
    sk = nv.nvfp4_calib_tensor_scale(to_dev(xk.reshape(-1), dtype))
    sv = nv.nvfp4_calib_tensor_scale(to_dev(xv.reshape(-1), dtype))
    xk_d, xv_d = to_dev(xk, dtype), to_dev(xv, dtype)
    planes = [nv.KVPlane.allocate(w.B, w.Hkv, S_max, w.D) for _ in range(4)]
    lens_a = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    lens_b = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_kv_quantize_append_kv(xk_d, xv_d, start, sk, sv, planes[0], planes[1], new_lens=lens_a,
                                   status=status)
    nv.nvfp4_kv_quantize_append(xk_d, start, sk, planes[2], new_lens=lens_b, status=status)
    nv.nvfp4_kv_quantize_append(xv_d, start, sv, planes[3], status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for a, b in ((planes[0], planes[2]), (planes[1], planes[3])):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
    assert lens_a.tolist() == [n_new, 5 + n_new, 100 + n_new] == lens_b.tolist()
    # oracle: sequence 1, K and V, with the oracle's own tensor scales (equal to the
    # device's bit for bit, which test_calib_bit_exact covers)
    rc_k, st_k_o = oracle.tensor_scale(xk.reshape(-1).numpy())
    rc_v, st_v_o = oracle.tensor_scale(xv.reshape(-1).numpy())
    assert rc_k == 0 and rc_v == 0
    assert np.float32(sk.item()).view(np.uint32) == st_k_o.view(np.uint32)
    assert np.float32(sv.item()).view(np.uint32) == st_v_o.view(np.uint32)
    for x, st_o, pl in ((xk, st_k_o, planes[0]), (xv, st_v_o, planes[1])):
        oc, os_ = oracle.new_planes(1, w.Hkv, S_max, w.D)
        assert oracle.quantize_append(x[1:2].numpy(), np.array([5], np.int32), st_o, oc, os_) == 0
        np.testing.assert_array_equal(pl.codes[1].cpu().numpy(), oc[0])
        np.testing.assert_array_equal(pl.scales[1].cpu().numpy(), os_[0])


# ---------------------------------------------------------------------------
# MXFP4 codec: the OCP format the pages compare NVFP4 with
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
def test_mxfp4_quantize_append_bit_exact(nv, dtype, D):
    w = synthetic.shrink(synthetic.get("long64k"), B=3, Hq=8, Hkv=2, D=D, dtype=dtype)
    n_new = 37
    x = synthetic.kv_tokens(w, n_new, "k")
    start = np.array([0, 5, 100], np.int32)
    S_max = synthetic.capacity(100 + n_new)
    plane = nv.KVPlane.allocate_mxfp4(w.B, w.Hkv, S_max, D)
    lens = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.mxfp4_kv_quantize_append(to_dev(x, dtype), torch.from_numpy(start).cuda(), plane, new_lens=lens,
                                status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert lens.tolist() == (start + n_new).tolist()
    oc, os_ = oracle.new_mxfp4_planes(w.B, w.Hkv, S_max, D)
    assert oracle.mxfp4_quantize_append(x.numpy(), start, oc, os_) == 0
    np.testing.assert_array_equal(plane.codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(plane.scales.cpu().numpy(), os_)


def test_mxfp4_special_blocks_bit_exact(nv):
    rows = synthetic.special_blocks(128)
    extra = torch.zeros(4, 128)
    extra[0, :3] = torch.tensor([3e38, -1.0, 1e-30])           # top of the exponent range
    extra[1, :2] = torch.tensor([7.346839692639297e-40, -3.6734198463196485e-40])   # subnormal amax
    extra[2, ::5] = 6.0 * 2.0 ** -100                         # exact grid values, low exponent
    extra[3, :] = torch.linspace(-8.0, 8.0, 128)              # every E2M1 tie within one block
    for dtype in ("f32", "bf16"):
        src = torch.cat([rows, extra]) if dtype == "f32" else rows
        x = src.to(torch.bfloat16).float() if dtype == "bf16" else src
        n = x.shape[0]
        x = x.view(1, n, 1, 128).contiguous()
        plane = nv.KVPlane.allocate_mxfp4(1, 1, 16, 128)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.mxfp4_kv_quantize_append(to_dev(x, dtype), torch.zeros(1, dtype=torch.int32, device="cuda"),
                                    plane, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        oc, os_ = oracle.new_mxfp4_planes(1, 1, 16, 128)
        assert oracle.mxfp4_quantize_append(x.numpy(), np.zeros(1, np.int32), oc, os_) == 0
        np.testing.assert_array_equal(plane.codes[0, 0, :n].cpu().numpy(), oc[0, 0, :n])
        np.testing.assert_array_equal(plane.scales[0, 0, :n].cpu().numpy(), os_[0, 0, :n])


def test_mxfp4_nonfinite_blocks_and_capacity(nv):
    B, H, S, D = 3, 2, 16, 64
    x = torch.ones(B, 2, H, D)
    x[0, 1, 1, 40] = float("nan")
    x[1, 0, 0, 3] = float("inf")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    plane = nv.KVPlane.allocate_mxfp4(B, H, S, D)
    start = np.array([0, 3, 6], np.int32)
    nv.mxfp4_kv_quantize_append(x.cuda(), torch.from_numpy(start).cuda(), plane, status=status)
    torch.cuda.synchronize()
    assert status.item() == nv.NVFP4_ERR_NONFINITE
    oc, os_ = oracle.new_mxfp4_planes(B, H, S, D)
    assert oracle.mxfp4_quantize_append(x.numpy(), start, oc, os_) == 4
    np.testing.assert_array_equal(plane.codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(plane.scales.cpu().numpy(), os_)
    assert os_[0, 1, 1, 1] == 0xFF and os_[1, 0, 3, 0] == 0xFF
    # a sequence past its capacity is skipped and reported; new_lens only for the others
    status.zero_()
    lens = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    start = np.array([0, 15, 14], np.int32)
    plane2 = nv.KVPlane.allocate_mxfp4(B, H, S, D)
    y = torch.ones(B, 2, H, D)
    nv.mxfp4_kv_quantize_append(y.cuda(), torch.from_numpy(start).cuda(), plane2, new_lens=lens,
                                status=status)
    torch.cuda.synchronize()
    assert status.item() == nv.NVFP4_ERR_CAPACITY
    assert lens.tolist() == [2, -7, 16]
    assert not plane2.codes[1].any().item() and not plane2.scales[1].any().item()


def test_mxfp4_error_above_nvfp4_on_device_codes(nv):
    # the pages' ordering (NVFP4 < MXFP4 quantization error) on the planes the
    # device wrote for the long-context K recipe
    w = synthetic.shrink(synthetic.get("long64k"), B=1, Hq=8, Hkv=2)
    n = 512
    x = synthetic.kv_tokens(w, n, "k")
    xd = to_dev(x, "bf16")
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = nv.nvfp4_calib_tensor_scale(xd)
    p16 = nv.KVPlane.allocate(1, w.Hkv, n, 128)
    p32 = nv.KVPlane.allocate_mxfp4(1, w.Hkv, n, 128)
    nv.nvfp4_kv_quantize_append(xd, start, st, p16)
    nv.mxfp4_kv_quantize_append(xd, start, p32)
    ref = x.numpy().transpose(0, 2, 1, 3).astype(np.float64)
    rec16 = oracle.nvfp4_reconstruct_planes(p16.codes.cpu().numpy(), p16.scales.cpu().numpy(),
                                            np.float32(st.item()), [n])
    rec32 = oracle.mxfp4_reconstruct_planes(p32.codes.cpu().numpy(), p32.scales.cpu().numpy(), [n])
    assert np.mean((rec16 - ref) ** 2) < np.mean((rec32 - ref) ** 2)


# ---------------------------------------------------------------------------
# Paged cache: a page pool and a block table in place of contiguous slabs
# ---------------------------------------------------------------------------
def _paged_setup(nv, B, H, D, page_tokens, max_pages, num_pages, seed):
    """A block table that hands out distinct pool pages in a shuffled order."""
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)[:B * max_pages]
    table = perm.view(B, max_pages).to(torch.int32).cuda()
    k = nv.PagedKVPlane.allocate(num_pages, H, page_tokens, D, table)
    v = nv.PagedKVPlane.allocate(num_pages, H, page_tokens, D, table)
    return table, k, v


def _gather(plane, table_np, S):
    """Contiguous [B][H][S][...] views of a paged plane, by following its table."""
    codes, scales = plane.codes.cpu().numpy(), plane.scales.cpu().numpy()
    B, M = table_np.shape
    P = codes.shape[2]
    oc = np.zeros((B, codes.shape[1], S, codes.shape[3]), np.uint8)
    os_ = np.zeros((B, scales.shape[1], S, scales.shape[3]), np.uint8)
    for b in range(B):
        for m in range(S // P):
            oc[b, :, m * P:(m + 1) * P] = codes[table_np[b, m]]
            os_[b, :, m * P:(m + 1) * P] = scales[table_np[b, m]]
    return oc, os_


@pytest.mark.parametrize("D,q_dtype", [(128, "bf16"), (128, "f32"), (64, "bf16")])
def test_paged_cache_matches_contiguous_and_oracle(nv, D, q_dtype):
    B, H, Hq, P, M = 3, 2, 8, 128, 4
    S = P * M
    w = synthetic.shrink(synthetic.get("long64k"), B=B, Hq=Hq, Hkv=H, D=D)
    table, kp, vp = _paged_setup(nv, B, H, D, P, M, 20, seed=D)
    lens = [300, 129, 511]
    xk = synthetic.kv_tokens(w, S, "k")
    xv = synthetic.kv_tokens(w, S, "v")
    sk = nv.nvfp4_calib_tensor_scale(to_dev(xk.reshape(-1), "bf16"))
    sv = nv.nvfp4_calib_tensor_scale(to_dev(xv.reshape(-1), "bf16"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    new_lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    # a prefill of 300 tokens, then the rest one chunk at a time: pages are crossed mid-append
    for lo, hi in ((0, 300), (300, 301), (301, S)):
        start = torch.full((B,), lo, dtype=torch.int32, device="cuda")
        nv.nvfp4_kv_quantize_append_paged(to_dev(xk[:, lo:hi], "bf16"), start, sk, kp, new_lens=new_lens,
                                          status=status)
        nv.nvfp4_kv_quantize_append_paged(to_dev(xv[:, lo:hi], "bf16"), start, sv, vp, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0 and new_lens.tolist() == [S] * B
    # the pages, read through the table, hold exactly the oracle's contiguous planes
    table_np = table.cpu().numpy()
    kc, ks = _gather(kp, table_np, S)
    vc, vs = _gather(vp, table_np, S)
    _, st_k = oracle.tensor_scale(xk.reshape(-1).numpy())
    _, st_v = oracle.tensor_scale(xv.reshape(-1).numpy())
    okc, oks = oracle.new_planes(B, H, S, D)
    ovc, ovs = oracle.new_planes(B, H, S, D)
    z = np.zeros(B, np.int32)
    assert oracle.quantize_append(xk.numpy(), z, st_k, okc, oks) == 0
    assert oracle.quantize_append(xv.numpy(), z, st_v, ovc, ovs) == 0
    for got, want in ((kc, okc), (ks, oks), (vc, ovc), (vs, ovs)):
        np.testing.assert_array_equal(got, want)
    # attention through the table equals attention over the same bytes laid out contiguously
    q = synthetic.queries(w)
    qd = to_dev(q, q_dtype)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    paged = nv.nvfp4_decode_attention_paged(qd, kp, vp, sk, sv, lens_d, status=status)
    kcont = nv.KVPlane(torch.from_numpy(kc).cuda(), torch.from_numpy(ks).cuda())
    vcont = nv.KVPlane(torch.from_numpy(vc).cuda(), torch.from_numpy(vs).cuda())
    cont = nv.nvfp4_decode_attention(qd, kcont, vcont, sk, sv, lens_d, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(paged, cont)
    want = oracle.decode_attention_nvfp4(q.numpy(), okc, oks, ovc, ovs, st_k, st_v, np.array(lens, np.int32))
    assert_attention_close(paged.cpu().numpy(), want)


def test_paged_bad_table_entries_are_reported(nv):
    B, H, D, P, M, NP = 2, 1, 128, 128, 2, 4
    table = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    kp = nv.PagedKVPlane.allocate(NP, H, P, D, table)
    vp = nv.PagedKVPlane.allocate(NP, H, P, D, table)
    x = torch.ones(B, 200, H, D, device="cuda")
    st = torch.tensor([0.01], device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_kv_quantize_append_paged(x, torch.zeros(B, dtype=torch.int32, device="cuda"), st, kp,
                                      status=status)
    nv.nvfp4_kv_quantize_append_paged(x, torch.zeros(B, dtype=torch.int32, device="cuda"), st, vp,
                                      status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # sequence 1's second page points outside the pool: appends skip it, attention
    # reads page 0 in its place; both report the bad entry
    bad = torch.tensor([[0, 1], [2, NP]], dtype=torch.int32, device="cuda")
    kb = nv.PagedKVPlane(kp.codes, kp.scales, bad)
    vb = nv.PagedKVPlane(vp.codes, vp.scales, bad)
    before = kp.codes.clone()
    nv.nvfp4_kv_quantize_append_paged(x[:, :1].contiguous(), torch.tensor([150, 150], dtype=torch.int32, device="cuda"),
                                      st, kb, status=status)
    torch.cuda.synchronize()
    assert status.item() == nv.NVFP4_ERR_INVALID_ARG
    assert torch.equal(kp.codes[3], before[3])
    status.zero_()
    q = torch.ones(B, 4, D, dtype=torch.bfloat16, device="cuda")
    out = nv.nvfp4_decode_attention_paged(q, kb, vb, st, st, torch.tensor([200, 200], dtype=torch.int32,
                                                                          device="cuda"), status=status)
    torch.cuda.synchronize()
    assert status.item() == nv.NVFP4_ERR_INVALID_ARG
    assert torch.isfinite(out).all()


def test_dequant_lookup_all_scale_bytes_many_tensor_scales(nv):
    """The FP8 lookup every dequant path shares, against the oracle: every
    (scale byte 0..126, code 0..15) pair -- one plane of 16 tokens x 8 blocks,
    block j holding all 16 codes under scale byte 8t + j -- under 600 tensor
    scales (log-uniform over 2^-40 .. 2^24, plus powers of two and values just
    above and below them), covering normal, subnormal, zero and saturated FP8
    results."""
    S, D = 16, 128
    codes = np.zeros((1, 1, S, D // 2), np.uint8)
    scales = np.zeros((1, 1, S, D // 16), np.uint8)
    nib = np.arange(16, dtype=np.uint8)
    for t in range(S):
        for j in range(D // 16):
            scales[0, 0, t, j] = min(8 * t + j, 0x7E)
            codes[0, 0, t, 8 * j:8 * j + 8] = nib[0::2] | (nib[1::2] << 4)
    plane = nv.KVPlane(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda())
    lens = np.array([S], np.int32)
    lens_d = torch.from_numpy(lens).cuda()
    rng = np.random.default_rng(5)
    sts = list(np.exp2(rng.uniform(-40, 24, 560)).astype(np.float32))
    for e in range(-30, 21, 5):
        p = np.float32(2.0 ** e)
        sts += [p, np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(np.inf)),
                np.float32(p * 1.5)]
    out = torch.empty(1, 1, S, D, dtype=torch.uint8, device="cuda")
    for st in sts:
        st = np.float32(st)
        s = torch.tensor([st], dtype=torch.float32, device="cuda")
        got = nv.nvfp4_kv_dequant_fp8(plane, s, lens_d, out=out).cpu().numpy()
        want = oracle.dequant_planes(codes, scales, st, lens)
        np.testing.assert_array_equal(got, want, err_msg="tensor scale %r" % float(st))


# ---------------------------------------------------------------------------
# append + attention in one call
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D,q_dtype", [(128, "bf16"), (128, "f32"), (64, "bf16")])
def test_append_attention_matches_two_calls_and_oracle(nv, D, q_dtype):
    """nvfp4_decode_attention_append equals quantize_append_kv + decode
    attention bit for bit (planes, new lengths, output), and the oracle within
    tolerance; sequences with 0, 1, 127 (the new token opens a tile), 700 and
    4100 cached tokens, and one whose slot is past the capacity."""
    w = synthetic.shrink(synthetic.get("gqa"), B=6, Hq=16, Hkv=2, D=D)
    lens = [700, 1, 127, 0, 4100, 50]
    S_max = synthetic.capacity(4101)
    c = Case(w, lens=lens, S_max=S_max, q_dtype=q_dtype)
    start = list(lens)
    start[5] = S_max                                      # past the capacity: not appended
    start_d = torch.tensor(start, dtype=torch.int32, device="cuda")
    xk = synthetic.kv_tokens(w, 1, "k", stream=9)
    xv = synthetic.kv_tokens(w, 1, "v", stream=9)
    xk_d, xv_d = to_dev(xk, w.dtype), to_dev(xv, w.dtype)
    planes = {}
    for key in ("two", "one"):
        planes[key] = (nv.KVPlane(c.k.codes.clone(), c.k.scales.clone()),
                       nv.KVPlane(c.v.codes.clone(), c.v.scales.clone()))
    st_two = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_one = torch.zeros(1, dtype=torch.int32, device="cuda")
    lens_two = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    lens_one = torch.full((w.B,), -5, dtype=torch.int32, device="cuda")
    k2, v2 = planes["two"]
    nv.nvfp4_kv_quantize_append_kv(xk_d, xv_d, start_d, c.sk, c.sv, k2, v2, new_lens=lens_two, status=st_two)
    att_lens = start_d + 1
    want_dev = nv.nvfp4_decode_attention(c.q_dev, k2, v2, c.sk, c.sv, att_lens, status=st_two)
    k1, v1 = planes["one"]
    got = nv.nvfp4_decode_attention_append(c.q_dev, xk_d, xv_d, start_d, k1, v1, c.sk, c.sv,
                                           new_lens=lens_one, status=st_one)
    torch.cuda.synchronize()
    assert st_two.item() == nv.NVFP4_ERR_CAPACITY and st_one.item() == nv.NVFP4_ERR_CAPACITY
    assert torch.equal(k1.codes, k2.codes) and torch.equal(k1.scales, k2.scales)
    assert torch.equal(v1.codes, v2.codes) and torch.equal(v1.scales, v2.scales)
    assert lens_one.tolist()[:5] == lens_two.tolist()[:5] == [s + 1 for s in start[:5]]
    assert torch.equal(got, want_dev)
    # oracle: the prefill planes, the new token at slot start, fp64 attention over start + 1
    got = got.cpu().numpy()
    for b in range(5):
        kc, ks, vc, vs = c.oracle_planes(b)
        at = np.array([start[b]], np.int32)
        assert oracle.quantize_append(xk[b:b + 1].numpy(), at, c.sk_o, kc, ks) == 0
        assert oracle.quantize_append(xv[b:b + 1].numpy(), at, c.sv_o, vc, vs) == 0
        want = oracle.decode_attention_nvfp4(c.q[b:b + 1].numpy(), kc, ks, vc, vs, c.sk_o, c.sv_o,
                                             np.array([start[b] + 1], np.int32))
        assert_attention_close(got[b:b + 1], want)


# ---------------------------------------------------------------------------
# failure path: a pipeline wait that gives up
# ---------------------------------------------------------------------------
def test_attention_wait_timeout_reports_and_recovers(nv):
    """With a zero wait limit the tensor-core kernel's first wait that is not
    already complete gives up: the call reports NVFP4_ERR_TIMEOUT through the
    status word, drains its copies and MMAs, releases tensor memory and
    returns (no hang, no fault), and the next call with the default limit is
    correct again.  The limit is set on the host; nothing on the device is
    made to fail."""
    c = Case(synthetic.shrink(synthetic.get("long64k"), L=3000, Hq=16, Hkv=2))
    want = c.oracle_attention()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        nv.nvfp4_set_wait_limit(0)
        nv.nvfp4_decode_attention(c.q_dev, c.k, c.v, c.sk, c.sv, c.seq_lens, status=status)
        torch.cuda.synchronize()
    finally:
        nv.nvfp4_set_wait_limit(-1)
    assert status.item() == nv.NVFP4_ERR_TIMEOUT
    status.zero_()
    got = nv.nvfp4_decode_attention(c.q_dev, c.k, c.v, c.sk, c.sv, c.seq_lens, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert_attention_close(got.cpu().numpy(), want)


# ---- chunked-prefill attention (tensor cores) ----
def _prefill_case(w, start, C, q_dtype=None):
    # the cache holds every sequence up to the end of its chunk
    case = Case(w, lens=[s + C for s in start], q_dtype=q_dtype)
    q = synthetic.prefill_queries(w, C)
    if q_dtype is not None and q_dtype != w.dtype:
        q = q.to(torch.bfloat16 if q_dtype == "bf16" else torch.float32).float()
    return case, q


def _check_prefill(nv, w, start, C, q_dtype=None, softmax_scale=0.0):
    case, q = _prefill_case(w, start, C, q_dtype)
    qd = q_dtype or w.dtype
    start_d = torch.tensor(start, dtype=torch.int32, device="cuda")
    got = nv.nvfp4_prefill_attention(to_dev(q, qd), case.k, case.v, case.sk, case.sv, start_d,
                                     softmax_scale=softmax_scale, status=case.status)
    torch.cuda.synchronize()
    assert case.status.item() == 0
    kc, ks, vc, vs = case.oracle_planes()
    want = oracle.prefill_attention_nvfp4(q.numpy(), kc, ks, vc, vs, case.sk_o, case.sv_o,
                                          np.array(start, np.int32), softmax_scale)
    return assert_attention_close(got.cpu().numpy(), want)


@pytest.mark.parametrize("g,C,start", [(4, 200, [0, 300]), (8, 130, [5, 129]), (1, 300, [77, 0]),
                                       (16, 40, [1000, 3]), (12, 97, [256, 511])])
def test_prefill_attention_parity(nv, g, C, start):
    w = synthetic.shrink(synthetic.get("gqa"), B=len(start), Hkv=2, Hq=2 * g)
    _check_prefill(nv, w, start, C)


def test_prefill_attention_softmax_scale_and_f32_rejected(nv):
    w = synthetic.shrink(synthetic.get("gqa"), B=2, Hkv=1, Hq=8)
    _check_prefill(nv, w, [100, 3], 150, softmax_scale=0.05)
    # fp32 queries are not taken by the tensor-core prefill
    case, q = _prefill_case(w, [0, 0], 16)
    start_d = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(nv.NativeError):
        nv.nvfp4_prefill_attention(q.cuda(), case.k, case.v, case.sk, case.sv, start_d)


def test_prefill_attention_2048_chunk_group12(nv):
    # the large-MoE shape's chunk: 2048 queries x a GQA group of 12, after
    # 1024 cached tokens (two KV heads keep the oracle to seconds)
    w = synthetic.shrink(synthetic.get("moe128k"), B=1, Hkv=2, Hq=24)
    _check_prefill(nv, w, [1024], 2048)


def test_prefill_attention_capacity_and_empty(nv):
    w = synthetic.shrink(synthetic.get("gqa"), B=2, Hkv=1, Hq=4)
    case, q = _prefill_case(w, [0, 0], 64)
    start_d = torch.tensor([0, case.S_max - 10], dtype=torch.int32, device="cuda")
    out = torch.full((2, 64, 4, 128), 7.0, device="cuda")
    nv.nvfp4_prefill_attention(to_dev(q, w.dtype), case.k, case.v, case.sk, case.sv, start_d, out=out,
                               status=case.status)
    torch.cuda.synchronize()
    assert case.status.item() == nv.NVFP4_ERR_CAPACITY
    assert torch.all(out[1] == 7.0).item()              # the over-long sequence is skipped
    kc, ks, vc, vs = case.oracle_planes(0)
    want = oracle.prefill_attention_nvfp4(q[:1].numpy(), kc, ks, vc, vs, case.sk_o, case.sv_o,
                                          np.zeros(1, np.int32))
    assert_attention_close(out[:1].cpu().numpy(), want)
    # an empty chunk is a no-op
    empty = torch.empty(2, 0, 4, 128, device="cuda", dtype=torch.bfloat16)
    nv.nvfp4_prefill_attention(empty, case.k, case.v, case.sk, case.sv, start_d)
