"""Shared test helpers: build the same NVFP4 cache on the GPU (through the
C-ABI binding) and in the oracle (CPU) from one set of seeded inputs, and
compare the two.  Inputs come only from `synthetic`; expected values come
only from `oracle`.
"""
import numpy as np
import torch

import oracle
import synthetic

ATOL_MAX = 2e-2    # attention: max-abs error vs the fp64 oracle
ATOL_MEAN = 2e-3   # attention: mean-abs error vs the fp64 oracle


def to_dev(x_f32: torch.Tensor, dtype: str) -> torch.Tensor:
    t = x_f32.to(torch.float32 if dtype == "f32" else torch.bfloat16)
    return t.contiguous().cuda()


class Case:
    """One workload: inputs, GPU cache and oracle cache built side by side."""

    def __init__(self, w: synthetic.Workload, lens=None, S_max=None, prefill_chunk=None,
                 q_dtype=None):
        import bit_decode_attention_b200 as nv
        self.w = w
        self.lens = list(lens if lens is not None else synthetic.seq_lens(w))
        Lmax = max(self.lens) if self.lens else 0
        self.S_max = S_max or synthetic.capacity(max(Lmax, 1))
        self.q_dtype = q_dtype or w.dtype
        B, H, D = w.B, w.Hkv, w.D
        # inputs (fp32 values exact in the workload dtype), token-major
        self.xk = synthetic.kv_tokens(w, Lmax, "k")
        self.xv = synthetic.kv_tokens(w, Lmax, "v")
        self.q = synthetic.queries(w)
        if self.q_dtype != w.dtype:
            self.q = self.q.to(torch.bfloat16 if self.q_dtype == "bf16" else torch.float32).float()
        # calibration over every token that will be stored (per tensor)
        mask = torch.zeros(B, Lmax, dtype=torch.bool)
        for b, L in enumerate(self.lens):
            mask[b, :L] = True
        self.mask = mask
        xk_used = self.xk[mask]
        xv_used = self.xv[mask]
        st, self.sk_o = oracle.tensor_scale(xk_used.numpy())
        assert st == 0
        st, self.sv_o = oracle.tensor_scale(xv_used.numpy())
        assert st == 0
        # GPU: calibrate on the same values, then append in chunks
        self.sk = nv.nvfp4_calib_tensor_scale(to_dev(xk_used, w.dtype))
        self.sv = nv.nvfp4_calib_tensor_scale(to_dev(xv_used, w.dtype))
        self.k = nv.KVPlane.allocate(B, H, self.S_max, D)
        self.v = nv.KVPlane.allocate(B, H, self.S_max, D)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        chunk = prefill_chunk or max(Lmax, 1)
        xk_d, xv_d = to_dev(self.xk, w.dtype), to_dev(self.xv, w.dtype)
        for b in range(B):
            sub_k = nv.KVPlane(self.k.codes[b:b + 1], self.k.scales[b:b + 1])
            sub_v = nv.KVPlane(self.v.codes[b:b + 1], self.v.scales[b:b + 1])
            for lo in range(0, self.lens[b], chunk):
                hi = min(self.lens[b], lo + chunk)
                start = torch.tensor([lo], dtype=torch.int32, device="cuda")
                nv.nvfp4_kv_quantize_append(xk_d[b:b + 1, lo:hi].contiguous(), start, self.sk, sub_k,
                                            status=self.status)
                nv.nvfp4_kv_quantize_append(xv_d[b:b + 1, lo:hi].contiguous(), start, self.sv, sub_v,
                                            status=self.status)
        self.seq_lens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")
        self.q_dev = to_dev(self.q, self.q_dtype)
        torch.cuda.synchronize()

    # ---- oracle side ----
    def oracle_planes(self, batch_index=None):
        """Oracle planes for all (or one) sequences, from the raw inputs."""
        w = self.w
        bs = range(w.B) if batch_index is None else [batch_index]
        kc, ks = oracle.new_planes(len(bs), w.Hkv, self.S_max, w.D)
        vc, vs = oracle.new_planes(len(bs), w.Hkv, self.S_max, w.D)
        for i, b in enumerate(bs):
            L = self.lens[b]
            if L == 0:
                continue
            z = np.zeros(1, np.int32)
            tk = oracle.new_planes(1, w.Hkv, self.S_max, w.D)
            tv = oracle.new_planes(1, w.Hkv, self.S_max, w.D)
            assert oracle.quantize_append(self.xk[b:b + 1, :L].numpy(), z, self.sk_o, *tk) == 0
            assert oracle.quantize_append(self.xv[b:b + 1, :L].numpy(), z, self.sv_o, *tv) == 0
            kc[i], ks[i], vc[i], vs[i] = tk[0][0], tk[1][0], tv[0][0], tv[1][0]
        return kc, ks, vc, vs

    def oracle_attention(self, batch_index=None, softmax_scale=0.0):
        w = self.w
        kc, ks, vc, vs = self.oracle_planes(batch_index)
        bs = list(range(w.B)) if batch_index is None else [batch_index]
        q = self.q[bs].numpy()
        lens = np.array([self.lens[b] for b in bs], np.int32)
        return oracle.decode_attention_nvfp4(q, kc, ks, vc, vs, self.sk_o, self.sv_o, lens,
                                             softmax_scale)

    def gpu_attention(self, softmax_scale=0.0, workspace=None):
        import bit_decode_attention_b200 as nv
        out = nv.nvfp4_decode_attention(self.q_dev, self.k, self.v, self.sk, self.sv, self.seq_lens,
                                        softmax_scale=softmax_scale, workspace=workspace,
                                        status=self.status)
        torch.cuda.synchronize()
        return out


def assert_attention_close(got, want, atol_max=ATOL_MAX, atol_mean=ATOL_MEAN):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got))
    err = np.abs(got - want)
    assert err.max() <= atol_max, "max-abs error %.3g" % err.max()
    assert err.mean() <= atol_mean, "mean-abs error %.3g" % err.mean()
    return err.max(), err.mean()
